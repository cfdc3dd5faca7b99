// Test-only probe library: exercises, one at a time, the sm_100a building
// blocks the fused IPA kernel relies on, so that a layout or descriptor
// mistake shows up as a failing small GEMM instead of a wrong attention
// output.  Built next to the tests; not part of the product library.
//
//   mode 0: D[128 x 64]  = A[128 x 64] . B[64 x 64]^T  A, B by TMA (128B swizzle), both K-major
//   mode 1: same, A written into tensor memory by the threads (A from TMEM)
//   mode 2: D[128 x N]   = A[128 x 64] . B[64 x N]     B by TMA, MN-major, N = 64 or 256
//   mode 3: same as 0, A written into shared memory by the threads with the
//           128B swizzle pattern the softmax warps use for P
// Plus a bounded-wait probe: a kernel waits on an mbarrier nothing arrives on
// and must come back with an error code instead of hanging.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "sm100.cuh"

using namespace sm100;

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                   CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

bool make_map(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {cols, rows, 1};
  const cuuint64_t str[2] = {cols * 2, cols * rows * 2};
  const cuuint32_t box[3] = {64, box_rows, 1};
  const cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void*>(base), dims, str, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

__global__ void __launch_bounds__(128, 1)
    probe_kernel(const __grid_constant__ CUtensorMap tma, const __grid_constant__ CUtensorMap tmb, int mode,
                 int nn, const __half* A, float* D, int* err) {
  extern __shared__ unsigned char raw[];
  const uint32_t r32 = smem_u32(raw);
  const uint32_t sb = (r32 + 1023u) & ~1023u;
  unsigned char* sm = raw + (sb - r32);
  const uint32_t SA = 0, SB = 16384;           // A 16 KB, B up to 32 KB
  const uint32_t BAR = 65536, SLOT = BAR + 64;
  const int tid = threadIdx.x, warp = tid >> 5;
  uint32_t* slot = reinterpret_cast<uint32_t*>(sm + SLOT);
  if (tid == 0) {
    mbar_init(sb + BAR, 1);
    mbar_init(sb + BAR + 8, 1);
    mbar_init(sb + BAR + 16, 128);
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *slot;
  const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;

  // stage A (threads) when the mode needs it
  if (mode == 1) {
    // row tid of A -> tensor memory columns [256, 288): 64 fp16 packed in pairs
    const uint4* src = reinterpret_cast<const uint4*>(A + tid * 64);
    uint32_t r[32];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const uint4 v = src[e];
      r[4 * e] = v.x; r[4 * e + 1] = v.y; r[4 * e + 2] = v.z; r[4 * e + 3] = v.w;
    }
    tmem_st32(tmem + 256 + lane_off, r);
    tmem_st_wait();
  } else if (mode == 3) {
    const uint4* src = reinterpret_cast<const uint4*>(A + tid * 64);
    unsigned char* row = sm + SA + tid * 128;
#pragma unroll
    for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4*>(row + ((c ^ (tid & 7)) << 4)) = src[c];
    fence_proxy_async_smem();
  }
  tc_fence_before();
  mbar_arrive(sb + BAR + 16);

  if (tid == 0) {
    uint32_t bytes = (mode == 2) ? static_cast<uint32_t>(nn) * 128u : 8192u;
    if (mode == 0 || mode == 2) bytes += 16384u;
    mbar_arrive_expect_tx(sb + BAR, bytes);
    if (mode == 0 || mode == 2) tma_load_3d(sb + SA, &tma, sb + BAR, 0, 0, 0);
    if (mode == 2) {
      for (int p = 0; p < nn / 64; ++p) tma_load_3d(sb + SB + 8192 * p, &tmb, sb + BAR, 64 * p, 0, 0);
    } else {
      tma_load_3d(sb + SB, &tmb, sb + BAR, 0, 0, 0);
    }
    bool ok = mbar_wait_bounded(sb + BAR, 0, nullptr, 200000000ull) &&
              mbar_wait_bounded(sb + BAR + 16, 0, nullptr, 200000000ull);
    if (!ok) {
      record_error(err, DEV_TIMEOUT_FULL);
    } else {
      tc_fence_after();
      if (mode == 2) {
        const uint32_t id = idesc_f16(128, nn, true);
        for (int k = 0; k < 4; ++k)
          umma_ss(tmem, smem_desc_sw128(sb + SA + 32 * k, 16, 1024), smem_desc_sw128(sb + SB + 2048 * k, 8192, 1024),
                  id, k > 0);
      } else {
        const uint32_t id = idesc_f16(128, 64, false);
        for (int k = 0; k < 4; ++k) {
          if (mode == 1)
            umma_ts(tmem, tmem + 256 + 8 * k, smem_desc_sw128(sb + SB + 32 * k, 16, 1024), id, k > 0);
          else
            umma_ss(tmem, smem_desc_sw128(sb + SA + 32 * k, 16, 1024), smem_desc_sw128(sb + SB + 32 * k, 16, 1024),
                    id, k > 0);
        }
      }
      umma_commit(sb + BAR + 8);
    }
  }
  __syncthreads();
  const bool done = mbar_wait_bounded(sb + BAR + 8, 0, nullptr, 200000000ull);
  if (!done) {
    if (tid == 0) record_error(err, DEV_TIMEOUT_MMA);
  } else {
    tc_fence_after();
    for (int c0 = 0; c0 < nn; c0 += 32) {
      uint32_t r[32];
      tmem_ld32(tmem + c0 + lane_off, r);
      tmem_ld_wait();
      for (int e = 0; e < 32; ++e) D[tid * nn + c0 + e] = __uint_as_float(r[e]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

__global__ void timeout_kernel(int* err, unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = smem_u32(&bar);
  if (threadIdx.x == 0) {
    mbar_init(b, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // nothing ever arrives on this barrier: the bounded wait must give up
    if (!mbar_wait_bounded(b, 0, nullptr, limit_ns)) record_error(err, DEV_TIMEOUT_PROBE);
  }
}

}  // namespace

extern "C" __attribute__((visibility("default"))) int probe_umma(int mode, int nn, const void* A, const void* B,
                                                               float* D, int* err, void* stream) {
  if (mode < 0 || mode > 3) return 1;
  if (mode != 2) nn = 64;
  if (nn != 64 && nn != 128 && nn != 256) return 1;
  CUtensorMap ma{}, mb{};
  if (!make_map(&ma, A, 64, 128, 128)) return 2;
  if (mode == 2) {
    if (!make_map(&mb, B, nn, 64, 64)) return 2;
  } else {
    if (!make_map(&mb, B, 64, 64, 64)) return 2;
  }
  const int smem = 65536 + 1024 + 1024;
  if (cudaFuncSetAttribute(probe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return 3;
  probe_kernel<<<1, 128, smem, static_cast<cudaStream_t>(stream)>>>(ma, mb, mode, nn,
                                                                     static_cast<const __half*>(A), D, err);
  return cudaGetLastError() == cudaSuccess ? 0 : 4;
}

extern "C" __attribute__((visibility("default"))) int probe_bounded_wait(int* err, unsigned long long limit_ns,
                                                                       void* stream) {
  timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(err, limit_ns);
  return cudaGetLastError() == cudaSuccess ? 0 : 4;
}
