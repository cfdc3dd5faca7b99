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

bool make_map(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint32_t box_rows,
              uint32_t box_cols = 64, CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_128B) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {cols, rows, 1};
  const cuuint64_t str[2] = {cols * 2, cols * rows * 2};
  const cuuint32_t box[3] = {box_cols, box_rows, 1};
  const cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void*>(base), dims, str, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// CTA-pair probe (cluster of 2, cta_group::2, M = 256):
//   mode 0: D[256 x 128] = A[256 x 64] . B[128 x 64]^T; A and B by pair TMA
//           (each CTA: its 128 rows of A, its 64 rows of B), both K-major;
//   mode 1: D[256 x 256] = A . B[64 x 256]; A written to tensor memory by the
//           threads, B MN-major 128-byte swizzle, each CTA 128 of the N columns;
//   mode 2: D[256 x 64]  = A . B[64 x 64]; like mode 1 with a 64-byte
//           swizzled B, each CTA 32 of the N columns.
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(128, 1)
    pair_probe_kernel(const __grid_constant__ CUtensorMap tma, const __grid_constant__ CUtensorMap tmb, int mode,
                      int nn, const __half* A, float* D, int* err) {
  extern __shared__ unsigned char raw[];
  const uint32_t r32 = smem_u32(raw);
  const uint32_t sb = (r32 + 1023u) & ~1023u;
  unsigned char* sm = raw + (sb - r32);
  const uint32_t SA = 0, SB = 16384, BAR = 65536, SLOT = BAR + 64;
  const uint32_t FULL = sb + BAR, DONE = sb + BAR + 8, READY = sb + BAR + 16;
  const int tid = threadIdx.x, warp = tid >> 5;
  const uint32_t rank = cluster_ctarank();
  uint32_t* slot = reinterpret_cast<uint32_t*>(sm + SLOT);
  if (tid == 0) {
    mbar_init(FULL, 2);
    mbar_init(DONE, 1);
    mbar_init(READY, 2);
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc_pair(smem_u32(slot), 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *slot;
  const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
  const int row0 = static_cast<int>(rank) * 128;
  if (mode != 0) {
    const uint4* src = reinterpret_cast<const uint4*>(A + (row0 + tid) * 64);
    uint32_t r[32];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const uint4 v = src[e];
      r[4 * e] = v.x; r[4 * e + 1] = v.y; r[4 * e + 2] = v.z; r[4 * e + 3] = v.w;
    }
    tmem_st32(tmem + 384 + lane_off, r);
    tmem_st_wait();
  }
  tc_fence_before();
  __syncthreads();
  if (tid == 0) {
    mbar_arrive_cluster(mapa_shared(READY, 0));
    uint32_t bytes = 0;
    const uint32_t full0 = mapa_shared(FULL, 0);
    if (mode == 0) bytes = 16384 + 8192;
    if (mode == 1) bytes = 2 * 8192;
    if (mode == 2) bytes = 4096;
    mbar_arrive_expect_tx_cluster(full0, bytes);
    if (mode == 0) {
      tma_load_3d_pair(sb + SA, &tma, full0, 0, row0, 0);
      tma_load_3d_pair(sb + SB, &tmb, full0, 0, 64 * static_cast<int>(rank), 0);
    } else if (mode == 1) {
      for (int p = 0; p < 2; ++p)
        tma_load_3d_pair(sb + SB + 8192 * p, &tmb, full0, 128 * static_cast<int>(rank) + 64 * p, 0, 0);
    } else {
      tma_load_3d_pair(sb + SB, &tmb, full0, 32 * static_cast<int>(rank), 0, 0);
    }
  }
  if (rank == 0 && tid == 0) {
    const bool ok = mbar_wait_bounded(FULL, 0, nullptr, 200000000ull) &&
                    mbar_wait_bounded(READY, 0, nullptr, 200000000ull);
    if (!ok) {
      record_error(err, DEV_TIMEOUT_FULL);
    } else {
      tc_fence_after();
      for (int k = 0; k < 4; ++k) {
        if (mode == 0)
          umma2_ss(tmem, smem_desc(sb + SA + 32 * k, 16, 1024, 2), smem_desc(sb + SB + 32 * k, 16, 1024, 2),
                   idesc_f16(256, 128, false), k > 0);
        else if (mode == 1)
          umma2_ts(tmem, tmem + 384 + 8 * k, smem_desc(sb + SB + 2048 * k, 8192, 1024, 2),
                   idesc_f16(256, 256, true), k > 0);
        else
          umma2_ts(tmem, tmem + 384 + 8 * k, smem_desc(sb + SB + 1024 * k, 8192, 512, 4),
                   idesc_f16(256, 64, true), k > 0);
      }
      umma2_commit_both(DONE);
    }
  }
  const bool done = mbar_wait_bounded(DONE, 0, nullptr, 300000000ull);
  if (!done) {
    if (tid == 0) record_error(err, DEV_TIMEOUT_MMA);
  } else {
    tc_fence_after();
    for (int c0 = 0; c0 < nn; c0 += 32) {
      uint32_t r[32];
      tmem_ld32(tmem + c0 + lane_off, r);
      tmem_ld_wait();
      for (int e = 0; e < 32; ++e) D[(row0 + tid) * nn + c0 + e] = __uint_as_float(r[e]);
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
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

// CTA-pair probe: mode 0 needs A [256 x 64] and B [128 x 64] (K contiguous);
// modes 1 / 2 need A [256 x 64] and B [64 x nn] (N contiguous), nn = 256 / 64.
extern "C" __attribute__((visibility("default"))) int probe_umma_pair(int mode, const void* A, const void* B,
                                                                    float* D, int* err, void* stream) {
  if (mode < 0 || mode > 2) return 1;
  const int nn = mode == 0 ? 128 : mode == 1 ? 256 : 64;
  CUtensorMap ma{}, mb{};
  if (!make_map(&ma, A, 64, 256, 128)) return 2;
  if (mode == 0 && !make_map(&mb, B, 64, 128, 64)) return 2;
  if (mode == 1 && !make_map(&mb, B, 256, 64, 64)) return 2;
  if (mode == 2 && !make_map(&mb, B, 64, 64, 64, 32, CU_TENSOR_MAP_SWIZZLE_64B)) return 2;
  const int smem = 65536 + 1024 + 1024;
  if (cudaFuncSetAttribute(pair_probe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return 3;
  pair_probe_kernel<<<2, 128, smem, static_cast<cudaStream_t>(stream)>>>(ma, mb, mode, nn,
                                                                         static_cast<const __half*>(A), D, err);
  return cudaGetLastError() == cudaSuccess ? 0 : 4;
}
