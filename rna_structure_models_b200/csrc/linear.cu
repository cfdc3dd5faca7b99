// Dense projection y = x W + b on the tensor cores (tcgen05, fp32
// accumulation in tensor memory).  The module around the IPA core uses it for
// the q / k / v / point projections of the single representation and for the
// output projection (Flash Invariant Point Attention keeps the IPA layer's
// projections; the factorised core sits between them).
//
// Two operand paths:
//   * tf32 (x row-major with 16-byte aligned rows, the common case): x is
//     read by TMA straight from the caller's fp32 array as K-major 128 x 32
//     tiles; W is transposed once per call into fp32 W^T [N, Kq] (Kq = K
//     rounded up to 4) by linear_pack_w_kernel<float>, read the same way, and
//     the two are multiplied with tcgen05.mma kind::tf32 (K = 8 per
//     instruction).  The copies zero-fill past M, N and K.
//   * fp16 (any other x strides):
//       linear_pack_x_kernel -- x -> fp16 [M, Kp], K zero-padded to 64
//       linear_pack_w_kernel -- W [K, N] -> W^T fp16 [N, Kp] (shared-memory
//                               transpose)
//     then K-major 128 x 64 tiles of both, kind::f16 (K = 16).
//   linear_kernel<TF32> -- one CTA per 128 x 128 tile of y, two CTAs per SM: a
//     three-stage TMA ring, one thread issuing the MMAs (M = N = 128), four
//     warps reading the accumulator back (+ b).
// Every mbarrier wait is bounded; on expiry the CTA records an error code,
// drains what it started, frees tensor memory and exits.
#include <cuda_fp16.h>

#include <cmath>
#include <cstdint>

#include "bounds.cuh"
#include "internal.h"
#include "sm100.cuh"

#define IPA_FILE_TAG 10

namespace fipa {

using namespace sm100;

namespace {

// Three stages: K is a few hundred to two thousand here, and 99 KB of shared
// memory lets two CTAs share an SM, so one CTA's epilogue overlaps the other's
// main loop (input projection at L = 4096: 41 -> 31 us; four stages kept one
// CTA per SM).
constexpr int LBM = 128, LBN = 128, LBK = 64, LST = 3;
constexpr uint32_t L_TILE = 16384;                 // 128 rows x 64 fp16
constexpr uint32_t L_STAGE = 2 * L_TILE;           // x tile | W^T tile
constexpr uint32_t L_AUX = LST * L_STAGE;
constexpr uint32_t L_SMEM = L_AUX + 256;
constexpr uint32_t L_ALLOC = L_SMEM + 1024;
enum { LB_FULL0 = 0, LB_EMPTY0 = LST, LB_DONE = 2 * LST, LB_DRAIN, LB_COUNT };
constexpr uint32_t L_TMEM_SLOT = 8 * LB_COUNT;
constexpr uint32_t L_ABORT = L_TMEM_SLOT + 8;

struct LinArgs {
  int M, N, nk;
  const float* bias;   // [N] or null
  float* y;            // [M, ldy]
  int64_t ldy;
  int* err;
};

__device__ __forceinline__ uint64_t kmaj(uint32_t saddr) { return smem_desc_sw128(saddr, 16, 1024); }

// Instruction descriptor for .kind::tf32 (A and B tf32, D f32): the fields of
// the .kind::f16 one with format 2 (tf32) for A and B.
__host__ __device__ __forceinline__ uint32_t idesc_tf32(int M, int N, bool b_mn_major) {
  uint32_t d = 0;
  d |= 1u << 4;
  d |= 2u << 7;
  d |= 2u << 10;
  d |= (b_mn_major ? 1u : 0u) << 16;
  d |= static_cast<uint32_t>(N >> 3) << 17;
  d |= static_cast<uint32_t>(M >> 4) << 24;
  return d;
}

__device__ __forceinline__ void umma_ss_tf32(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// K blocks of 128 bytes per row (32 tf32 or 64 fp16), both operands K-major
// with the 128-byte swizzle.
template <bool TF32>
__global__ void __launch_bounds__(192, 2)
    linear_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                  const LinArgs a) {
  extern __shared__ unsigned char lin_smem_raw[];
  const uint32_t raw = smem_u32(lin_smem_raw);
  const uint32_t sb = (raw + 1023u) & ~1023u;
  unsigned char* smem = lin_smem_raw + (sb - raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int m0 = blockIdx.y * LBM, n0 = blockIdx.x * LBN;
  auto bar = [&](int k) -> uint32_t { return sb + L_AUX + 8u * k; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L_AUX + L_ABORT);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L_AUX + L_TMEM_SLOT);

  if (tid == 0) {
    for (int s = 0; s < LST; ++s) {
      mbar_init(bar(LB_FULL0 + s), 1);
      mbar_init(bar(LB_EMPTY0 + s), 1);
    }
    mbar_init(bar(LB_DONE), 1);
    mbar_init(bar(LB_DRAIN), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(tmem_slot), LBN);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_w);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  auto fail = [&](int code) {
    record_error(a.err, code);
    *abort_flag = 1;
  };

  if (warp == 4) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      int issued = 0;
      for (int kt = 0; kt < a.nk; ++kt) {
        const int s = kt % LST;
        if (kt >= LST && !mbar_wait_bounded(bar(LB_EMPTY0 + s), ((kt / LST) - 1) & 1, abort_flag)) {
          fail(DEV_TIMEOUT_EMPTY);
          break;
        }
        const uint32_t st = sb + s * L_STAGE;
        mbar_arrive_expect_tx(bar(LB_FULL0 + s), L_STAGE);
        const int kx = kt * (TF32 ? 32 : LBK);   // first K element of the block
        tma_load_3d(st, &tm_x, bar(LB_FULL0 + s), kx, m0, 0);
        tma_load_3d(st + L_TILE, &tm_w, bar(LB_FULL0 + s), kx, n0, 0);
        issued = kt + 1;
      }
      if (*abort_flag)   // let the copies already started land before the CTA exits
        for (int kt = (issued > LST ? issued - LST : 0); kt < issued; ++kt)
          mbar_wait_bounded(bar(LB_FULL0 + kt % LST), (kt / LST) & 1, nullptr, 100000000ull);
    }
  } else if (warp == 5) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = TF32 ? idesc_tf32(LBM, LBN, false) : idesc_f16(LBM, LBN, false);
      bool ok = true, issued_any = false;
      for (int kt = 0; kt < a.nk; ++kt) {
        const int s = kt % LST;
        if (!mbar_wait_bounded(bar(LB_FULL0 + s), (kt / LST) & 1, abort_flag)) {
          fail(DEV_TIMEOUT_FULL);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t st = sb + s * L_STAGE;
#pragma unroll
        for (int k = 0; k < 4; ++k) {   // 32 bytes of K per instruction: 8 tf32 or 16 fp16
          const uint32_t acc = (kt > 0 || k > 0) ? 1u : 0u;
          if (TF32)
            umma_ss_tf32(tmem, kmaj(st + 32 * k), kmaj(st + L_TILE + 32 * k), idesc, acc);
          else
            umma_ss(tmem, kmaj(st + 32 * k), kmaj(st + L_TILE + 32 * k), idesc, acc);
        }
        umma_commit(bar(LB_EMPTY0 + s));
        issued_any = true;
      }
      if (ok) {
        umma_commit(bar(LB_DONE));
      } else if (issued_any) {
        umma_commit(bar(LB_DRAIN));
        mbar_wait_bounded(bar(LB_DRAIN), 0, nullptr, 100000000ull);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ epilogue: rows m0 + 32 warp + lane
    const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(bar(LB_DONE), 0, abort_flag));
    if (ok) {
      tc_fence_after();
      const int row = m0 + warp * 32 + lane;
      const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
      // this CTA's columns [n0, n0 + LBN) of the row, within [M - 1 rows of ldy, then N]
      const int ncol = a.N - n0 < LBN ? a.N - n0 : LBN;
      float* yr = IPA_SPAN(a.y, static_cast<int64_t>(row < a.M ? row : 0) * a.ldy + n0, ncol,
                           static_cast<int64_t>(a.M - 1) * a.ldy + a.N, a.err) - n0;
      for (int c0 = 0; c0 < LBN; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(tmem + c0 + lane_off, v);
        tmem_ld_wait();
        const int col0 = n0 + c0;
        if (row >= a.M || col0 >= a.N) continue;
        if (col0 + 32 <= a.N && (a.ldy & 3) == 0) {
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            float4 o = make_float4(__uint_as_float(v[e]), __uint_as_float(v[e + 1]), __uint_as_float(v[e + 2]),
                                   __uint_as_float(v[e + 3]));
            if (a.bias) {
              o.x += a.bias[col0 + e];
              o.y += a.bias[col0 + e + 1];
              o.z += a.bias[col0 + e + 2];
              o.w += a.bias[col0 + e + 3];
            }
            *reinterpret_cast<float4*>(yr + col0 + e) = o;
          }
        } else {
          for (int e = 0; e < 32 && col0 + e < a.N; ++e)
            yr[col0 + e] = __uint_as_float(v[e]) + (a.bias ? a.bias[col0 + e] : 0.f);
        }
      }
    } else if (lane == 0) {
      fail(DEV_TIMEOUT_MMA);
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, LBN);
  }
}

struct PackX {
  int M, K, Kp;
  View x;          // [M, K] fp32 (strides s[0], s[1])
  __half* out;     // [M, Kp]
  int* err;
};

// One thread per 8 consecutive elements of a row (Kp is a multiple of 64, so
// a group never straddles rows): two 16-byte loads when the row is dense and
// the group lies inside K and 16-byte aligned, element loads otherwise; one
// 16-byte store of the 8 fp16 values.
__global__ void __launch_bounds__(256) linear_pack_x_kernel(const PackX a) {
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t n = static_cast<int64_t>(a.M) * (a.Kp / 8);
  if (t >= n) return;
  const int m = static_cast<int>(t / (a.Kp / 8)), k = 8 * static_cast<int>(t % (a.Kp / 8));
  const float* x = static_cast<const float*>(a.x.p) + m * a.x.s[0];
  float v[8];
  if (a.x.s[1] == 1 && k + 8 <= a.K && (reinterpret_cast<uintptr_t>(x + k) & 15u) == 0) {
    const float4 lo = __ldg(reinterpret_cast<const float4*>(x + k)), hi = __ldg(reinterpret_cast<const float4*>(x + k) + 1);
    v[0] = lo.x; v[1] = lo.y; v[2] = lo.z; v[3] = lo.w; v[4] = hi.x; v[5] = hi.y; v[6] = hi.z; v[7] = hi.w;
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = k + e < a.K ? x[(k + e) * a.x.s[1]] : 0.f;
  }
  *IPA_AT(reinterpret_cast<uint4*>(a.out), t, n, a.err) =
      make_uint4(pack_half2(v[0], v[1]), pack_half2(v[2], v[3]), pack_half2(v[4], v[5]), pack_half2(v[6], v[7]));
}

template <class T>
struct PackW {
  int K, N, Kp;
  View w;          // [K, N] fp32
  T* out;          // [N, Kp]
  int* err;
};

__device__ __forceinline__ void store_elem(__half* p, float v) { *p = __float2half_rn(v); }
__device__ __forceinline__ void store_elem(float* p, float v) { *p = v; }

// 32 x 32 tiles: read along n (contiguous in W), write along k (contiguous in
// W^T); fp16 W^T for the fp16 path, fp32 for the tf32 one
template <class T>
__global__ void __launch_bounds__(256) linear_pack_w_kernel(const PackW<T> a) {
  __shared__ float tile[32][33];
  const int k0 = blockIdx.x * 32, n0 = blockIdx.y * 32;
  const float* w = static_cast<const float*>(a.w.p);
  for (int r = threadIdx.y; r < 32; r += 8) {
    const int k = k0 + r, n = n0 + threadIdx.x;
    tile[r][threadIdx.x] = (k < a.K && n < a.N) ? w[k * a.w.s[0] + n * a.w.s[1]] : 0.f;
  }
  __syncthreads();
  for (int r = threadIdx.y; r < 32; r += 8) {
    const int n = n0 + r, k = k0 + threadIdx.x;
    if (n < a.N && k < a.Kp)
      store_elem(IPA_AT(a.out, static_cast<int64_t>(n) * a.Kp + k, static_cast<int64_t>(a.N) * a.Kp, a.err),
                 tile[threadIdx.x][r]);
  }
}

}  // namespace

LinearWorkspace linear_workspace_layout(int M, int K, int N) {
  auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  LinearWorkspace w{};
  const size_t Kp = (static_cast<size_t>(K) + 63) / 64 * 64;
  size_t o = 0;
  w.x16 = o; o = up(o + static_cast<size_t>(M) * Kp * 2);
  w.w16 = o; o = up(o + static_cast<size_t>(N) * Kp * 2);
  // tf32 path: fp32 W^T [N, Kq] from offset 0 (the fp16 buffers are unused there)
  const size_t Kq = (static_cast<size_t>(K) + 3) / 4 * 4;
  w.w32 = 0;
  w.total = o > up(static_cast<size_t>(N) * Kq * 4) ? o : up(static_cast<size_t>(N) * Kq * 4);
  return w;
}

namespace {
bool tf32_rows(const View& v) {
  return v.dtype == 0 && v.s[1] == 1 && v.s[0] % 4 == 0 && (reinterpret_cast<uintptr_t>(v.p) & 15u) == 0;
}
}  // namespace

cudaError_t linear_launch(const LinearLaunch& a, cudaStream_t st) {
  cudaError_t e;
  if (tf32_rows(a.x)) {
    // x [M, K] straight from the caller's array, W^T [N, Kq] fp32 from the
    // workspace: both as 128 x 32 K-major boxes
    const int Kq = (a.K + 3) / 4 * 4;
    float* w32 = reinterpret_cast<float*>(a.ws + a.lay.w32);
    CUtensorMap tx, tw;
    const uint64_t xd[3] = {static_cast<uint64_t>(a.K), static_cast<uint64_t>(a.M), 1};
    const uint64_t xs[2] = {static_cast<uint64_t>(a.x.s[0]) * 4, static_cast<uint64_t>(a.x.s[0]) * 4 * a.M};
    const uint32_t xb[3] = {32, LBM, 1};
    const uint64_t wd[3] = {static_cast<uint64_t>(a.K), static_cast<uint64_t>(a.N), 1};
    const uint64_t wsb[2] = {static_cast<uint64_t>(Kq) * 4, static_cast<uint64_t>(Kq) * 4 * a.N};
    const uint32_t wb[3] = {32, LBN, 1};
    if (encode_tmap_f32_sw128(&tx, a.x.p, 3, xd, xs, xb) && encode_tmap_f32_sw128(&tw, w32, 3, wd, wsb, wb)) {
      PackW<float> pw{a.K, a.N, Kq, a.w, w32, a.err};
      linear_pack_w_kernel<float><<<dim3((Kq + 31) / 32, (a.N + 31) / 32), dim3(32, 8), 0, st>>>(pw);
      e = cudaFuncSetAttribute(linear_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(L_ALLOC));
      if (e != cudaSuccess) return e;
      LinArgs la{a.M, a.N, (a.K + 31) / 32, a.bias, a.y, a.ldy, a.err};
      linear_kernel<true><<<dim3((a.N + LBN - 1) / LBN, (a.M + LBM - 1) / LBM), 192, L_ALLOC, st>>>(tx, tw, la);
      return cudaGetLastError();
    }
  }
  const int Kp = (a.K + 63) / 64 * 64;
  __half* x16 = reinterpret_cast<__half*>(a.ws + a.lay.x16);
  __half* w16 = reinterpret_cast<__half*>(a.ws + a.lay.w16);
  {
    PackX p{a.M, a.K, Kp, a.x, x16, a.err};
    const int64_t n = static_cast<int64_t>(a.M) * (Kp / 8);
    linear_pack_x_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, st>>>(p);
  }
  {
    PackW<__half> p{a.K, a.N, Kp, a.w, w16, a.err};
    linear_pack_w_kernel<__half><<<dim3(Kp / 32, (a.N + 31) / 32), dim3(32, 8), 0, st>>>(p);
  }
  CUtensorMap tx, tw;
  if (!encode_tmap_f16_3d(&tx, x16, Kp, a.M, 1, static_cast<uint64_t>(Kp) * 2,
                          static_cast<uint64_t>(Kp) * 2 * a.M, LBK, LBM) ||
      !encode_tmap_f16_3d(&tw, w16, Kp, a.N, 1, static_cast<uint64_t>(Kp) * 2,
                          static_cast<uint64_t>(Kp) * 2 * a.N, LBK, LBN))
    return cudaErrorInvalidValue;
  e = cudaFuncSetAttribute(linear_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(L_ALLOC));
  if (e != cudaSuccess) return e;
  LinArgs la{a.M, a.N, Kp / LBK, a.bias, a.y, a.ldy, a.err};
  linear_kernel<false><<<dim3((a.N + LBN - 1) / LBN, (a.M + LBM - 1) / LBM), 192, L_ALLOC, st>>>(tx, tw, la);
  return cudaGetLastError();
}

}  // namespace fipa
