// Fused attention pass of the IPA core for sm_100a: one CTA per
// (batch, head, 128-query tile), a flash-style loop over 64-key tiles.
//
// Warp roles (320 threads):
//   warps 0-7  softmax and epilogue, two threads per query row (column halves
//              of S; tensor-memory lane = row);
//   warp 8     producer: per key tile, the fp32 column term and the TMA loads
//              of K_h, V_h and the shared Z2 tile into a 3-stage ring;
//   warp 9     tensor-memory allocation and the single MMA-issuing thread.
// A pair width of 0 (no pair block) skips every Q_pair / Z2 step.
//
// Per key tile j (MMA issue order QK(0), QK(1), PV(0), QK(2), PV(1), ...):
//   S  = Q_h . K_h^T (A from shared memory, K = 64)
//      + Q_pair . Z2^T (A from tensor memory, K = DZ)        -> TMEM, 64 cols
//   softmax warps: x = S + col_j, online max with lazy rescaling (only when
//      the running max grows by more than tau = 8 in log2 units; exact since
//      the final division uses the same stale max), P = exp2(x - m) rounded to
//      fp16 into shared memory, l summed from the ROUNDED P so that the
//      normalisation matches what the MMA aggregates;
//   O += P . [V_h | Z2]   (N = 64 and N = DZ, B operand MN-major)      -> TMEM
// Epilogue: O / l, value points mapped back with R_i^T (relative to the
// centroid), their norms, the pair output sum_r z1_i[r] (P Z2)[r], zero rows
// for queries without an allowed key; staged through shared memory and
// written with coalesced row stores.
//
// Tensor memory (512 columns): O [0, 64+DZ) | S [320, 384) | Q_pair [384, 384+DZ/2).
// Shared memory: Q_h 16 KB | 3 x (K_h 8 KB | V_h 8 KB | Z2 DZ*128 B) | 2 x P 16 KB.
// Every mbarrier wait is bounded (2 s); on expiry the CTA records an error
// code, raises a CTA-wide abort flag, drains its in-flight copies and MMAs,
// frees tensor memory and exits.
#include <cuda_fp16.h>

#include <cmath>
#include <cstdint>

#include "internal.h"
#include "bounds.cuh"
#include "ipa_epilogue.cuh"

#define IPA_FILE_TAG 2
#include "sm100.cuh"

#ifdef IPA_TRACE
// Per-tile event timestamps (SM clock) of two CTAs, read back by the tracing
// build only.
__device__ unsigned long long g_ipa_trace[2][64][16];
#define IPA_TR(slot, j, ev)                                                              \
  do {                                                                                   \
    if (trace_slot >= 0 && (j) < 64) g_ipa_trace[trace_slot][(j)][(ev)] = clock64();     \
  } while (0)
#else
#define IPA_TR(slot, j, ev) \
  do {                      \
  } while (0)
#endif

namespace fipa {

using namespace sm100;

namespace {

struct AttnArgs {
  int B, L, H, DZ, RCz, Cz, nqt, nkt, F;
  float tau;
  const float4* rowq;
  const float4* colk;
  const float4* oq;
  const float4* ok;
  const float4* cen;
  const float* headc;
  const float* wqp;    // [H, DZ]
  const float4* frame; // [B, L, 4]
  const float* z1f;    // [B, L, DZ]
  float* out;
  float* lse;           // training forward: [B, H, L] log-sum-exp (natural log), else null
  float* uagg;          // training forward: [B, L, H, R Cz] pair aggregate, else null
  int* err;
  int trace_cta0, trace_cta1;
};

// shared-memory map (offsets from a 1024-byte aligned base)
constexpr uint32_t SM_QH = 0;                          // 128 x 64 fp16, SW128
constexpr uint32_t STG_BYTES = 16384 + 8192 * 4;       // Kh | Vh | Z2 (<= 4 panels)
constexpr uint32_t SM_STG = 16384;
constexpr uint32_t SM_P = SM_STG + NSTAGE * STG_BYTES; // 2 x (128 x 64 fp16, SW128)
constexpr uint32_t SM_AUX = SM_P + 2 * 16384;
constexpr uint32_t AUX_COL = 0;                        // float [NSTAGE][64]
constexpr uint32_t AUX_D = 1024;                       // float4 [NSTAGE]
constexpr uint32_t AUX_BAR = 1152;                     // mbarriers
constexpr uint32_t AUX_XCH = 2048;                     // float [2][2][128] row maxima + [2][128] row sums
constexpr uint32_t SMEM_BYTES = SM_AUX + AUX_XCH + 4096;
constexpr uint32_t SMEM_ALLOC = SMEM_BYTES + 1024;     // + alignment slack
// the epilogue stage (128 rows x stage_pitch(DZ) floats) reuses the K/V stages and P
static_assert(SM_STG + 128u * stage_pitch(MAX_DZ) * 4u <= SM_AUX, "epilogue stage overlaps the aux area");

// barrier slots
enum { B_Q = 0, B_QP, B_SFULL, B_SFREE, B_FULL0, B_EMPTY0 = B_FULL0 + NSTAGE,
       B_PFULL0 = B_EMPTY0 + NSTAGE, B_PFREE0 = B_PFULL0 + 2, B_DRAIN = B_PFREE0 + 2,
       B_COUNT = B_DRAIN + 1 };
constexpr uint32_t AUX_TMEM = AUX_BAR + 8 * B_COUNT;
constexpr uint32_t AUX_ABORT = AUX_TMEM + 8;

// tensor memory columns
constexpr uint32_t TM_O = 0;
constexpr uint32_t TM_S = 320;
constexpr uint32_t TM_QP = 384;
constexpr uint32_t TM_COLS = 512;

__device__ __forceinline__ uint64_t kdesc(uint32_t saddr) {  // K-major SW128
  return smem_desc_sw128(saddr, 16, 1024);
}
__device__ __forceinline__ uint64_t mndesc(uint32_t saddr) {  // MN-major SW128, 64-col panels 8 KB apart
  return smem_desc_sw128(saddr, 8192, 1024);
}

constexpr int NTHREADS = 320;   // 8 softmax warps, producer warp, MMA warp
constexpr int NSOFT = 256;      // softmax threads: two per query row (column halves)
constexpr int W_PROD = 8, W_MMA = 9;

__global__ void __launch_bounds__(NTHREADS, 1)
    ipa_attention_kernel(const __grid_constant__ CUtensorMap tm_qh,
                         const __grid_constant__ CUtensorMap tm_kh,
                         const __grid_constant__ CUtensorMap tm_vh,
                         const __grid_constant__ CUtensorMap tm_z2, const AttnArgs a) {
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  const uint32_t sb = (raw_u32 + 1023u) & ~1023u;
  unsigned char* smem = smem_raw + (sb - raw_u32);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int I = blockIdx.x % a.nqt;
  const int bh = blockIdx.x / a.nqt;
  const int b = bh / a.H, h = bh % a.H;
  const int L = a.L, nt = a.nkt, DZ = a.DZ;
#ifdef IPA_TRACE
  const int trace_slot = blockIdx.x == a.trace_cta0 ? 0 : blockIdx.x == a.trace_cta1 ? 1 : -1;
#endif

  float* col_s = reinterpret_cast<float*>(smem + SM_AUX + AUX_COL);
  float4* dinfo = reinterpret_cast<float4*>(smem + SM_AUX + AUX_D);
  float* xch = reinterpret_cast<float*>(smem + SM_AUX + AUX_XCH);   // [2 parity][2 halves][128]
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + SM_AUX + AUX_ABORT);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SM_AUX + AUX_TMEM);
  auto bar = [&](int k) -> uint32_t { return sb + SM_AUX + AUX_BAR + 8u * k; };

  if (tid == 0) {
    mbar_init(bar(B_Q), 1);
    mbar_init(bar(B_QP), NSOFT);
    mbar_init(bar(B_SFULL), 1);
    mbar_init(bar(B_SFREE), NSOFT);
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(bar(B_FULL0 + s), 1);
      mbar_init(bar(B_EMPTY0 + s), 1);
    }
    for (int p = 0; p < 2; ++p) {
      mbar_init(bar(B_PFULL0 + p), NSOFT);
      mbar_init(bar(B_PFREE0 + p), 1);
    }
    mbar_init(bar(B_DRAIN), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == W_MMA) {
    tmem_alloc(smem_u32(tmem_slot), TM_COLS);
    tmem_relinquish();
  }
  if (warp == W_PROD && lane == 0) {
    tma_prefetch_desc(&tm_qh);
    tma_prefetch_desc(&tm_kh);
    tma_prefetch_desc(&tm_vh);
    tma_prefetch_desc(&tm_z2);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  auto fail = [&](int code) {
    record_error(a.err, code);
    *abort_flag = 1;
  };

  if (warp == W_PROD) {
    // ------------------------------------------------ TMA producer warp
    const float4 oqv = a.oq[b * a.nqt + I];
    if (lane == 0) {
      mbar_arrive_expect_tx(bar(B_Q), 16384);
      tma_load_3d(sb + SM_QH, &tm_qh, bar(B_Q), 0, I * QT, bh);
    }
    int issued = 0;
    float cv_next[2];
    float4 dnext;
    auto load_cols = [&](int J) {
      const float4 okv = a.ok[b * nt + J];
      const float dx = okv.x - oqv.x, dy = okv.y - oqv.y, dz = okv.z - oqv.z;
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const int key = J * KT + lane + 32 * t;
        float cv = -INFINITY;
        if (key < L) {
          const float4 ck = a.colk[static_cast<int64_t>(bh) * L + key];
          cv = ck.w - fmaf(ck.x, dx, fmaf(ck.y, dy, ck.z * dz));
        }
        cv_next[t] = cv;
      }
      dnext = make_float4(dx, dy, dz, fmaf(dx, dx, fmaf(dy, dy, dz * dz)));
    };
    load_cols((2 * I) % nt);
    for (int j = 0; j < nt; ++j) {
      const int s = j % NSTAGE;
      const int J = (2 * I + j) % nt;
      if (j >= NSTAGE) {
        int ok = 1;
        if (lane == 0) ok = mbar_wait_bounded(bar(B_EMPTY0 + s), ((j / NSTAGE) - 1) & 1, abort_flag);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) {
          if (lane == 0) fail(DEV_TIMEOUT_EMPTY);
          break;
        }
      }
      if (lane == 0) IPA_TR(0, j, 13);
#pragma unroll
      for (int t = 0; t < 2; ++t) col_s[s * KT + lane + 32 * t] = cv_next[t];
      if (lane == 0) dinfo[s] = dnext;
      __syncwarp();
      if (lane == 0) {
        const uint32_t st = sb + SM_STG + s * STG_BYTES;
        mbar_arrive_expect_tx(bar(B_FULL0 + s), 16384u + static_cast<uint32_t>(DZ) * 128u);
        tma_load_3d(st, &tm_kh, bar(B_FULL0 + s), 0, J * KT, bh);
        tma_load_3d(st + 8192, &tm_vh, bar(B_FULL0 + s), 0, J * KT, bh);
        for (int p = 0; p < DZ / 64; ++p)
          tma_load_3d(st + 16384 + 8192 * p, &tm_z2, bar(B_FULL0 + s), 64 * p, J * KT, b);
        IPA_TR(0, j, 14);
      }
      __syncwarp();
      issued = j + 1;
      // column terms of the following tile, loaded while its stage is still busy
      if (j + 1 < nt) load_cols((2 * I + j + 1) % nt);
    }
    if (lane == 0 && *abort_flag) {
      for (int j = (issued > NSTAGE ? issued - NSTAGE : 0); j < issued; ++j)
        mbar_wait_bounded(bar(B_FULL0 + j % NSTAGE), (j / NSTAGE) & 1, nullptr, 100000000ull);
    }
  } else if (warp == W_MMA) {
    // ------------------------------------------------ MMA issuer (one thread)
    // Issue order QK(0), QK(1), PV(0), QK(2), PV(1), ...: QK(j) as soon as the
    // softmax warps have read S(j-1), PV(j-1) as soon as P(j-1) is written, so
    // S(j) is computed while the softmax of tile j-1 runs.
    if (lane == 0) {
      bool ok = mbar_wait_bounded(bar(B_Q), 0, abort_flag) && mbar_wait_bounded(bar(B_QP), 0, abort_flag);
      if (!ok) fail(DEV_TIMEOUT_SOFTMAX);
      tc_fence_after();
      const uint32_t idq = idesc_f16(128, KT, false);
      const uint32_t idv1 = idesc_f16(128, 64, true);
      const uint32_t idv2 = idesc_f16(128, DZ, true);
      const uint32_t tS = tmem + TM_S, tO = tmem + TM_O, tQP = tmem + TM_QP;
      bool issued_any = false;
      for (int j = 0; ok && j <= nt; ++j) {
        if (j < nt) {
          const int s = j % NSTAGE;
          ok = mbar_wait_bounded(bar(B_FULL0 + s), (j / NSTAGE) & 1, abort_flag);
          IPA_TR(0, j, 0);
          if (ok && j > 0) ok = mbar_wait_bounded(bar(B_SFREE), (j - 1) & 1, abort_flag);
          IPA_TR(0, j, 1);
          if (!ok) { fail(DEV_TIMEOUT_FULL); break; }
          tc_fence_after();
          const uint32_t st = sb + SM_STG + s * STG_BYTES;
#pragma unroll
          for (int k = 0; k < 4; ++k)
            umma_ss(tS, kdesc(sb + SM_QH + 32 * k), kdesc(st + 32 * k), idq, k > 0 ? 1u : 0u);
          for (int kk = 0; kk < DZ / 16; ++kk)
            umma_ts(tS, tQP + 8 * kk, kdesc(st + 16384 + 8192 * (kk >> 2) + 32 * (kk & 3)), idq, 1u);
          umma_commit(bar(B_SFULL));
          IPA_TR(0, j, 2);
          issued_any = true;
        }
        if (j > 0) {
          const int jj = j - 1, pb = jj & 1, s2 = jj % NSTAGE;
          ok = mbar_wait_bounded(bar(B_PFULL0 + pb), (jj >> 1) & 1, abort_flag);
          IPA_TR(0, jj, 3);
          if (!ok) { fail(DEV_TIMEOUT_SOFTMAX); break; }
          tc_fence_after();
          const uint32_t pbase = sb + SM_P + 16384 * pb;
          const uint32_t st = sb + SM_STG + s2 * STG_BYTES;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint32_t acc = (jj > 0 || k > 0) ? 1u : 0u;
            umma_ss(tO, kdesc(pbase + 32 * k), mndesc(st + 8192 + 2048 * k), idv1, acc);
            if (DZ > 0) umma_ss(tO + 64, kdesc(pbase + 32 * k), mndesc(st + 16384 + 2048 * k), idv2, acc);
          }
          umma_commit(bar(B_PFREE0 + pb));
          umma_commit(bar(B_EMPTY0 + s2));
          IPA_TR(0, jj, 4);
        }
      }
      if (!ok && issued_any) {
        umma_commit(bar(B_DRAIN));
        mbar_wait_bounded(bar(B_DRAIN), 0, nullptr, 100000000ull);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ softmax + epilogue (256 threads)
    // Thread (half, r): query row r of the tile, S columns [32 half, 32 half + 32).
    const int quarter = warp & 3, half = warp >> 2;
    const int r = quarter * 32 + lane;
    const int row = I * QT + r;
    const bool in_range = row < L;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t pair_bar = 2 + quarter;   // named barrier of the two warps sharing these rows
    const float ch = a.headc[h];
    const float4 sq = in_range ? a.rowq[static_cast<int64_t>(bh) * L + row] : make_float4(0, 0, 0, 0);
    const float pq = static_cast<float>(IPA_PQ);
    const bool tr = (tid == 0 || tid == 96);
    const int tev = tid == 0 ? 0 : 1;
    (void)tr; (void)tev;

    // Q_pair row = log2(e) w_L w_bias[:, h] * z1_i -> tensor memory; this thread writes half the columns
    {
      const float4* zr = reinterpret_cast<const float4*>(a.z1f + (static_cast<int64_t>(b) * L + (in_range ? row : 0)) * DZ);
      const float4* wr = reinterpret_cast<const float4*>(a.wqp + static_cast<int64_t>(h) * DZ);
      // 32-column chunks of the DZ / 2 packed columns, alternating between the
      // two halves (every chunk lies inside the row's DZ pair factors)
      float qmax = 0.f;   // largest |Q_pair| before rounding (NaN if any is NaN)
      for (int c0 = 32 * half; c0 < DZ / 2; c0 += 64) {
        uint32_t rg[32];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float4 z = in_range ? zr[c0 / 2 + e] : make_float4(0, 0, 0, 0);
          const float4 w = wr[c0 / 2 + e];
          const float4 y = make_float4(z.x * w.x, z.y * w.y, z.z * w.z, z.w * w.w);
          qmax = fmax_nan(qmax, fmax_nan(fmax_nan(fabsf(y.x), fabsf(y.y)), fmax_nan(fabsf(y.z), fabsf(y.w))));
          rg[2 * e] = pack_half2(y.x, y.y);
          rg[2 * e + 1] = pack_half2(y.z, y.w);
        }
        tmem_st32(tmem + TM_QP + c0 + lane_off, rg);
      }
      if (!(qmax < 65520.f)) record_error(a.err, DEV_NONFINITE);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(B_QP));
    }

    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    const int OW = 64 + DZ;
    const int o_lo = half * (OW / 2), o_hi = o_lo + OW / 2;   // O columns this thread rescales / stages
    for (int j = 0; j < nt && ok; ++j) {
      const int s = j % NSTAGE, pb = j & 1;
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(bar(B_SFULL), j & 1, abort_flag))) {
        if (lane == 0) fail(DEV_TIMEOUT_MMA);
        ok = false;
        break;
      }
      if (tr) IPA_TR(0, j, tev ? 11 : 5);
      tc_fence_after();
      uint32_t sr[32];
      tmem_ld32(tmem + TM_S + 32 * half + lane_off, sr);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(bar(B_SFREE));
      if (tid == 0) IPA_TR(0, j, 6);
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(bar(B_FULL0 + s), (j / NSTAGE) & 1, abort_flag))) {
        if (lane == 0) fail(DEV_TIMEOUT_FULL);
        ok = false;
        break;
      }
      if (tid == 0) IPA_TR(0, j, 7);

      const float4* colv = reinterpret_cast<const float4*>(col_s + s * KT + 32 * half);
      const float4 dd = dinfo[s];
      const float rt = ch * (2.f * fmaf(sq.x, dd.x, fmaf(sq.y, dd.y, sq.z * dd.z)) - pq * dd.w);
      float2 x[16];
      float mxa = -INFINITY, mxb = -INFINITY;
#pragma unroll
      for (int k4 = 0; k4 < 8; ++k4) {
        const float4 cv = colv[k4];
        x[2 * k4] = add_f32x2(make_float2(__uint_as_float(sr[4 * k4]), __uint_as_float(sr[4 * k4 + 1])),
                              make_float2(cv.x, cv.y));
        x[2 * k4 + 1] = add_f32x2(make_float2(__uint_as_float(sr[4 * k4 + 2]), __uint_as_float(sr[4 * k4 + 3])),
                                  make_float2(cv.z, cv.w));
        mxa = fmax3(mxa, x[2 * k4].x, x[2 * k4].y);
        mxb = fmax3(mxb, x[2 * k4 + 1].x, x[2 * k4 + 1].y);
      }
      // row max over both halves (exchange through shared memory)
      const float mine = fmaxf(mxa, mxb);
      float* xb = xch + (j & 1) * 256;
      xb[half * 128 + r] = mine;
      named_bar_sync(pair_bar, 64);
      const float mt = fmaxf(mine, xb[(1 - half) * 128 + r]) + rt;
      const bool need = mt > m_used + a.tau;
      const bool resc = need && (m_used != -INFINITY);
      const float scale = resc ? ex2(m_used - mt) : 1.f;
      if (need) m_used = mt;
      l *= scale;
      // while no key of the row has been allowed, every x is -inf and the
      // exponent base 0 gives P = 0
      const float nbase = (m_used != -INFINITY) ? rt - m_used : 0.f;
      const float2 nb2 = make_float2(nbase, nbase);
      uint32_t pk[16];
      float ls4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        // P rounded to fp16 (nearest even) by the pack: the value the tensor
        // core multiplies; the row sum adds exactly those values
        const float2 y = add_f32x2(x[k], nb2);
        pk[k] = pack_half2(ex2(y.x), ex2(y.y));
        ls4[k & 3] = add_half2_to_f32(pk[k], ls4[k & 3]);
      }
      l += (ls4[0] + ls4[1]) + (ls4[2] + ls4[3]);
      if (tid == 0) IPA_TR(0, j, 8);
      if (j >= 2) {
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(bar(B_PFREE0 + pb), ((j - 2) >> 1) & 1, abort_flag))) {
          if (lane == 0) fail(DEV_TIMEOUT_MMA);
          ok = false;
          break;
        }
      }
      if (tid == 0) IPA_TR(0, j, 9);
      unsigned char* prow = smem + SM_P + 16384 * pb + r * 128;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int chunk = 4 * half + c;
        *reinterpret_cast<uint4*>(prow + ((chunk ^ (r & 7)) << 4)) =
            make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      }
      fence_proxy_async_smem();
      if (__any_sync(0xffffffffu, resc)) {
        // O must hold exactly tiles < j when it is rescaled: wait for PV(j-1)
        if (!__all_sync(0xffffffffu,
                        mbar_wait_bounded(bar(B_PFREE0 + ((j - 1) & 1)), ((j - 1) >> 1) & 1, abort_flag))) {
          if (lane == 0) fail(DEV_TIMEOUT_MMA);
          ok = false;
          break;
        }
        tc_fence_after();
        for (int c0 = o_lo; c0 < o_hi; c0 += 32) {
          uint32_t o[32];
          tmem_ld32(tmem + TM_O + c0 + lane_off, o);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * scale);
          tmem_st32(tmem + TM_O + c0 + lane_off, o);
        }
        tmem_st_wait();
        tc_fence_before();
      }
      mbar_arrive(bar(B_PFULL0 + pb));
      if (tr) IPA_TR(0, j, tev ? 12 : 10);
    }

    // ------------------------------------------------ epilogue
    // frame of this row (rotation, translation, valid), loaded while the last
    // P.V runs
    const float4* fgr = a.frame + (static_cast<int64_t>(b) * L + (in_range ? row : 0)) * 4;
    const float4 f3 = fgr[3];
    float4 g0 = make_float4(0.f, 0.f, 0.f, 0.f), g1 = g0, g2 = g0, cn = g0;
    if (half == 0) {
      g0 = fgr[0];
      g1 = fgr[1];
      g2 = fgr[2];
      cn = a.cen[b];
    }
    if (ok && !__all_sync(0xffffffffu, mbar_wait_bounded(bar(B_PFREE0 + ((nt - 1) & 1)),
                                                          ((nt - 1) >> 1) & 1, abort_flag))) {
      if (lane == 0) fail(DEV_TIMEOUT_MMA);
      ok = false;
    }
    const bool all_ok = __all_sync(0xffffffffu, ok);
    // total row sum over the two halves
    xch[512 + half * 128 + r] = l;
    named_bar_sync(pair_bar, 64);
    const float lt = l + xch[512 + (1 - half) * 128 + r];
    const bool dead = !(in_range && f3.x != 0.f && lt > 0.f);
    // training forward: log-sum-exp of the true logits; the pass left the row
    // constant c sum_p |gq'_p|^2 (rowq.w) out of its logits
    if (a.lse != nullptr && half == 0 && in_range)
      *IPA_AT(a.lse, static_cast<int64_t>(bh) * L + row, static_cast<int64_t>(a.B) * a.H * L, a.err) = dead ? INFINITY : (m_used + log2f(lt) - sq.w) * 0.69314718055994531f;
    const int pitch = stage_pitch(DZ);
    float* stage = reinterpret_cast<float*>(smem + SM_STG);
    if (all_ok) {
      tc_fence_after();
      const float inv = dead ? 0.f : 1.f / lt;
      float* orow = stage + r * pitch;
      for (int c0 = o_lo; c0 < o_hi; c0 += 32) {
        uint32_t o[32];
        tmem_ld32(tmem + TM_O + c0 + lane_off, o);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; e += 4)
          *reinterpret_cast<float4*>(orow + c0 + e) =
              make_float4(__uint_as_float(o[e]) * inv, __uint_as_float(o[e + 1]) * inv,
                          __uint_as_float(o[e + 2]) * inv, __uint_as_float(o[e + 3]) * inv);
      }
      if (half == 0) stage_frame(orow + 64 + DZ, g0, g1, g2, cn, dead);
    }
    tc_fence_before();
    named_bar_sync(1, NSOFT);
    if (!*abort_flag) {
      EpilogueArgs ea{stage, DZ, a.Cz, a.RCz, a.F, a.H, L, b, h, I * QT, a.z1f, a.out};
      ea.uagg = a.uagg;
      ea.rows = static_cast<int64_t>(a.B) * L * a.H;
      ea.err = a.err;
      write_rows<IPA_C, IPA_PV>(ea, warp, lane);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == W_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, TM_COLS);
  }
}

}  // namespace

cudaError_t ipa_launch_core(const IpaLaunch& a, cudaStream_t stream) {
  // the CTA-pair kernel covers pair widths 128 and 256; this kernel the rest
  if (ipa_pair_supported(a.DZ)) return ipa_launch_core_pair(a, stream);
  unsigned char* ws = a.ws;
  const IpaWorkspace& w = a.lay;
  CUtensorMap tqh, tkh, tvh, tz2;
  const uint64_t bh = static_cast<uint64_t>(a.B) * a.H;
  const uint64_t rowb = static_cast<uint64_t>(a.L) * DH * 2;
  bool ok = encode_tmap_f16_3d(&tqh, ws + w.qh, DH, a.L, bh, DH * 2, rowb, 64, QT) &&
            encode_tmap_f16_3d(&tkh, ws + w.kh, DH, a.L, bh, DH * 2, rowb, 64, KT) &&
            encode_tmap_f16_3d(&tvh, ws + w.vh, DH, a.L, bh, DH * 2, rowb, 64, KT) &&
            (a.DZ == 0 ? (tz2 = tvh, true) :   // no pair block: the Z2 map is never read
             encode_tmap_f16_3d(&tz2, ws + w.z2, a.DZ, a.L, a.B, static_cast<uint64_t>(a.DZ) * 2,
                                static_cast<uint64_t>(a.L) * a.DZ * 2, 64, KT));
  if (!ok) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(ipa_attention_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(SMEM_ALLOC));
  if (e != cudaSuccess) return e;
  AttnArgs t{};
  t.B = a.B; t.L = a.L; t.H = a.H; t.DZ = a.DZ; t.RCz = a.RCz; t.Cz = a.Cz;
  t.nqt = a.nqt; t.nkt = a.nkt; t.F = a.F; t.tau = 8.f;
  t.rowq = reinterpret_cast<const float4*>(ws + w.rowq);
  t.colk = reinterpret_cast<const float4*>(ws + w.colk);
  t.oq = reinterpret_cast<const float4*>(ws + w.oq);
  t.ok = reinterpret_cast<const float4*>(ws + w.ok);
  t.cen = reinterpret_cast<const float4*>(ws + w.cen);
  t.headc = reinterpret_cast<const float*>(ws + w.headc);
  t.wqp = reinterpret_cast<const float*>(ws + w.wqp);
  t.frame = reinterpret_cast<const float4*>(ws + w.frame);
  t.z1f = reinterpret_cast<const float*>(ws + w.z1f);
  t.out = a.out; t.err = a.err; t.lse = a.lse; t.uagg = a.uagg;
  t.trace_cta0 = 0;
  t.trace_cta1 = static_cast<int>(bh * a.nqt) / 2;
  ipa_attention_kernel<<<static_cast<unsigned>(bh * a.nqt), NTHREADS, SMEM_ALLOC, stream>>>(tqh, tkh, tvh, tz2, t);
  return cudaGetLastError();
}

#ifdef IPA_TRACE
bool ipa_trace_read(void* host, size_t bytes) {
  if (bytes < sizeof(g_ipa_trace)) return false;
  return cudaMemcpyFromSymbol(host, g_ipa_trace, sizeof(g_ipa_trace)) == cudaSuccess;
}
#endif

}  // namespace fipa
