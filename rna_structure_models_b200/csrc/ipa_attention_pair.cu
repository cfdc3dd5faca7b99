// Fused attention pass of the IPA core on a CTA pair (cta_group::2).
//
// A cluster of two CTAs owns 256 query rows of one (batch, head); CTA r of
// the pair owns rows [256 I + 128 r, +128).  Key tiles are 128 keys.  The MMAs
// are issued by one thread of CTA 0 for both CTAs (M = 256): each CTA
// supplies its own 128 rows of A and HALF of every B operand from its own
// shared memory, which halves the per-CTA shared-memory footprint and the
// operand traffic of a key tile and allows N = 128 keys per Q.K^T MMA
// (N = 64 MMAs run well below the tensor rate on this GPU).
//
//   S = [Q_h | Q_pair] . [K_h | Z2]^T      N = 128: CTA r supplies keys [64 r, 64 r + 64)
//   O_pair += P . Z2                        N = DZ: CTA r supplies features [r DZ/2, (r+1) DZ/2)
//   O_v    += P . V_h                       N = 64: CTA r supplies V_h columns [32 r, 32 r + 32)
//
// P (fp16, 128 keys) lives in tensor memory and is the A operand of the P.V
// MMAs.  Per CTA, tensor memory: O_pair [0, DZ) | O_v [DZ, DZ+64) | S [320, 448)
// | P [448, 512); shared memory: Q_h 16 KB | Q_pair DZ*256 B | 2 x K slot
// (own 64 keys: K_h 8 KB + Z2 DZ*128 B) | 1 x V slot (all 128 keys: own Z2
// panels DZ*128 B + own V_h columns 8 KB, 64-byte swizzle).
//
// Warps: 0-7 softmax and epilogue (two threads per query row), 8 K producer
// (K_h / Z2 key-half copies, then the fp32 column terms), 9 MMA issuer (one
// thread of CTA 0) and tensor-memory owner, 10 V producer.  K and V copies
// have their own threads so that neither waits for the other's slot.
//
// Synchronisation: barriers the MMA thread waits on live in CTA 0 (K/V slots
// full: TMA bytes of both CTAs; S read and P written: one arrival per softmax
// warp of both CTAs); barriers the softmax and producer warps wait on live in
// each CTA and are signalled by multicast tcgen05.commit.  Every wait is
// bounded (2 s) and reports into the error word.
//
// The softmax, lazy rescaling, rounded row sums, tile-local point terms and
// the epilogue are those of the single-CTA kernel (ipa_attention.cu).
//
// Key-split tail (inference only): the pair tiles of the last, partial wave
// may each run as 2-5 CTA pairs over consecutive key-tile ranges.  Each
// stores its un-normalised accumulators, row maximum and half sums; the one
// that takes the last ticket merges the chunks in chunk order into tensor
// memory (flash-decoding style rescale by 2^(m_s - max m)) and runs the
// output pass.  ipa_split_plan chooses the chunk count on the host.
#include <cuda_fp16.h>

#include <cmath>
#include <cstdint>

#include "bounds.cuh"
#include "internal.h"
#include "ipa_epilogue.cuh"

#define IPA_FILE_TAG 3
#include "sm100.cuh"

#ifdef IPA_TRACE
__device__ unsigned long long g_pair_trace[2][64][32];
__device__ unsigned long long g_pair_span[4096][64];  // per CTA: globaltimer start/end, clock64 start/end, smid, phase clocks
#define PAIR_SPAN(k)                                                  \
  do {                                                                \
    if (blockIdx.x < 4096) g_pair_span[blockIdx.x][(k)] = clock64();  \
  } while (0)
#define PAIR_TR(j, ev)                                                               \
  do {                                                                               \
    if (trace_slot >= 0 && (j) < 64) g_pair_trace[trace_slot][(j)][(ev)] = clock64(); \
  } while (0)
#else
#define PAIR_TR(j, ev) \
  do {                 \
  } while (0)
#define PAIR_SPAN(k) \
  do {               \
  } while (0)
#endif

namespace fipa {

using namespace sm100;

namespace {

struct PairArgs {
  int B, L, H, DZ, RCz, Cz, nqt, nkt, nqp, nkp, F;  // nqt/nkt: 128-row / 64-key tiles; nqp/nkp: 256 / 128
  float tau;
  const float4* rowq;
  const float4* colk;
  const float4* oq;     // [B, nqt]   128-row query tile origins
  const float4* ok;     // [B, nkt]   64-key tile origins
  const float4* cen;
  const float* headc;
  const float* wqp;     // [H, DZ]
  const float4* frame;
  const float* z1f;     // [B, L, DZ]
  float* out;
  float* lse;           // training forward: [B, H, L] log-sum-exp (natural log), else null
  float* uagg;          // training forward: [B, L, H, R Cz] pair aggregate, else null
  int* err;
  int tma_epi;          // 1: the output pass stages the pair features and stores them with TMA
  // key-split tail: pair tiles [split_first, T) are each run as split_s
  // chunks of consecutive key tiles by split_s CTA pairs (split_s == 1: none)
  int split_first, split_s;
  int64_t part_extent;  // floats in part (bounds-checked build)
  int ticket_extent;    // ints in ticket
  float* part;          // per (chunk, CTA rank): [DZ + 64 + 3][128] partial accumulators, max, two half sums
  int* ticket;          // per (split tile, CTA rank): chunks finished (zero between calls)
  int trace_cta0, trace_cta1;
};

constexpr int NT = 352;            // 8 softmax warps, K producer, MMA issuer, V producer
constexpr int NSOFT = 256;
constexpr int W_PROD = 8, W_MMA = 9, W_VPROD = 10;
constexpr int NCOL = 4;            // column-term ring
constexpr int MAX_SPLIT = 5;       // key chunks of a split tile

// shared memory (offsets from a 1024-byte aligned base)
constexpr uint32_t SP_QH = 0;
constexpr uint32_t SP_QP = 16384;                 // DZ/64 panels x 16 KB
constexpr uint32_t KSLOT = 8192 + 4 * 8192;       // K_h half + Z2 half (<= 4 panels)
constexpr uint32_t SP_K = SP_QP + 4 * 16384;      // 2 slots
constexpr uint32_t SP_V = SP_K + 2 * KSLOT;       // Z2 own panels (<= 2 x 16 KB) | V_h 8 KB
constexpr uint32_t V_VH = 32768;
constexpr uint32_t VSLOT = V_VH + 8192;
constexpr uint32_t SP_AUX = SP_V + VSLOT;
constexpr uint32_t AX_COL = 0;                    // float [NCOL][128]
constexpr uint32_t AX_D = 2048;                   // float4 [NCOL][2]
constexpr uint32_t AX_XCH = 2304;                 // float [2][2][128] maxima + [2][128] sums
constexpr uint32_t AX_BAR = 5376;
constexpr uint32_t SP_BYTES = SP_AUX + 6144;
constexpr uint32_t SP_ALLOC = SP_BYTES + 1024;
// the epilogue stage (128 rows x (64 + DZ + 20) floats) reuses Q_pair, K and V
static_assert(SP_QP + 128u * stage_pitch(MAX_DZ) * 4u <= SP_AUX, "epilogue stage overlaps the aux area");

enum {
  // local barriers (waited on in each CTA)
  P_QFULL = 0, P_SFULL, P_PFREE, P_KEMPTY0, P_COLFULL0 = P_KEMPTY0 + 2, P_DRAIN = P_COLFULL0 + NCOL,
  // barriers waited on by the MMA thread (used in CTA 0)
  P_KFULL0, P_VFULL = P_KFULL0 + 2, P_SFREE, P_PFULL, P_QREADY, P_ZFULL, P_COUNT
};
constexpr uint32_t AX_TMEM = AX_BAR + 8 * P_COUNT;
constexpr uint32_t AX_ABORT = AX_TMEM + 8;
constexpr uint32_t AX_LAST = AX_ABORT + 4;        // int: this CTA finishes its split tile

constexpr uint32_t TM_S = 320, TM_P = 448, TM_COLS = 512;

__device__ __forceinline__ uint64_t k128(uint32_t a) { return smem_desc(a, 16, 1024, 2); }           // K-major SW128
__device__ __forceinline__ uint64_t mn128(uint32_t a) { return smem_desc(a, 16384, 1024, 2); }       // MN-major SW128, 16 KB panels
__device__ __forceinline__ uint64_t mn64(uint32_t a) { return smem_desc(a, 16384, 512, 4); }         // MN-major SW64

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NT, 1)
    ipa_attention_pair_kernel(const __grid_constant__ CUtensorMap tm_qh,
                              const __grid_constant__ CUtensorMap tm_kh,
                              const __grid_constant__ CUtensorMap tm_z2k,
                              const __grid_constant__ CUtensorMap tm_z2v,
                              const __grid_constant__ CUtensorMap tm_vh,
                              const __grid_constant__ CUtensorMap tm_z1,
                              const __grid_constant__ CUtensorMap tm_z1f,
                              const __grid_constant__ CUtensorMap tm_out, const PairArgs a) {
  extern __shared__ unsigned char smem_raw[];
#ifdef IPA_TRACE
  if (threadIdx.x == 0 && blockIdx.x < 4096) {
    uint32_t smid;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
    g_pair_span[blockIdx.x][0] = globaltimer_ns();
    g_pair_span[blockIdx.x][2] = clock64();
    g_pair_span[blockIdx.x][4] = smid;
  }
#endif
  const uint32_t raw_u32 = smem_u32(smem_raw);
  const uint32_t sb = (raw_u32 + 1023u) & ~1023u;
  unsigned char* smem = smem_raw + (sb - raw_u32);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1;
  // a split tile's chunk c covers key tiles [c nkp / S, (c + 1) nkp / S)
  int tile = pair, chunk = -1, kbeg = 0, nt = a.nkp;
  if (pair >= a.split_first) {
    const int q = pair - a.split_first;
    tile = a.split_first + q / a.split_s;
    chunk = q % a.split_s;
    kbeg = chunk * a.nkp / a.split_s;
    nt = (chunk + 1) * a.nkp / a.split_s - kbeg;
  }
  const int I2 = tile % a.nqp;
  const int bh = tile / a.nqp;
  const int b = bh / a.H, h = bh % a.H;
  const int L = a.L, DZ = a.DZ, np = DZ / 64;
  const int row0 = 256 * I2 + 128 * static_cast<int>(rank);   // first query row of this CTA
  const int I = row0 / QT;                                      // its 128-row query tile
#ifdef IPA_TRACE
  const int trace_slot = (blockIdx.x == a.trace_cta0) ? 0 : (blockIdx.x == a.trace_cta1) ? 1 : -1;
#endif

  float* col_s = reinterpret_cast<float*>(smem + SP_AUX + AX_COL);
  float4* dinfo = reinterpret_cast<float4*>(smem + SP_AUX + AX_D);
  float* xch = reinterpret_cast<float*>(smem + SP_AUX + AX_XCH);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + SP_AUX + AX_ABORT);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SP_AUX + AX_TMEM);
  auto bar = [&](int k) -> uint32_t { return sb + SP_AUX + AX_BAR + 8u * k; };
  auto bar0 = [&](int k) -> uint32_t { return mapa_shared(bar(k), 0); };   // the barrier in CTA 0

  if (tid == 0) {
    mbar_init(bar(P_QFULL), 1);
    mbar_init(bar(P_SFULL), 1);
    mbar_init(bar(P_PFREE), 1);
    mbar_init(bar(P_KEMPTY0), 1);
    mbar_init(bar(P_KEMPTY0 + 1), 1);
    for (int s = 0; s < NCOL; ++s) mbar_init(bar(P_COLFULL0 + s), 1);
    mbar_init(bar(P_DRAIN), 1);
    mbar_init(bar(P_KFULL0), 2);
    mbar_init(bar(P_KFULL0 + 1), 2);
    mbar_init(bar(P_VFULL), 2);
    mbar_init(bar(P_SFREE), 16);
    mbar_init(bar(P_PFULL), 16);
    mbar_init(bar(P_QREADY), 2);
    mbar_init(bar(P_ZFULL), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == W_MMA) {
    tmem_alloc_pair(smem_u32(tmem_slot), TM_COLS);
    tmem_relinquish_pair();
  }
  if (warp == W_PROD && lane == 0) {
    tma_prefetch_desc(&tm_qh);
    tma_prefetch_desc(&tm_kh);
    tma_prefetch_desc(&tm_z2k);
    tma_prefetch_desc(&tm_z2v);
    tma_prefetch_desc(&tm_vh);
    tma_prefetch_desc(&tm_z1);
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (tid == 0) PAIR_SPAN(5);

  auto fail = [&](int code) {
    record_error(a.err, code);
    *abort_flag = 1;
  };
  const int start = chunk < 0 ? (2 * I2) % a.nkp : kbeg;   // a whole tile starts at its diagonal key tile

  if (warp == W_PROD) {
    // ------------------------------------------------ producer (each CTA)
    const float4 oqv = a.oq[b * a.nqt + (I < a.nqt ? I : a.nqt - 1)];
    if (lane == 0) {
      // Q_h rows and the fp16 z1 rows of this CTA (scaled into Q_pair in place)
      mbar_arrive_expect_tx(bar(P_QFULL), 16384u * static_cast<uint32_t>(1 + np));
      tma_load_3d(sb + SP_QH, &tm_qh, bar(P_QFULL), 0, row0, bh);
      tma_load_4d(sb + SP_QP, &tm_z1, bar(P_QFULL), 0, row0, 0, b);   // all np panels
    }
    const uint32_t kbytes = 8192u + static_cast<uint32_t>(np) * 8192u;
    // inputs of the column terms of the next tile, loaded one tile ahead so
    // that their global-load latency overlaps the wait for a free K slot
    float4 ckn[4], okn[4], odn = make_float4(0.f, 0.f, 0.f, 0.f);
    auto fetch_cols = [&](int j) {
      const int J2 = (start + j) % a.nkp;
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int key = J2 * 128 + lane + 32 * t;
        const bool in = j < nt && key < L;
        ckn[t] = in ? a.colk[static_cast<int64_t>(bh) * L + key] : make_float4(0.f, 0.f, 0.f, -INFINITY);
        okn[t] = in ? a.ok[b * a.nkt + key / KT] : make_float4(0.f, 0.f, 0.f, 0.f);
      }
      const int jt = 2 * J2 + (lane & 1);
      odn = (j < nt && jt < a.nkt) ? a.ok[b * a.nkt + jt] : make_float4(0.f, 0.f, 0.f, 0.f);
    };
    auto load_k = [&](int j) {
      const int J2 = (start + j) % a.nkp;
      const int s = j & 1;
      if (lane == 0) {
        const uint32_t kf = bar0(P_KFULL0 + s);
        const uint32_t st = sb + SP_K + s * KSLOT;
        const int krow = J2 * 128 + 64 * static_cast<int>(rank);
        mbar_arrive_expect_tx_remote(kf, kbytes);
        PAIR_TR(j, 10);
        tma_load_3d_pair(st, &tm_kh, kf, 0, krow, bh);
        PAIR_TR(j, 9);
        tma_load_4d_pair(st + 8192, &tm_z2k, kf, 0, krow, 0, b);   // all np panels of the key half
        PAIR_TR(j, 13);
      }
      // column terms of this CTA's rows for the 128 keys of the tile (-inf
      // for keys past L and for masked keys, whose colk.w is -inf)
      const int cs = j % NCOL;
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const float4 ck = ckn[t], okv = okn[t];
        col_s[cs * 128 + lane + 32 * t] =
            ck.w - fmaf(ck.x, okv.x - oqv.x, fmaf(ck.y, okv.y - oqv.y, ck.z * (okv.z - oqv.z)));
      }
      if (lane < 2) {
        const float dx = odn.x - oqv.x, dy = odn.y - oqv.y, dz = odn.z - oqv.z;
        dinfo[cs * 2 + lane] = make_float4(dx, dy, dz, fmaf(dx, dx, fmaf(dy, dy, dz * dz)));
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(P_COLFULL0 + cs));
      __syncwarp();
      fetch_cols(j + 1);
    };
    auto wait_local = [&](int barid, uint32_t parity, int code) -> bool {
      int ok = 1;
      if (lane == 0) ok = mbar_wait_bounded(bar(barid), parity, abort_flag);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok && lane == 0) fail(code);
      return ok != 0;
    };
    fetch_cols(0);
    // K(0), K(1); then K(j) as soon as QK(j-2) has released its slot.  The
    // column terms of tile j reuse ring entry j mod 4: QK(j-2) was issued
    // after the softmax released S(j-3), so it has finished tile j-4.
    load_k(0);
    if (nt > 1) load_k(1);
    for (int j = 2; j < nt; ++j) {
      if (!wait_local(P_KEMPTY0 + (j & 1), ((j - 2) >> 1) & 1, DEV_TIMEOUT_EMPTY)) break;
      if (lane == 0) PAIR_TR(j, 12);
      load_k(j);
    }
    // the epilogue's z1 rows (fp32, contiguous), brought into L2 while the
    // last tiles run
    if (lane == 0 && row0 < L) {
      const int nrows = L - row0 < 128 ? L - row0 : 128;
      bulk_prefetch_l2(a.z1f + (static_cast<int64_t>(b) * L + row0) * DZ, static_cast<uint32_t>(nrows * DZ * 4));
    }
    // staged output pass: the z1 rows into the Q_pair / K area (DZ / 32 boxes
    // of 16 KB from SP_QP) once the last Q.K has completed and released both
    if (a.tma_epi && !*abort_flag && wait_local(P_KEMPTY0 + ((nt - 1) & 1), ((nt - 1) >> 1) & 1, DEV_TIMEOUT_EMPTY) &&
        lane == 0) {
      mbar_arrive_expect_tx(bar(P_ZFULL), static_cast<uint32_t>(DZ / 32) * 16384u);
      for (int k = 0; k < DZ / 32; ++k) tma_load_3d(sb + SP_QP + 16384u * k, &tm_z1f, bar(P_ZFULL), 32 * k, row0, b);
    }
  } else if (warp == W_VPROD) {
#ifdef IPA_TRACE
    // tracing build only: one idle lane of CTA 0 records when each K slot fills
    if (lane == 1 && rank == 0 && trace_slot >= 0) {
      for (int j = 0; j < nt; ++j) {
        if (!mbar_wait_bounded_cluster(bar(P_KFULL0 + (j & 1)), (j >> 1) & 1, abort_flag)) break;
        PAIR_TR(j, 11);
      }
    }
#endif
    // ------------------------------------------------ V producer (each CTA, one thread)
    if (lane == 0) {
      const uint32_t vbytes = static_cast<uint32_t>(np / 2) * 16384u + 8192u;
      for (int j = 0; j < nt; ++j) {
        // the V slot is free once P.V(j-1) has completed, which PFREE
        // signals; this thread cannot fall two phases behind because P.V(j)
        // needs V(j) first
        if (j > 0 && !mbar_wait_bounded(bar(P_PFREE), (j - 1) & 1, abort_flag)) {
          fail(DEV_TIMEOUT_EMPTY);
          break;
        }
        PAIR_TR(j, 15);
        const int J2 = (start + j) % a.nkp;
        const uint32_t vf = bar0(P_VFULL);
        const uint32_t st = sb + SP_V;
        mbar_arrive_expect_tx_remote(vf, vbytes);
        tma_load_4d_pair(st, &tm_z2v, vf, 0, J2 * 128, static_cast<int>(rank) * (np / 2), b);   // own np/2 panels
        tma_load_3d_pair(st + V_VH, &tm_vh, vf, 32 * static_cast<int>(rank), J2 * 128, bh);
        PAIR_TR(j, 14);
      }
    }
    __syncwarp();
  } else if (warp == W_MMA) {
    // ------------------------------------------------ MMA issuer (CTA 0, one thread)
    if (rank == 0 && lane == 0) {
      bool ok = mbar_wait_bounded_cluster(bar(P_QREADY), 0, abort_flag);
      if (!ok) fail(DEV_TIMEOUT_SOFTMAX);
      PAIR_SPAN(7);
      tc_fence_after();
      const uint32_t idq = idesc_f16(256, 128, false);
      const uint32_t idz = idesc_f16(256, DZ, true);
      const uint32_t idv = idesc_f16(256, 64, true);
      const uint32_t tS = tmem + TM_S, tP = tmem + TM_P, tOz = tmem, tOv = tmem + DZ;
      bool issued_any = false;
      // Q.K(j) as soon as its K tile is in and S(j-1) has been read, then
      // P.V(j-1) once P(j-1) and V(j-1) are in
      for (int j = 0; ok && j <= nt; ++j) {
        if (j < nt) {
          const int s = j & 1;
          ok = mbar_wait_bounded(bar(P_KFULL0 + s), (j >> 1) & 1, abort_flag);
          PAIR_TR(j, 0);
          if (ok && j > 0) ok = mbar_wait_bounded(bar(P_SFREE), (j - 1) & 1, abort_flag);
          PAIR_TR(j, 1);
          if (!ok) { fail(DEV_TIMEOUT_FULL); break; }
          tc_fence_after();
          const uint32_t st = sb + SP_K + s * KSLOT;
#pragma unroll
          for (int k = 0; k < 4; ++k)
            umma2_ss(tS, k128(sb + SP_QH + 32 * k), k128(st + 32 * k), idq, k > 0 ? 1u : 0u);
          for (int kk = 0; kk < 4 * np; ++kk)
            umma2_ss(tS, k128(sb + SP_QP + 16384 * (kk >> 2) + 32 * (kk & 3)),
                     k128(st + 8192 + 8192 * (kk >> 2) + 32 * (kk & 3)), idq, 1u);
          umma2_commit_both(bar(P_SFULL));
          umma2_commit_both(bar(P_KEMPTY0 + s));
          PAIR_TR(j, 2);
          if (j == 0) PAIR_SPAN(8);
          issued_any = true;
        }
        if (j > 0) {
          const int jj = j - 1;
          ok = mbar_wait_bounded(bar(P_PFULL), jj & 1, abort_flag);
          if (ok) ok = mbar_wait_bounded(bar(P_VFULL), jj & 1, abort_flag);
          PAIR_TR(jj, 3);
          if (!ok) { fail(DEV_TIMEOUT_SOFTMAX); break; }
          tc_fence_after();
          const uint32_t st = sb + SP_V;
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint32_t acc = (jj > 0 || k > 0) ? 1u : 0u;
            umma2_ts(tOz, tP + 8 * k, mn128(st + 2048 * k), idz, acc);
            umma2_ts(tOv, tP + 8 * k, mn64(st + V_VH + 1024 * k), idv, acc);
          }
          umma2_commit_both(bar(P_PFREE));   // P and the V slot are free
          PAIR_TR(jj, 4);
        }
      }
      PAIR_SPAN(9);
      if (!ok && issued_any) {
        umma2_commit_both(bar(P_DRAIN));
        mbar_wait_bounded(bar(P_DRAIN), 0, nullptr, 100000000ull);
      }
    }
    __syncwarp();
  } else if (warp < 8) {
    // ------------------------------------------------ softmax + epilogue (256 threads)
    const int quarter = warp & 3, half = warp >> 2;
    const int r = quarter * 32 + lane;
    const int row = row0 + r;
    const bool in_range = row < L;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t pair_bar = 2 + quarter;
    const float ch = a.headc[h];
    const float4 sq = in_range ? a.rowq[static_cast<int64_t>(bh) * L + row] : make_float4(0, 0, 0, 0);
    const float pq = static_cast<float>(IPA_PQ);
    const int tev = (tid == 0) ? 0 : (tid == 96) ? 1 : -1;
    (void)tev;

    // Q_pair = (log2(e) w_L w_bias[:, h]) * z1_i: the z1 rows arrive by TMA in
    // the 128-byte swizzled K-major panels the MMA reads; each thread scales
    // half of the panels of its row in place (fp32 product, one fp16 rounding)
    {
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(bar(P_QFULL), 0, abort_flag)) && lane == 0)
        fail(DEV_TIMEOUT_FULL);
      const float* wr = a.wqp + static_cast<int64_t>(h) * DZ;
      float qmax = 0.f;   // largest |Q_pair| before rounding (NaN if any is NaN)
      for (int p = half * (np / 2); p < (half + 1) * (np / 2); ++p) {
        unsigned char* prow = smem + SP_QP + 16384 * p + r * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint4* ptr = reinterpret_cast<uint4*>(prow + ((c ^ (r & 7)) << 4));
          uint4 u = *ptr;
          const float4 w0 = __ldg(reinterpret_cast<const float4*>(wr + 64 * p + 8 * c));
          const float4 w1 = __ldg(reinterpret_cast<const float4*>(wr + 64 * p + 8 * c + 4));
          const float2 z0 = unpack_half2(u.x), z1 = unpack_half2(u.y), z2 = unpack_half2(u.z), z3 = unpack_half2(u.w);
          const float e[8] = {z0.x * w0.x, z0.y * w0.y, z1.x * w0.z, z1.y * w0.w,
                              z2.x * w1.x, z2.y * w1.y, z3.x * w1.z, z3.y * w1.w};
#pragma unroll
          for (int t = 0; t < 8; ++t) qmax = fmax_nan(qmax, fabsf(e[t]));
          u = make_uint4(pack_half2(e[0], e[1]), pack_half2(e[2], e[3]), pack_half2(e[4], e[5]), pack_half2(e[6], e[7]));
          *ptr = u;
        }
      }
      if (in_range && !(qmax < 65520.f)) record_error(a.err, DEV_NONFINITE);
      fence_proxy_async_smem();
      named_bar_sync(1, NSOFT);
      if (tid == 0) PAIR_SPAN(6);
      if (tid == 0) mbar_arrive_cluster(bar0(P_QREADY));
    }

    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    const int OW = DZ + 64;
    const int o_lo = half * (OW / 2), o_hi = o_lo + OW / 2;
    for (int j = 0; j < nt && ok; ++j) {
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(bar(P_SFULL), j & 1, abort_flag))) {
        if (lane == 0) fail(DEV_TIMEOUT_MMA);
        ok = false;
        break;
      }
      if (tev >= 0) PAIR_TR(j, tev ? 26 : 16);
      tc_fence_after();
      uint32_t sr[64];
      {
        uint32_t r0[32], r1[32];
        tmem_ld32(tmem + TM_S + 64 * half + lane_off, r0);
        tmem_ld32(tmem + TM_S + 64 * half + 32 + lane_off, r1);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; ++e) { sr[e] = r0[e]; sr[32 + e] = r1[e]; }
      }
      tc_fence_before();
      if (tid == 0) PAIR_TR(j, 17);
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(bar0(P_SFREE));
      if (tid == 0) PAIR_TR(j, 18);
      const int cs = j % NCOL;
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(bar(P_COLFULL0 + cs), (j / NCOL) & 1, abort_flag))) {
        if (lane == 0) fail(DEV_TIMEOUT_FULL);
        ok = false;
        break;
      }
      if (tid == 0) PAIR_TR(j, 19);
      const float4* colv = reinterpret_cast<const float4*>(col_s + cs * 128 + 64 * half);
      const float4 dd = dinfo[cs * 2 + half];
      const float rt = ch * (2.f * fmaf(sq.x, dd.x, fmaf(sq.y, dd.y, sq.z * dd.z)) - pq * dd.w);
      // x = S + column term (packed pairs), running maximum over this half's keys
      float2 x[32];
      float mxa = -INFINITY, mxb = -INFINITY;
#pragma unroll
      for (int k4 = 0; k4 < 16; ++k4) {
        const float4 cv = colv[k4];
        x[2 * k4] = add_f32x2(make_float2(__uint_as_float(sr[4 * k4]), __uint_as_float(sr[4 * k4 + 1])),
                              make_float2(cv.x, cv.y));
        x[2 * k4 + 1] = add_f32x2(make_float2(__uint_as_float(sr[4 * k4 + 2]), __uint_as_float(sr[4 * k4 + 3])),
                                  make_float2(cv.z, cv.w));
        mxa = fmax3(mxa, x[2 * k4].x, x[2 * k4].y);
        mxb = fmax3(mxb, x[2 * k4 + 1].x, x[2 * k4 + 1].y);
      }
      // this half's max in full logit units (the row term differs between the key halves)
      const float mine = fmaxf(mxa, mxb) + rt;
      float* xb = xch + (j & 1) * 256;
      xb[half * 128 + r] = mine;
      if (tid == 0) PAIR_TR(j, 20);
      named_bar_sync(pair_bar, 64);
      if (tid == 0) PAIR_TR(j, 21);
      const float mt = fmaxf(mine, xb[(1 - half) * 128 + r]);
      const bool need = mt > m_used + a.tau;
      const bool resc = need && (m_used != -INFINITY);
      const float scale = resc ? ex2(m_used - mt) : 1.f;
      if (need) m_used = mt;
      l *= scale;
      // while no key of the row has been allowed, every x is -inf and the
      // exponent base 0 gives P = 0
      const float nbase = (m_used != -INFINITY) ? rt - m_used : 0.f;
      const float2 nb2 = make_float2(nbase, nbase);
      // P = 2^(x - base) rounded to fp16 (round to nearest even) in the pack;
      // the row sum adds exactly the fp16 values the P.V MMA consumes
      uint32_t pk[32];
      float ls4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        const float2 y = add_f32x2(x[k], nb2);
        pk[k] = pack_half2(ex2(y.x), ex2(y.y));
        ls4[k & 3] = add_half2_to_f32(pk[k], ls4[k & 3]);
      }
      l += (ls4[0] + ls4[1]) + (ls4[2] + ls4[3]);
      if (tid == 0) PAIR_TR(j, 22);
      // PV(j-1) must have finished reading P and accumulating O
      if (j >= 1 && !__all_sync(0xffffffffu, mbar_wait_bounded(bar(P_PFREE), (j - 1) & 1, abort_flag))) {
        if (lane == 0) fail(DEV_TIMEOUT_MMA);
        ok = false;
        break;
      }
      if (tid == 0) PAIR_TR(j, 23);
      tc_fence_after();
      if (__any_sync(0xffffffffu, resc)) {
        for (int c0 = o_lo; c0 < o_hi; c0 += 32) {
          uint32_t o[32];
          tmem_ld32(tmem + c0 + lane_off, o);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * scale);
          tmem_st32(tmem + c0 + lane_off, o);
        }
      }
      tmem_st32(tmem + TM_P + 32 * half + lane_off, pk);
      tmem_st_wait();
      tc_fence_before();
      if (tid == 0) PAIR_TR(j, 24);
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(bar0(P_PFULL));
      if (tid == 0) PAIR_TR(j, 25);
      if (tid == 96) PAIR_TR(j, 27);
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
    if (ok && !__all_sync(0xffffffffu, mbar_wait_bounded(bar(P_PFREE), (nt - 1) & 1, abort_flag))) {
      if (lane == 0) fail(DEV_TIMEOUT_MMA);
      ok = false;
    }
    if (tid == 0) PAIR_SPAN(10);
    const bool all_ok = __all_sync(0xffffffffu, ok);
    // key-split tail: each chunk stores its partial accumulators, row
    // maximum and half sums; the chunk that finishes its tile last (ticket)
    // merges all chunks in chunk order into tensor memory, so the result does
    // not depend on which chunk that is, and runs the output pass.  A chunk's
    // block holds the accumulators as groups of four columns,
    // [OW / 4][128 rows][4] (a warp's float4 stores cover 512 contiguous
    // bytes), then the row maximum and the two half sums, [3][128].
    bool epi = true;
    if (chunk >= 0) {
      const int OW3 = OW + 3;
      const int64_t qc = pair - a.split_first;   // (split tile) S + chunk
      const int64_t blk_floats = static_cast<int64_t>(OW3) * 128;
      const int64_t mine = (2 * qc + rank) * blk_floats;   // this chunk-CTA's block in part
      if (all_ok) {
        tc_fence_after();
        for (int c0 = o_lo; c0 < o_hi; c0 += 32) {
          uint32_t o[32];
          tmem_ld32(tmem + c0 + lane_off, o);
          tmem_ld_wait();
          float4* m4 = IPA_SPAN(reinterpret_cast<float4*>(a.part), mine / 4 + (c0 / 4) * 128, 8 * 128,
                                a.part_extent / 4, a.err);
#pragma unroll
          for (int g = 0; g < 8; ++g)
            m4[g * 128 + r] = make_float4(__uint_as_float(o[4 * g]), __uint_as_float(o[4 * g + 1]),
                                          __uint_as_float(o[4 * g + 2]), __uint_as_float(o[4 * g + 3]));
        }
        if (half == 0) *IPA_AT(a.part, mine + OW * 128 + r, a.part_extent, a.err) = m_used;
        *IPA_AT(a.part, mine + (OW + 1 + half) * 128 + r, a.part_extent, a.err) = l;
      }
      // the barrier orders every thread's stores before thread 0's device-
      // scope fence, which orders them before the ticket (fences are
      // cumulative); the merging CTA fences after reading the ticket
      named_bar_sync(1, NSOFT);
      volatile int* last = reinterpret_cast<volatile int*>(smem + SP_AUX + AX_LAST);
      if (tid == 0) {
        int* tk = IPA_AT(a.ticket, 2 * (qc / a.split_s) + rank, a.ticket_extent, a.err);
        __threadfence();
        const bool fin = atomicAdd(tk, 1) == a.split_s - 1;
        if (fin) {
          *tk = 0;   // every chunk of the tile has counted: ready for the next call
          __threadfence();
        }
        *last = fin ? 1 : 0;
      }
      named_bar_sync(1, NSOFT);
      epi = *last != 0;
      if (epi) {
        const float* c0p = a.part + (2 * (qc - chunk) + rank) * blk_floats;   // chunk 0 of this tile
        const int S = a.split_s;
        float ms[MAX_SPLIT], wt[MAX_SPLIT];
        float M = -INFINITY;
#pragma unroll
        for (int s = 0; s < MAX_SPLIT; ++s) {
          ms[s] = s < S ? (s == chunk ? m_used : __ldcg(c0p + 2 * s * blk_floats + OW * 128 + r)) : -INFINITY;
          M = fmaxf(M, ms[s]);
        }
        float ln = 0.f;
#pragma unroll
        for (int s = 0; s < MAX_SPLIT; ++s) {
          wt[s] = (s < S && M != -INFINITY) ? ex2(ms[s] - M) : 0.f;
          if (s < S) ln = fmaf(wt[s], s == chunk ? l : __ldcg(c0p + 2 * s * blk_floats + (OW + 1 + half) * 128 + r), ln);
        }
        tc_fence_after();
        // 16 columns at a time: the loads of every other chunk are issued
        // together (one L2 round trip per group), then summed in chunk order
        for (int c0 = o_lo; c0 < o_hi; c0 += 16) {
          uint32_t o[16];
          tmem_ld16(tmem + c0 + lane_off, o);
          float v[MAX_SPLIT][16];
#pragma unroll
          for (int s = 0; s < MAX_SPLIT; ++s) {
            const float4* src = reinterpret_cast<const float4*>(c0p + 2 * s * blk_floats) + (c0 / 4) * 128 + r;
            const bool other = s < S && s != chunk;
#pragma unroll
            for (int g = 0; g < 4; ++g) {
              const float4 x = other ? __ldcg(src + g * 128) : make_float4(0.f, 0.f, 0.f, 0.f);
              v[s][4 * g] = x.x;
              v[s][4 * g + 1] = x.y;
              v[s][4 * g + 2] = x.z;
              v[s][4 * g + 3] = x.w;
            }
          }
          tmem_ld_wait();
          float acc[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) acc[e] = 0.f;
#pragma unroll
          for (int s = 0; s < MAX_SPLIT; ++s) {
            if (s < S) {
#pragma unroll
              for (int e = 0; e < 16; ++e) acc[e] = fmaf(wt[s], s == chunk ? __uint_as_float(o[e]) : v[s][e], acc[e]);
            }
          }
#pragma unroll
          for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(acc[e]);
          tmem_st16(tmem + c0 + lane_off, o);
        }
        tmem_st_wait();
        m_used = M;
        l = ln;
        // the output pass reads columns of both halves of a row
        tc_fence_before();
        named_bar_sync(pair_bar, 64);
        tc_fence_after();
      }
    }
    if (epi) {
      xch[512 + half * 128 + r] = l;
      named_bar_sync(pair_bar, 64);
      if (tid == 0) PAIR_SPAN(20);
      const float lt = l + xch[512 + (1 - half) * 128 + r];
      const bool dead = !(in_range && f3.x != 0.f && lt > 0.f);
      // training forward: log-sum-exp of the true logits; the pass left the row
      // constant c sum_p |gq'_p|^2 (rowq.w) out of its logits
      if (a.lse != nullptr && half == 0 && in_range)
        *IPA_AT(a.lse, static_cast<int64_t>(bh) * L + row, static_cast<int64_t>(a.B) * a.H * L, a.err) = dead ? INFINITY : (m_used + log2f(lt) - sq.w) * 0.69314718055994531f;
      // direct output pass when the pair block has no padding and whole
      // 64-column factors (the staged pass below handles every other shape)
      if (a.tma_epi) {
        // staged pair features (z1 from the boxes the producer loaded, the
        // output through staging boxes and a TMA store), scalars and points direct
        const bool zok = __all_sync(0xffffffffu, mbar_wait_bounded(bar(P_ZFULL), 0, abort_flag));
        if (!zok && lane == 0) fail(DEV_TIMEOUT_FULL);
        const int nz = DZ / 32;
        if (all_ok && zok && !*abort_flag) {
          tc_fence_after();
          const float inv = dead ? 0.f : 1.f / lt;
          const int rrow = in_range ? row : 0;
          const int64_t orow = (static_cast<int64_t>(b) * L + rrow) * a.H + h;
          const int64_t nrows = static_cast<int64_t>(a.B) * L * a.H;
          auto z1box = [&](int k) -> const unsigned char* { return smem + SP_QP + 16384u * k; };
          auto obox = [&](int k) -> unsigned char* {
            return smem + (k == 0 ? SP_QH : SP_QP + 16384u * (nz + k - 1));
          };
          stage_row_pair(tmem + lane_off, half, a.Cz, a.RCz / a.Cz, inv, r,
                         a.uagg != nullptr ? IPA_SPAN(a.uagg, orow * a.RCz, a.RCz, nrows * a.RCz, a.err) : nullptr,
                         in_range, z1box, obox);
          if (tid == 0) PAIR_SPAN(22);
          if (half == 0)
            write_row_points<IPA_C, IPA_PV>(tmem + DZ + lane_off, inv, dead, in_range,
                                            IPA_SPAN(a.out, orow * a.F, a.F, nrows * a.F, a.err), g0, g1, g2, cn);
          fence_proxy_async_smem();   // the staging writes, before the TMA store reads them
        }
        named_bar_sync(1, NSOFT);
        // a tile past the last row (the pair's second CTA when L <= 128) has
        // nothing to store; the tensor map clips the rest of a ragged tile
        if (tid == 0 && all_ok && zok && !*abort_flag && row0 < L &&
            IPA_CHECK(row0 >= 0 && b >= 0 && b < a.B && h >= 0 && h < a.H, a.err)) {
          for (int k = 0; k < a.Cz / 32; ++k)
            tma_store_4d(&tm_out, sb + (k == 0 ? SP_QH : SP_QP + 16384u * (nz + k - 1)), IPA_C + 4 * IPA_PV + 32 * k, h,
                         row0, b);
          bulk_commit_group();
          bulk_wait_read_all();   // the staging boxes must outlive the reads, not the writes
        }
        if (tid == 0) PAIR_SPAN(21);
      } else if (a.RCz == DZ && (a.Cz & 63) == 0) {
        if (all_ok && !*abort_flag) {
          tc_fence_after();
          const float inv = dead ? 0.f : 1.f / lt;
          const int rrow = in_range ? row : 0;
          const int64_t orow = (static_cast<int64_t>(b) * L + rrow) * a.H + h;
          const int64_t nrows = static_cast<int64_t>(a.B) * L * a.H;
          unsigned long long* etr = nullptr;
#ifdef IPA_TRACE
          if (tid == 0 && blockIdx.x < 4096) etr = &g_pair_span[blockIdx.x][22];
#endif
          write_row_direct<IPA_C, IPA_PV>(tmem + lane_off, half, DZ, a.Cz, a.RCz / a.Cz, inv, dead, in_range,
                                          a.z1f + (static_cast<int64_t>(b) * L + rrow) * DZ,
                                          IPA_SPAN(a.out, orow * a.F, a.F, nrows * a.F, a.err),
                                          a.uagg != nullptr ? IPA_SPAN(a.uagg, orow * a.RCz, a.RCz, nrows * a.RCz, a.err)
                                                            : nullptr,
                                          g0, g1, g2, cn, etr);
          if (tid == 0) PAIR_SPAN(21);
        }
      } else {
        const int pitch = stage_pitch(DZ);
        float* stage = reinterpret_cast<float*>(smem + SP_QP);
        if (all_ok) {
          tc_fence_after();
          const float inv = dead ? 0.f : 1.f / lt;
          float* orow = stage + r * pitch;
          // tensor memory holds [O_pair | O_v]; the stage row is [O_v | O_pair | frame]
          for (int c0 = o_lo; c0 < o_hi; c0 += 32) {
            uint32_t o[32];
            tmem_ld32(tmem + c0 + lane_off, o);
            tmem_ld_wait();
            const int dstc = c0 < DZ ? 64 + c0 : c0 - DZ;
#pragma unroll
            for (int e = 0; e < 32; e += 4)
              *reinterpret_cast<float4*>(orow + dstc + e) =
                  make_float4(__uint_as_float(o[e]) * inv, __uint_as_float(o[e + 1]) * inv,
                              __uint_as_float(o[e + 2]) * inv, __uint_as_float(o[e + 3]) * inv);
          }
          if (half == 0) stage_frame(orow + 64 + DZ, g0, g1, g2, cn, dead);
        }
        tc_fence_before();
        named_bar_sync(1, NSOFT);
        if (tid == 0) PAIR_SPAN(11);
        if (!*abort_flag) {
          EpilogueArgs ea{stage, DZ, a.Cz, a.RCz, a.F, a.H, L, b, h, row0, a.z1f, a.out};
          ea.uagg = a.uagg;
          ea.rows = static_cast<int64_t>(a.B) * L * a.H;
          ea.err = a.err;
#ifdef IPA_TRACE
          ea.trace = (blockIdx.x < 4096 && warp == 0) ? &g_pair_span[blockIdx.x][16] : nullptr;
#endif
          write_rows<IPA_C, IPA_PV>(ea, warp, lane);
        }
      }
    } else if (a.tma_epi) {
      // the z1 boxes the producer loaded must land before the CTA ends
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(bar(P_ZFULL), 0, abort_flag)) && lane == 0)
        fail(DEV_TIMEOUT_FULL);
    }
  }

  if (tid == 0) PAIR_SPAN(12);
  tc_fence_before();
  __syncthreads();
  if (tid == 0) PAIR_SPAN(13);
  cluster_sync();
  if (tid == 0) PAIR_SPAN(14);
  if (warp == W_MMA) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, TM_COLS);
  }
#ifdef IPA_TRACE
  if (threadIdx.x == 0 && blockIdx.x < 4096) {
    g_pair_span[blockIdx.x][3] = clock64();
    g_pair_span[blockIdx.x][1] = globaltimer_ns();
  }
#endif
}

}  // namespace

bool ipa_pair_supported(int DZ) { return DZ == 128 || DZ == 256; }

// Key split of the last, partial wave.  T pair tiles on P resident CTA pairs
// run floor(T / P) full waves and a tail of r = T mod P tiles that leaves
// P - r pairs idle for a whole tile.  Splitting each tail tile's nkp key
// tiles into S chunks runs the tail as ceil(r S / P) rounds of
// ceil(nkp / S) key tiles.  In units of one key tile's time, a CTA pair's
// set-up, Q load and output pass cost about 5 (event clocks of the tracing
// build: ~10 us against ~2 us per key tile), and the merge about
// 1 + (S - 1) / 2.  S is the cheapest of 2 .. MAX_SPLIT under that cost,
// taken when it saves at least a tenth of the tail and the partials fit the
// workspace's reserve.
SplitPlan ipa_split_plan(int T, int nkp, int P, int64_t max_tiles, int64_t max_chunks) {
  SplitPlan none{T, 1};
  if (T <= 0 || P <= 0 || nkp < 2) return none;
  const int r = T % P;
  if (r == 0) return none;
  constexpr double kFixed = 5.0;
  double best = 0.9 * (nkp + kFixed);
  int bs = 1;
  for (int S = 2; S <= MAX_SPLIT && S <= nkp; ++S) {
    if (r > max_tiles || static_cast<int64_t>(r) * S > max_chunks) break;
    const int rounds = (r * S + P - 1) / P;
    const double cost = rounds * ((nkp + S - 1) / S + kFixed) + 1.0 + 0.5 * (S - 1);
    if (cost < best) {
      best = cost;
      bs = S;
    }
  }
  return bs == 1 ? none : SplitPlan{T - r, bs};
}

cudaError_t ipa_launch_core_pair(const IpaLaunch& a, cudaStream_t stream) {
  unsigned char* ws = a.ws;
  const IpaWorkspace& w = a.lay;
  CUtensorMap tqh, tkh, tz2k, tz2v, tvh, tz1;
  const uint64_t bh = static_cast<uint64_t>(a.B) * a.H;
  const uint64_t rowb = static_cast<uint64_t>(a.L) * DH * 2;
  bool ok = encode_tmap_f16_3d(&tqh, ws + w.qh, DH, a.L, bh, DH * 2, rowb, 64, QT) &&
            encode_tmap_f16_3d(&tkh, ws + w.kh, DH, a.L, bh, DH * 2, rowb, 64, 64) &&
            encode_tmap_f16_panels(&tz2k, ws + w.z2, a.DZ, a.L, a.B, 64, a.DZ / 64) &&
            encode_tmap_f16_panels(&tz2v, ws + w.z2, a.DZ, a.L, a.B, 128, a.DZ / 128) &&
            encode_tmap_f16_3d(&tvh, ws + w.vh, DH, a.L, bh, DH * 2, rowb, 32, 128, 64) &&
            encode_tmap_f16_panels(&tz1, ws + w.z1h, a.DZ, a.L, a.B, 128, a.DZ / 64);
  if (!ok) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(ipa_attention_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(SP_ALLOC));
  if (e != cudaSuccess) return e;
  PairArgs t{};
  t.B = a.B; t.L = a.L; t.H = a.H; t.DZ = a.DZ; t.RCz = a.RCz; t.Cz = a.Cz;
  t.nqt = a.nqt; t.nkt = a.nkt; t.nqp = (a.L + 255) / 256; t.nkp = (a.L + 127) / 128; t.F = a.F; t.tau = 8.f;
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
  // staged output pass: whole 32-column factors, the pair block unpadded, and
  // the z1 boxes plus the staging boxes inside the freed operand area
  CUtensorMap tz1f = tz1, tout = tz1;
  t.tma_epi = 0;
  if (a.RCz == a.DZ && a.Cz % 32 == 0 &&
      SP_QP + 16384u * static_cast<uint32_t>(a.DZ / 32 + a.Cz / 32 - 1) <= SP_AUX) {
    const uint64_t zd[3] = {static_cast<uint64_t>(a.DZ), static_cast<uint64_t>(a.L), static_cast<uint64_t>(a.B)};
    const uint64_t zs[2] = {static_cast<uint64_t>(a.DZ) * 4, static_cast<uint64_t>(a.L) * a.DZ * 4};
    const uint32_t zb[3] = {32, 128, 1};
    const uint64_t od[4] = {static_cast<uint64_t>(a.F), static_cast<uint64_t>(a.H), static_cast<uint64_t>(a.L),
                            static_cast<uint64_t>(a.B)};
    const uint64_t os[3] = {static_cast<uint64_t>(a.F) * 4, static_cast<uint64_t>(a.H) * a.F * 4,
                            static_cast<uint64_t>(a.L) * a.H * a.F * 4};
    const uint32_t ob[4] = {32, 1, 128, 1};
    if (encode_tmap_f32_sw128(&tz1f, ws + w.z1f, 3, zd, zs, zb) && encode_tmap_f32_sw128(&tout, a.out, 4, od, os, ob))
      t.tma_epi = 1;
  }
  const int pairs = static_cast<int>(bh) * t.nqp;
  // one CTA per SM (shared memory), so P = SMs / 2 resident pairs; the
  // training forward (log-sum-exp and pair aggregate of whole rows) is not split
  SplitPlan plan{pairs, 1};
  if (a.lse == nullptr && a.uagg == nullptr && w.split_tiles > 0) {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess)
      plan = ipa_split_plan(pairs, t.nkp, sms / 2, w.split_tiles, w.split_chunks);
  }
  t.split_first = plan.first;
  t.split_s = plan.S;
  t.part = reinterpret_cast<float*>(ws + w.split);
  t.ticket = reinterpret_cast<int*>(ws + w.ticket);
  t.part_extent = w.split_chunks * 2 * (a.DZ + 67) * 128;
  t.ticket_extent = static_cast<int>(2 * w.split_tiles);
  const int blocks = plan.first + (pairs - plan.first) * plan.S;
  t.trace_cta0 = 0;
  t.trace_cta1 = 1;   // the peer CTA of the first pair
  ipa_attention_pair_kernel<<<static_cast<unsigned>(2 * blocks), NT, SP_ALLOC, stream>>>(tqh, tkh, tz2k, tz2v, tvh, tz1,
                                                                                          tz1f, tout, t);
  return cudaGetLastError();
}

#ifdef IPA_TRACE
bool ipa_pair_trace_read(void* host, size_t bytes) {
  if (bytes < sizeof(g_pair_trace)) return false;
  return cudaMemcpyFromSymbol(host, g_pair_trace, sizeof(g_pair_trace)) == cudaSuccess;
}
bool ipa_pair_span_read(void* host, size_t bytes) {
  if (bytes < sizeof(g_pair_span)) return false;
  return cudaMemcpyFromSymbol(host, g_pair_span, sizeof(g_pair_span)) == cudaSuccess;
}
int ipa_pair_max_clusters() {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(2 * 192);
  cfg.blockDim = dim3(NT);
  cfg.dynamicSmemBytes = SP_ALLOC;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  int n = -1;
  cudaFuncSetAttribute(ipa_attention_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(SP_ALLOC));
  if (cudaOccupancyMaxActiveClusters(&n, ipa_attention_pair_kernel, &cfg) != cudaSuccess) return -1;
  return n;
}
#endif

}  // namespace fipa
