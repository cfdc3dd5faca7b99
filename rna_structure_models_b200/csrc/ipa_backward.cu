// Gradients of the fused IPA core on sm_100a (Flash Invariant Point
// Attention is a drop-in replacement for IPA in training: TL;DR, Abstract,
// Figure 3).  Flash-style recomputation on the augmented operands of the
// forward pass; no L x L array is stored.
//
// Notation (log2 units, per batch b and head h): x_ij = log2(e) l_ij is the
// true logit, recomputed exactly as the forward pass computed it:
//   x_ij = Q_h,i . K_h,j + Q_pair,i . Z2_j + col_j(I) + rt_i(J) - w_i
// with the forward prologue's rows (Q_h unscaled tile-local query points,
// K_h 2c-scaled tile-local key points, V_h centroid-relative value points),
// col / rt the per-key / per-row tile-origin terms and w_i = c |gq'_i|^2 the
// row constant the forward pass leaves out.  With lse2_i the training
// forward's log-sum-exp (log2 units), p_ij = 2^(x_ij - lse2_i) = a_ij and
//   dP_ij = dO_i . V_h,j + dU_i . Z2_j     dO_i = [g_o | R_i d_opt | R_i d_opt],
//                                          dU_i = z1_i (.) g_pair_i
//   dS_ij = ln 2 p_ij (dP_ij - D_i)        D_i = sum_j p_ij dP_ij, from the
//                                          forward output and U
// dS is dL/dx.  The kernels:
//   ipa_bwd_rows_kernel  one warp per (b, i, h): dO, dU, Q_pair (fp16 rows;
//                        DZ / 32 columns per lane with 16-byte accesses for
//                        contiguous fp32 rows),
//                        the row constant -(w_i + lse2_i), D_i and the query
//                        and key points relative to the centroid (fp32);
//   query pass           one CTA per (b, h, 128 queries), 32-key tiles:
//                        S, dP (tcgen05, TMEM), dS (fp16, TMEM), then
//                        dQ_h += dS K_h, dQ_pair += dS Z2 (A = dS from TMEM),
//                        row sums rs_i = sum_j dS_ij, RSo_i = sum_j dS_ij o_J;
//   key pass             one CTA per (b, h, 128 keys), 32-query tiles:
//                        S^T, dP^T, then P^T and dS^T (fp16, in place in
//                        TMEM) as A operands of dV += P^T dO,
//                        dZ2 += P^T dU + dS^T Q_pair, dK_h += dS^T Q_h, column
//                        sums cs_j, CSo_j = sum_i dS_ij o_I, and the d gamma
//                        sum_i dS_ij |gq_i - gk_j|^2 from fp32 points (CUDA
//                        cores, inside the dS loop);
//   (both passes run as one grid, ipa_bwd_kernel, so that the key-pass CTAs
//   fill the SMs the query pass leaves idle in its last wave; key-pass CTAs
//   of the grid's last, partial wave may run as chunks of consecutive query
//   tiles whose partial sums the chunk with the last ticket adds in chunk
//   order, ipa_bwd_split_plan)
//   ipa_bwd_map_kernel   per residue, all heads: the augmented gradients
//                        mapped back to q, k, v, the local points and the
//                        frames (sums over heads), per-block d gamma partials;
//   ipa_bwd_pair_kernel  per pair column and residue: d z1, d z2
//                        (sums over heads) and d w_bias partials
//                        (ipa_bwd_pair4_kernel: four columns per thread,
//                        16-byte accesses, for contiguous fp32 rows);
//   ipa_bwd_reduce_kernel  fixed-order sums of the partials, one block per
//                        (head, 32 pair columns).
// Every mbarrier wait is bounded (2 s) and reports into the error word.
#include <cuda_fp16.h>

#include <cmath>
#include <cstdint>

#include "bounds.cuh"
#include "internal.h"
#include "sm100.cuh"

#define IPA_FILE_TAG 11

#ifdef IPA_TRACE
// Tracing build only: per-tile event clocks of the first CTA of each pass,
// [pass][tile][event] (events listed where they are taken).
__device__ unsigned long long g_bwd_trace[2][256][16];
#define BWD_TR(pass, j, ev)                                                         \
  do {                                                                              \
    if (blk == 0 && (j) >= 0 && (j) < 256) g_bwd_trace[(pass)][(j)][(ev)] = clock64(); \
  } while (0)
#else
#define BWD_TR(pass, j, ev) \
  do {                      \
  } while (0)
#endif

namespace fipa {

using namespace sm100;

namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.69314718055994531f;

struct BwdArgs {
  int B, L, H, DZ, RCz, Cz, R, nqt, nkt, ns;
  int qp_stage;          // query pass: 1 if its last stage lives in the Q_pair area (free once Q_pair is in TMEM)
  float qscale, w_L, w_C;
  // forward prologue outputs (workspace)
  const float4* rowq;    // [B*H, L] (sum_p gq', c |gq'|^2)
  const float4* colk;    // [B*H, L] (2c sum_p gk', 0 or -inf)
  const float4* oq;      // [B, nqt] 128-row tile origins
  const float4* ok;      // [B, nkt] 64-row tile origins
  const float4* cen;     // [B]
  const float* headc;    // [H] c = log2(e) w_L gamma w_C / 2
  const float* wqp;      // [H, DZ] log2(e) w_L w_bias
  const float4* frame;   // [B, L, 4]
  const float* z1f;      // [B, L, DZ]
  const __half* z1h;     // [B, L, DZ]
  // backward prologue outputs
  const float2* rowd;    // [B*H, L] (-(w + lse2), D)
  // pass outputs
  float* dqh;            // [B*H, L, 64]
  float* dqp;            // [B*H, L, DZ]
  float4* rsq;           // [B*H, L] (rs, RSo)
  float* dkh;            // [B*H, L, 64]
  float* dva;            // [B*H, L, 64]
  float* dz2;            // [B*H, L, DZ]
  float4* csk;           // [B*H, L] (cs, CSo)
  const float* pts;      // [B*H, L, 24]: query points gq - cen (12) | key points gk - cen (12), fp32
  float* gsum;           // [B*H, L]: sum_i dS_ij |gq_i - gk_j|^2 per key (the d gamma sum, one side only)
  int* err;
  // key pass, query split of the last wave: key tiles [split_first, nkb) run
  // as split_s chunks of consecutive 32-query tiles (split_s == 1: none)
  int split_first, split_s;
  float* part;           // per chunk: [DZ + 128][128] accumulators (float4 groups), [2][5][128] half sums
  int64_t part_extent;   // floats in part
  int* ticket;           // per split key tile: chunks finished (zero between calls)
  int ticket_extent;
};

__device__ __forceinline__ uint64_t kd128(uint32_t a) { return smem_desc(a, 16, 1024, 2); }      // K-major SW128
__device__ __forceinline__ uint64_t mnd(uint32_t a, uint32_t panel) { return smem_desc(a, panel, 1024, 2); }  // MN-major SW128

__device__ __forceinline__ float ldf(const View& v, int64_t off) {
  return v.dtype == 1 ? static_cast<float>(reinterpret_cast<const double*>(v.p)[off])
                      : reinterpret_cast<const float*>(v.p)[off];
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(r[0]),
               "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}

// ------------------------------------------------------------------ prologue
struct RowsArgs {
  int B, L, H, DZ, RCz, Cz, F;
  bool z1_half;          // Q_pair from the fp16 z1 (as the CTA-pair forward core), else from fp32 z1
  int pair_cpl;          // 4 or 8: pair columns per lane from 16-byte loads (contiguous fp32 rows, R Cz = DZ); 0: per element
  View g_out, out, lse, uagg;
  const float4* frame;
  const float4* cen;
  const float4* rowq;
  const float* wqp;
  const float* z1f;
  const __half* z1h;
  __half* doh;           // [B*H, L, 64]
  __half* du;            // [B*H, L, DZ]
  __half* qp;            // [B*H, L, DZ]
  float2* rowd;          // [B*H, L]
  View q_pts, k_pts;
  float* pts;            // [B*H, L, 24]
  int* err;
  int* kticket;          // the key pass's split tickets, zeroed here (nkticket ints)
  int nkticket;
};

// Pair block of one row when its rows are contiguous fp32 and R Cz = DZ:
// lane l owns the CPL = DZ / 32 consecutive columns [CPL l, CPL l + CPL) (one
// factor r, features cc .. cc + CPL - 1), every operand read with 16-byte
// loads issued together; the same per-element arithmetic as the general loop.
template <int CPL>
__device__ __forceinline__ void bwd_pair_cols(const RowsArgs& a, int lane, bool live, int64_t gbase, int64_t ubase,
                                              int64_t bi, int h, __half* dur, __half* qpr, float& part) {
  const int c0 = CPL * lane, r = c0 / a.Cz, cc = c0 % a.Cz;
  float z[CPL], w[CPL], gp[CPL], u[CPL], zh[CPL];
  const float4* z4 = reinterpret_cast<const float4*>(a.z1f + bi * a.DZ + c0);
  const float4* w4 = reinterpret_cast<const float4*>(a.wqp + static_cast<int64_t>(h) * a.DZ + c0);
  const float4* g4 = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(a.g_out.p) + gbase +
                                                     (IPA_C + 4 * IPA_PV + cc));
  const float4* u4 = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(a.uagg.p) + ubase +
                                                     r * a.uagg.s[3] + cc);
#pragma unroll
  for (int q = 0; q < CPL / 4; ++q) {
    const float4 zv = z4[q], wv = w4[q];
    const float4 gv = live ? g4[q] : make_float4(0.f, 0.f, 0.f, 0.f);
    const float4 uv = live ? u4[q] : make_float4(0.f, 0.f, 0.f, 0.f);
    z[4 * q] = zv.x; z[4 * q + 1] = zv.y; z[4 * q + 2] = zv.z; z[4 * q + 3] = zv.w;
    w[4 * q] = wv.x; w[4 * q + 1] = wv.y; w[4 * q + 2] = wv.z; w[4 * q + 3] = wv.w;
    gp[4 * q] = gv.x; gp[4 * q + 1] = gv.y; gp[4 * q + 2] = gv.z; gp[4 * q + 3] = gv.w;
    u[4 * q] = uv.x; u[4 * q + 1] = uv.y; u[4 * q + 2] = uv.z; u[4 * q + 3] = uv.w;
  }
  if (a.z1_half) {
    const __half* zr = a.z1h + bi * a.DZ + c0;
    uint32_t hw[CPL / 2];
    if constexpr (CPL == 8) {
      const uint4 t = *reinterpret_cast<const uint4*>(zr);
      hw[0] = t.x; hw[1] = t.y; hw[2] = t.z; hw[3] = t.w;
    } else {
      const uint2 t = *reinterpret_cast<const uint2*>(zr);
      hw[0] = t.x; hw[1] = t.y;
    }
#pragma unroll
    for (int e = 0; e < CPL / 2; ++e) {
      const float2 f = unpack_half2(hw[e]);
      zh[2 * e] = f.x;
      zh[2 * e + 1] = f.y;
    }
  } else {
#pragma unroll
    for (int e = 0; e < CPL; ++e) zh[e] = z[e];
  }
  uint32_t dw[CPL / 2], qw[CPL / 2];
#pragma unroll
  for (int e = 0; e < CPL; e += 2) {
    float d2v[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      d2v[k] = 0.f;
      if (live) {
        d2v[k] = __half2float(__float2half_rn(z[e + k] * gp[e + k]));
        part = fmaf(d2v[k], u[e + k], part);
      }
    }
    dw[e / 2] = pack_half2(d2v[0], d2v[1]);
    qw[e / 2] = pack_half2(zh[e] * w[e], zh[e + 1] * w[e + 1]);
  }
  if constexpr (CPL == 8) {
    *reinterpret_cast<uint4*>(dur + c0) = make_uint4(dw[0], dw[1], dw[2], dw[3]);
    *reinterpret_cast<uint4*>(qpr + c0) = make_uint4(qw[0], qw[1], qw[2], qw[3]);
  } else {
    *reinterpret_cast<uint2*>(dur + c0) = make_uint2(dw[0], dw[1]);
    *reinterpret_cast<uint2*>(qpr + c0) = make_uint2(qw[0], qw[1]);
  }
}

// One warp per (b, i, h), heads fastest.  Lane l: scalar channel l (< 16),
// point coordinate l (< 24: point l / 3, axis l % 3), pair columns l + 32 k
// (or, for contiguous fp32 rows, the lane's run of DZ / 32 columns).
__global__ void __launch_bounds__(256) ipa_bwd_rows_kernel(const RowsArgs a) {
  const int64_t wid = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (blockIdx.x == 0)
    for (int e = threadIdx.x; e < a.nkticket; e += blockDim.x) *IPA_AT(a.kticket, e, a.nkticket, a.err) = 0;
  if (wid >= static_cast<int64_t>(a.B) * a.L * a.H) return;
  const int h = static_cast<int>(wid % a.H);
  const int64_t bi = wid / a.H;
  const int i = static_cast<int>(bi % a.L), b = static_cast<int>(bi / a.L);
  const int64_t bhl = (static_cast<int64_t>(b) * a.H + h) * a.L + i;
  const float4* fr = a.frame + bi * 4;
  const float4 f0 = fr[0], f1 = fr[1], f2 = fr[2], f3 = fr[3];
  const bool live = f3.x != 0.f;
  const int C = IPA_C, PV = IPA_PV;
  const int64_t gbase = b * a.g_out.s[0] + i * a.g_out.s[1] + h * a.g_out.s[2];
  const int64_t obase = b * a.out.s[0] + i * a.out.s[1] + h * a.out.s[2];
  float part = 0.f;   // this lane's share of D_i
  // scalar channels
  float g_o = 0.f;     // rounded to fp16 as the dP MMA sees it, in D too
  if (lane < C && live) {
    g_o = __half2float(__float2half_rn(ldf(a.g_out, gbase + lane * a.g_out.s[3])));
    part = g_o * ldf(a.out, obase + lane * a.out.s[3]);
  }
  // value points: d_opt = g_pt + g_n unit(o_pt), dog = R d_opt (global frame)
  const int l = lane < 3 * PV ? lane : 0;
  const int x = l % 3, p3 = l - x;
  float opt = 0.f, gpt = 0.f, gn = 0.f;
  if (live) {
    opt = ldf(a.out, obase + (C + l) * a.out.s[3]);
    gpt = ldf(a.g_out, gbase + (C + l) * a.g_out.s[3]);
    gn = ldf(a.g_out, gbase + (C + 3 * PV + l / 3) * a.g_out.s[3]);
  }
  const float o0 = __shfl_sync(0xffffffffu, opt, p3), o1 = __shfl_sync(0xffffffffu, opt, p3 + 1),
              o2 = __shfl_sync(0xffffffffu, opt, p3 + 2);
  const float nrm = sqrtf(o0 * o0 + o1 * o1 + o2 * o2);
  const float dopt = gpt + (nrm > 0.f ? gn * opt / nrm : 0.f);
  const float d0 = __shfl_sync(0xffffffffu, dopt, p3), d1 = __shfl_sync(0xffffffffu, dopt, p3 + 1),
              d2 = __shfl_sync(0xffffffffu, dopt, p3 + 2);
  const float Rm[9] = {f0.x, f0.y, f0.z, f0.w, f1.x, f1.y, f1.z, f1.w, f2.x};
  const float4 cn = a.cen[b];
  const float tc[3] = {f2.y - cn.x, f2.z - cn.y, f2.w - cn.z};
  const float dog = fmaf(Rm[3 * x], d0, fmaf(Rm[3 * x + 1], d1, Rm[3 * x + 2] * d2));
  const float dog16 = __half2float(__float2half_rn(dog));
  const float og = fmaf(Rm[3 * x], o0, fmaf(Rm[3 * x + 1], o1, Rm[3 * x + 2] * o2)) + tc[x];   // og - centroid
  if (lane < 3 * PV && live) part = fmaf(dog16, og, part);
  // dO row: column l and 32 + l; dog coordinate e is held by lane e
  const float dg_a = __shfl_sync(0xffffffffu, dog16, (lane - 16) & 31);   // col l = 16 + e, e = l - 16
  const float dg_b = __shfl_sync(0xffffffffu, dog16, lane < 8 ? lane + 16 : lane - 8);
  const float c_lo = lane < C ? g_o : dg_a;
  const float c_hi = dg_b;                 // col 32 + l: l < 8 -> dog[16 + l], else dog[l - 8]
  const int64_t nbhl = static_cast<int64_t>(a.B) * a.H * a.L;
  __half* drow = IPA_SPAN(a.doh, bhl * 64, 64, nbhl * 64, a.err);
  drow[lane] = __float2half_rn(live ? c_lo : 0.f);
  drow[32 + lane] = __float2half_rn(live ? c_hi : 0.f);
  // pair block: dU = z1 (.) g_pair (fp16), Q_pair = fp16(w_qp z1), D += dU . U
  const float* z1r = a.z1f + bi * a.DZ;
  const __half* z1hr = a.z1h + bi * a.DZ;
  const float* wr = a.wqp + static_cast<int64_t>(h) * a.DZ;
  __half* dur = IPA_SPAN(a.du, bhl * a.DZ, a.DZ, nbhl * a.DZ, a.err);
  __half* qpr = IPA_SPAN(a.qp, bhl * a.DZ, a.DZ, nbhl * a.DZ, a.err);
  const int64_t ubase = b * a.uagg.s[0] + i * a.uagg.s[1] + h * a.uagg.s[2];
  if (a.pair_cpl == 8) bwd_pair_cols<8>(a, lane, live, gbase, ubase, bi, h, dur, qpr, part);
  else if (a.pair_cpl == 4) bwd_pair_cols<4>(a, lane, live, gbase, ubase, bi, h, dur, qpr, part);
  else for (int c = lane; c < a.DZ; c += 32) {
    float duv = 0.f;
    if (c < a.RCz && live) {
      const int r = c / a.Cz, cc = c % a.Cz;
      const float gp = ldf(a.g_out, gbase + (C + 4 * PV + cc) * a.g_out.s[3]);
      const __half d16 = __float2half_rn(z1r[c] * gp);
      duv = __half2float(d16);
      part = fmaf(duv, ldf(a.uagg, ubase + r * a.uagg.s[3] + cc * a.uagg.s[4]), part);
    }
    dur[c] = __float2half_rn(duv);
    const float zq = a.z1_half ? __half2float(z1hr[c]) : z1r[c];
    qpr[c] = __float2half_rn(zq * wr[c]);
  }
  // query and key points relative to the centroid (fp32), for the key
  // pass's d gamma sum: lane e < 12 query coordinate e, 12 <= lane < 24 key
  // coordinate e - 12
  if (lane < 24) {
    const bool isq = lane < 12;
    const int e = isq ? lane : lane - 12, pp = e / 3, xx = e % 3;
    const View& pv = isq ? a.q_pts : a.k_pts;
    const int64_t pb = b * pv.s[0] + i * pv.s[1] + h * pv.s[2] + pp * pv.s[3];
    const float x0 = ldf(pv, pb), x1 = ldf(pv, pb + pv.s[4]), x2 = ldf(pv, pb + 2 * pv.s[4]);
    const float v = fmaf(Rm[3 * xx], x0, fmaf(Rm[3 * xx + 1], x1, Rm[3 * xx + 2] * x2)) + tc[xx];
    *IPA_AT(a.pts, bhl * 24 + lane, nbhl * 24, a.err) = live ? v : 0.f;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
  if (lane == 0) {
    float rowc = -INFINITY, D = 0.f;
    if (live) {
      const float lse = ldf(a.lse, b * a.lse.s[0] + h * a.lse.s[1] + i * a.lse.s[2]);
      rowc = -(a.rowq[bhl].w + lse * kLog2e);
      D = part;
    }
    *IPA_AT(a.rowd, bhl, nbhl, a.err) = make_float2(rowc, D);
  }
}

// --------------------------------------------------------------- query pass
// Warps 0-7: two threads per query row (keys [16 half, 16 half + 16) of a
// 32-key tile); warp 8: TMA producer and the per-key column terms; warp 9:
// tensor memory and the MMA-issuing thread.
constexpr int NTH = 320, NSOFT = 256, W_PROD = 8, W_MMA = 9;
constexpr int MAX_NS = 3;
// Streamed tiles are 32 rows (keys in the query pass, queries in the key
// pass): at R Cz = 256 a 64-row stage left room for one stage only, which put
// every tile's load in series with its MMAs; 32-row stages fit two (query
// pass) and three (key pass).
constexpr int BT = 32;

// tensor memory (512 columns)
// Q_TM_QPT: the first QPT_COLS columns of the Q_pair rows (fp16 pairs), the
// A operand of most of S's pair part, so that its MMAs read only the key
// tile from shared memory
constexpr uint32_t Q_TM_DQP = 0, Q_TM_DQH = 256, Q_TM_S = 320, Q_TM_DP = 352, Q_TM_DS = 384, Q_TM_QPT = 400;
constexpr int QPT_COLS = 112;

struct QLayout {
  uint32_t qh, qp, dO, du, stg, stg_bytes, aux, total;
};
__host__ __device__ inline QLayout q_layout(int DZ, int ns) {
  QLayout s{};
  const uint32_t np = DZ / 64;
  s.qh = 0;
  s.qp = 16384;
  s.dO = s.qp + np * 16384;
  s.du = s.dO + 16384;
  s.stg = s.du + np * 16384;
  s.stg_bytes = 8192 + np * 4096;           // K_h 4 KB | V_h 4 KB | Z2 np x 4 KB (32 keys)
  s.aux = s.stg + ns * s.stg_bytes;
  s.total = s.aux + 2048;
  return s;
}
// aux area: col terms [MAX_NS][32] floats (384 B, from 0) | tile info [MAX_NS][2] float4 (96 B) | barriers
constexpr uint32_t QA_COL = 0, QA_INFO = 768, QA_BAR = 896;
enum { QB_QFULL = 0, QB_QTM, QB_SFULL, QB_SFREE, QB_DSFULL, QB_DSFREE, QB_DRAIN, QB_FULL0, QB_EMPTY0 = QB_FULL0 + MAX_NS,
       QB_COUNT = QB_EMPTY0 + MAX_NS };
constexpr uint32_t QA_TMEM = QA_BAR + 8 * QB_COUNT, QA_ABORT = QA_TMEM + 8;

__device__ __forceinline__ void bwd_q_body(const int blk, const CUtensorMap& tm_qh, const CUtensorMap& tm_qp,
                                           const CUtensorMap& tm_do, const CUtensorMap& tm_du,
                                           const CUtensorMap& tm_kh, const CUtensorMap& tm_vh,
                                           const CUtensorMap& tm_z2, const BwdArgs& a) {
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  const uint32_t sb = (raw_u32 + 1023u) & ~1023u;
  unsigned char* smem = smem_raw + (sb - raw_u32);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int I = blk % a.nqt;
  const int bh = blk / a.nqt;
  const int b = bh / a.H, h = bh % a.H;
  const int L = a.L, nt = (a.L + BT - 1) / BT, DZ = a.DZ, np = DZ / 64, NS = a.ns;   // nt 32-key tiles
  const int nreg = NS - a.qp_stage;   // stages in the stage area; stage nreg (if any) in the Q_pair area
  const QLayout lay = q_layout(DZ, nreg);
  auto stage_at = [&](int s) -> uint32_t { return s < nreg ? sb + lay.stg + s * lay.stg_bytes : sb + lay.qp; };
  float* col_s = reinterpret_cast<float*>(smem + lay.aux + QA_COL);
  float4* info = reinterpret_cast<float4*>(smem + lay.aux + QA_INFO);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + lay.aux + QA_ABORT);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + lay.aux + QA_TMEM);
  auto bar = [&](int k) -> uint32_t { return sb + lay.aux + QA_BAR + 8u * k; };

  if (tid == 0) {
    mbar_init(bar(QB_QFULL), 1);
    mbar_init(bar(QB_QTM), NSOFT);
    mbar_init(bar(QB_SFULL), 1);
    mbar_init(bar(QB_SFREE), NSOFT);
    mbar_init(bar(QB_DSFULL), NSOFT);
    mbar_init(bar(QB_DSFREE), 1);
    mbar_init(bar(QB_DRAIN), 1);
    for (int s = 0; s < MAX_NS; ++s) {
      mbar_init(bar(QB_FULL0 + s), 2);   // the copy's expect-tx arrive and the column-term arrive
      mbar_init(bar(QB_EMPTY0 + s), 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == W_MMA) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
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
    const float4 oqv = a.oq[b * a.nqt + I];
    if (lane == 0) {
      mbar_arrive_expect_tx(bar(QB_QFULL), 2u * 16384u * static_cast<uint32_t>(1 + np));
      tma_load_3d(sb + lay.qh, &tm_qh, bar(QB_QFULL), 0, I * QT, bh);
      tma_load_4d(sb + lay.qp, &tm_qp, bar(QB_QFULL), 0, I * QT, 0, bh);
      tma_load_3d(sb + lay.dO, &tm_do, bar(QB_QFULL), 0, I * QT, bh);
      tma_load_4d(sb + lay.du, &tm_du, bar(QB_QFULL), 0, I * QT, 0, bh);
    }
    // A stage's copy is issued as soon as the stage is free.  The global
    // values its column terms need (the key tile's origin, the keys' column
    // terms) are loaded one tile ahead; FULL completes on the copy and on a
    // second arrive after the terms are in shared memory.
    int issued = 0;
    auto fetch = [&](int j, float4& okv, float4& ck) {
      okv = a.ok[b * a.nkt + j * BT / KT];   // the 64-key origin tile holding these keys
      const int key = j * BT + lane;
      ck = key < L ? a.colk[static_cast<int64_t>(bh) * L + key] : make_float4(0.f, 0.f, 0.f, 0.f);
    };
    float4 ok_next, ck_next;
    fetch(0, ok_next, ck_next);
    for (int j = 0; j < nt; ++j) {
      const int s = j % NS;
      if (j >= NS) {
        int ok = 1;
        if (lane == 0) ok = mbar_wait_bounded(bar(QB_EMPTY0 + s), ((j / NS) - 1) & 1, abort_flag);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (lane == 0) BWD_TR(0, j, 10);   // stage free
        if (!ok) {
          if (lane == 0) fail(DEV_TIMEOUT_EMPTY);
          break;
        }
      }
      issued = j + 1;
      if (lane == 0) {
        // the Q_pair-area stage is first filled once every thread has copied
        // its Q_pair row into tensor memory
        if (s == nreg && j == nreg && !mbar_wait_bounded(bar(QB_QTM), 0, abort_flag)) {
          fail(DEV_TIMEOUT_EMPTY);
          issued = j;
        }
      }
      issued = __shfl_sync(0xffffffffu, issued, 0);
      if (issued == j) break;
      if (lane == 0) {
        const uint32_t st = stage_at(s);
        mbar_arrive_expect_tx(bar(QB_FULL0 + s), lay.stg_bytes);
        tma_load_3d(st, &tm_kh, bar(QB_FULL0 + s), 0, j * BT, bh);
        tma_load_3d(st + 4096, &tm_vh, bar(QB_FULL0 + s), 0, j * BT, bh);
        tma_load_4d(st + 8192, &tm_z2, bar(QB_FULL0 + s), 0, j * BT, 0, b);
        BWD_TR(0, j, 11);                  // copy issued
      }
      const float4 okv = ok_next, ck = ck_next;
      if (j + 1 < nt) fetch(j + 1, ok_next, ck_next);
      const float dx = okv.x - oqv.x, dy = okv.y - oqv.y, dz = okv.z - oqv.z;
      col_s[s * BT + lane] = j * BT + lane < L ? ck.w - fmaf(ck.x, dx, fmaf(ck.y, dy, ck.z * dz)) : -INFINITY;
      if (lane == 0) {
        info[2 * s] = make_float4(dx, dy, dz, fmaf(dx, dx, fmaf(dy, dy, dz * dz)));
        info[2 * s + 1] = okv;
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(bar(QB_FULL0 + s));
        BWD_TR(0, j, 12);                  // column terms in
      }
    }
    if (lane == 0 && *abort_flag) {
      // copies still in flight must land before the CTA exits
      mbar_wait_bounded(bar(QB_QFULL), 0, nullptr, 100000000ull);
      for (int j = (issued > NS ? issued - NS : 0); j < issued; ++j)
        mbar_wait_bounded(bar(QB_FULL0 + j % NS), (j / NS) & 1, nullptr, 100000000ull);
    }
  } else if (warp == W_MMA) {
    if (lane == 0) {
      bool ok = mbar_wait_bounded(bar(QB_QFULL), 0, abort_flag) && mbar_wait_bounded(bar(QB_QTM), 0, abort_flag);
      if (!ok) fail(DEV_TIMEOUT_FULL);
      tc_fence_after();
      const uint32_t id32 = idesc_f16(128, BT, false);
      const uint32_t id64mn = idesc_f16(128, 64, true);
      const uint32_t idz = idesc_f16(128, DZ, true);
      const int ntm = 4 * np < 2 * QPT_COLS / 16 ? 4 * np : 2 * QPT_COLS / 16;   // S pair K-steps with A in TMEM
      const uint32_t tS = tmem + Q_TM_S, tDP = tmem + Q_TM_DP, tDS = tmem + Q_TM_DS;
      const uint32_t tDQH = tmem + Q_TM_DQH, tDQP = tmem + Q_TM_DQP;
      bool issued_any = false;
      auto issue_sdp = [&](int j) -> bool {
        const int s = j % NS;
        bool w = mbar_wait_bounded(bar(QB_FULL0 + s), (j / NS) & 1, abort_flag);
        BWD_TR(0, j, 0);                   // stage j landed
        if (w && j > 0) w = mbar_wait_bounded(bar(QB_SFREE), (j - 1) & 1, abort_flag);
        BWD_TR(0, j, 1);                   // S(j-1), dP(j-1) read
        if (!w) { fail(DEV_TIMEOUT_FULL); return false; }
        tc_fence_after();
        const uint32_t st = stage_at(s);
#pragma unroll
        for (int k = 0; k < 4; ++k) umma_ss(tS, kd128(sb + lay.qh + 32 * k), kd128(st + 32 * k), id32, k > 0 ? 1u : 0u);
        for (int kk = 0; kk < ntm; ++kk)
          umma_ts(tS, tmem + Q_TM_QPT + 8 * kk, kd128(st + 8192 + 4096 * (kk >> 2) + 32 * (kk & 3)), id32, 1u);
        for (int kk = ntm; kk < 4 * np; ++kk)
          umma_ss(tS, kd128(sb + lay.qp + 16384 * (kk >> 2) + 32 * (kk & 3)),
                  kd128(st + 8192 + 4096 * (kk >> 2) + 32 * (kk & 3)), id32, 1u);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          umma_ss(tDP, kd128(sb + lay.dO + 32 * k), kd128(st + 4096 + 32 * k), id32, k > 0 ? 1u : 0u);
        for (int kk = 0; kk < 4 * np; ++kk)
          umma_ss(tDP, kd128(sb + lay.du + 16384 * (kk >> 2) + 32 * (kk & 3)),
                  kd128(st + 8192 + 4096 * (kk >> 2) + 32 * (kk & 3)), id32, 1u);
        umma_commit(bar(QB_SFULL));
        BWD_TR(0, j, 2);                   // S(j), dP(j) issued
        issued_any = true;
        return true;
      };
      auto issue_dq = [&](int jj) -> bool {
        if (!mbar_wait_bounded(bar(QB_DSFULL), jj & 1, abort_flag)) { fail(DEV_TIMEOUT_SOFTMAX); return false; }
        BWD_TR(0, jj, 3);                  // dS(jj) written
        tc_fence_after();
        const int s = jj % NS;
        const uint32_t st = stage_at(s);
#pragma unroll
        for (int k = 0; k < BT / 16; ++k) {
          const uint32_t acc = (jj > 0 || k > 0) ? 1u : 0u;
          umma_ts(tDQH, tDS + 8 * k, mnd(st + 2048 * k, 4096), id64mn, acc);
          umma_ts(tDQP, tDS + 8 * k, mnd(st + 8192 + 2048 * k, 4096), idz, acc);
        }
        umma_commit(bar(QB_DSFREE));
        umma_commit(bar(QB_EMPTY0 + s));
        BWD_TR(0, jj, 4);                  // dQ(jj) issued
        return true;
      };
      // Three stages (the third in the Q_pair area): S(j), dP(j) before
      // dQ(j-1), so the tensor pipe works on tile j while the threads finish
      // j - 1, and the copy of tile j + 2 has a whole tile to land.  Two
      // stages: dQ(j-1) first, since tile j + 1 reuses the stage dQ(j-1)
      // releases (S(j), dP(j) first left each copy exposed).
      for (int j = 0; ok && j <= nt; ++j) {
        if (NS >= 3) {
          if (j < nt) ok = issue_sdp(j);
          if (ok && j > 0) ok = issue_dq(j - 1);
        } else {
          if (j > 0) ok = issue_dq(j - 1);
          if (ok && j < nt) ok = issue_sdp(j);
        }
      }
      if (!ok && issued_any) {
        umma_commit(bar(QB_DRAIN));
        mbar_wait_bounded(bar(QB_DRAIN), 0, nullptr, 100000000ull);
      }
    }
    __syncwarp();
  } else {
    const int quarter = warp & 3, half = warp >> 2;
    const int r = quarter * 32 + lane;
    const int row = I * QT + r;
    const bool in_range = row < L;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const float ch = a.headc[h];
    const float4 sq = in_range ? a.rowq[static_cast<int64_t>(bh) * L + row] : make_float4(0.f, 0.f, 0.f, 0.f);
    const float2 rd = in_range ? a.rowd[static_cast<int64_t>(bh) * L + row] : make_float2(-INFINITY, 0.f);
    const float pq = static_cast<float>(IPA_PQ);
    float rs = 0.f, ro0 = 0.f, ro1 = 0.f, ro2 = 0.f;
    bool ok = true;
    // the first QPT_COLS columns of this row's Q_pair into tensor memory
    // (from the 128-byte swizzled panels TMA wrote: 16-byte chunk c of row r
    // at 16 (c ^ (r & 7))), half 0 the first half of them
    if (__all_sync(0xffffffffu, mbar_wait_bounded(bar(QB_QFULL), 0, abort_flag))) {
      const int nw = DZ / 2 < QPT_COLS ? DZ / 2 : QPT_COLS;   // words (fp16 pairs) in tensor memory
      for (int w0 = half * (QPT_COLS / 2); w0 < (half + 1) * (QPT_COLS / 2) && w0 < nw; w0 += 8) {
        const int pnl = w0 >> 5, c0 = (w0 & 31) >> 2;
        const unsigned char* rowp = smem + lay.qp + 16384u * pnl + r * 128;
        const uint4 u0 = *reinterpret_cast<const uint4*>(rowp + ((c0 ^ (r & 7)) << 4));
        const uint4 u1 = *reinterpret_cast<const uint4*>(rowp + (((c0 + 1) ^ (r & 7)) << 4));
        const uint32_t v[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
        tmem_st8(tmem + Q_TM_QPT + w0 + lane_off, v);
      }
      tmem_st_wait();
    } else {
      if (lane == 0) fail(DEV_TIMEOUT_FULL);
    }
    tc_fence_before();
    mbar_arrive(bar(QB_QTM));
    for (int j = 0; j < nt && ok; ++j) {
      const int s = j % NS;
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(bar(QB_SFULL), j & 1, abort_flag))) {
        if (lane == 0) fail(DEV_TIMEOUT_MMA);
        ok = false;
        break;
      }
      tc_fence_after();
      if (tid == 0) BWD_TR(0, j, 5);     // S(j), dP(j) complete
      uint32_t sv[16], dv[16];
      tmem_ld16(tmem + Q_TM_S + 16 * half + lane_off, sv);
      tmem_ld16(tmem + Q_TM_DP + 16 * half + lane_off, dv);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(bar(QB_SFREE));
      if (tid == 0) BWD_TR(0, j, 6);     // read
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(bar(QB_FULL0 + s), (j / NS) & 1, abort_flag))) {
        if (lane == 0) fail(DEV_TIMEOUT_FULL);
        ok = false;
        break;
      }
      if (tid == 0) BWD_TR(0, j, 7);     // column terms visible
      const float4 dd = info[2 * s], oj = info[2 * s + 1];
      const float rt = ch * (2.f * fmaf(sq.x, dd.x, fmaf(sq.y, dd.y, sq.z * dd.z)) - pq * dd.w);
      const float base = rt + rd.x;                        // row terms - (w + lse2); -inf on dead rows
      const float* cv = col_s + s * BT + 16 * half;
      uint32_t pk[8];
      float tsum = 0.f;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const float x0 = __uint_as_float(sv[2 * k]) + cv[2 * k] + base;
        const float x1 = __uint_as_float(sv[2 * k + 1]) + cv[2 * k + 1] + base;
        const float p0 = ex2(x0), p1 = ex2(x1);
        const float g0 = p0 * (__uint_as_float(dv[2 * k]) - rd.y) * kLn2;
        const float g1 = p1 * (__uint_as_float(dv[2 * k + 1]) - rd.y) * kLn2;
        pk[k] = pack_half2(g0, g1);
        tsum = add_half2_to_f32(pk[k], tsum);
      }
      rs += tsum;
      ro0 = fmaf(tsum, oj.x, ro0);
      ro1 = fmaf(tsum, oj.y, ro1);
      ro2 = fmaf(tsum, oj.z, ro2);
      // dQ(j-1) must have finished reading dS(j-1)
      if (j >= 1 && !__all_sync(0xffffffffu, mbar_wait_bounded(bar(QB_DSFREE), (j - 1) & 1, abort_flag))) {
        if (lane == 0) fail(DEV_TIMEOUT_MMA);
        ok = false;
        break;
      }
      if (tid == 0) BWD_TR(0, j, 8);     // dQ(j-1) done with dS
      tc_fence_after();
      tmem_st8(tmem + Q_TM_DS + 8 * half + lane_off, pk);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(QB_DSFULL));
      if (tid == 0) BWD_TR(0, j, 9);     // dS(j) written
    }
    if (ok && !__all_sync(0xffffffffu, mbar_wait_bounded(bar(QB_DSFREE), (nt - 1) & 1, abort_flag))) {
      if (lane == 0) fail(DEV_TIMEOUT_MMA);
      ok = false;
    }
    const bool all_ok = __all_sync(0xffffffffu, ok);
    // row sums of the two halves
    // (the first stage's area is free: every MMA that read it has completed)
    named_bar_sync(1, NSOFT);
    if (half == 1) reinterpret_cast<float4*>(smem + lay.stg)[r] = make_float4(rs, ro0, ro1, ro2);
    named_bar_sync(1, NSOFT);
    if (all_ok && !*abort_flag) {
      tc_fence_after();
      if (half == 0 && in_range) {
        const float4 o = reinterpret_cast<const float4*>(smem + lay.stg)[r];
        *IPA_AT(a.rsq, static_cast<int64_t>(bh) * L + row, static_cast<int64_t>(a.B) * a.H * L, a.err) =
            make_float4(rs + o.x, ro0 + o.y, ro1 + o.z, ro2 + o.w);
      }
      // accumulators: dQ_h (64 columns, 32 per half) and dQ_pair (DZ, DZ / 2 per half)
      {
        uint32_t v[32];
        tmem_ld32(tmem + Q_TM_DQH + 32 * half + lane_off, v);
        tmem_ld_wait();
        if (in_range) {
          float4* dst = reinterpret_cast<float4*>(IPA_SPAN(a.dqh, (static_cast<int64_t>(bh) * L + row) * 64 + 32 * half,
                                                           32, static_cast<int64_t>(a.B) * a.H * L * 64, a.err));
#pragma unroll
          for (int e = 0; e < 8; ++e)
            dst[e] = make_float4(__uint_as_float(v[4 * e]), __uint_as_float(v[4 * e + 1]),
                                 __uint_as_float(v[4 * e + 2]), __uint_as_float(v[4 * e + 3]));
        }
      }
      for (int c0 = half * (DZ / 2); c0 < (half + 1) * (DZ / 2); c0 += 32) {
        uint32_t v[32];
        tmem_ld32(tmem + Q_TM_DQP + c0 + lane_off, v);
        tmem_ld_wait();
        if (in_range) {
          float4* dst = reinterpret_cast<float4*>(IPA_SPAN(a.dqp, (static_cast<int64_t>(bh) * L + row) * DZ + c0, 32,
                                                           static_cast<int64_t>(a.B) * a.H * L * DZ, a.err));
#pragma unroll
          for (int e = 0; e < 8; ++e)
            dst[e] = make_float4(__uint_as_float(v[4 * e]), __uint_as_float(v[4 * e + 1]),
                                 __uint_as_float(v[4 * e + 2]), __uint_as_float(v[4 * e + 3]));
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == W_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ----------------------------------------------------------------- key pass
// Warps 0-7: two threads per key row (queries [16 half, 16 half + 16) of a
// 32-query tile); warp 8: TMA producer and the per-query terms; warp 9: MMA.
// S^T and dP^T are double-buffered (buffer i & 1, 32 columns each), so that
// the MMAs of tile i + 1 run while the threads work on tile i.
// S^T / dP^T buffer t: S^T at K_TM_SD + 64 t, dP^T right after it (one N = 64
// accumulator for their pair parts)
constexpr uint32_t K_TM_DZ2 = 0, K_TM_DKH = 256, K_TM_DVA = 320, K_TM_SD = 384;
constexpr int MAX_KSPLIT = 5;   // query chunks of a split key tile

struct KLayout {
  uint32_t kh, vh, z2, stg, stg_bytes, aux, total;
};
__host__ __device__ inline KLayout k_layout(int DZ, int ns) {
  KLayout s{};
  const uint32_t np = DZ / 64;
  s.kh = 0;
  s.vh = 16384;
  s.z2 = 32768;
  s.stg = s.z2 + np * 16384;
  // Q_h 4 KB | dO 4 KB | np x (Q_pair panel 4 KB | dU panel 4 KB) (32 queries): each
  // Q_pair panel with its dU panel is one 64-row K-major B operand
  s.stg_bytes = 8192 + 2 * np * 4096;
  s.aux = s.stg + ns * s.stg_bytes;
  s.total = s.aux + 6656;
  return s;
}
// aux: per-query terms [MAX_NS][32] float4 (1.5 KB) | stage query-tile origin [MAX_NS] float4 | barriers |
// tensor-memory slot, abort flag, pair flags | per-stage query points [MAX_NS][32][12] floats (4.5 KB, from 2048)
constexpr uint32_t KA_Q = 0, KA_OQ = 1536, KA_BAR = 1600, KA_QPTS = 2048;
enum { KB_KFULL = 0, KB_SFULL0, KB_PFULL0 = KB_SFULL0 + 2, KB_ACC0 = KB_PFULL0 + 2, KB_DRAIN = KB_ACC0 + 2,
       KB_FULL0, KB_EMPTY0 = KB_FULL0 + MAX_NS, KB_COUNT = KB_EMPTY0 + MAX_NS };
constexpr uint32_t KA_TMEM = KA_BAR + 8 * KB_COUNT, KA_ABORT = KA_TMEM + 8, KA_PAIR = KA_ABORT + 8;
constexpr uint32_t KA_LAST = KA_PAIR + 64;   // int: this CTA finishes its split key tile
static_assert(KA_LAST + 4 <= KA_QPTS, "key-pass aux area overlaps the query points");

__device__ __forceinline__ void bwd_k_body(const int blk, const CUtensorMap& tm_kh, const CUtensorMap& tm_vh,
                                           const CUtensorMap& tm_z2, const CUtensorMap& tm_qh,
                                           const CUtensorMap& tm_do, const CUtensorMap& tm_qp,
                                           const CUtensorMap& tm_du, const BwdArgs& a) {
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  const uint32_t sb = (raw_u32 + 1023u) & ~1023u;
  unsigned char* smem = smem_raw + (sb - raw_u32);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nkp = (a.L + 127) / 128;
  // a split key tile's chunk c covers query tiles [c nqa / S, (c + 1) nqa / S)
  const int nqa = (a.L + BT - 1) / BT;          // 32-query tiles in all
  int tile = blk, chunk = -1, ib = 0, nq = nqa;  // nq: query tiles this CTA runs, from ib
  if (blk >= a.split_first) {
    const int q = blk - a.split_first;
    tile = a.split_first + q / a.split_s;
    chunk = q % a.split_s;
    ib = chunk * nqa / a.split_s;
    nq = (chunk + 1) * nqa / a.split_s - ib;
  }
  const int J2 = tile % nkp;                    // 128-key tile
  const int bh = tile / nkp;
  const int b = bh / a.H, h = bh % a.H;
  const int L = a.L, DZ = a.DZ, np = DZ / 64, NS = a.ns;
  const KLayout lay = k_layout(DZ, NS);
  float4* qinfo = reinterpret_cast<float4*>(smem + lay.aux + KA_Q);
  float4* oqs = reinterpret_cast<float4*>(smem + lay.aux + KA_OQ);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + lay.aux + KA_ABORT);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + lay.aux + KA_TMEM);
  auto bar = [&](int k) -> uint32_t { return sb + lay.aux + KA_BAR + 8u * k; };

  if (tid == 0) {
    mbar_init(bar(KB_KFULL), 1);
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(KB_SFULL0 + t), 1);
      mbar_init(bar(KB_PFULL0 + t), NSOFT);
      mbar_init(bar(KB_ACC0 + t), 1);
    }
    mbar_init(bar(KB_DRAIN), 1);
    for (int s = 0; s < MAX_NS; ++s) {
      mbar_init(bar(KB_FULL0 + s), 2);   // the copy's expect-tx arrive and the row-term arrive
      mbar_init(bar(KB_EMPTY0 + s), 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == W_MMA) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
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
    if (lane == 0) {
      mbar_arrive_expect_tx(bar(KB_KFULL), 2u * 16384u + static_cast<uint32_t>(np) * 16384u);
      tma_load_3d(sb + lay.kh, &tm_kh, bar(KB_KFULL), 0, J2 * 128, bh);
      tma_load_3d(sb + lay.vh, &tm_vh, bar(KB_KFULL), 0, J2 * 128, bh);
      tma_load_4d(sb + lay.z2, &tm_z2, bar(KB_KFULL), 0, J2 * 128, 0, b);
    }
    const float ch = a.headc[h];
    const float pq = static_cast<float>(IPA_PQ);
    const int js0 = 2 * J2, js1 = 2 * J2 + 1;   // the two 64-key origin tiles of this CTA
    const float4 ok0 = a.ok[b * a.nkt + js0];
    const float4 ok1 = js1 < a.nkt ? a.ok[b * a.nkt + js1] : ok0;
    // As in the query pass: each stage's copy goes out as soon as the stage
    // is free, the global row values of a tile (its query-tile origin, row
    // terms and the 32 query points, 12 floats = 3 float4 per query) are
    // loaded one tile ahead, and FULL completes on the copy and on a second
    // arrive after they are in shared memory.
    int issued = 0;
    struct RowVals {
      float4 oqv, sq, v[3];
      float2 rd;
    };
    auto fetch = [&](int il, RowVals& r) {
      const int i = ib + il;                    // global 32-query tile
      r.oqv = a.oq[b * a.nqt + (i * BT) / QT];
      const int qi = i * BT + lane;
      r.sq = qi < L ? a.rowq[static_cast<int64_t>(bh) * L + qi] : make_float4(0.f, 0.f, 0.f, 0.f);
      r.rd = qi < L ? a.rowd[static_cast<int64_t>(bh) * L + qi] : make_float2(0.f, 0.f);
      const float4* src = reinterpret_cast<const float4*>(a.pts) + (static_cast<int64_t>(bh) * L + i * BT) * 6;
#pragma unroll
      for (int u = 0; u < 3; ++u) {
        const int f = lane + 32 * u, row = f / 3;
        r.v[u] = i * BT + row < L ? src[row * 6 + f % 3] : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    };
    RowVals nxt;
    fetch(0, nxt);
    for (int i = 0; i < nq; ++i) {
      const int s = i % NS;
      if (i >= NS) {
        int ok = 1;
        if (lane == 0) ok = mbar_wait_bounded(bar(KB_EMPTY0 + s), ((i / NS) - 1) & 1, abort_flag);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (lane == 0) BWD_TR(1, i, 10);
        if (!ok) {
          if (lane == 0) fail(DEV_TIMEOUT_EMPTY);
          break;
        }
      }
      issued = i + 1;
      if (lane == 0) {
        const uint32_t st = sb + lay.stg + s * lay.stg_bytes;
        mbar_arrive_expect_tx(bar(KB_FULL0 + s), lay.stg_bytes);
        const int q0 = (ib + i) * BT;
        tma_load_3d(st, &tm_qh, bar(KB_FULL0 + s), 0, q0, bh);
        tma_load_3d(st + 4096, &tm_do, bar(KB_FULL0 + s), 0, q0, bh);
        for (int p = 0; p < np; ++p) {   // interleaved panels: Q_pair p, then dU p
          tma_load_4d(st + 8192 + 8192 * p, &tm_qp, bar(KB_FULL0 + s), 0, q0, p, bh);
          tma_load_4d(st + 8192 + 8192 * p + 4096, &tm_du, bar(KB_FULL0 + s), 0, q0, p, bh);
        }
        BWD_TR(1, i, 11);
      }
      const RowVals cur = nxt;
      if (i + 1 < nq) fetch(i + 1, nxt);
      const float4 oqv = cur.oqv;
      const float d0x = ok0.x - oqv.x, d0y = ok0.y - oqv.y, d0z = ok0.z - oqv.z;
      const float d1x = ok1.x - oqv.x, d1y = ok1.y - oqv.y, d1z = ok1.z - oqv.z;
      const float n0 = fmaf(d0x, d0x, fmaf(d0y, d0y, d0z * d0z)), n1 = fmaf(d1x, d1x, fmaf(d1y, d1y, d1z * d1z));
      {
        float4 e = make_float4(-INFINITY, -INFINITY, 0.f, 0.f);
        if ((ib + i) * BT + lane < L) {
          const float4 sq = cur.sq;
          const float rt0 = ch * (2.f * fmaf(sq.x, d0x, fmaf(sq.y, d0y, sq.z * d0z)) - pq * n0);
          const float rt1 = ch * (2.f * fmaf(sq.x, d1x, fmaf(sq.y, d1y, sq.z * d1z)) - pq * n1);
          e = make_float4(rt0 + cur.rd.x, rt1 + cur.rd.x, cur.rd.y, 0.f);
        }
        qinfo[s * BT + lane] = e;
      }
      if (lane == 0) oqs[s] = oqv;
      float4* qp = reinterpret_cast<float4*>(smem + lay.aux + KA_QPTS) + s * BT * 3;
#pragma unroll
      for (int u = 0; u < 3; ++u) qp[lane + 32 * u] = cur.v[u];
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(bar(KB_FULL0 + s));
        BWD_TR(1, i, 12);
      }
    }
    if (lane == 0 && *abort_flag) {
      mbar_wait_bounded(bar(KB_KFULL), 0, nullptr, 100000000ull);
      for (int i = (issued > NS ? issued - NS : 0); i < issued; ++i)
        mbar_wait_bounded(bar(KB_FULL0 + i % NS), (i / NS) & 1, nullptr, 100000000ull);
    }
  } else if (warp == W_MMA) {
    if (lane == 0) {
      bool ok = mbar_wait_bounded(bar(KB_KFULL), 0, abort_flag);
      if (!ok) fail(DEV_TIMEOUT_FULL);
      tc_fence_after();
      const uint32_t id32 = idesc_f16(128, BT, false);
      const uint32_t id64mn = idesc_f16(128, 64, true);
      const uint32_t id64 = idesc_f16(128, 2 * BT, false);   // [Q_pair ; dU] rows of a stage
      const uint32_t idz = idesc_f16(128, DZ, true);
      bool issued_any = false;
      // S^T(i), dP^T(i) into buffer i & 1, once stage i has landed and the
      // accumulation MMAs of tile i - 2 (which read P^T / dS^T in place from
      // that buffer) have completed
      auto issue_sdp = [&](int i) -> bool {
        const int s = i % NS, t = i & 1;
        bool w = mbar_wait_bounded(bar(KB_FULL0 + s), (i / NS) & 1, abort_flag);
        BWD_TR(1, i, 0);
        if (w && i >= 2) w = mbar_wait_bounded(bar(KB_ACC0 + t), ((i - 2) >> 1) & 1, abort_flag);
        BWD_TR(1, i, 1);
        if (!w) { fail(DEV_TIMEOUT_FULL); return false; }
        tc_fence_after();
        const uint32_t st = sb + lay.stg + s * lay.stg_bytes;
        const uint32_t sQh = st, sDO = st + 4096, sPair = st + 8192;
        const uint32_t tS = tmem + K_TM_SD + 64 * t, tDP = tS + 32;
        // the pair parts of S^T and dP^T share their A operand (Z2): one
        // N = 64 MMA per K-step against [Q_pair ; dU], into [S^T | dP^T]
        for (int kk = 0; kk < 4 * np; ++kk)
          umma_ss(tS, kd128(sb + lay.z2 + 16384 * (kk >> 2) + 32 * (kk & 3)),
                  kd128(sPair + 8192 * (kk >> 2) + 32 * (kk & 3)), id64, kk > 0 ? 1u : 0u);
#pragma unroll
        for (int k = 0; k < 4; ++k) umma_ss(tS, kd128(sb + lay.kh + 32 * k), kd128(sQh + 32 * k), id32, 1u);
#pragma unroll
        for (int k = 0; k < 4; ++k) umma_ss(tDP, kd128(sb + lay.vh + 32 * k), kd128(sDO + 32 * k), id32, 1u);
        umma_commit(bar(KB_SFULL0 + t));
        BWD_TR(1, i, 2);
        issued_any = true;
        return true;
      };
      // dV += P^T dO, dZ2 += P^T dU + dS^T Q_pair, dK_h += dS^T Q_h for tile
      // i, once its threads have written P^T / dS^T (fp16, in place)
      auto issue_acc = [&](int i) -> bool {
        const int s = i % NS, t = i & 1;
        if (!mbar_wait_bounded(bar(KB_PFULL0 + t), (i >> 1) & 1, abort_flag)) { fail(DEV_TIMEOUT_SOFTMAX); return false; }
        BWD_TR(1, i, 3);
        tc_fence_after();
        const uint32_t st = sb + lay.stg + s * lay.stg_bytes;
        const uint32_t sQh = st, sDO = st + 4096, sQP = st + 8192, sDU = st + 8192 + 4096;   // panels 8 KB apart
        const uint32_t tS = tmem + K_TM_SD + 64 * t, tDP = tS + 32;
#pragma unroll
        for (int k = 0; k < BT / 16; ++k) {
          const uint32_t acc = (i > 0 || k > 0) ? 1u : 0u;
          umma_ts(tmem + K_TM_DVA, tS + 8 * k, mnd(sDO + 2048 * k, 4096), id64mn, acc);
          umma_ts(tmem + K_TM_DZ2, tS + 8 * k, mnd(sDU + 2048 * k, 8192), idz, acc);
          umma_ts(tmem + K_TM_DZ2, tDP + 8 * k, mnd(sQP + 2048 * k, 8192), idz, 1u);
          umma_ts(tmem + K_TM_DKH, tDP + 8 * k, mnd(sQh + 2048 * k, 4096), id64mn, acc);
        }
        umma_commit(bar(KB_ACC0 + t));
        umma_commit(bar(KB_EMPTY0 + s));
        BWD_TR(1, i, 4);
        return true;
      };
      // with two or more stages S^T / dP^T(i) are issued before the
      // accumulation of tile i - 1; with one, tile i cannot load until that
      // accumulation has released the stage
      for (int i = 0; ok && i <= nq; ++i) {
        if (NS == 1) {
          if (i > 0) ok = issue_acc(i - 1);
          if (ok && i < nq) ok = issue_sdp(i);
        } else {
          if (i < nq) ok = issue_sdp(i);
          if (ok && i > 0) ok = issue_acc(i - 1);
        }
      }
      if (!ok && issued_any) {
        umma_commit(bar(KB_DRAIN));
        mbar_wait_bounded(bar(KB_DRAIN), 0, nullptr, 100000000ull);
      }
    }
    __syncwarp();
  } else {
    const int quarter = warp & 3, half = warp >> 2;
    const int r = quarter * 32 + lane;
    const int key = J2 * 128 + r;
    const bool in_range = key < L;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t pair_bar = 2 + quarter;
    volatile int* pair_ok = reinterpret_cast<volatile int*>(smem + lay.aux + KA_PAIR);   // [2 parities][4][2]
    const float4 ck = in_range ? a.colk[static_cast<int64_t>(bh) * L + key] : make_float4(0.f, 0.f, 0.f, -INFINITY);
    const int sub = r >> 6;                      // which 64-key origin tile
    const float4 okj = a.ok[b * a.nkt + (in_range ? key / 64 : 0)];
    float2 kc[6];                                // this key's points relative to the centroid, in pairs
    {
      const float4* kp = reinterpret_cast<const float4*>(a.pts + (static_cast<int64_t>(bh) * L + (in_range ? key : 0)) * 24 + 12);
#pragma unroll
      for (int u = 0; u < 3; ++u) {
        const float4 w = in_range ? kp[u] : make_float4(0.f, 0.f, 0.f, 0.f);
        kc[2 * u] = make_float2(w.x, w.y);
        kc[2 * u + 1] = make_float2(w.z, w.w);
      }
    }
    float cs = 0.f, co0 = 0.f, co1 = 0.f, co2 = 0.f, gsum = 0.f;
    bool ok = true;
    for (int i = 0; i < nq && ok; ++i) {
      const int s = i % NS;
      // the two warps of these lanes decide together whether to go on, so
      // that neither waits at their shared barrier for one that has left
      const int tb = i & 1;                   // tensor-memory buffer of this tile
      const bool got = __all_sync(0xffffffffu, mbar_wait_bounded(bar(KB_SFULL0 + tb), (i >> 1) & 1, abort_flag));
      if (tid == 0) BWD_TR(1, i, 5);
      uint32_t sv[16], dv[16];
      if (got) {
        tc_fence_after();
        tmem_ld16(tmem + K_TM_SD + 64 * tb + 16 * half + lane_off, sv);
        tmem_ld16(tmem + K_TM_SD + 64 * tb + 32 + 16 * half + lane_off, dv);
        tmem_ld_wait();
        tc_fence_before();
      }
      if (tid == 0) BWD_TR(1, i, 6);
      if (lane == 0) pair_ok[(i & 1) * 8 + quarter * 2 + half] = got ? 1 : 0;
      named_bar_sync(pair_bar, 64);           // both halves have read before either overwrites
      if (!(pair_ok[(i & 1) * 8 + quarter * 2] && pair_ok[(i & 1) * 8 + quarter * 2 + 1])) {
        if (lane == 0) fail(DEV_TIMEOUT_MMA);
        ok = false;
        break;
      }
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(bar(KB_FULL0 + s), (i / NS) & 1, abort_flag))) {
        if (lane == 0) fail(DEV_TIMEOUT_FULL);
        ok = false;
        break;
      }
      if (tid == 0) BWD_TR(1, i, 7);
      const float4 oqv = oqs[s];
      const float colv = ck.w - fmaf(ck.x, okj.x - oqv.x, fmaf(ck.y, okj.y - oqv.y, ck.z * (okj.z - oqv.z)));
      const float4* qi = qinfo + s * BT + 16 * half;
      // this half's 16 query points relative to the centroid, 12 floats each
      const float4* qc = reinterpret_cast<const float4*>(smem + lay.aux + KA_QPTS) + (s * BT + 16 * half) * 3;
      // |gq_i - gk_j|^2, two coordinates per packed instruction
      auto dist2 = [&](const int k) {
        const float4 g0 = qc[3 * k], g1 = qc[3 * k + 1], g2 = qc[3 * k + 2];
        const float2 d0 = sub_f32x2(make_float2(g0.x, g0.y), kc[0]), d1 = sub_f32x2(make_float2(g0.z, g0.w), kc[1]);
        const float2 d2 = sub_f32x2(make_float2(g1.x, g1.y), kc[2]), d3 = sub_f32x2(make_float2(g1.z, g1.w), kc[3]);
        const float2 d4 = sub_f32x2(make_float2(g2.x, g2.y), kc[4]), d5 = sub_f32x2(make_float2(g2.z, g2.w), kc[5]);
        float2 acc = mul_f32x2(d0, d0);
        acc = fma_f32x2(d1, d1, acc);
        acc = fma_f32x2(d2, d2, acc);
        acc = fma_f32x2(d3, d3, acc);
        acc = fma_f32x2(d4, d4, acc);
        acc = fma_f32x2(d5, d5, acc);
        return acc.x + acc.y;
      };
      uint32_t pp[8], pd[8];
      float tsum = 0.f;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const float4 e0 = qi[2 * k], e1 = qi[2 * k + 1];
        const float x0 = __uint_as_float(sv[2 * k]) + colv + (sub ? e0.y : e0.x);
        const float x1 = __uint_as_float(sv[2 * k + 1]) + colv + (sub ? e1.y : e1.x);
        const float p0 = ex2(x0), p1 = ex2(x1);
        pp[k] = pack_half2(p0, p1);
        const float ds0 = p0 * (__uint_as_float(dv[2 * k]) - e0.z) * kLn2;
        const float ds1 = p1 * (__uint_as_float(dv[2 * k + 1]) - e1.z) * kLn2;
        pd[k] = pack_half2(ds0, ds1);
        tsum = add_half2_to_f32(pd[k], tsum);
        // d gamma: sum_i dS_ij |gq_i - gk_j|^2 (dS before its fp16 rounding)
        gsum = fmaf(ds0, dist2(2 * k), gsum);
        gsum = fmaf(ds1, dist2(2 * k + 1), gsum);
      }
      cs += tsum;
      co0 = fmaf(tsum, oqv.x, co0);
      co1 = fmaf(tsum, oqv.y, co1);
      co2 = fmaf(tsum, oqv.z, co2);
      if (tid == 0) BWD_TR(1, i, 8);
      tc_fence_after();
      tmem_st8(tmem + K_TM_SD + 64 * tb + 8 * half + lane_off, pp);
      tmem_st8(tmem + K_TM_SD + 64 * tb + 32 + 8 * half + lane_off, pd);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(KB_PFULL0 + tb));
      if (tid == 0) BWD_TR(1, i, 9);
    }
    // the commit after the last accumulation tracks every earlier MMA of the issuing thread
    if (ok && !__all_sync(0xffffffffu, mbar_wait_bounded(bar(KB_ACC0 + ((nq - 1) & 1)), ((nq - 1) >> 1) & 1, abort_flag))) {
      if (lane == 0) fail(DEV_TIMEOUT_MMA);
      ok = false;
    }
    const bool all_ok = __all_sync(0xffffffffu, ok);
    // query split: each chunk stores its accumulators (partial column pc:
    // dZ2 [0, DZ) | dK_h [DZ, DZ + 64) | dV [DZ + 64, DZ + 128), as float4
    // groups of columns, [(DZ + 128) / 4][128 rows][4]) and its five half
    // sums ([2 halves][5][128]); the chunk that takes the last ticket adds the
    // chunks in chunk order (its own from tensor memory and registers), so
    // the result does not depend on which chunk that is, and writes the rows
    // as a whole tile does.  No CTA waits for another.
    bool epi = true;
    if (chunk >= 0) {
      constexpr int NSUM = 5;
      const int OWK = DZ + 128;
      const int64_t qc = blk - a.split_first;   // (split tile) S + chunk
      const int64_t blk_floats = static_cast<int64_t>(OWK + 2 * NSUM) * 128;
      const int64_t mine = qc * blk_floats;
      auto tcol = [&](int pc) -> uint32_t {
        return pc < DZ ? K_TM_DZ2 + pc : pc < DZ + 64 ? K_TM_DKH + (pc - DZ) : K_TM_DVA + (pc - DZ - 64);
      };
      // this thread's 32-column groups: its half of dZ2, of dK_h and of dV
      const int ngrp = DZ / 64 + 2;
      auto grp = [&](int g) -> int { return g < DZ / 64 ? half * (DZ / 2) + 32 * g : DZ + 64 * (g - DZ / 64) + 32 * half; };
      float sums[NSUM] = {cs, co0, co1, co2, gsum};
      if (all_ok) {
        tc_fence_after();
        for (int g = 0; g < ngrp; ++g) {
          const int pc0 = grp(g);
          uint32_t v[32];
          tmem_ld32(tmem + tcol(pc0) + lane_off, v);
          tmem_ld_wait();
          float4* m4 = IPA_SPAN(reinterpret_cast<float4*>(a.part), mine / 4 + (pc0 / 4) * 128, 8 * 128,
                                a.part_extent / 4, a.err);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            m4[e * 128 + r] = make_float4(__uint_as_float(v[4 * e]), __uint_as_float(v[4 * e + 1]),
                                          __uint_as_float(v[4 * e + 2]), __uint_as_float(v[4 * e + 3]));
        }
#pragma unroll
        for (int k = 0; k < NSUM; ++k)
          *IPA_AT(a.part, mine + (OWK + half * NSUM + k) * 128 + r, a.part_extent, a.err) = sums[k];
      }
      // the barrier orders every thread's stores before thread 0's device-
      // scope fence and ticket; the merging CTA fences after its ticket
      named_bar_sync(1, NSOFT);
      volatile int* last = reinterpret_cast<volatile int*>(smem + lay.aux + KA_LAST);
      if (tid == 0) {
        int* tk = IPA_AT(a.ticket, qc / a.split_s, a.ticket_extent, a.err);
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
      if (epi && all_ok) {
        const float* c0p = a.part + (qc - chunk) * blk_floats;   // chunk 0 of this tile
        const int S = a.split_s;
#pragma unroll
        for (int k = 0; k < NSUM; ++k) {
          float acc = 0.f;
#pragma unroll
          for (int sc = 0; sc < MAX_KSPLIT; ++sc)
            if (sc < S) acc += sc == chunk ? sums[k] : __ldcg(c0p + sc * blk_floats + (OWK + half * NSUM + k) * 128 + r);
          sums[k] = acc;
        }
        cs = sums[0]; co0 = sums[1]; co1 = sums[2]; co2 = sums[3]; gsum = sums[4];
        tc_fence_after();
        for (int g = 0; g < ngrp; ++g) {
#pragma unroll
          for (int hsub = 0; hsub < 2; ++hsub) {   // 16 columns at a time, the other chunks' loads together
            const int pc0 = grp(g) + 16 * hsub;
            uint32_t o[16];
            tmem_ld16(tmem + tcol(pc0) + lane_off, o);
            float v[MAX_KSPLIT][16];
#pragma unroll
            for (int sc = 0; sc < MAX_KSPLIT; ++sc) {
              const float4* src = reinterpret_cast<const float4*>(c0p + sc * blk_floats) + (pc0 / 4) * 128 + r;
              const bool other = sc < S && sc != chunk;
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const float4 x = other ? __ldcg(src + q * 128) : make_float4(0.f, 0.f, 0.f, 0.f);
                v[sc][4 * q] = x.x; v[sc][4 * q + 1] = x.y; v[sc][4 * q + 2] = x.z; v[sc][4 * q + 3] = x.w;
              }
            }
            tmem_ld_wait();
            float acc[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) acc[e] = 0.f;
#pragma unroll
            for (int sc = 0; sc < MAX_KSPLIT; ++sc)
              if (sc < S) {
#pragma unroll
                for (int e = 0; e < 16; ++e) acc[e] += sc == chunk ? __uint_as_float(o[e]) : v[sc][e];
              }
#pragma unroll
            for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(acc[e]);
            tmem_st16(tmem + tcol(pc0) + lane_off, o);
          }
        }
        tmem_st_wait();
        tc_fence_before();
      }
    }
    if (epi) {
    named_bar_sync(1, NSOFT);   // every thread is past its last read of the stage area
    if (half == 1) {
      reinterpret_cast<float4*>(smem + lay.stg)[r] = make_float4(cs, co0, co1, co2);
      reinterpret_cast<float*>(smem + lay.stg + 2048)[r] = gsum;
    }
    named_bar_sync(1, NSOFT);
    if (all_ok && !*abort_flag) {
      tc_fence_after();
      if (half == 0 && in_range) {
        const float4 o = reinterpret_cast<const float4*>(smem + lay.stg)[r];
        const int64_t nbhl = static_cast<int64_t>(a.B) * a.H * L;
        *IPA_AT(a.csk, static_cast<int64_t>(bh) * L + key, nbhl, a.err) =
            make_float4(cs + o.x, co0 + o.y, co1 + o.z, co2 + o.w);
        *IPA_AT(a.gsum, static_cast<int64_t>(bh) * L + key, nbhl, a.err) =
            gsum + reinterpret_cast<const float*>(smem + lay.stg + 2048)[r];
      }
      auto store32 = [&](uint32_t tcol, float* dst_row) {
        uint32_t v[32];
        tmem_ld32(tmem + tcol + lane_off, v);
        tmem_ld_wait();
        if (in_range) {
          float4* dst = reinterpret_cast<float4*>(dst_row);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            dst[e] = make_float4(__uint_as_float(v[4 * e]), __uint_as_float(v[4 * e + 1]),
                                 __uint_as_float(v[4 * e + 2]), __uint_as_float(v[4 * e + 3]));
        }
      };
      const int64_t rowi = static_cast<int64_t>(bh) * L + (in_range ? key : 0);
      const int64_t nrow = static_cast<int64_t>(a.B) * a.H * L;
      store32(K_TM_DKH + 32 * half, IPA_SPAN(a.dkh, rowi * 64 + 32 * half, 32, nrow * 64, a.err));
      store32(K_TM_DVA + 32 * half, IPA_SPAN(a.dva, rowi * 64 + 32 * half, 32, nrow * 64, a.err));
      for (int c0 = half * (DZ / 2); c0 < (half + 1) * (DZ / 2); c0 += 32)
        store32(K_TM_DZ2 + c0, IPA_SPAN(a.dz2, rowi * DZ + c0, 32, nrow * DZ, a.err));
    }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == W_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Both passes in one grid: blocks [0, nqb) run the query pass, the rest the
// key pass.  Each pass alone is 2.6 waves of one CTA per SM; in one grid the
// key-pass CTAs fill the SMs the query pass leaves idle in its last wave.
struct BwdMaps {
  CUtensorMap q_qh, q_qp, q_do, q_du, q_kh, q_vh, q_z2;   // query pass
  CUtensorMap k_kh, k_vh, k_z2, k_qh, k_do, k_qp, k_du;   // key pass
};

// One CTA of NTH = 320 threads per SM (shared memory).  Registers are
// allocated to warps in groups of four, so the 10 warps count as 12 and the
// bound is 65536 / (12 x 32) -> 168 per thread.
__global__ void __launch_bounds__(NTH, 1)
    ipa_bwd_kernel(const __grid_constant__ BwdMaps m, const BwdArgs aq, const BwdArgs ak, const int nqb) {
  if (static_cast<int>(blockIdx.x) < nqb)
    bwd_q_body(blockIdx.x, m.q_qh, m.q_qp, m.q_do, m.q_du, m.q_kh, m.q_vh, m.q_z2, aq);
  else
    bwd_k_body(blockIdx.x - nqb, m.k_kh, m.k_vh, m.k_z2, m.k_qh, m.k_do, m.k_qp, m.k_du, ak);
}

// ------------------------------------------------------------------ mapping
struct MapArgs {
  int B, L, H, DZ, RCz, Cz, R, rb, nblk;
  float qscale, w_L, w_C;
  View q_pts, k_pts, v_pts, g_out, out, uagg;
  const float4* frame;
  const float4* cen;
  const float4* oq;
  const float4* ok;
  const float* headc;
  const float* wqp;
  const float* z1f;
  const float* dqh;
  const float* dqp;
  const float4* rsq;
  const float* dkh;
  const float* dva;
  const float* dz2;
  const float4* csk;
  const float* gsum;     // [B*H, L] sum_i dS_ij |gq_i - gk_j|^2 per key
  int nqt, nkt;
  // gradients (contiguous fp32)
  float *d_q, *d_k, *d_v, *d_qpts, *d_kpts, *d_vpts, *d_rot, *d_trans, *d_z1, *d_z2;
  float* wb_part;        // [B][pair-column blocks][H][DZ]
  double* g_part;        // [nblk * B][H]
  int* err;
};

// Block: rb residues of one batch, all heads.  Phase 1: thread (residue,
// head) -> scalar and point gradients, per-head frame contributions and
// d gamma terms; phase 2: frame gradients summed over heads in a fixed
// order, and the block's d gamma partial (the pair columns are
// ipa_bwd_pair_kernel's).
__global__ void __launch_bounds__(256) ipa_bwd_map_kernel(const MapArgs a) {
  extern __shared__ float sm_map[];   // [rb][H][12] frame terms, then [rb][H] d gamma (double)
  const int blk = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int H = a.H, rb = a.rb;
  const int i0 = blk * rb;
  float* fterm = sm_map;
  double* gterm = reinterpret_cast<double*>(sm_map + ((rb * H * 12 + 1) & ~1));
  const int C = IPA_C, PQ = IPA_PQ, PV = IPA_PV;
  const float4 cn = a.cen[b];
  if (tid < rb * H) {
    const int il = tid / H, h = tid % H;
    const int i = i0 + il;
    float fr[12];
#pragma unroll
    for (int e = 0; e < 12; ++e) fr[e] = 0.f;
    double gsum = 0.0;
    if (i < a.L) {
      const int64_t bi = static_cast<int64_t>(b) * a.L + i;
      const int64_t bhl = (static_cast<int64_t>(b) * H + h) * a.L + i;
      const float4* fp = a.frame + bi * 4;
      const float4 f0 = fp[0], f1 = fp[1], f2 = fp[2];
      const float Rm[9] = {f0.x, f0.y, f0.z, f0.w, f1.x, f1.y, f1.z, f1.w, f2.x};
      const float tc[3] = {f2.y - cn.x, f2.z - cn.y, f2.w - cn.z};
      const float c = a.headc[h];
      const float* dq = a.dqh + bhl * 64;
      const float* dk = a.dkh + bhl * 64;
      const float* dv = a.dva + bhl * 64;
      const float4 rq = a.rsq[bhl], ck = a.csk[bhl];
      const int64_t o3 = bi * H + h;
      const int64_t nblh = static_cast<int64_t>(a.B) * a.L * H;
      float* dqo = IPA_SPAN(a.d_q, o3 * C, C, nblh * C, a.err);
      float* dko = IPA_SPAN(a.d_k, o3 * C, C, nblh * C, a.err);
      float* dvo = IPA_SPAN(a.d_v, o3 * C, C, nblh * C, a.err);
      float* dqpo = IPA_SPAN(a.d_qpts, o3 * PQ * 3, PQ * 3, nblh * PQ * 3, a.err);
      float* dkpo = IPA_SPAN(a.d_kpts, o3 * PQ * 3, PQ * 3, nblh * PQ * 3, a.err);
      float* dvpo = IPA_SPAN(a.d_vpts, o3 * PV * 3, PV * 3, nblh * PV * 3, a.err);
      for (int e = 0; e < C; ++e) {
        dqo[e] = a.qscale * dq[e];
        dko[e] = dk[e];
        dvo[e] = dv[e];
      }
      // query and key points: d gq = Gq2c + 2c (RSo - rs gq_c), d gk = 2c (Gk' + CSo - cs gk_c)
      for (int p = 0; p < PQ; ++p) {
        float lq[3], lk[3], gqc[3], gkc[3], dgq[3], dgk[3];
        for (int y = 0; y < 3; ++y) {
          lq[y] = ldf(a.q_pts, b * a.q_pts.s[0] + i * a.q_pts.s[1] + h * a.q_pts.s[2] + p * a.q_pts.s[3] + y * a.q_pts.s[4]);
          lk[y] = ldf(a.k_pts, b * a.k_pts.s[0] + i * a.k_pts.s[1] + h * a.k_pts.s[2] + p * a.k_pts.s[3] + y * a.k_pts.s[4]);
        }
        for (int x = 0; x < 3; ++x) {
          gqc[x] = fmaf(Rm[3 * x], lq[0], fmaf(Rm[3 * x + 1], lq[1], Rm[3 * x + 2] * lq[2])) + tc[x];
          gkc[x] = fmaf(Rm[3 * x], lk[0], fmaf(Rm[3 * x + 1], lk[1], Rm[3 * x + 2] * lk[2])) + tc[x];
        }
        const float rso[3] = {rq.y, rq.z, rq.w}, cso[3] = {ck.y, ck.z, ck.w};
        for (int x = 0; x < 3; ++x) {
          const int e = C + 3 * p + x;
          const float gq2c = dq[e] + dq[e + 3 * PQ];                   // hi + lo key columns
          const float gk1 = dk[e] + dk[e + 6 * PQ];                    // query hi + lo columns
          dgq[x] = gq2c + 2.f * c * (rso[x] - rq.x * gqc[x]);
          dgk[x] = 2.f * c * (gk1 + cso[x] - ck.x * gkc[x]);
        }
        for (int y = 0; y < 3; ++y) {
          dqpo[p * 3 + y] = Rm[y] * dgq[0] + Rm[3 + y] * dgq[1] + Rm[6 + y] * dgq[2];
          dkpo[p * 3 + y] = Rm[y] * dgk[0] + Rm[3 + y] * dgk[1] + Rm[6 + y] * dgk[2];
        }
        for (int x = 0; x < 3; ++x) {
          for (int y = 0; y < 3; ++y) fr[3 * x + y] += dgq[x] * lq[y] + dgk[x] * lk[y];
          fr[9 + x] += dgq[x] + dgk[x];
        }
      }
      // d gamma: x_ij holds -(log2(e) w_L w_C / 2) gamma sum_p |gq_ip - gk_jp|^2
      gsum = -static_cast<double>(kLog2e) * a.w_L * a.w_C * 0.5 * static_cast<double>(a.gsum[bhl]);
      // value points
      for (int p = 0; p < PV; ++p) {
        float lv[3], dgv[3];
        for (int y = 0; y < 3; ++y)
          lv[y] = ldf(a.v_pts, b * a.v_pts.s[0] + i * a.v_pts.s[1] + h * a.v_pts.s[2] + p * a.v_pts.s[3] + y * a.v_pts.s[4]);
        for (int x = 0; x < 3; ++x) dgv[x] = dv[C + 3 * p + x];
        for (int y = 0; y < 3; ++y)
          dvpo[p * 3 + y] = Rm[y] * dgv[0] + Rm[3 + y] * dgv[1] + Rm[6 + y] * dgv[2];
        for (int x = 0; x < 3; ++x) {
          for (int y = 0; y < 3; ++y) fr[3 * x + y] += dgv[x] * lv[y];
          fr[9 + x] += dgv[x];
        }
      }
      // output side: o_pt = R^T (og - t): dR += (R o_pt) d_opt^T, dt -= R d_opt
      if (fp[3].x != 0.f) {
        const int64_t gb = b * a.g_out.s[0] + i * a.g_out.s[1] + h * a.g_out.s[2];
        const int64_t ob = b * a.out.s[0] + i * a.out.s[1] + h * a.out.s[2];
        for (int p = 0; p < PV; ++p) {
          float op[3], dopt[3];
          for (int y = 0; y < 3; ++y) op[y] = ldf(a.out, ob + (C + 3 * p + y) * a.out.s[3]);
          const float nrm = sqrtf(op[0] * op[0] + op[1] * op[1] + op[2] * op[2]);
          const float gn = ldf(a.g_out, gb + (C + 3 * PV + p) * a.g_out.s[3]);
          for (int y = 0; y < 3; ++y)
            dopt[y] = ldf(a.g_out, gb + (C + 3 * p + y) * a.g_out.s[3]) + (nrm > 0.f ? gn * op[y] / nrm : 0.f);
          for (int x = 0; x < 3; ++x) {
            const float rop = Rm[3 * x] * op[0] + Rm[3 * x + 1] * op[1] + Rm[3 * x + 2] * op[2];
            const float rdo = Rm[3 * x] * dopt[0] + Rm[3 * x + 1] * dopt[1] + Rm[3 * x + 2] * dopt[2];
            for (int y = 0; y < 3; ++y) fr[3 * x + y] += rop * dopt[y];
            fr[9 + x] -= rdo;
          }
        }
      }
    }
    for (int e = 0; e < 12; ++e) fterm[(il * H + h) * 12 + e] = fr[e];
    gterm[il * H + h] = gsum;
  }
  __syncthreads();
  // frame gradients: sum over heads in order
  for (int t = tid; t < rb * 12; t += blockDim.x) {
    const int il = t / 12, e = t % 12;
    const int i = i0 + il;
    if (i >= a.L) continue;
    float s = 0.f;
    for (int h = 0; h < H; ++h) s += fterm[(il * H + h) * 12 + e];
    const int64_t bi = static_cast<int64_t>(b) * a.L + i;
    const int64_t nbl = static_cast<int64_t>(a.B) * a.L;
    if (e < 9) *IPA_AT(a.d_rot, bi * 9 + e, nbl * 9, a.err) = s;
    else *IPA_AT(a.d_trans, bi * 3 + (e - 9), nbl * 3, a.err) = s;
  }
  // d gamma partial of this block: residues in order
  for (int h = tid; h < H; h += blockDim.x) {
    double s = 0.0;
    for (int il = 0; il < rb; ++il) s += gterm[il * H + h];
    *IPA_AT(a.g_part, (static_cast<int64_t>(b) * a.nblk + blk) * H + h, static_cast<int64_t>(a.B) * a.nblk * H, a.err) = s;
  }
}

// Pair columns: a block covers 32 columns x PAIR_RB = 8 residues, one thread
// per (column, residue): d z1 and d z2 (sums over heads, heads in order);
// the per-residue terms z1 dQ_pair of every head are summed over the block's
// residues in order through shared memory (d w_bias partials).  Warps read
// 32 consecutive columns of one row.
constexpr int PAIR_RB = 8;
constexpr int PAIR_HC = 16;

__global__ void __launch_bounds__(256) ipa_bwd_pair_kernel(const MapArgs a) {
  __shared__ float wsm[PAIR_RB][PAIR_HC][33];
  const int tid = threadIdx.x, cl = tid & 31, il = tid >> 5;
  const int col = blockIdx.x * 32 + cl;
  const int blk = blockIdx.y, b = blockIdx.z;
  const int i = blk * PAIR_RB + il;
  const int H = a.H, C = IPA_C, PV = IPA_PV;
  const bool valid = i < a.L && col < a.DZ;
  const int ic = valid ? i : 0, cc0 = col < a.DZ ? col : 0;
  const int cc = cc0 % a.Cz, rr = cc0 / a.Cz;
  const bool inpair = valid && col < a.RCz;
  const int64_t bi = static_cast<int64_t>(b) * a.L + ic;
  const bool live = valid && a.frame[bi * 4 + 3].x != 0.f;
  const float z1 = valid ? a.z1f[bi * a.DZ + cc0] : 0.f;
  float s1 = 0.f, s2 = 0.f;
  for (int h0 = 0; h0 < H; h0 += PAIR_HC) {
    const int nh = H - h0 < PAIR_HC ? H - h0 : PAIR_HC;
#pragma unroll 4
    for (int hh = 0; hh < nh; ++hh) {
      const int h = h0 + hh;
      const int64_t bhl = (static_cast<int64_t>(b) * H + h) * a.L + ic;
      const float dq = valid ? a.dqp[bhl * a.DZ + cc0] : 0.f;
      if (inpair) {
        const float gp = ldf(a.g_out, b * a.g_out.s[0] + ic * a.g_out.s[1] + h * a.g_out.s[2] +
                                          (C + 4 * PV + cc) * a.g_out.s[3]);
        const float u = ldf(a.uagg, b * a.uagg.s[0] + ic * a.uagg.s[1] + h * a.uagg.s[2] + rr * a.uagg.s[3] +
                                        cc * a.uagg.s[4]);
        s1 += a.wqp[h * a.DZ + cc0] * dq + (live ? gp * u : 0.f);
        s2 += a.dz2[bhl * a.DZ + cc0];
      }
      wsm[il][hh][cl] = z1 * dq;
    }
    __syncthreads();
    for (int t = tid; t < nh * 32; t += blockDim.x) {
      const int hh = t >> 5, c = t & 31;
      float w = 0.f;
#pragma unroll
      for (int q = 0; q < PAIR_RB; ++q) w += wsm[q][hh][c];
      if (blockIdx.x * 32 + c < a.DZ)
        *IPA_AT(a.wb_part, ((static_cast<int64_t>(b) * gridDim.y + blk) * H + h0 + hh) * a.DZ + blockIdx.x * 32 + c,
                static_cast<int64_t>(a.B) * gridDim.y * H * a.DZ, a.err) = w;
    }
    __syncthreads();
  }
  if (inpair) {
    const int64_t nz = static_cast<int64_t>(a.B) * a.L * a.RCz;
    *IPA_AT(a.d_z1, bi * a.RCz + col, nz, a.err) = s1;
    *IPA_AT(a.d_z2, bi * a.RCz + col, nz, a.err) = s2;
  }
}

// The same sums with 16-byte accesses, when every operand row is contiguous
// fp32 on 16-byte boundaries and the pair block has no padding (R Cz = DZ,
// DZ % 128 == 0): thread (residue il, lane) owns columns [128 x + 4 lane,
// +4) of block column x, so a warp reads 512 contiguous bytes per operand.
// The per-element arithmetic and every summation order are those of
// ipa_bwd_pair_kernel (heads in order for d z1 / d z2, the block's residues
// in order for the d w_bias partials), eight heads per shared-memory round.
constexpr int PAIR4_HC = 8;
__global__ void __launch_bounds__(256) ipa_bwd_pair4_kernel(const MapArgs a) {
  __shared__ float4 wsm4[PAIR_RB][PAIR4_HC][33];
  const int tid = threadIdx.x, cl = tid & 31, il = tid >> 5;
  const int col = blockIdx.x * 128 + 4 * cl;
  const int blk = blockIdx.y, b = blockIdx.z;
  const int i = blk * PAIR_RB + il;
  const int H = a.H, C = IPA_C, PV = IPA_PV;
  const bool valid = i < a.L;
  const int ic = valid ? i : 0;
  const int cc = col % a.Cz, rr = col / a.Cz;
  const int64_t bi = static_cast<int64_t>(b) * a.L + ic;
  const bool live = valid && a.frame[bi * 4 + 3].x != 0.f;
  const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
  const float4 z1 = valid ? *reinterpret_cast<const float4*>(a.z1f + bi * a.DZ + col) : zero;
  const float* gbase = reinterpret_cast<const float*>(a.g_out.p) + b * a.g_out.s[0] + ic * a.g_out.s[1] + (C + 4 * PV + cc);
  const float* ubase = reinterpret_cast<const float*>(a.uagg.p) + b * a.uagg.s[0] + ic * a.uagg.s[1] + rr * a.uagg.s[3] + cc;
  float4 s1 = zero, s2 = zero;
  for (int h0 = 0; h0 < H; h0 += PAIR4_HC) {
    const int nh = H - h0 < PAIR4_HC ? H - h0 : PAIR4_HC;
#pragma unroll 4
    for (int hh = 0; hh < nh; ++hh) {
      const int h = h0 + hh;
      const int64_t bhl = (static_cast<int64_t>(b) * H + h) * a.L + ic;
      const float4 dq = valid ? *reinterpret_cast<const float4*>(a.dqp + bhl * a.DZ + col) : zero;
      if (valid) {
        const float4 gp = *reinterpret_cast<const float4*>(gbase + h * a.g_out.s[2]);
        const float4 u = *reinterpret_cast<const float4*>(ubase + h * a.uagg.s[2]);
        const float4 w = *reinterpret_cast<const float4*>(a.wqp + h * a.DZ + col);
        const float4 d2 = *reinterpret_cast<const float4*>(a.dz2 + bhl * a.DZ + col);
        s1.x += w.x * dq.x + (live ? gp.x * u.x : 0.f);
        s1.y += w.y * dq.y + (live ? gp.y * u.y : 0.f);
        s1.z += w.z * dq.z + (live ? gp.z * u.z : 0.f);
        s1.w += w.w * dq.w + (live ? gp.w * u.w : 0.f);
        s2.x += d2.x; s2.y += d2.y; s2.z += d2.z; s2.w += d2.w;
      }
      wsm4[il][hh][cl] = make_float4(z1.x * dq.x, z1.y * dq.y, z1.z * dq.z, z1.w * dq.w);
    }
    __syncthreads();
    for (int t = tid; t < nh * 32; t += blockDim.x) {
      const int hh = t >> 5, c = t & 31;
      float4 w = zero;
#pragma unroll
      for (int q = 0; q < PAIR_RB; ++q) {
        const float4 v = wsm4[q][hh][c];
        w.x += v.x; w.y += v.y; w.z += v.z; w.w += v.w;
      }
      float4* dst = reinterpret_cast<float4*>(
          IPA_SPAN(a.wb_part, ((static_cast<int64_t>(b) * gridDim.y + blk) * H + h0 + hh) * a.DZ + blockIdx.x * 128 + 4 * c,
                   4, static_cast<int64_t>(a.B) * gridDim.y * H * a.DZ, a.err));
      *dst = w;
    }
    __syncthreads();
  }
  if (valid) {
    const int64_t nz = static_cast<int64_t>(a.B) * a.L * a.RCz;
    *reinterpret_cast<float4*>(IPA_SPAN(a.d_z1, bi * a.RCz + col, 4, nz, a.err)) = s1;
    *reinterpret_cast<float4*>(IPA_SPAN(a.d_z2, bi * a.RCz + col, 4, nz, a.err)) = s2;
  }
}

// One block of 1024 threads per (head, 32 columns).  Thread (c, g): group g
// of 32 sums parts g, g + 32, ... (factors r in order, four running sums
// over parts 128 apart) for column c; the 32 group sums are then added in
// group order.  Warp 0 of the first column
// block sums the d gamma parts, lane l taking parts l, l + 32, ..., then a
// fixed shuffle tree.  The order of every sum depends on the sizes alone, so
// the result is reproducible.
constexpr int RED_THREADS = 1024;
__global__ void __launch_bounds__(RED_THREADS) ipa_bwd_reduce_kernel(const float* wb_part, int nwb, const double* g_part,
                                                                     int ng, int H, int DZ, int Cz, int R, float scale,
                                                                     float* d_wb, float* d_gamma, int* err) {
  __shared__ double red[32][33];
  const int h = blockIdx.x, t = threadIdx.x, cl = t & 31, g = t >> 5;
  const int c = blockIdx.y * 32 + cl;
  // four independent running sums (parts p, p + 32, p + 64, p + 96 of each
  // step of 128), so that four loads are in flight; combined in a fixed order
  double acc0 = 0.0, acc1 = 0.0, acc2 = 0.0, acc3 = 0.0;
  if (c < Cz) {
    const int64_t pstride = static_cast<int64_t>(H) * DZ;
    const float* col = wb_part + static_cast<int64_t>(h) * DZ + c;
    int p = g;
    for (; p + 96 < nwb; p += 128)
      for (int r = 0; r < R; ++r) {
        const float* q = col + r * Cz + p * pstride;
        acc0 += q[0];
        acc1 += q[32 * pstride];
        acc2 += q[64 * pstride];
        acc3 += q[96 * pstride];
      }
    for (; p < nwb; p += 32)
      for (int r = 0; r < R; ++r) acc0 += col[r * Cz + p * pstride];
  }
  red[g][cl] = (acc0 + acc1) + (acc2 + acc3);
  __syncthreads();
  if (t < 32 && c < Cz) {
    double sum = 0.0;
    for (int q = 0; q < 32; ++q) sum += red[q][t];
    *IPA_AT(d_wb, c * H + h, static_cast<int64_t>(Cz) * H, err) = static_cast<float>(sum * scale);
  }
  if (blockIdx.y == 0 && t >= 32 && t < 64) {
    const int l = t - 32;
    double g0 = 0.0, g1 = 0.0, g2 = 0.0, g3 = 0.0;
    int p = l;
    for (; p + 96 < ng; p += 128) {
      g0 += g_part[static_cast<int64_t>(p) * H + h];
      g1 += g_part[static_cast<int64_t>(p + 32) * H + h];
      g2 += g_part[static_cast<int64_t>(p + 64) * H + h];
      g3 += g_part[static_cast<int64_t>(p + 96) * H + h];
    }
    for (; p < ng; p += 32) g0 += g_part[static_cast<int64_t>(p) * H + h];
    double gs = (g0 + g1) + (g2 + g3);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) gs += __shfl_xor_sync(0xffffffffu, gs, off);
    if (l == 0) *IPA_AT(d_gamma, h, H, err) = static_cast<float>(gs);
  }
}

int stages_for(uint32_t resident, uint32_t stage, uint32_t aux) {
  const uint32_t budget = 227u * 1024u - 1024u - aux;
  int ns = static_cast<int>((budget - resident) / stage);
  return ns > MAX_NS ? MAX_NS : ns;
}

}  // namespace

#ifdef IPA_TRACE
bool ipa_bwd_trace_read(void* host, size_t bytes) {
  if (bytes < sizeof(g_bwd_trace)) return false;
  return cudaMemcpyFromSymbol(host, g_bwd_trace, sizeof(g_bwd_trace)) == cudaSuccess;
}
#endif

// Residues per block of ipa_bwd_map_kernel (one thread per residue and
// head): about 64 threads, so that a long sequence spreads as many small
// blocks evenly over the SMs (with 256-thread blocks, L = 4096 and H = 12
// gave 196 blocks on 148 SMs, and the SMs holding two set the time).
static int map_residues_per_block(int H) {
  const int rb = 64 / H;
  return rb < 1 ? 1 : rb > 32 ? 32 : rb;
}

IpaBwdWorkspace ipa_bwd_workspace_layout(int B, int L, int H, int DZ, int RCz) {
  auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  IpaBwdWorkspace w{};
  w.fwd = ipa_workspace_layout(B, L, H, DZ, RCz);
  size_t o = up(w.fwd.total);
  const size_t bhl = static_cast<size_t>(B) * H * L;
  const int rb = map_residues_per_block(H);
  const size_t nblk = (L + rb - 1) / rb;                // per-residue mapping blocks
  const size_t npb = (L + PAIR_RB - 1) / PAIR_RB;        // pair-column blocks
  w.doh = o; o = up(o + bhl * 64 * 2);
  w.du = o; o = up(o + bhl * DZ * 2);
  w.qp = o; o = up(o + bhl * DZ * 2);
  w.rowd = o; o = up(o + bhl * 8);
  w.dqh = o; o = up(o + bhl * 64 * 4);
  w.dqp = o; o = up(o + bhl * DZ * 4);
  w.rsq = o; o = up(o + bhl * 16);
  w.dkh = o; o = up(o + bhl * 64 * 4);
  w.dva = o; o = up(o + bhl * 64 * 4);
  w.dz2 = o; o = up(o + bhl * DZ * 4);
  w.csk = o; o = up(o + bhl * 16);
  w.pts = o; o = up(o + bhl * 24 * 4);
  w.gsum = o; o = up(o + bhl * 4);
  w.wb_part = o; o = up(o + static_cast<size_t>(B) * npb * H * DZ * 4);
  w.g_part = o; o = up(o + static_cast<size_t>(B) * nblk * H * 8);
  const int64_t nkb = static_cast<int64_t>(B) * H * ((L + 127) / 128);
  w.ksplit_chunks = nkb < kBwdSlots ? nkb : kBwdSlots;
  w.ksplit_tiles = w.ksplit_chunks / 2;
  w.kpart = o; o = up(o + static_cast<size_t>(w.ksplit_chunks) * (DZ + 138) * 128 * 4);
  w.kticket = o; o = up(o + static_cast<size_t>(w.ksplit_tiles) * 4 + 4);
  w.total = o;
  return w;
}

// Query split of the key pass.  The grid is nqb query-pass CTAs, then nkb
// key-pass CTAs, one per SM at a time (P resident).  When the last, partial
// wave (r = (nqb + nkb) mod P CTAs) holds key-pass CTAs only, each of them
// can run as S chunks of consecutive 32-query tiles, all chunks in one round
// (r S <= P).  Cost in units of one 32-query tile (~2 us): a chunk pays
// ceil(nq / S) tiles plus ~5 of set-up and output; the merging one ~1 + S / 2
// more.  S is the cheapest of 2 .. MAX_KSPLIT when it saves a tenth.
SplitPlan ipa_bwd_split_plan(int nqb, int nkb, int nq, int P, int64_t max_tiles, int64_t max_chunks) {
  const int T = nqb + nkb;
  SplitPlan none{nkb, 1};
  if (P <= 0 || T < P || nq < 2) return none;
  const int r = T % P;
  if (r == 0 || r > nkb || r > max_tiles) return none;
  constexpr double kFixed = 5.0;
  double best = 0.9 * (nq + kFixed);
  int bs = 1;
  for (int S = 2; S <= MAX_KSPLIT && S <= nq && static_cast<int64_t>(r) * S <= max_chunks && r * S <= P; ++S) {
    const double cost = (nq + S - 1) / S + kFixed + 1.0 + 0.5 * S;
    if (cost < best) {
      best = cost;
      bs = S;
    }
  }
  return bs == 1 ? none : SplitPlan{nkb - r, bs};
}

cudaError_t ipa_launch_bwd(const IpaBwdLaunch& a, cudaStream_t stream) {
  const IpaLaunch& f = a.f;
  unsigned char* ws = f.ws;
  const IpaBwdWorkspace& w = a.lay;
  const IpaWorkspace& fw = w.fwd;
  const int B = f.B, L = f.L, H = f.H, DZ = f.DZ, np = DZ / 64;
  const uint64_t bh = static_cast<uint64_t>(B) * H;

  // 1. the forward prologue again (frames, augmented rows, tile origins)
  cudaError_t e = ipa_launch_prologue(f, stream);
  if (e != cudaSuccess) return e;

  // 2. backward rows
  RowsArgs ra{};
  ra.B = B; ra.L = L; ra.H = H; ra.DZ = DZ; ra.RCz = f.RCz; ra.Cz = f.Cz; ra.F = f.F;
  ra.z1_half = ipa_pair_supported(DZ);
  ra.g_out = a.g_out; ra.out = a.out; ra.lse = a.lse; ra.uagg = a.uagg;
  {
    // 16-byte pair-block loads: fp32 rows with unit feature stride, every
    // row start and factor start on a 16-byte boundary, whole columns per lane
    auto al16 = [](const View& v, int n) {
      bool ok = (reinterpret_cast<uintptr_t>(v.p) & 15u) == 0;
      for (int d = 0; d < n; ++d) ok = ok && (v.s[d] % 4 == 0);
      return ok;
    };
    const bool vec = f.RCz == DZ && (DZ == 128 || DZ == 256) && f.Cz % 8 == 0 && a.g_out.dtype == 0 &&
                     a.g_out.s[3] == 1 && al16(a.g_out, 3) && (IPA_C + 4 * IPA_PV) % 4 == 0 && a.uagg.dtype == 0 &&
                     a.uagg.s[4] == 1 && al16(a.uagg, 4);
    ra.pair_cpl = vec ? DZ / 32 : 0;
  }
  ra.frame = reinterpret_cast<const float4*>(ws + fw.frame);
  ra.cen = reinterpret_cast<const float4*>(ws + fw.cen);
  ra.rowq = reinterpret_cast<const float4*>(ws + fw.rowq);
  ra.wqp = reinterpret_cast<const float*>(ws + fw.wqp);
  ra.z1f = reinterpret_cast<const float*>(ws + fw.z1f);
  ra.z1h = reinterpret_cast<const __half*>(ws + fw.z1h);
  ra.doh = reinterpret_cast<__half*>(ws + w.doh);
  ra.du = reinterpret_cast<__half*>(ws + w.du);
  ra.qp = reinterpret_cast<__half*>(ws + w.qp);
  ra.rowd = reinterpret_cast<float2*>(ws + w.rowd);
  ra.q_pts = f.q_pts; ra.k_pts = f.k_pts;
  ra.pts = reinterpret_cast<float*>(ws + w.pts);
  ra.err = f.err;
  ra.kticket = reinterpret_cast<int*>(ws + w.kticket);
  ra.nkticket = static_cast<int>(w.ksplit_tiles);
  const int64_t warps = static_cast<int64_t>(B) * L * H;
  ipa_bwd_rows_kernel<<<static_cast<unsigned>((warps + 7) / 8), 256, 0, stream>>>(ra);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  BwdArgs ba{};
  ba.B = B; ba.L = L; ba.H = H; ba.DZ = DZ; ba.RCz = f.RCz; ba.Cz = f.Cz; ba.R = f.R;
  ba.nqt = f.nqt; ba.nkt = f.nkt;
  ba.qscale = kLog2e * f.w_L * f.scalar_scale; ba.w_L = f.w_L; ba.w_C = f.w_C;
  ba.rowq = reinterpret_cast<const float4*>(ws + fw.rowq);
  ba.colk = reinterpret_cast<const float4*>(ws + fw.colk);
  ba.oq = reinterpret_cast<const float4*>(ws + fw.oq);
  ba.ok = reinterpret_cast<const float4*>(ws + fw.ok);
  ba.cen = reinterpret_cast<const float4*>(ws + fw.cen);
  ba.headc = reinterpret_cast<const float*>(ws + fw.headc);
  ba.wqp = reinterpret_cast<const float*>(ws + fw.wqp);
  ba.frame = reinterpret_cast<const float4*>(ws + fw.frame);
  ba.z1f = reinterpret_cast<const float*>(ws + fw.z1f);
  ba.z1h = reinterpret_cast<const __half*>(ws + fw.z1h);
  ba.rowd = reinterpret_cast<const float2*>(ws + w.rowd);
  ba.dqh = reinterpret_cast<float*>(ws + w.dqh);
  ba.dqp = reinterpret_cast<float*>(ws + w.dqp);
  ba.rsq = reinterpret_cast<float4*>(ws + w.rsq);
  ba.dkh = reinterpret_cast<float*>(ws + w.dkh);
  ba.dva = reinterpret_cast<float*>(ws + w.dva);
  ba.dz2 = reinterpret_cast<float*>(ws + w.dz2);
  ba.csk = reinterpret_cast<float4*>(ws + w.csk);
  ba.pts = reinterpret_cast<const float*>(ws + w.pts);
  ba.gsum = reinterpret_cast<float*>(ws + w.gsum);
  ba.err = f.err;
  ba.split_first = 1 << 30;   // the query pass runs whole tiles
  ba.split_s = 1;

  const uint64_t rowb = static_cast<uint64_t>(L) * DH * 2;
  // 3.-4. query and key passes, one grid
  {
    BwdMaps mp;
    bool ok = encode_tmap_f16_3d(&mp.q_qh, ws + fw.qh, DH, L, bh, DH * 2, rowb, 64, 128) &&
              encode_tmap_f16_panels(&mp.q_qp, ws + w.qp, DZ, L, bh, 128, np) &&
              encode_tmap_f16_3d(&mp.q_do, ws + w.doh, DH, L, bh, DH * 2, rowb, 64, 128) &&
              encode_tmap_f16_panels(&mp.q_du, ws + w.du, DZ, L, bh, 128, np) &&
              encode_tmap_f16_3d(&mp.q_kh, ws + fw.kh, DH, L, bh, DH * 2, rowb, 64, BT) &&
              encode_tmap_f16_3d(&mp.q_vh, ws + fw.vh, DH, L, bh, DH * 2, rowb, 64, BT) &&
              encode_tmap_f16_panels(&mp.q_z2, ws + fw.z2, DZ, L, B, BT, np) &&
              encode_tmap_f16_3d(&mp.k_kh, ws + fw.kh, DH, L, bh, DH * 2, rowb, 64, 128) &&
              encode_tmap_f16_3d(&mp.k_vh, ws + fw.vh, DH, L, bh, DH * 2, rowb, 64, 128) &&
              encode_tmap_f16_panels(&mp.k_z2, ws + fw.z2, DZ, L, B, 128, np) &&
              encode_tmap_f16_3d(&mp.k_qh, ws + fw.qh, DH, L, bh, DH * 2, rowb, 64, BT) &&
              encode_tmap_f16_3d(&mp.k_do, ws + w.doh, DH, L, bh, DH * 2, rowb, 64, BT) &&
              encode_tmap_f16_panels(&mp.k_qp, ws + w.qp, DZ, L, bh, BT, 1) &&
              encode_tmap_f16_panels(&mp.k_du, ws + w.du, DZ, L, bh, BT, 1);
    if (!ok) return cudaErrorInvalidValue;
    const QLayout l1 = q_layout(DZ, 1);
    const int nreg = stages_for(l1.stg, l1.stg_bytes, 2048);
    // one more stage in the Q_pair area: the columns in tensor memory free at
    // least its first stg_bytes (all of it when every K-step is there, the
    // first three panels at DZ = 256)
    ba.qp_stage = nreg < MAX_NS ? 1 : 0;
    ba.ns = nreg + ba.qp_stage;
    const KLayout k1 = k_layout(DZ, 1);
    BwdArgs kb = ba;
    kb.ns = stages_for(k1.stg, k1.stg_bytes, 6656);
    kb.qp_stage = 0;
    const uint32_t sq = q_layout(DZ, nreg).total, sk = k_layout(DZ, kb.ns).total;
    const uint32_t smem = (sq > sk ? sq : sk) + 1024;
    e = cudaFuncSetAttribute(ipa_bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    const int nqb = static_cast<int>(bh) * f.nqt;
    const int nkb = static_cast<int>(bh) * ((L + 127) / 128);
    int dev = 0, sms = 0;
    SplitPlan plan{nkb, 1};
    if (cudaGetDevice(&dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess)
      plan = ipa_bwd_split_plan(nqb, nkb, (L + BT - 1) / BT, sms, w.ksplit_tiles, w.ksplit_chunks);
    kb.split_first = plan.first;
    kb.split_s = plan.S;
    kb.part = reinterpret_cast<float*>(ws + w.kpart);
    kb.part_extent = w.ksplit_chunks * (DZ + 138) * 128;
    kb.ticket = reinterpret_cast<int*>(ws + w.kticket);
    kb.ticket_extent = static_cast<int>(w.ksplit_tiles);
    const int kblocks = plan.first + (nkb - plan.first) * plan.S;
    ipa_bwd_kernel<<<static_cast<unsigned>(nqb + kblocks), NTH, smem, stream>>>(mp, ba, kb, nqb);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  // 5. per-residue mapping and the reductions
  MapArgs m{};
  m.B = B; m.L = L; m.H = H; m.DZ = DZ; m.RCz = f.RCz; m.Cz = f.Cz; m.R = f.R;
  m.rb = map_residues_per_block(H);
  m.nblk = (L + m.rb - 1) / m.rb;
  m.qscale = ba.qscale; m.w_L = f.w_L; m.w_C = f.w_C;
  m.q_pts = f.q_pts; m.k_pts = f.k_pts; m.v_pts = f.v_pts; m.g_out = a.g_out; m.out = a.out; m.uagg = a.uagg;
  m.frame = ba.frame; m.cen = ba.cen; m.oq = ba.oq; m.ok = ba.ok; m.headc = ba.headc; m.wqp = ba.wqp;
  m.z1f = ba.z1f; m.dqh = ba.dqh; m.dqp = ba.dqp; m.rsq = ba.rsq; m.dkh = ba.dkh; m.dva = ba.dva;
  m.dz2 = ba.dz2; m.csk = ba.csk; m.gsum = ba.gsum; m.nqt = f.nqt; m.nkt = f.nkt;
  m.d_q = a.d_q; m.d_k = a.d_k; m.d_v = a.d_v; m.d_qpts = a.d_q_pts; m.d_kpts = a.d_k_pts; m.d_vpts = a.d_v_pts;
  m.d_rot = a.d_rot; m.d_trans = a.d_trans; m.d_z1 = a.d_z1; m.d_z2 = a.d_z2;
  m.wb_part = reinterpret_cast<float*>(ws + w.wb_part);
  m.g_part = reinterpret_cast<double*>(ws + w.g_part);
  m.err = f.err;
  const size_t msmem = static_cast<size_t>((m.rb * H * 12 + 1) & ~1) * 4 + static_cast<size_t>(m.rb) * H * 8;
  const unsigned mthreads = static_cast<unsigned>((m.rb * H + 31) / 32 * 32);
  ipa_bwd_map_kernel<<<dim3(static_cast<unsigned>(m.nblk), static_cast<unsigned>(B)), mthreads, msmem, stream>>>(m);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int npb = (L + PAIR_RB - 1) / PAIR_RB;
  if (ra.pair_cpl != 0 && (reinterpret_cast<uintptr_t>(a.d_z1) & 15u) == 0 &&
      (reinterpret_cast<uintptr_t>(a.d_z2) & 15u) == 0)
    // the rows kernel's 16-byte conditions (fp32 rows on 16-byte boundaries,
    // R Cz = DZ, DZ = 128 or 256) and aligned gradient outputs
    ipa_bwd_pair4_kernel<<<dim3(static_cast<unsigned>(DZ / 128), static_cast<unsigned>(npb), static_cast<unsigned>(B)),
                           256, 0, stream>>>(m);
  else
    ipa_bwd_pair_kernel<<<dim3(static_cast<unsigned>((DZ + 31) / 32), static_cast<unsigned>(npb), static_cast<unsigned>(B)),
                          256, 0, stream>>>(m);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const dim3 rgrid(static_cast<unsigned>(H), static_cast<unsigned>((f.Cz + 31) / 32));
  ipa_bwd_reduce_kernel<<<rgrid, RED_THREADS, 0, stream>>>(m.wb_part, B * npb, m.g_part, B * m.nblk, H, DZ, f.Cz, f.R,
                                                          kLog2e * f.w_L, a.d_w_bias, a.d_gamma, f.err);
  return cudaGetLastError();
}

}  // namespace fipa
