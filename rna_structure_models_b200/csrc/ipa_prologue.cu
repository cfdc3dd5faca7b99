// Prologue of the fused IPA core: applies the residue frames and writes the
// fp16 augmented operands that the attention kernel streams with TMA.
//
//   ipa_tile_kernel   -- one CTA per (batch, 64-residue key tile): frame rows
//                        (R, t, valid), partial sums of the valid origins, and
//                        the pair factors z2 (fp16) and z1 (fp32 and fp16)
//                        padded to DZ.
//   ipa_rows_kernel   -- one thread per (b, i, h), heads fastest: the
//                        centroid of the valid origins (each block reduces
//                        the tile partial sums of its batches), query-tile
//                        (128) and key-tile (64) origins relative to it, the
//                        Q_h, K_h, V_h rows (64 fp16 each) and the two small
//                        fp32 row terms; designated threads also write the
//                        centroid, tile origins, per-head point coefficient
//                        and pair-bias weights w_L log2(e) w_bias[c, h] that
//                        the core kernel reads.
//
// Augmented row layout for the (C, Pq, Pv) = (16, 4, 8) head shape, with
// c = log2(e) w_L gamma_h w_C / 2, gq' / gk' the global query / key points
// relative to their tile origin and gv the value points relative to the
// centroid (hi = fp16(x), lo = fp16(x - hi)):
//   Q_h: [ log2(e) w_L s q (16) | gq'hi (12) | gq'hi (12) | gq'lo (12) | -1 -1 | 0 (10) ]
//   K_h: [ k (16) | 2c gk' hi (12) | lo (12) | hi (12) | c|gk'|^2 hi, lo | 0 (10) ]
//   V_h: [ v (16) | gv hi (24) | gv lo (24) ]
// so Q_h . K_h = log2(e) w_L s q.k + 2c gq'.gk' - c sum_p |gk'_p|^2 (the
// lo*lo product is dropped; every kept product is exact in fp32).
#include <cuda_fp16.h>

#include <cmath>
#include <cstdint>

#include "bounds.cuh"
#include "internal.h"
#include "sm100.cuh"

#define IPA_FILE_TAG 1

namespace fipa {

using namespace sm100;

namespace {

constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ float ldf(const View& v, int64_t off) {
  return reinterpret_cast<const float*>(v.p)[off];
}
__device__ __forceinline__ bool ldb(const View& v, int64_t off) {
  return reinterpret_cast<const unsigned char*>(v.p)[off] != 0;
}

struct TileArgs {
  int B, L, R, Cz, RCz, DZ, nkt;
  View rot, trans, mask, z1, z2;
  float4* frame;   // [B, L, 4]: (R00 R01 R02 R10) (R11 R12 R20 R21) (R22 tx ty tz) (valid 0 0 0)
  float4* part;    // [B, nkt]: sum of valid origins, count
  float* z1f;      // [B, L, DZ]
  __half* z1h;     // [B, L, DZ]
  __half* z2h;     // [B, L, DZ]
  int* err;        // DEV_NONFINITE when a pair factor does not survive the fp16 rounding
  int* ticket;     // the core's key-split tickets, zeroed here (nticket ints)
  int nticket;
};

// |x| >= 65520 (or NaN) does not survive the rounding to fp16
__device__ __forceinline__ void check_fp16_range(const TileArgs& a, float vmax) {
  if (!(vmax < 65520.f)) record_error(a.err, DEV_NONFINITE);
}

// Pair factors of 64 residues x one 64-column panel, zero-padded beyond
// R*Cz and zero for masked residues: 4 residues x 64 columns per pass, all
// loads of a thread issued before its stores.
// Vector form of the copy below for the dense layout (unit column stride,
// Cz % 4 == 0, 16-byte aligned rows): 16 residues x 64 columns per pass,
// four columns per thread.
__device__ __forceinline__ bool ipa_tile_copy_pairs_vec(const TileArgs& a, int b, int i0, int panel, int tid) {
  if (a.z1.s[3] != 1 || a.z2.s[3] != 1 || (a.Cz & 3) != 0 || a.z1.s[2] != a.Cz || a.z2.s[2] != a.Cz ||
      ((reinterpret_cast<uintptr_t>(a.z1.p) | reinterpret_cast<uintptr_t>(a.z2.p)) & 15) != 0 ||
      ((a.z1.s[0] | a.z1.s[1] | a.z2.s[0] | a.z2.s[1]) & 3) != 0)
    return false;
  const int col = panel * 64 + 4 * (tid & 15);       // first of this thread's 4 columns
  const bool inpair = col < a.RCz;                    // RCz % 16 == 0: all 4 or none
  constexpr int NP = KT / 16;
  float4 v1[NP], v2[NP];
#pragma unroll
  for (int q = 0; q < NP; ++q) {
    const int i = i0 + 16 * q + (tid >> 4);
    v1[q] = make_float4(0.f, 0.f, 0.f, 0.f);
    v2[q] = v1[q];
    if (i < a.L && inpair && ldb(a.mask, b * a.mask.s[0] + i * a.mask.s[1])) {
      v1[q] = __ldg(reinterpret_cast<const float4*>(static_cast<const float*>(a.z1.p) + b * a.z1.s[0] + i * a.z1.s[1] + col));
      v2[q] = __ldg(reinterpret_cast<const float4*>(static_cast<const float*>(a.z2.p) + b * a.z2.s[0] + i * a.z2.s[1] + col));
    }
  }
  float vmax = 0.f;
#pragma unroll
  for (int q = 0; q < NP; ++q) {
    vmax = fmax_nan(vmax, fmax_nan(fmax_nan(fabsf(v1[q].x), fabsf(v1[q].y)), fmax_nan(fabsf(v1[q].z), fabsf(v1[q].w))));
    vmax = fmax_nan(vmax, fmax_nan(fmax_nan(fabsf(v2[q].x), fabsf(v2[q].y)), fmax_nan(fabsf(v2[q].z), fabsf(v2[q].w))));
  }
  check_fp16_range(a, vmax);
#pragma unroll
  for (int q = 0; q < NP; ++q) {
    const int i = i0 + 16 * q + (tid >> 4);
    if (i < a.L) {
      const int64_t o = (static_cast<int64_t>(b) * a.L + i) * a.DZ + col;
      const int64_t ext = static_cast<int64_t>(a.B) * a.L * a.DZ;
      *reinterpret_cast<float4*>(IPA_SPAN(a.z1f, o, 4, ext, a.err)) = v1[q];
      *reinterpret_cast<uint2*>(IPA_SPAN(a.z1h, o, 4, ext, a.err)) =
          make_uint2(pack_half2(v1[q].x, v1[q].y), pack_half2(v1[q].z, v1[q].w));
      *reinterpret_cast<uint2*>(IPA_SPAN(a.z2h, o, 4, ext, a.err)) =
          make_uint2(pack_half2(v2[q].x, v2[q].y), pack_half2(v2[q].z, v2[q].w));
    }
  }
  return true;
}

__device__ __forceinline__ void ipa_tile_copy_pairs(const TileArgs& a, int b, int i0, int panel, int tid) {
  if (ipa_tile_copy_pairs_vec(a, b, i0, panel, tid)) return;
  const int col = panel * 64 + (tid & 63);
  const bool inpair = col < a.RCz;
  const int rr = inpair ? col / a.Cz : 0, cc = inpair ? col % a.Cz : 0;
  constexpr int NR = KT / 4;
  float v1[NR], v2[NR];
#pragma unroll
  for (int q = 0; q < NR; ++q) {
    const int i = i0 + 4 * q + (tid >> 6);
    v1[q] = 0.f;
    v2[q] = 0.f;
    if (i < a.L && inpair && ldb(a.mask, b * a.mask.s[0] + i * a.mask.s[1])) {
      v1[q] = ldf(a.z1, b * a.z1.s[0] + i * a.z1.s[1] + rr * a.z1.s[2] + cc * a.z1.s[3]);
      v2[q] = ldf(a.z2, b * a.z2.s[0] + i * a.z2.s[1] + rr * a.z2.s[2] + cc * a.z2.s[3]);
    }
  }
  float vmax = 0.f;
#pragma unroll
  for (int q = 0; q < NR; ++q) vmax = fmax_nan(vmax, fmax_nan(fabsf(v1[q]), fabsf(v2[q])));
  check_fp16_range(a, vmax);
#pragma unroll
  for (int q = 0; q < NR; ++q) {
    const int i = i0 + 4 * q + (tid >> 6);
    if (i < a.L) {
      const int64_t o = (static_cast<int64_t>(b) * a.L + i) * a.DZ + col;
      const int64_t ext = static_cast<int64_t>(a.B) * a.L * a.DZ;
      *IPA_AT(a.z1f, o, ext, a.err) = v1[q];
      *IPA_AT(a.z1h, o, ext, a.err) = __float2half_rn(v1[q]);
      *IPA_AT(a.z2h, o, ext, a.err) = __float2half_rn(v2[q]);
    }
  }
}

__global__ void __launch_bounds__(256) ipa_tile_kernel(const TileArgs a) {
  const int J = blockIdx.x, b = blockIdx.y, panel = blockIdx.z, tid = threadIdx.x;
  const int i0 = J * KT;
  __shared__ float red[2][4];
  if ((J | b | panel) == 0)
    for (int e = tid; e < a.nticket; e += blockDim.x) *IPA_AT(a.ticket, e, a.nticket, a.err) = 0;
  if (panel > 0) {
    ipa_tile_copy_pairs(a, b, i0, panel, tid);
    return;
  }
  const bool pairs = a.DZ > 0;   // no pair block (distance-aware attention): frames and sums only
  if (tid < KT) {
    const int i = i0 + tid;
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
    if (i < a.L) {
      const bool valid = ldb(a.mask, b * a.mask.s[0] + i * a.mask.s[1]);
      const int64_t ro = b * a.rot.s[0] + i * a.rot.s[1];
      float Rm[9];
#pragma unroll
      for (int x = 0; x < 3; ++x)
#pragma unroll
        for (int y = 0; y < 3; ++y) Rm[3 * x + y] = ldf(a.rot, ro + x * a.rot.s[2] + y * a.rot.s[3]);
      const int64_t to = b * a.trans.s[0] + i * a.trans.s[1];
      const float tx = ldf(a.trans, to), ty = ldf(a.trans, to + a.trans.s[2]), tz = ldf(a.trans, to + 2 * a.trans.s[2]);
      float4* f = IPA_SPAN(a.frame, (static_cast<int64_t>(b) * a.L + i) * 4, 4, static_cast<int64_t>(a.B) * a.L * 4, a.err);
      f[0] = make_float4(Rm[0], Rm[1], Rm[2], Rm[3]);
      f[1] = make_float4(Rm[4], Rm[5], Rm[6], Rm[7]);
      f[2] = make_float4(Rm[8], tx, ty, tz);
      f[3] = make_float4(valid ? 1.f : 0.f, 0.f, 0.f, 0.f);
      if (valid) s = make_float4(tx, ty, tz, 1.f);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      s.x += __shfl_xor_sync(0xffffffffu, s.x, off);
      s.y += __shfl_xor_sync(0xffffffffu, s.y, off);
      s.z += __shfl_xor_sync(0xffffffffu, s.z, off);
      s.w += __shfl_xor_sync(0xffffffffu, s.w, off);
    }
    if ((tid & 31) == 0) {
      red[tid >> 5][0] = s.x; red[tid >> 5][1] = s.y; red[tid >> 5][2] = s.z; red[tid >> 5][3] = s.w;
    }
  }
  __syncthreads();
  if (tid == 0)
    *IPA_AT(a.part, b * a.nkt + J, static_cast<int64_t>(a.B) * a.nkt, a.err) =
        make_float4(red[0][0] + red[1][0], red[0][1] + red[1][1], red[0][2] + red[1][2], red[0][3] + red[1][3]);
  if (pairs) ipa_tile_copy_pairs(a, b, i0, 0, tid);
}

struct RowArgs {
  int B, L, H, nqt, nkt, Cz, RCz, DZ;
  int rb;          // residues per block (128 / H)
  float qscale;    // log2(e) w_L scalar_scale
  float w_L, w_C;
  View q, k, v, q_pts, k_pts, v_pts, gamma, w_bias;
  const float4* frame;
  const float4* part;   // [B, nkt] sum of valid origins and count per 64-residue tile
  float4* cen;     // [B]        written here for the core kernel
  float4* oq;      // [B, nqt]
  float4* ok;      // [B, nkt]
  float* headc;    // [H]
  float* wqp;      // [H, DZ]
  uint4* qh;       // [B*H, L, 64] fp16 (8 x uint4 per row)
  uint4* kh;
  uint4* vh;
  float4* rowq;    // [B*H, L]: (sum_p gq'_p, c sum_p |gq'_p|^2)
  float4* colk;    // [B*H, L]
  int* err;
};

// N consecutive elements of a row: float4 loads when the row is contiguous
// and 16-byte aligned (the common dense layout), element loads otherwise.
template <int N>
__device__ __forceinline__ void load_row(const View& v, int64_t base, int64_t st, float (&out)[N]) {
  const float* p = reinterpret_cast<const float*>(v.p) + base;
  if (N % 4 == 0 && st == 1 && (reinterpret_cast<uintptr_t>(p) & 15u) == 0) {
#pragma unroll
    for (int e = 0; e < N; e += 4) {
      const float4 x = __ldg(reinterpret_cast<const float4*>(p) + e / 4);
      out[e] = x.x; out[e + 1] = x.y; out[e + 2] = x.z; out[e + 3] = x.w;
    }
  } else {
#pragma unroll
    for (int e = 0; e < N; ++e) out[e] = p[e * st];
  }
}

// Origin (mean of the valid centred frame origins) of a run of 64-residue
// tiles [J0, J1) of batch b, from their partial sums; 0 for an empty run.
__device__ __forceinline__ float4 tile_origin(const float4* part, int J0, int J1, float4 cen) {
  float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int J = J0; J < J1; ++J) {
    const float4 p = part[J];
    s.x += p.x; s.y += p.y; s.z += p.z; s.w += p.w;
  }
  if (!(s.w > 0.f)) return make_float4(0.f, 0.f, 0.f, 0.f);
  const float inv = 1.f / s.w;
  return make_float4(s.x * inv - cen.x, s.y * inv - cen.y, s.z * inv - cen.z, 0.f);
}

template <int C, int PQ, int PV>
__global__ void __launch_bounds__(128, 4) ipa_rows_kernel(const RowArgs a) {
  static_assert(C + 9 * PQ + 2 <= DH && C + 6 * PV <= DH, "augmented rows wider than 64");
  // a block owns rb consecutive residues of one batch, all heads (heads
  // fastest: the threads of a residue read its contiguous [H, ...] input
  // rows together); its output rows are staged in shared memory and written
  // as one contiguous run of rb rows per head plane
  extern __shared__ uint4 stage_rows[];    // [3][H][rb][8] fp16 rows, then [2][H][rb] float4 terms
  const int rb = a.rb, H = a.H;
  const int b = blockIdx.y;
  const int i0 = blockIdx.x * rb;
  const int il = threadIdx.x / H, h = threadIdx.x % H;
  const int i = i0 + il;
  const bool active = il < rb && i < a.L;
  const int nrow = a.L - i0 < rb ? a.L - i0 : rb;

  // centroid of the batch's valid origins (double sums over the per-tile
  // partial sums of the tile kernel)
  __shared__ double red[4][4];
  __shared__ float4 cen_s;
  {
    double sx = 0, sy = 0, sz = 0, sn = 0;
    for (int J = threadIdx.x; J < a.nkt; J += blockDim.x) {
      const float4 p = a.part[static_cast<int64_t>(b) * a.nkt + J];
      sx += p.x; sy += p.y; sz += p.z; sn += p.w;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      sx += __shfl_xor_sync(0xffffffffu, sx, off);
      sy += __shfl_xor_sync(0xffffffffu, sy, off);
      sz += __shfl_xor_sync(0xffffffffu, sz, off);
      sn += __shfl_xor_sync(0xffffffffu, sn, off);
    }
    if ((threadIdx.x & 31) == 0) {
      const int w = threadIdx.x >> 5;
      red[w][0] = sx; red[w][1] = sy; red[w][2] = sz; red[w][3] = sn;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      double tx = 0, ty = 0, tz = 0, tn = 0;
      for (int w = 0; w < 4; ++w) { tx += red[w][0]; ty += red[w][1]; tz += red[w][2]; tn += red[w][3]; }
      const double inv = tn > 0 ? 1.0 / tn : 0.0;
      cen_s = make_float4(static_cast<float>(tx * inv), static_cast<float>(ty * inv), static_cast<float>(tz * inv),
                          static_cast<float>(tn));
    }
    __syncthreads();
  }
  const int slot = h * rb + il;                                   // row of this thread in a staged plane
  uint4* sq_rows = stage_rows + static_cast<size_t>(0 * H * rb + slot) * 8;
  uint4* sk_rows = stage_rows + static_cast<size_t>(1 * H * rb + slot) * 8;
  uint4* sv_rows = stage_rows + static_cast<size_t>(2 * H * rb + slot) * 8;
  float4* sterm = reinterpret_cast<float4*>(stage_rows + static_cast<size_t>(3 * H * rb) * 8);
  // the [H, DZ] pair-bias weights, one entry per thread of batch 0
  if (b == 0 && active)
    for (int64_t e = static_cast<int64_t>(i) * H + h; e < static_cast<int64_t>(H) * a.DZ;
         e += static_cast<int64_t>(H) * a.L) {
      const int he = static_cast<int>(e / a.DZ), col = static_cast<int>(e % a.DZ);
      *IPA_AT(a.wqp, e, static_cast<int64_t>(H) * a.DZ, a.err) = col < a.RCz ? kLog2e * a.w_L * ldf(a.w_bias, (col % a.Cz) * a.w_bias.s[0] + he * a.w_bias.s[1]) : 0.f;
    }
  if (active) {
  const float4 cn = cen_s;
  const float4* partb = a.part + static_cast<int64_t>(b) * a.nkt;
  const int Jq = (i / QT) * (QT / KT);
  const float4 oqv = tile_origin(partb, Jq, Jq + QT / KT < a.nkt ? Jq + QT / KT : a.nkt, cn);
  const float4 okv = tile_origin(partb, i / KT, i / KT + 1, cn);
  // the values the core kernel reads per batch / tile / head, one writer each
  if (h == 0) {
    if (i == 0) *IPA_AT(a.cen, b, a.B, a.err) = cn;
    if (i % QT == 0) *IPA_AT(a.oq, b * a.nqt + i / QT, static_cast<int64_t>(a.B) * a.nqt, a.err) = oqv;
    if (i % KT == 0) *IPA_AT(a.ok, b * a.nkt + i / KT, static_cast<int64_t>(a.B) * a.nkt, a.err) = okv;
  }
  if (b == 0 && i == 0) *IPA_AT(a.headc, h, H, a.err) = kLog2e * a.w_L * ldf(a.gamma, h * a.gamma.s[0]) * a.w_C * 0.5f;
  const float c = kLog2e * a.w_L * ldf(a.gamma, h * a.gamma.s[0]) * a.w_C * 0.5f;

  const float4* fr = a.frame + (static_cast<int64_t>(b) * a.L + i) * 4;
  const float4 f0 = fr[0], f1 = fr[1], f2 = fr[2], f3 = fr[3];
  const float Rm[9] = {f0.x, f0.y, f0.z, f0.w, f1.x, f1.y, f1.z, f1.w, f2.x};
  const float tc[3] = {f2.y - cn.x, f2.z - cn.y, f2.w - cn.z};
  const bool valid = f3.x != 0.f;
  const float oqa[3] = {oqv.x, oqv.y, oqv.z}, oka[3] = {okv.x, okv.y, okv.z};

  float qs[C], ks[C], vs[C], qp[PQ * 3], kp[PQ * 3], vp[PV * 3];
  load_row(a.q, b * a.q.s[0] + i * a.q.s[1] + h * a.q.s[2], a.q.s[3], qs);
  load_row(a.k, b * a.k.s[0] + i * a.k.s[1] + h * a.k.s[2], a.k.s[3], ks);
  load_row(a.v, b * a.v.s[0] + i * a.v.s[1] + h * a.v.s[2], a.v.s[3], vs);
  auto load_pts = [&](const View& v, auto& dst) {
    const int64_t base = b * v.s[0] + i * v.s[1] + h * v.s[2];
    if (v.s[4] == 1 && v.s[3] == 3) {
      load_row(v, base, 1, dst);             // [points, xyz] dense
    } else {
      constexpr int NP = sizeof(dst) / sizeof(float) / 3;
#pragma unroll
      for (int p = 0; p < NP; ++p)
#pragma unroll
        for (int y = 0; y < 3; ++y) dst[3 * p + y] = ldf(v, base + p * v.s[3] + y * v.s[4]);
    }
  };
  load_pts(a.q_pts, qp);
  load_pts(a.k_pts, kp);
  load_pts(a.v_pts, vp);

  // frames applied: gq' = R q + t' - o_I, gk' = R k + t' - o_J, gv = R v + t'
  float gq[PQ * 3], gk[PQ * 3], gv[PV * 3];
#pragma unroll
  for (int p = 0; p < PQ; ++p)
#pragma unroll
    for (int x = 0; x < 3; ++x) {
      gq[3 * p + x] = fmaf(Rm[3 * x], qp[3 * p], fmaf(Rm[3 * x + 1], qp[3 * p + 1], Rm[3 * x + 2] * qp[3 * p + 2])) + tc[x] - oqa[x];
      gk[3 * p + x] = fmaf(Rm[3 * x], kp[3 * p], fmaf(Rm[3 * x + 1], kp[3 * p + 1], Rm[3 * x + 2] * kp[3 * p + 2])) + tc[x] - oka[x];
    }
#pragma unroll
  for (int p = 0; p < PV; ++p)
#pragma unroll
    for (int x = 0; x < 3; ++x)
      gv[3 * p + x] = fmaf(Rm[3 * x], vp[3 * p], fmaf(Rm[3 * x + 1], vp[3 * p + 1], Rm[3 * x + 2] * vp[3 * p + 2])) + tc[x];

  // rows are built and stored one after the other to keep few values live
  float sq[3] = {0.f, 0.f, 0.f}, sk[3] = {0.f, 0.f, 0.f}, nk = 0.f, nq = 0.f;
#pragma unroll
  for (int e = 0; e < 3 * PQ; ++e) {
    sq[e % 3] += gq[e];
    sk[e % 3] += gk[e];
    nk = fmaf(gk[e], gk[e], nk);
    nq = fmaf(gq[e], gq[e], nq);
  }
  // largest fp16 exponent field written, per half-word lane: a value that
  // does not survive the rounding (|x| >= 65520 -> inf, or NaN) has all
  // exponent bits set
  uint32_t emax = 0u;
  auto store_row = [&](uint4* dst, auto value_of) {
#pragma unroll
    for (int u = 0; u < DH / 8; ++u) {
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float x0 = value_of(8 * u + 2 * e), x1 = value_of(8 * u + 2 * e + 1);
        const uint32_t pk = pack_half2(x0, x1);
        emax = __vmaxu2(emax, pk & 0x7c007c00u);
        w[e] = valid ? pk : 0u;
      }
      dst[u] = make_uint4(w[0], w[1], w[2], w[3]);
    }
  };
  auto hi_of = [](float x) { return __half2float(__float2half_rn(x)); };
  // Q_h: [ scaled q | gq' hi | gq' hi | gq' lo | -1 -1 | 0 ]
  store_row(sq_rows, [&](int col) -> float {
    if (col < C) return a.qscale * qs[col];
    if (col < C + 9 * PQ) {
      const int u = col - C, part = u / (3 * PQ), e = u % (3 * PQ);
      const float hi = hi_of(gq[e]);
      return part < 2 ? hi : gq[e] - hi;
    }
    return col < C + 9 * PQ + 2 ? -1.f : 0.f;
  });
  // K_h: [ k | 2c gk' hi | lo | hi | c|gk'|^2 hi, lo | 0 ]
  store_row(sk_rows, [&](int col) -> float {
    if (col < C) return ks[col];
    if (col < C + 9 * PQ) {
      const int u = col - C, part = u / (3 * PQ), e = u % (3 * PQ);
      const float g = 2.f * c * gk[e], hi = hi_of(g);
      return part == 1 ? g - hi : hi;
    }
    if (col < C + 9 * PQ + 2) {
      const float n = c * nk, hi = hi_of(n);
      return col == C + 9 * PQ ? hi : n - hi;
    }
    return 0.f;
  });
  // V_h: [ v | gv hi | gv lo ]
  store_row(sv_rows, [&](int col) -> float {
    if (col < C) return vs[col];
    if (col < C + 6 * PV) {
      const int u = col - C, part = u / (3 * PV), e = u % (3 * PV);
      const float hi = hi_of(gv[e]);
      return part == 0 ? hi : gv[e] - hi;
    }
    return 0.f;
  });
  if (!valid) {
    sq[0] = sq[1] = sq[2] = 0.f;
    sk[0] = sk[1] = sk[2] = 0.f;
    nq = 0.f;
  }
  // .w: the row constant c sum_p |gq'_p|^2 that the fused pass leaves out of
  // its logits (it cancels in the softmax); a training forward adds it back
  // to report the log-sum-exp of the true logits
  sterm[slot] = make_float4(sq[0], sq[1], sq[2], c * nq);
  sterm[H * rb + slot] = make_float4(2.f * c * sk[0], 2.f * c * sk[1], 2.f * c * sk[2], valid ? 0.f : -INFINITY);
  // |x| >= 65520 (or NaN) does not survive the fp16 rounding
  if (valid && ((emax & 0xffffu) == 0x7c00u || (emax >> 16) == 0x7c00u)) record_error(a.err, DEV_NONFINITE);
  }
  __syncthreads();
  // each head plane's run of nrow rows, 16-byte stores, consecutive threads on
  // consecutive addresses
  uint4* const outs[3] = {a.qh, a.kh, a.vh};
  const int run = nrow * 8;                                        // uint4 per plane run
#pragma unroll
  for (int kind = 0; kind < 3; ++kind) {
    const uint4* src = stage_rows + static_cast<size_t>(kind * H * rb) * 8;
    for (int e = threadIdx.x; e < H * run; e += blockDim.x) {
      const int hh = e / run, r = e % run;
      *IPA_AT(outs[kind], (static_cast<int64_t>(b * H + hh) * a.L + i0) * 8 + r, static_cast<int64_t>(a.B) * H * a.L * 8,
              a.err) = src[hh * rb * 8 + r];
    }
  }
  for (int e = threadIdx.x; e < 2 * H * nrow; e += blockDim.x) {
    const int which = e / (H * nrow), rem = e % (H * nrow);
    const int hh = rem / nrow, r = rem % nrow;
    float4* dst = which == 0 ? a.rowq : a.colk;
    *IPA_AT(dst, static_cast<int64_t>(b * H + hh) * a.L + i0 + r, static_cast<int64_t>(a.B) * H * a.L, a.err) =
        sterm[which * H * rb + hh * rb + r];
  }
}

}  // namespace

cudaError_t ipa_launch_prologue(const IpaLaunch& a, cudaStream_t stream) {
  unsigned char* ws = a.ws;
  const IpaWorkspace& w = a.lay;

  TileArgs ta{};
  ta.B = a.B; ta.L = a.L; ta.R = a.R; ta.Cz = a.Cz; ta.RCz = a.RCz; ta.DZ = a.DZ; ta.nkt = a.nkt;
  ta.rot = a.rot; ta.trans = a.trans; ta.mask = a.mask; ta.z1 = a.z1; ta.z2 = a.z2;
  ta.frame = reinterpret_cast<float4*>(ws + w.frame);
  ta.part = reinterpret_cast<float4*>(ws + w.part);
  ta.z1f = reinterpret_cast<float*>(ws + w.z1f);
  ta.z2h = reinterpret_cast<__half*>(ws + w.z2);
  ta.z1h = reinterpret_cast<__half*>(ws + w.z1h);
  ta.err = a.err;
  ta.ticket = reinterpret_cast<int*>(ws + w.ticket);
  ta.nticket = static_cast<int>(2 * w.split_tiles);
  ipa_tile_kernel<<<dim3(a.nkt, a.B, a.DZ > 0 ? a.DZ / 64 : 1), 256, 0, stream>>>(ta);

  RowArgs r{};
  r.B = a.B; r.L = a.L; r.H = a.H; r.nqt = a.nqt; r.nkt = a.nkt; r.Cz = a.Cz; r.RCz = a.RCz; r.DZ = a.DZ;
  r.qscale = kLog2e * a.w_L * a.scalar_scale;
  r.w_L = a.w_L; r.w_C = a.w_C;
  r.q = a.q; r.k = a.k; r.v = a.v; r.q_pts = a.q_pts; r.k_pts = a.k_pts; r.v_pts = a.v_pts;
  r.gamma = a.gamma; r.w_bias = a.w_bias;
  r.frame = ta.frame; r.part = ta.part;
  r.cen = reinterpret_cast<float4*>(ws + w.cen);
  r.oq = reinterpret_cast<float4*>(ws + w.oq);
  r.ok = reinterpret_cast<float4*>(ws + w.ok);
  r.headc = reinterpret_cast<float*>(ws + w.headc);
  r.wqp = reinterpret_cast<float*>(ws + w.wqp);
  r.qh = reinterpret_cast<uint4*>(ws + w.qh);
  r.kh = reinterpret_cast<uint4*>(ws + w.kh);
  r.vh = reinterpret_cast<uint4*>(ws + w.vh);
  r.rowq = reinterpret_cast<float4*>(ws + w.rowq);
  r.colk = reinterpret_cast<float4*>(ws + w.colk);
  r.err = a.err;
  r.rb = 128 / a.H;
  const size_t smem = static_cast<size_t>(a.H) * r.rb * (3 * DH * 2 + 2 * 16);
  // the largest request is 128 rows x 416 B
  const cudaError_t e = cudaFuncSetAttribute(ipa_rows_kernel<IPA_C, IPA_PQ, IPA_PV>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, 128 * (3 * DH * 2 + 2 * 16));
  if (e != cudaSuccess) return e;
  const dim3 grid(static_cast<unsigned>((a.L + r.rb - 1) / r.rb), static_cast<unsigned>(a.B));
  ipa_rows_kernel<IPA_C, IPA_PQ, IPA_PV><<<grid, 128, smem, stream>>>(r);
  return cudaGetLastError();
}

IpaWorkspace ipa_workspace_layout(int B, int L, int H, int DZ, int RCz, bool with_split) {
  (void)RCz;
  auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  IpaWorkspace w{};
  size_t o = 0;
  const size_t bhl = static_cast<size_t>(B) * H * L, bl = static_cast<size_t>(B) * L;
  const int nqt = (L + QT - 1) / QT, nkt = (L + KT - 1) / KT;
  w.qh = o; o = up(o + bhl * DH * 2);
  w.kh = o; o = up(o + bhl * DH * 2);
  w.vh = o; o = up(o + bhl * DH * 2);
  w.z2 = o; o = up(o + bl * DZ * 2);
  w.z1h = o; o = up(o + bl * DZ * 2);
  w.z1f = o; o = up(o + bl * DZ * 4);
  w.rowq = o; o = up(o + bhl * 16);
  w.colk = o; o = up(o + bhl * 16);
  w.frame = o; o = up(o + bl * 64);
  w.part = o; o = up(o + static_cast<size_t>(B) * nkt * 16);
  w.cen = o; o = up(o + static_cast<size_t>(B) * 16);
  w.oq = o; o = up(o + static_cast<size_t>(B) * nqt * 16);
  w.ok = o; o = up(o + static_cast<size_t>(B) * nkt * 16);
  w.headc = o; o = up(o + static_cast<size_t>(H) * 4);
  w.wqp = o; o = up(o + static_cast<size_t>(H) * DZ * 4);
  w.err = o; o = up(o + 16);
  w.split = w.ticket = o;
  if (with_split && ipa_pair_supported(DZ)) {
    const int64_t T = static_cast<int64_t>(B) * H * ((L + 255) / 256);
    w.split_tiles = T < kSplitPairs ? T : kSplitPairs;
    w.split_chunks = 2 * w.split_tiles;
    w.split = o; o = up(o + static_cast<size_t>(w.split_chunks) * 2 * (DZ + 67) * 128 * 4);
    w.ticket = o; o = up(o + static_cast<size_t>(w.split_tiles) * 2 * 4);
  }
  w.total = o;
  return w;
}

}  // namespace fipa
