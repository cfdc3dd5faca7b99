// Gradients of the geometric direction-and-distance attention for sm_100a
// ("Geometric direction-and-distance attention", Required behavior: the
// operator is differentiated with the derivative of the unsquared distance
// at a zero displacement defined as the zero vector).
//
// With s_ij = (A <qd_i, kd_j> - B |qp_i - kp_j|) / sqrt(3), a = masked
// softmax_j(s), agg_i = sum_j a_ij vr_j and upstream gradients g_output,
// g_attention, g_vectors:
//   g_vec_i  = g_vectors_i + [i has an allowed key] g_output_i W^T
//   dagg_i   = R_i g_vec_i,   da_ij = <dagg_i, vr_j> + g_attention_ij
//   ds_ij    = a_ij (da_ij - D_i),  D_i = sum_j a_ij da_ij
//            = <dagg_i, agg_i> + sum_j a_ij g_attention_ij
//   d qd_i   =  A/sqrt3 sum_j ds_ij kd_j,   d qp_i = -B/sqrt3 sum_j ds_ij u_ij
//   d kd_j   =  A/sqrt3 sum_i ds_ij qd_i,   d kp_j =  B/sqrt3 sum_i ds_ij u_ij
//   d vr_j   =  sum_i a_ij dagg_i,  u_ij = (qp_i - kp_j) / |qp_i - kp_j| or 0
// Launches (all fp32 on CUDA cores; the per-pair terms are recomputed, no
// N x N array is stored):
//   0. the forward statistics (scales, rotated inputs, row max / sum, agg)
//   1. geo_gvec_kernel     -- g_vec (a register-tiled product, 64 rows x 32
//                             columns per block) and whether any head is live
//   2. geo_dagg_kernel     -- per (b, n, h): dagg = R g_vec, <dagg, agg>
//   3. geo_dw_part_kernel / geo_dw_sum_kernel -- dW = vec^T g_output and
//                             db = sum g_output over live rows, per 128-row
//                             chunk (register-tiled), then summed in a fixed
//                             order
//   4. geo_bwd_rows_kernel -- per (b, h, 128 queries) x 4 key splits: D_i,
//                             then d qd, d qp and the per-head sums of
//                             ds <qd, kd> and ds |qp - kp|
//   5. geo_bwd_cols_kernel -- per (b, h, 128 keys) x 4 query splits: d kd,
//                             d kp, d vr
//   6. geo_bwd_frame_kernel -- per (b, n, h): local gradients R^T (...) and
//                             the head's frame terms, summed over heads in
//                             order into the rotation and translation
//                             gradients; block 0 also writes the scale
//                             gradients.
#include <cmath>
#include <cstdint>

#include "bounds.cuh"
#include "geo_common.cuh"
#include "internal.h"
#include "sm100.cuh"

#define IPA_FILE_TAG 6

namespace fipa {

using namespace sm100;
using namespace geo;

namespace {

constexpr int BW_ROWS = 128;
constexpr int BW_SPLIT = 4;
constexpr int BW_CHUNK = 32;
constexpr float kInvSqrt3 = 0.57735026918962576f;

struct GvecArgs {
  int B, N, H, HM3, Cout;
  View g_output, g_vectors;
  bool has_g_vectors;
  const unsigned char* live;   // [B, N, H]
  const float* wt;             // [Cout, HM3]
  float* gvec;                 // [B*N, HM3]
  unsigned char* rowlive;      // [B*N]
  int* err;
};

// g_vec = g_vectors + [row live] g_output W^T: a 64-row x 32-column tile of
// g_vec per block (tile_product over the Cout columns of g_output); rows with
// no live head pass no g_output on.
constexpr int GV_TM = 64, GV_TN = 32;
__global__ void __launch_bounds__(256) geo_gvec_kernel(const GvecArgs a) {
  __shared__ int64_t goff[GV_TM];   // g_output offset of each row, -1 if it passes nothing on
  const int64_t rows = static_cast<int64_t>(a.B) * a.N;
  const int r0 = blockIdx.x * GV_TM, c0 = blockIdx.y * GV_TN;
  if (threadIdx.x < GV_TM) {
    const int64_t row = r0 + static_cast<int>(threadIdx.x);
    int l = 0;
    if (row < rows)
      for (int h = 0; h < a.H; ++h) l |= a.live[row * a.H + h] != 0;
    const int b = static_cast<int>(row / a.N), n = static_cast<int>(row % a.N);
    goff[threadIdx.x] = (row < rows && l) ? b * a.g_output.s[0] + n * a.g_output.s[1] : -1;
    if (blockIdx.y == 0 && row < rows) *IPA_AT(a.rowlive, row, rows, a.err) = l ? 1 : 0;
  }
  __syncthreads();
  const int64_t sc = a.g_output.s[2];
  float acc[GV_TM / 16][GV_TN / 16];
  tile_product<GV_TM, GV_TN>(
      r0, c0, a.Cout,
      [&](int r, int c) {
        const int64_t off = goff[r - r0];
        return (c < a.Cout && off >= 0) ? ldf(a.g_output, off + c * sc) : 0.f;
      },
      [&](int c, int kx) { return (c < a.Cout && kx < a.HM3) ? a.wt[static_cast<int64_t>(c) * a.HM3 + kx] : 0.f; },
      acc);
  const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
#pragma unroll
  for (int j = 0; j < GV_TN / 16; ++j) {
    const int kx = c0 + tx + 16 * j;
    if (kx >= a.HM3) continue;
    const int h = kx / (a.HM3 / a.H), mx = kx % (a.HM3 / a.H), m = mx / 3, x = mx % 3;
#pragma unroll
    for (int i = 0; i < GV_TM / 16; ++i) {
      const int64_t row = r0 + ty + 16 * i;
      if (row >= rows) continue;
      float g = acc[i][j];
      if (a.has_g_vectors) {
        const int b = static_cast<int>(row / a.N), n = static_cast<int>(row % a.N);
        const View& v = a.g_vectors;
        g += ldf(v, b * v.s[0] + n * v.s[1] + h * v.s[2] + m * v.s[3] + x * v.s[4]);
      }
      *IPA_AT(a.gvec, row * a.HM3 + kx, rows * a.HM3, a.err) = g;
    }
  }
}

struct DaggArgs {
  int B, N, H, M, VW, HM3;
  const float* gvec;   // [B*N, HM3]
  const float* rotf;   // [B, N, 9]
  const float* agg;    // [B*H, N, VW]
  float* dagg;         // [B*H, N, VW]
  float4* rowinfo;     // [B*H, N]: .z <- <dagg, agg>
  int* err;
};

__global__ void __launch_bounds__(256) geo_dagg_kernel(const DaggArgs a) {
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= static_cast<int64_t>(a.B) * a.N * a.H) return;
  const int h = static_cast<int>(t % a.H);
  const int64_t bn = t / a.H;
  const int b = static_cast<int>(bn / a.N), n = static_cast<int>(bn % a.N);
  const float* R = a.rotf + bn * 9;
  const float* g = a.gvec + bn * a.HM3 + h * 3 * a.M;
  const int64_t row = (static_cast<int64_t>(b) * a.H + h) * a.N + n;
  const float* ag = a.agg + row * a.VW;
  const int64_t nbhn = static_cast<int64_t>(a.B) * a.N * a.H;
  float* dst = IPA_SPAN(a.dagg, row * a.VW, 3 * a.M, nbhn * a.VW, a.err);
  float d1 = 0.f;
  for (int m = 0; m < a.M; ++m) {
#pragma unroll
    for (int x = 0; x < 3; ++x) {
      const float v = fmaf(R[3 * x], g[3 * m], fmaf(R[3 * x + 1], g[3 * m + 1], R[3 * x + 2] * g[3 * m + 2]));
      dst[3 * m + x] = v;
      d1 = fmaf(v, ag[3 * m + x], d1);
    }
  }
  *IPA_AT(a.rowinfo, row, nbhn, a.err) = make_float4(0.f, 0.f, d1, 0.f);
}

constexpr int DW_ROWS = 128;

struct DwArgs {
  int64_t rows;
  int HM3, Cout, N, nchunk;
  View g_output;
  const float* vec;                // [rows, HM3]
  const unsigned char* rowlive;    // [rows]
  float* part_w;                   // [nchunk, HM3, Cout]
  float* part_b;                   // [nchunk, Cout]
  float* d_w;                      // [HM3, Cout]
  float* d_b;                      // [Cout] or null
  int* err;
};

// Partial dW over one chunk of 128 rows: the 32 x 64 tile (k, c) of
// vec^T g_output summed over the chunk's rows in order (tile_product, rows
// that pass nothing on contribute zeros); the first k tile also sums the
// chunk's g_output rows for db.
constexpr int DW_TM = 32, DW_TN = 64;
__global__ void __launch_bounds__(256) geo_dw_part_kernel(const DwArgs a) {
  __shared__ int64_t goff[DW_ROWS];   // g_output offset of each row, -1 if it passes nothing on
  const int k0 = blockIdx.x * DW_TM, c0 = blockIdx.y * DW_TN;
  const int64_t r0 = static_cast<int64_t>(blockIdx.z) * DW_ROWS;
  for (int rr = threadIdx.x; rr < DW_ROWS; rr += blockDim.x) {
    const int64_t row = r0 + rr;
    int64_t off = -1;
    if (row < a.rows && a.rowlive[row]) {
      const int b = static_cast<int>(row / a.N), n = static_cast<int>(row % a.N);
      off = b * a.g_output.s[0] + n * a.g_output.s[1];
    }
    goff[rr] = off;
  }
  __syncthreads();
  const int64_t sc = a.g_output.s[2];
  float acc[DW_TM / 16][DW_TN / 16];
  tile_product<DW_TM, DW_TN>(
      k0, c0, DW_ROWS,
      [&](int k, int rr) { return (k < a.HM3 && r0 + rr < a.rows) ? a.vec[(r0 + rr) * a.HM3 + k] : 0.f; },
      [&](int rr, int c) { return (c < a.Cout && goff[rr] >= 0) ? ldf(a.g_output, goff[rr] + c * sc) : 0.f; },
      acc);
  const int64_t nwc = static_cast<int64_t>(a.HM3) * a.Cout;
  const int64_t pw0 = static_cast<int64_t>(blockIdx.z) * nwc;
  const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
#pragma unroll
  for (int i = 0; i < DW_TM / 16; ++i) {
    const int k = k0 + ty + 16 * i;
    if (k >= a.HM3) continue;
#pragma unroll
    for (int j = 0; j < DW_TN / 16; ++j) {
      const int c = c0 + tx + 16 * j;
      if (c < a.Cout) *IPA_AT(a.part_w, pw0 + static_cast<int64_t>(k) * a.Cout + c, a.nchunk * nwc, a.err) = acc[i][j];
    }
  }
  if (blockIdx.x == 0 && threadIdx.x < DW_TN && c0 + static_cast<int>(threadIdx.x) < a.Cout) {
    const int c = c0 + threadIdx.x;
    float accb = 0.f;
    for (int rr = 0; rr < DW_ROWS; ++rr)
      if (goff[rr] >= 0) accb += ldf(a.g_output, goff[rr] + c * sc);
    *IPA_AT(a.part_b, static_cast<int64_t>(blockIdx.z) * a.Cout + c, static_cast<int64_t>(a.nchunk) * a.Cout, a.err) = accb;
  }
}

// dW and db: the chunk partials summed in a fixed order (deterministic).
__global__ void __launch_bounds__(256) geo_dw_sum_kernel(const DwArgs a) {
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t nw = static_cast<int64_t>(a.HM3) * a.Cout;
  if (t < nw) {
    float s = 0.f;
    for (int z = 0; z < a.nchunk; ++z) s += a.part_w[z * nw + t];
    *IPA_AT(a.d_w, t, nw, a.err) = s;
  }
  if (t < a.Cout && a.d_b) {
    float s = 0.f;
    for (int z = 0; z < a.nchunk; ++z) s += a.part_b[static_cast<int64_t>(z) * a.Cout + t];
    *IPA_AT(a.d_b, t, a.Cout, a.err) = s;
  }
}

struct PairArgs {
  int B, N, H, VW;
  const float4* qg;      // [B*H, N, 2]
  const float4* kg;      // [B*H, N, 2]
  const float* vg;       // [B*H, N, VW]
  const float2* sc;      // [H]
  const float2* ml;      // [B*H, N]
  const float* dagg;     // [B*H, N, VW]
  float4* rowinfo;       // [B*H, N]: (m, 1/l or 0, D, 0)
  const unsigned char* pm;
  int64_t pms[4];
  View g_att;
  bool has_g_att;
  float4* dq;            // [B*H, N, 2]: (d qd, 0), (d qp, 0) in the global frame
  float4* dk;            // [B*H, N, 2]
  float* dvr;            // [B*H, N, VW]
  float* acc;            // [B, H, row blocks, 4 warps, 2]: per-warp sums of ds <qd, kd> and ds |qp - kp|
  int* err;
};

__device__ __forceinline__ float g_att_at(const PairArgs& a, int b, int h, int i, int j) {
  const View& v = a.g_att;
  return ldf(v, b * v.s[0] + h * v.s[1] + static_cast<int64_t>(i) * v.s[2] + static_cast<int64_t>(j) * v.s[3]);
}

// two 512-thread blocks per SM (<= 64 registers) where the accumulators allow it
template <int M>
__global__ void __launch_bounds__(BW_ROWS * BW_SPLIT, M <= 4 ? 2 : 1) geo_bwd_rows_kernel(const PairArgs a) {
  constexpr int V = 3 * M;
  const int tid = threadIdx.x;
  const int r = tid % BW_ROWS, split = tid / BW_ROWS;
  const int h = blockIdx.y, b = blockIdx.z;
  const int i = blockIdx.x * BW_ROWS + r;
  const int N = a.N;
  const int64_t bh = static_cast<int64_t>(b) * a.H + h;
  const float2 sc = a.sc[h];
  const bool in_range = i < N;
  float4 q0 = make_float4(0, 0, 0, 0), q1 = q0;
  float m = 0.f, inv = 0.f, d1 = 0.f;
  float dg[V];
#pragma unroll
  for (int e = 0; e < V; ++e) dg[e] = 0.f;
  if (in_range) {
    const float2 st = a.ml[bh * N + i];
    if (st.y > 0.f) {
      m = st.x;
      inv = 1.f / st.y;
      q0 = a.qg[2 * (bh * N + i)];
      q1 = a.qg[2 * (bh * N + i) + 1];
      d1 = a.rowinfo[bh * N + i].z;
#pragma unroll
      for (int e = 0; e < V; ++e) dg[e] = a.dagg[(bh * N + i) * a.VW + e];
    }
  }
  const bool live = inv > 0.f;
  const unsigned char* pmrow =
      a.pm ? a.pm + b * a.pms[0] + h * a.pms[1] + static_cast<int64_t>(in_range ? i : 0) * a.pms[2] : nullptr;
  const int nchunk = (N + BW_CHUNK - 1) / BW_CHUNK;
  extern __shared__ float bw_merge[];   // [BW_SPLIT][8][BW_ROWS], the staged keys, the g_attention tiles
  auto sm_at = [&](int s2, int e) -> float& { return bw_merge[(s2 * 8 + e) * BW_ROWS + r]; };

  // keys of one 32-key chunk staged per split group: [k0 | k1 | vr (padded)];
  // with g_attention, also the group's 128 x 32 tile of it (rows padded to 33
  // floats), loaded row-contiguous so a warp reads 128 consecutive bytes
  constexpr int SW = 8 + ((V + 3) & ~3);
  constexpr int GP = BW_CHUNK + 1;
  float* stg = bw_merge + BW_SPLIT * 8 * BW_ROWS + split * BW_CHUNK * SW;
  float* gst = bw_merge + BW_SPLIT * (8 * BW_ROWS + BW_CHUNK * SW) + split * BW_ROWS * GP;
  const uint32_t gbar = 1 + split;
  const int row0 = blockIdx.x * BW_ROWS;
  auto stage_chunk = [&](int j0) {
    named_bar_sync(gbar, BW_ROWS);                 // the previous chunk has been read
    for (int e = r; e < BW_CHUNK * SW; e += BW_ROWS) {
      const int it = e / SW, f = e % SW, j = j0 + it;
      float v = 0.f;
      if (j < N) {
        if (f < 8) v = reinterpret_cast<const float*>(a.kg)[8 * (bh * N + j) + f];
        else if (f - 8 < V) v = a.vg[(bh * N + j) * a.VW + (f - 8)];
      } else if (f == 3) {
        v = -INFINITY;                             // beyond N: never allowed
      }
      stg[e] = v;
    }
    if (a.has_g_att)
      for (int e = r; e < BW_ROWS * BW_CHUNK; e += BW_ROWS) {
        const int rr = e / BW_CHUNK, kk = e % BW_CHUNK, ii = row0 + rr, jj = j0 + kk;
        gst[rr * GP + kk] = (ii < N && jj < N) ? g_att_at(a, b, h, ii, jj) : 0.f;
      }
    named_bar_sync(gbar, BW_ROWS);
  };
  // bit k: key j0 + k allowed by the pair mask (a dense, 16-byte aligned
  // row of 32 bytes is read as two 16-byte words)
  auto chunk_mask = [&](int j0) -> uint32_t {
    uint32_t allowed = 0xffffffffu;
    if (pmrow) {
      allowed = 0u;
      const unsigned char* pr = pmrow + static_cast<int64_t>(j0) * a.pms[3];
      if (a.pms[3] == 1 && j0 + BW_CHUNK <= N && (reinterpret_cast<uintptr_t>(pr) & 15u) == 0) {
        const uint4 u0 = *reinterpret_cast<const uint4*>(pr);
        const uint4 u1 = *reinterpret_cast<const uint4*>(pr + 16);
        const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
        for (int q = 0; q < BW_CHUNK / 4; ++q) allowed |= nonzero_byte_bits(w[q]) << (4 * q);
      } else {
        for (int k = 0; k < BW_CHUNK && j0 + k < N; ++k) allowed |= pr[k * a.pms[3]] ? (1u << k) : 0u;
      }
    }
    return allowed;
  };

  // D_i = <dagg_i, agg_i> + sum_j a_ij g_attention_ij
  float dsum = 0.f;
  if (a.has_g_att) {
    for (int ch = split; ch < nchunk; ch += BW_SPLIT) {
      const int j0 = ch * BW_CHUNK;
      stage_chunk(j0);
      if (!live) continue;
      const uint32_t allowed = chunk_mask(j0);
      for (int k = 0; k < BW_CHUNK; ++k) {
        if (!((allowed >> k) & 1u)) continue;
        const float4 k0 = *reinterpret_cast<const float4*>(stg + k * SW);
        const float4 k1 = *reinterpret_cast<const float4*>(stg + k * SW + 4);
        const float p = ex2(geo_score(q0, q1, k0, k1, sc.x, sc.y) - m) * inv;   // 0 beyond N
        dsum = fmaf(p, gst[r * GP + k], dsum);
      }
    }
  }
  sm_at(split, 0) = dsum;
  __syncthreads();
  float D = d1;
#pragma unroll
  for (int s2 = 0; s2 < BW_SPLIT; ++s2) D += sm_at(s2, 0);
  __syncthreads();

  float cq[3] = {0.f, 0.f, 0.f}, cp[3] = {0.f, 0.f, 0.f}, sdot = 0.f, sdist = 0.f;
  for (int ch = split; ch < nchunk; ch += BW_SPLIT) {
    const int j0 = ch * BW_CHUNK;
    stage_chunk(j0);
    if (!live) continue;
    const uint32_t allowed = chunk_mask(j0);
    for (int k = 0; k < BW_CHUNK; ++k) {
      if (!((allowed >> k) & 1u)) continue;
      const float* kk = stg + k * SW;
      const float4 k0 = *reinterpret_cast<const float4*>(kk), k1 = *reinterpret_cast<const float4*>(kk + 4);
      const GeoPair g = geo_pair(q0, q1, k0, k1, sc.x, sc.y);
      const float p = ex2(g.s - m) * inv;
      if (p == 0.f) continue;
      float da = a.has_g_att ? gst[r * GP + k] : 0.f;
      {
        // the key's V rotated values as 16-byte loads (rows of SW floats, SW % 4 == 0)
        const float4* kv = reinterpret_cast<const float4*>(kk + 8);
#pragma unroll
        for (int e4 = 0; e4 < (V + 3) / 4; ++e4) {
          const float4 w = kv[e4];
          const float wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int u = 0; u < 4; ++u)
            if (4 * e4 + u < V) da = fmaf(dg[4 * e4 + u], wv[u], da);
        }
      }
      const float ds = p * (da - D);
      cq[0] = fmaf(ds, k0.x, cq[0]);
      cq[1] = fmaf(ds, k0.y, cq[1]);
      cq[2] = fmaf(ds, k0.z, cq[2]);
      const float ru = g.dist > 0.f ? __fdividef(ds, g.dist) : 0.f;   // zero displacement: zero derivative
      cp[0] = fmaf(ru, g.dx, cp[0]);
      cp[1] = fmaf(ru, g.dy, cp[1]);
      cp[2] = fmaf(ru, g.dz, cp[2]);
      sdot = fmaf(ds, g.dot, sdot);
      sdist = fmaf(ds, g.dist, sdist);
    }
  }
  sm_at(split, 0) = cq[0]; sm_at(split, 1) = cq[1]; sm_at(split, 2) = cq[2];
  sm_at(split, 3) = cp[0]; sm_at(split, 4) = cp[1]; sm_at(split, 5) = cp[2];
  sm_at(split, 6) = sdot;  sm_at(split, 7) = sdist;
  __syncthreads();
  if (split != 0) return;
  float t[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    t[e] = 0.f;
#pragma unroll
    for (int s2 = 0; s2 < BW_SPLIT; ++s2) t[e] += sm_at(s2, e);
  }
  const float Ar = sc.x / kLog2e, Br = sc.y / kLog2e;   // A / sqrt3, B / sqrt3
  if (in_range) {
    const int64_t nbhn = static_cast<int64_t>(a.B) * a.H * N;
    float4* dq = IPA_SPAN(a.dq, 2 * (bh * N + i), 2, 2 * nbhn, a.err);
    dq[0] = make_float4(Ar * t[0], Ar * t[1], Ar * t[2], 0.f);
    dq[1] = make_float4(-Br * t[3], -Br * t[4], -Br * t[5], 0.f);
    *IPA_AT(a.rowinfo, bh * N + i, nbhn, a.err) = make_float4(m, inv, D, 0.f);
  }
  // per-head sums over the block's rows (warps 0-3 hold split 0)
  float s6 = t[6], s7 = t[7];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    s6 += __shfl_xor_sync(0xffffffffu, s6, o);
    s7 += __shfl_xor_sync(0xffffffffu, s7, o);
  }
  if ((tid & 31) == 0) {     // one slot per (b, h, row block, warp), summed in a fixed order later
    const int64_t slot = ((bh * gridDim.x + blockIdx.x) * 4 + (tid >> 5)) * 2;
    float* ap = IPA_SPAN(a.acc, slot, 2, static_cast<int64_t>(a.B) * a.H * gridDim.x * 8, a.err);
    ap[0] = s6;
    ap[1] = s7;
  }
}

template <int M>
__global__ void __launch_bounds__(BW_ROWS * BW_SPLIT, M <= 4 ? 2 : 1) geo_bwd_cols_kernel(const PairArgs a) {
  constexpr int V = 3 * M;
  const int tid = threadIdx.x;
  const int r = tid % BW_ROWS, split = tid / BW_ROWS;
  const int h = blockIdx.y, b = blockIdx.z;
  const int j = blockIdx.x * BW_ROWS + r;
  const int N = a.N;
  const int64_t bh = static_cast<int64_t>(b) * a.H + h;
  const float2 sc = a.sc[h];
  const bool in_range = j < N;
  float4 k0 = make_float4(0, 0, 0, -INFINITY), k1 = make_float4(0, 0, 0, 0);
  float vr[V];
#pragma unroll
  for (int e = 0; e < V; ++e) vr[e] = 0.f;
  if (in_range) {
    k0 = a.kg[2 * (bh * N + j)];
    k1 = a.kg[2 * (bh * N + j) + 1];
#pragma unroll
    for (int e = 0; e < V; ++e) vr[e] = a.vg[(bh * N + j) * a.VW + e];
  }
  float ck[3] = {0.f, 0.f, 0.f}, cp[3] = {0.f, 0.f, 0.f}, dv[V];
#pragma unroll
  for (int e = 0; e < V; ++e) dv[e] = 0.f;
  const unsigned char* pmcol =
      a.pm ? a.pm + b * a.pms[0] + h * a.pms[1] + static_cast<int64_t>(in_range ? j : 0) * a.pms[3] : nullptr;
  const int nchunk = (N + BW_CHUNK - 1) / BW_CHUNK;
  const bool active = in_range && k0.w == 0.f;
  extern __shared__ float bw_merge[];   // [BW_SPLIT][6 + V][BW_ROWS], then the staged queries
  // queries of one 32-query chunk staged per split group: [rowinfo | q0 | q1 | dagg (padded)]
  constexpr int SW = 12 + ((V + 3) & ~3);
  float* stg = bw_merge + BW_SPLIT * (6 + V) * BW_ROWS + split * BW_CHUNK * SW;
  const uint32_t gbar = 1 + split;
  for (int ch = split; ch < nchunk; ch += BW_SPLIT) {
    const int i0 = ch * BW_CHUNK;
    named_bar_sync(gbar, BW_ROWS);
    for (int e = r; e < BW_CHUNK * SW; e += BW_ROWS) {
      const int it = e / SW, f = e % SW, i = i0 + it;
      float v = 0.f;
      if (i < N) {
        if (f < 4) v = reinterpret_cast<const float*>(a.rowinfo)[4 * (bh * N + i) + f];
        else if (f < 12) v = reinterpret_cast<const float*>(a.qg)[8 * (bh * N + i) + (f - 4)];
        else if (f - 12 < V) v = a.dagg[(bh * N + i) * a.VW + (f - 12)];
      }
      stg[e] = v;                                  // beyond N: rowinfo.y = 0, skipped
    }
    named_bar_sync(gbar, BW_ROWS);
    if (!active) continue;
    // bit k: query i0 + k allowed with this key by the pair mask (the 32
    // bytes down this key's column loaded together)
    uint32_t allowed = 0xffffffffu;
    if (pmcol) {
      allowed = 0u;
#pragma unroll
      for (int k = 0; k < BW_CHUNK; ++k)
        if (i0 + k < N && pmcol[static_cast<int64_t>(i0 + k) * a.pms[2]]) allowed |= 1u << k;
    }
    for (int k = 0; k < BW_CHUNK; ++k) {
      const float* qq = stg + k * SW;
      const float4 info = *reinterpret_cast<const float4*>(qq);
      if (info.y == 0.f) continue;                 // query without an allowed key
      const int i = i0 + k;
      if (!((allowed >> k) & 1u)) continue;
      const float4 q0 = *reinterpret_cast<const float4*>(qq + 4), q1 = *reinterpret_cast<const float4*>(qq + 8);
      const GeoPair g = geo_pair(q0, q1, k0, k1, sc.x, sc.y);
      const float p = ex2(g.s - info.x) * info.y;
      if (p == 0.f) continue;
      float da = a.has_g_att ? g_att_at(a, b, h, i, j) : 0.f;
      // the query's V dagg values as 16-byte loads (rows of SW floats, SW % 4 == 0)
      float dq[(V + 3) & ~3];
#pragma unroll
      for (int e4 = 0; e4 < (V + 3) / 4; ++e4) {
        const float4 w = reinterpret_cast<const float4*>(qq + 12)[e4];
        dq[4 * e4] = w.x; dq[4 * e4 + 1] = w.y; dq[4 * e4 + 2] = w.z; dq[4 * e4 + 3] = w.w;
      }
#pragma unroll
      for (int e = 0; e < V; ++e) da = fmaf(dq[e], vr[e], da);
      const float ds = p * (da - info.z);
      ck[0] = fmaf(ds, q0.x, ck[0]);
      ck[1] = fmaf(ds, q0.y, ck[1]);
      ck[2] = fmaf(ds, q0.z, ck[2]);
      const float ru = g.dist > 0.f ? __fdividef(ds, g.dist) : 0.f;
      cp[0] = fmaf(ru, g.dx, cp[0]);
      cp[1] = fmaf(ru, g.dy, cp[1]);
      cp[2] = fmaf(ru, g.dz, cp[2]);
#pragma unroll
      for (int e = 0; e < V; ++e) dv[e] = fmaf(p, dq[e], dv[e]);
    }
  }
  __syncthreads();
  auto sm_at = [&](int s2, int e) -> float& { return bw_merge[(s2 * (6 + V) + e) * BW_ROWS + r]; };
#pragma unroll
  for (int e = 0; e < 3; ++e) {
    sm_at(split, e) = ck[e];
    sm_at(split, 3 + e) = cp[e];
  }
#pragma unroll
  for (int e = 0; e < V; ++e) sm_at(split, 6 + e) = dv[e];
  __syncthreads();
  if (split != 0 || !in_range) return;
  float t[6 + V];
#pragma unroll
  for (int e = 0; e < 6 + V; ++e) {
    t[e] = 0.f;
#pragma unroll
    for (int s2 = 0; s2 < BW_SPLIT; ++s2) t[e] += sm_at(s2, e);
  }
  const float Ar = sc.x / kLog2e, Br = sc.y / kLog2e;
  const int64_t nbhn = static_cast<int64_t>(a.B) * a.H * N;
  float4* dk = IPA_SPAN(a.dk, 2 * (bh * N + j), 2, 2 * nbhn, a.err);
  dk[0] = make_float4(Ar * t[0], Ar * t[1], Ar * t[2], 0.f);
  dk[1] = make_float4(Br * t[3], Br * t[4], Br * t[5], 0.f);   // u points from kp to qp
  float* dvr = IPA_SPAN(a.dvr, (bh * N + j) * a.VW, V, nbhn * a.VW, a.err);
#pragma unroll
  for (int e = 0; e < V; ++e) dvr[e] = t[6 + e];
}

struct FrameArgs {
  int B, N, H, M, VW, HM3;
  View qd, kd, qp, kp, val, dscale, xscale;
  const float* rotf;
  const float* agg;      // [B*H, N, VW]
  const float* gvec;     // [B*N, HM3]
  const float4* dq;
  const float4* dk;
  const float* dvr;
  const float* acc;      // [B, H, nrb, 4, 2] per-warp partial sums (geo_bwd_rows_kernel)
  int nrb;               // row blocks per (b, h)
  float *d_qd, *d_kd, *d_qp, *d_kp, *d_val, *d_rot, *d_trans, *d_dscale, *d_xscale;
  int* err;
};

// Block: rb = 128 / H residues x all heads, thread (residue, head): the
// local-frame gradients of its head's inputs and that head's terms of the
// frame gradient, which are then summed over heads in order (through shared
// memory) into d R and d t of the residue.  Block 0 also finishes the two
// scale gradients.
__global__ void __launch_bounds__(128) geo_bwd_frame_kernel(const FrameArgs a) {
  __shared__ float fterm[128 * 12];   // [rb][H][12]: d R (9), d t (3) per head
  const int H = a.H, rb = 128 / H;
  const int il = threadIdx.x / H, h = threadIdx.x % H;
  const int64_t rows = static_cast<int64_t>(a.B) * a.N;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * rb + il;
  const bool active = il < rb && t < rows;
  if (blockIdx.x == 0)
    for (int hh = threadIdx.x; hh < H; hh += blockDim.x) {
      // d scale = dA sigmoid(scale); dA = sum ds dot / sqrt3, dB = -sum ds dist / sqrt3
      const float xd = ldf(a.dscale, hh * a.dscale.s[0]), xx = ldf(a.xscale, hh * a.xscale.s[0]);
      double sd = 0.0, sx = 0.0;   // fixed summation order: batch, row block, warp
      for (int b = 0; b < a.B; ++b)
        for (int k = 0; k < a.nrb * 4; ++k) {
          const int64_t slot = ((static_cast<int64_t>(b) * H + hh) * a.nrb * 4 + k) * 2;
          sd += a.acc[slot];
          sx += a.acc[slot + 1];
        }
      *IPA_AT(a.d_dscale, hh, H, a.err) = static_cast<float>(sd) * kInvSqrt3 / (1.f + expf(-xd));
      *IPA_AT(a.d_xscale, hh, H, a.err) = -static_cast<float>(sx) * kInvSqrt3 / (1.f + expf(-xx));
    }
  if (active) {
    const int b = static_cast<int>(t / a.N), n = static_cast<int>(t % a.N);
    const float* R = a.rotf + t * 9;
    float Rm[9];
#pragma unroll
    for (int e = 0; e < 9; ++e) Rm[e] = R[e];
    float dR[9], dT[3];
#pragma unroll
    for (int e = 0; e < 9; ++e) dR[e] = 0.f;
    // local gradient R^T g and dR += g x^T for one rotated 3-vector x
    auto back = [&](const float g[3], const View& v, int64_t base, int64_t sx, float* out) {
      const float x0 = ldf(v, base), x1 = ldf(v, base + sx), x2 = ldf(v, base + 2 * sx);
#pragma unroll
      for (int y = 0; y < 3; ++y) out[y] = fmaf(Rm[y], g[0], fmaf(Rm[3 + y], g[1], Rm[6 + y] * g[2]));
#pragma unroll
      for (int x = 0; x < 3; ++x) {
        dR[3 * x] = fmaf(g[x], x0, dR[3 * x]);
        dR[3 * x + 1] = fmaf(g[x], x1, dR[3 * x + 1]);
        dR[3 * x + 2] = fmaf(g[x], x2, dR[3 * x + 2]);
      }
    };
    const int64_t row = (static_cast<int64_t>(b) * H + h) * a.N + n;
    const int64_t o3 = (t * H + h) * 3;
    const float4 q0 = a.dq[2 * row], q1 = a.dq[2 * row + 1], k0 = a.dk[2 * row], k1 = a.dk[2 * row + 1];
    const float gqd[3] = {q0.x, q0.y, q0.z}, gqp[3] = {q1.x, q1.y, q1.z};
    const float gkd[3] = {k0.x, k0.y, k0.z}, gkp[3] = {k1.x, k1.y, k1.z};
    const int64_t n3 = rows * H * 3;
    back(gqd, a.qd, b * a.qd.s[0] + n * a.qd.s[1] + h * a.qd.s[2], a.qd.s[3], IPA_SPAN(a.d_qd, o3, 3, n3, a.err));
    back(gkd, a.kd, b * a.kd.s[0] + n * a.kd.s[1] + h * a.kd.s[2], a.kd.s[3], IPA_SPAN(a.d_kd, o3, 3, n3, a.err));
    back(gqp, a.qp, b * a.qp.s[0] + n * a.qp.s[1] + h * a.qp.s[2], a.qp.s[3], IPA_SPAN(a.d_qp, o3, 3, n3, a.err));
    back(gkp, a.kp, b * a.kp.s[0] + n * a.kp.s[1] + h * a.kp.s[2], a.kp.s[3], IPA_SPAN(a.d_kp, o3, 3, n3, a.err));
#pragma unroll
    for (int x = 0; x < 3; ++x) dT[x] = gqp[x] + gkp[x];
    for (int m = 0; m < a.M; ++m) {
      const float* dv = a.dvr + row * a.VW + 3 * m;
      const float gv[3] = {dv[0], dv[1], dv[2]};
      back(gv, a.val, b * a.val.s[0] + n * a.val.s[1] + h * a.val.s[2] + m * a.val.s[3], a.val.s[4],
           IPA_SPAN(a.d_val, (t * H + h) * a.VW + 3 * m, 3, rows * H * a.VW, a.err));
      // vectors = R^T agg: dR += agg g_vec^T
      const float* ag = a.agg + row * a.VW + 3 * m;
      const float* gq = a.gvec + t * a.HM3 + h * a.VW + 3 * m;
#pragma unroll
      for (int x = 0; x < 3; ++x)
#pragma unroll
        for (int y = 0; y < 3; ++y) dR[3 * x + y] = fmaf(ag[x], gq[y], dR[3 * x + y]);
    }
    float* ft = fterm + (il * H + h) * 12;
#pragma unroll
    for (int e = 0; e < 9; ++e) ft[e] = dR[e];
#pragma unroll
    for (int x = 0; x < 3; ++x) ft[9 + x] = dT[x];
  }
  __syncthreads();
  // sums over heads in order, one (residue, entry) per thread
  for (int e = threadIdx.x; e < rb * 12; e += blockDim.x) {
    const int r = e / 12, k = e % 12;
    const int64_t tr = static_cast<int64_t>(blockIdx.x) * rb + r;
    if (tr >= rows) continue;
    float sum = 0.f;
    for (int hh = 0; hh < H; ++hh) sum += fterm[(r * H + hh) * 12 + k];
    if (k < 9) *IPA_AT(a.d_rot, tr * 9 + k, rows * 9, a.err) = sum;
    else *IPA_AT(a.d_trans, tr * 3 + (k - 9), rows * 3, a.err) = sum;
  }
}

struct TransposeArgs {
  int HM3, Cout;
  View w;
  float* wt;   // [Cout, HM3]
  int* err;
};

__global__ void geo_wt_kernel(const TransposeArgs a) {
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= static_cast<int64_t>(a.HM3) * a.Cout) return;
  const int c = static_cast<int>(t / a.HM3), k = static_cast<int>(t % a.HM3);
  *IPA_AT(a.wt, t, static_cast<int64_t>(a.HM3) * a.Cout, a.err) = ldf(a.w, k * a.w.s[0] + c * a.w.s[1]);
}

template <int M>
cudaError_t launch_pairs(const PairArgs& p, int B, int N, int H, cudaStream_t st) {
  dim3 grid((N + BW_ROWS - 1) / BW_ROWS, H, B);
  constexpr int V4 = (3 * M + 3) & ~3;
  const size_t smem_r = sizeof(float) * BW_SPLIT *
                        (8 * BW_ROWS + BW_CHUNK * (8 + V4) + (p.has_g_att ? BW_ROWS * (BW_CHUNK + 1) : 0));
  const size_t smem_c = sizeof(float) * BW_SPLIT * ((6 + 3 * M) * BW_ROWS + BW_CHUNK * (12 + V4));
  if (smem_r > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(geo_bwd_rows_kernel<M>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem_r));
    if (e != cudaSuccess) return e;
  }
  if (smem_c > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(geo_bwd_cols_kernel<M>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem_c));
    if (e != cudaSuccess) return e;
  }
  geo_bwd_rows_kernel<M><<<grid, BW_ROWS * BW_SPLIT, smem_r, st>>>(p);
  geo_bwd_cols_kernel<M><<<grid, BW_ROWS * BW_SPLIT, smem_c, st>>>(p);
  return cudaGetLastError();
}

}  // namespace

GeoBwdWorkspace geo_bwd_workspace_layout(int B, int N, int H, int M, int Cout) {
  auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  GeoBwdWorkspace w{};
  w.fwd = geo_workspace_layout(B, N, H, M, Cout);
  size_t o = w.fwd.total;
  const size_t bn = static_cast<size_t>(B) * N, bhn = bn * H;
  const size_t VW = 3 * static_cast<size_t>(M), HM3 = static_cast<size_t>(H) * VW;
  w.vec = o; o = up(o + bn * HM3 * 4);
  w.agg = o; o = up(o + bhn * VW * 4);
  w.gvec = o; o = up(o + bn * HM3 * 4);
  w.rowlive = o; o = up(o + bn);
  w.dagg = o; o = up(o + bhn * VW * 4);
  w.rowinfo = o; o = up(o + bhn * 16);
  w.dq = o; o = up(o + bhn * 32);
  w.dk = o; o = up(o + bhn * 32);
  w.dvr = o; o = up(o + bhn * VW * 4);
  w.acc = o; o = up(o + static_cast<size_t>(B) * H * ((N + BW_ROWS - 1) / BW_ROWS) * 4 * 2 * 4);
  w.wt = o; o = up(o + HM3 * static_cast<size_t>(Cout) * 4);
  const size_t nchunk = (bn + 127) / 128;
  w.dwpart = o; o = up(o + nchunk * HM3 * static_cast<size_t>(Cout) * 4);
  w.dbpart = o; o = up(o + nchunk * static_cast<size_t>(Cout) * 4);
  w.total = o;
  return w;
}

cudaError_t geo_launch_bwd(const GeoBwdLaunch& a, cudaStream_t st) {
  const GeoBwdWorkspace& w = a.lay;
  unsigned char* ws = a.ws;
  const int B = a.f.B, N = a.f.N, H = a.f.H, M = a.f.M, HM3 = a.f.HM3, Cout = a.f.Cout, VW = 3 * M;
  const int64_t rows = static_cast<int64_t>(B) * N;

  // 0. forward statistics: scales, rotated inputs, (m, l), agg, vectors
  GeoLaunch f = a.f;
  f.ws = ws;
  f.lay = w.fwd;
  f.out_vectors = reinterpret_cast<float*>(ws + w.vec);
  f.out_output = nullptr;
  f.out_attention = nullptr;
  f.out_agg = reinterpret_cast<float*>(ws + w.agg);
  f.skip_readout = true;
  cudaError_t e = geo_launch_all(f, st);
  if (e != cudaSuccess) return e;

  {
    TransposeArgs ta{HM3, Cout, a.f.output_weight, reinterpret_cast<float*>(ws + w.wt), a.f.err};
    const int64_t n = static_cast<int64_t>(HM3) * Cout;
    geo_wt_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, st>>>(ta);
  }
  GvecArgs ga{};
  ga.B = B; ga.N = N; ga.H = H; ga.HM3 = HM3; ga.Cout = Cout;
  ga.g_output = a.g_output; ga.g_vectors = a.g_vectors; ga.has_g_vectors = a.has_g_vectors;
  ga.live = ws + w.fwd.live;
  ga.wt = reinterpret_cast<const float*>(ws + w.wt);
  ga.gvec = reinterpret_cast<float*>(ws + w.gvec);
  ga.rowlive = ws + w.rowlive;
  ga.err = a.f.err;
  geo_gvec_kernel<<<dim3(static_cast<unsigned>((rows + GV_TM - 1) / GV_TM), (HM3 + GV_TN - 1) / GV_TN), 256, 0, st>>>(ga);

  DaggArgs da{};
  da.B = B; da.N = N; da.H = H; da.M = M; da.VW = VW; da.HM3 = HM3;
  da.gvec = ga.gvec;
  da.rotf = reinterpret_cast<const float*>(ws + w.fwd.rotf);
  da.agg = f.out_agg;
  da.dagg = reinterpret_cast<float*>(ws + w.dagg);
  da.rowinfo = reinterpret_cast<float4*>(ws + w.rowinfo);
  da.err = a.f.err;
  geo_dagg_kernel<<<static_cast<unsigned>((rows * H + 255) / 256), 256, 0, st>>>(da);

  DwArgs dw{};
  dw.rows = rows; dw.HM3 = HM3; dw.Cout = Cout; dw.g_output = a.g_output; dw.N = N;
  dw.nchunk = static_cast<int>((rows + DW_ROWS - 1) / DW_ROWS);
  dw.vec = f.out_vectors; dw.rowlive = ga.rowlive;
  dw.part_w = reinterpret_cast<float*>(ws + w.dwpart);
  dw.part_b = reinterpret_cast<float*>(ws + w.dbpart);
  dw.d_w = a.d_output_weight; dw.d_b = a.d_output_bias;
  dw.err = a.f.err;
  geo_dw_part_kernel<<<dim3((HM3 + DW_TM - 1) / DW_TM, (Cout + DW_TN - 1) / DW_TN, dw.nchunk), 256, 0, st>>>(dw);
  {
    int64_t n = static_cast<int64_t>(HM3) * Cout;
    geo_dw_sum_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, st>>>(dw);
  }

  PairArgs p{};
  p.B = B; p.N = N; p.H = H; p.VW = VW;
  p.qg = reinterpret_cast<const float4*>(ws + w.fwd.qg);
  p.kg = reinterpret_cast<const float4*>(ws + w.fwd.kg);
  p.vg = reinterpret_cast<const float*>(ws + w.fwd.vg);
  p.sc = reinterpret_cast<const float2*>(ws + w.fwd.sc);
  p.ml = reinterpret_cast<const float2*>(ws + w.fwd.ml);
  p.dagg = da.dagg;
  p.rowinfo = da.rowinfo;
  p.pm = a.f.has_pair_mask ? reinterpret_cast<const unsigned char*>(a.f.pair_mask.p) : nullptr;
  for (int d = 0; d < 4; ++d) p.pms[d] = a.f.has_pair_mask ? a.f.pair_mask.s[d] : 0;
  p.g_att = a.g_attention;
  p.has_g_att = a.has_g_attention;
  p.dq = reinterpret_cast<float4*>(ws + w.dq);
  p.dk = reinterpret_cast<float4*>(ws + w.dk);
  p.dvr = reinterpret_cast<float*>(ws + w.dvr);
  p.acc = reinterpret_cast<float*>(ws + w.acc);
  p.err = a.f.err;
  switch (M) {
    case 1: e = launch_pairs<1>(p, B, N, H, st); break;
    case 2: e = launch_pairs<2>(p, B, N, H, st); break;
    case 3: e = launch_pairs<3>(p, B, N, H, st); break;
    case 4: e = launch_pairs<4>(p, B, N, H, st); break;
    case 5: e = launch_pairs<5>(p, B, N, H, st); break;
    case 6: e = launch_pairs<6>(p, B, N, H, st); break;
    case 7: e = launch_pairs<7>(p, B, N, H, st); break;
    case 8: e = launch_pairs<8>(p, B, N, H, st); break;
    default: e = cudaErrorInvalidValue; break;
  }
  if (e != cudaSuccess) return e;

  FrameArgs fa{};
  fa.B = B; fa.N = N; fa.H = H; fa.M = M; fa.VW = VW; fa.HM3 = HM3;
  fa.qd = a.f.q_direction; fa.kd = a.f.k_direction; fa.qp = a.f.q_point; fa.kp = a.f.k_point;
  fa.val = a.f.values; fa.dscale = a.f.direction_scale; fa.xscale = a.f.distance_scale;
  fa.rotf = da.rotf; fa.agg = f.out_agg; fa.gvec = ga.gvec;
  fa.dq = p.dq; fa.dk = p.dk; fa.dvr = p.dvr; fa.acc = p.acc; fa.nrb = (N + BW_ROWS - 1) / BW_ROWS;
  fa.d_qd = a.d_q_direction; fa.d_kd = a.d_k_direction; fa.d_qp = a.d_q_point; fa.d_kp = a.d_k_point;
  fa.d_val = a.d_values; fa.d_rot = a.d_rotation; fa.d_trans = a.d_translation;
  fa.d_dscale = a.d_direction_scale; fa.d_xscale = a.d_distance_scale;
  fa.err = a.f.err;
  geo_bwd_frame_kernel<<<static_cast<unsigned>((rows + 128 / H - 1) / (128 / H)), 128, 0, st>>>(fa);
  return cudaGetLastError();
}

}  // namespace fipa
