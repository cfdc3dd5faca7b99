// Geometric direction-and-distance attention for sm_100a ("Geometric
// direction-and-distance attention", Required behavior).
//
// The score uses the UNSQUARED distance |qp_i - kp_j|, which does not
// factorise into query and key columns, so the per-pair score is evaluated on
// CUDA cores inside the key loop (fp32, MUFU sqrt / exp2).  Launches:
//   1. geo_weights_kernel -- softplus scales per head, readout weight / bias
//      converted to fp32.
//   2. geo_prep_kernel    -- per (b, n, h): rotated directions, transformed
//      points, R_j-rotated values (no translation), frame-mask bias.
//   3. geo_attn_kernel<M> -- per (b, h, 128 queries) x 4 key splits (each split
//      group of four warps stages its 32-key chunks in shared memory, double
//      buffered): scores and the value aggregation two keys per packed fp32
//      instruction, online masked softmax in the log2 domain with lazy
//      rescaling; splits merged through shared memory; R_i^T back-rotation.
//   4. geo_map_kernel     -- optional: recomputes each score and writes the
//      normalised attention map, 16 query rows per block, 16-byte stores.
//   5. geo_readout_kernel -- output = flatten(vectors) . W (+ b) as a
//      register-tiled product (64 x 64 per block), forced to zero for
//      queries where no head has an allowed key.
#include <cuda_fp16.h>

#include <cmath>
#include <cstdint>

#include "bounds.cuh"
#include "geo_common.cuh"
#include "internal.h"
#include "sm100.cuh"

#define IPA_FILE_TAG 5

namespace fipa {

using namespace sm100;
using namespace geo;

namespace {

constexpr int GEO_ROWS = 128;
constexpr int GEO_SPLIT = 4;
constexpr int GEO_CHUNK = 32;

struct WArgs {
  int H, HM3, Cout;
  bool has_bias;
  View dscale, xscale, w, bias;
  float2* sc;   // [H]: (log2e softplus(direction)/sqrt3, log2e softplus(distance)/sqrt3)
  float* wf;    // [HM3, Cout]
  float* bf;    // [Cout]
  int* err;
};

__global__ void geo_weights_kernel(const WArgs a) {
  const int64_t n = static_cast<int64_t>(a.HM3) * a.Cout;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t < n) {
    const int r = static_cast<int>(t / a.Cout), c = static_cast<int>(t % a.Cout);
    *IPA_AT(a.wf, t, n, a.err) = ldf(a.w, r * a.w.s[0] + c * a.w.s[1]);
  }
  if (t < a.Cout) *IPA_AT(a.bf, t, a.Cout, a.err) = a.has_bias ? ldf(a.bias, t * a.bias.s[0]) : 0.f;
  if (t < a.H) {
    const float k = kLog2e * 0.57735026918962576f;  // log2(e) / sqrt(3)
    *IPA_AT(a.sc, t, a.H, a.err) = make_float2(k * softplus_stable(ldf(a.dscale, t * a.dscale.s[0])),
                          k * softplus_stable(ldf(a.xscale, t * a.xscale.s[0])));
  }
}

struct PrepArgs {
  int B, N, H, M, VW;
  View qd, kd, qp, kp, val, rot, trans, fmask;
  float4* qg;   // [B*H, N, 2]: (qd, bias) (qp, 0)
  float4* kg;   // [B*H, N, 2]: (kd, bias) (kp, 0)
  float* vg;    // [B*H, N, VW]
  float* rotf;  // [B, N, 9]
  int* err;
};

__global__ void geo_prep_kernel(const PrepArgs a) {
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t total = static_cast<int64_t>(a.B) * a.N * a.H;
  if (t >= total) return;
  const int h = static_cast<int>(t % a.H);
  const int n = static_cast<int>((t / a.H) % a.N);
  const int b = static_cast<int>(t / (static_cast<int64_t>(a.H) * a.N));
  float R[9];
  const int64_t ro = b * a.rot.s[0] + n * a.rot.s[1];
#pragma unroll
  for (int x = 0; x < 3; ++x)
#pragma unroll
    for (int y = 0; y < 3; ++y) R[x * 3 + y] = ldf(a.rot, ro + x * a.rot.s[2] + y * a.rot.s[3]);
  const int64_t to = b * a.trans.s[0] + n * a.trans.s[1];
  const float T[3] = {ldf(a.trans, to), ldf(a.trans, to + a.trans.s[2]), ldf(a.trans, to + 2 * a.trans.s[2])};
  const bool valid = ldb(a.fmask, b * a.fmask.s[0] + n * a.fmask.s[1]);
  const float bias = valid ? 0.f : -INFINITY;

  auto rot3 = [&](const View& v, int64_t base, float out[3]) {
    const float p0 = ldf(v, base), p1 = ldf(v, base + v.s[3]), p2 = ldf(v, base + 2 * v.s[3]);
#pragma unroll
    for (int x = 0; x < 3; ++x) out[x] = fmaf(R[x * 3], p0, fmaf(R[x * 3 + 1], p1, R[x * 3 + 2] * p2));
  };
  float qd[3], kd[3], qp[3], kp[3];
  rot3(a.qd, b * a.qd.s[0] + n * a.qd.s[1] + h * a.qd.s[2], qd);
  rot3(a.kd, b * a.kd.s[0] + n * a.kd.s[1] + h * a.kd.s[2], kd);
  rot3(a.qp, b * a.qp.s[0] + n * a.qp.s[1] + h * a.qp.s[2], qp);
  rot3(a.kp, b * a.kp.s[0] + n * a.kp.s[1] + h * a.kp.s[2], kp);
  const int64_t row = (static_cast<int64_t>(b) * a.H + h) * a.N + n;
  float4* qo = IPA_SPAN(a.qg, 2 * row, 2, 2 * total, a.err);
  float4* ko = IPA_SPAN(a.kg, 2 * row, 2, 2 * total, a.err);
  qo[0] = make_float4(qd[0], qd[1], qd[2], bias);
  qo[1] = make_float4(qp[0] + T[0], qp[1] + T[1], qp[2] + T[2], 0.f);
  ko[0] = make_float4(kd[0], kd[1], kd[2], bias);
  ko[1] = make_float4(kp[0] + T[0], kp[1] + T[1], kp[2] + T[2], 0.f);
  float* vo = IPA_SPAN(a.vg, row * a.VW, a.VW, total * a.VW, a.err);
  for (int m = 0; m < a.M; ++m) {
    float vr[3];
    const int64_t vb = b * a.val.s[0] + n * a.val.s[1] + h * a.val.s[2] + m * a.val.s[3];
    const float p0 = ldf(a.val, vb), p1 = ldf(a.val, vb + a.val.s[4]), p2 = ldf(a.val, vb + 2 * a.val.s[4]);
#pragma unroll
    for (int x = 0; x < 3; ++x) vr[x] = fmaf(R[x * 3], p0, fmaf(R[x * 3 + 1], p1, R[x * 3 + 2] * p2));
    vo[3 * m] = vr[0];
    vo[3 * m + 1] = vr[1];
    vo[3 * m + 2] = vr[2];
  }
  for (int e = 3 * a.M; e < a.VW; ++e) vo[e] = 0.f;
  if (h == 0) {
    float* rf = IPA_SPAN(a.rotf, (static_cast<int64_t>(b) * a.N + n) * 9, 9, static_cast<int64_t>(a.B) * a.N * 9, a.err);
#pragma unroll
    for (int e = 0; e < 9; ++e) rf[e] = R[e];
  }
}

struct AttnArgs {
  int B, N, H, VW;
  float tau;
  const float4* qg;
  const float4* kg;
  const float* vg;
  const float2* sc;
  const float* rotf;
  const unsigned char* pm;   // may be null
  int64_t pms[4];            // element (byte) strides b, h, i, j
  float* out_vectors;        // [B, N, H, M, 3]
  float2* ml;                // [B*H, N]
  unsigned char* live;       // [B, N, H]
  float* agg;                // [B*H, N, VW] aggregated global-frame values, or null
  int* err;
};

// Staged chunk of 32 keys (one split group), laid out for packed pairs of
// keys (a, b) = (2t, 2t + 1): per pair four float4
//   (kd.x_a, kd.x_b, kd.y_a, kd.y_b) (kd.z_a, kd.z_b, bias_a, bias_b)
//   (kp.x_a, kp.x_b, kp.y_a, kp.y_b) (kp.z_a, kp.z_b, 0, 0)
// then the V rotated values as (v_e,a, v_e,b) pairs, padded to a multiple of
// four floats so that every pair record starts 16-byte aligned.
template <int V>
struct GeoChunk {
  static constexpr int PAIR = 16 + ((2 * V + 3) & ~3);   // floats per key pair, a multiple of 4 (float4 loads)
  static constexpr int FLOATS = (GEO_CHUNK / 2) * PAIR;
};

// One 512-thread block per SM: the packed-pair loop keeps its working set in
// registers without spilling (two blocks per SM at 64 registers spilled and
// measured 9 % slower at B=2 N=2048 H=8 M=4, despite the single wave).
template <int M>
__global__ void __launch_bounds__(GEO_ROWS * GEO_SPLIT, 1) geo_attn_kernel(const AttnArgs a) {
  constexpr int V = 3 * M;
  constexpr int PAIR = GeoChunk<V>::PAIR, CF = GeoChunk<V>::FLOATS;
  const int tid = threadIdx.x;
  const int r = tid % GEO_ROWS, split = tid / GEO_ROWS;
  const int h = blockIdx.y, b = blockIdx.z;
  const int i = blockIdx.x * GEO_ROWS + r;
  const int N = a.N;
  const int64_t bh = static_cast<int64_t>(b) * a.H + h;
  const bool in_range = i < N;
  const float2 sc = a.sc[h];

  float4 q0 = make_float4(0, 0, 0, -INFINITY), q1 = make_float4(0, 0, 0, 0);
  if (in_range) {
    q0 = a.qg[2 * (bh * N + i)];
    q1 = a.qg[2 * (bh * N + i) + 1];
  }
  const unsigned char* pmrow =
      a.pm ? a.pm + b * a.pms[0] + h * a.pms[1] + static_cast<int64_t>(in_range ? i : 0) * a.pms[2] : nullptr;
  const int64_t pj = a.pms[3];
  const float2 qx = make_float2(q0.x, q0.x), qy = make_float2(q0.y, q0.y), qz = make_float2(q0.z, q0.z);
  // a query whose frame is invalid (bias -inf) has no allowed key at all
  const bool qdead = !(q0.w == 0.f);
  const float2 px = make_float2(q1.x, q1.x), py = make_float2(q1.y, q1.y), pz = make_float2(q1.z, q1.z);
  const float2 A2 = make_float2(sc.x, sc.x), nB2 = make_float2(-sc.y, -sc.y);

  float m = -INFINITY;
  float2 l2 = make_float2(0.f, 0.f);
  float2 acc[V];                                // (sum over even keys, sum over odd keys)
#pragma unroll
  for (int e = 0; e < V; ++e) acc[e] = make_float2(0.f, 0.f);

  extern __shared__ float geo_merge[];  // [GEO_SPLIT][2 + V][GEO_ROWS], then 2 staged chunks per split
  float* stg0 = geo_merge + GEO_SPLIT * (2 + V) * GEO_ROWS + split * 2 * CF;
  const uint32_t gbar = 1 + split;
  const int nchunk = (N + GEO_CHUNK - 1) / GEO_CHUNK;
  // this thread's share of a chunk: source element e = (key, field) of the
  // [32 keys][8 + V] chunk, staged into the packed-pair layout
  constexpr int SRCW = 8 + V;
  constexpr int PER = (GEO_CHUNK * SRCW + GEO_ROWS - 1) / GEO_ROWS;
  auto fetch = [&](int ch, float (&vals)[PER]) {
    const int j0 = ch * GEO_CHUNK;
#pragma unroll
    for (int u = 0; u < PER; ++u) {
      const int e = r + u * GEO_ROWS;
      const int key = e / SRCW, f = e % SRCW, j = j0 + key;
      float v = 0.f;
      if (e < GEO_CHUNK * SRCW && ch < nchunk && j < N) {
        if (f < 8) v = reinterpret_cast<const float*>(a.kg)[8 * (bh * N + j) + f];
        else v = a.vg[(bh * N + j) * a.VW + (f - 8)];
      }
      vals[u] = v;
    }
  };
  auto stage = [&](float* dst, const float (&vals)[PER]) {
#pragma unroll
    for (int u = 0; u < PER; ++u) {
      const int e = r + u * GEO_ROWS;
      if (e >= GEO_CHUNK * SRCW) break;
      const int key = e / SRCW, f = e % SRCW, t = key >> 1, q = key & 1;
      // kg fields 0..7: kd.x kd.y kd.z bias kp.x kp.y kp.z 0
      int pos;
      if (f < 8) pos = (f >> 1) * 4 + (f & 1) * 2 + q;
      else pos = 16 + 2 * (f - 8) + q;
      dst[t * PAIR + pos] = vals[u];
    }
  };
  float pre[PER];
  int buf = 0;
  fetch(split, pre);
  stage(stg0, pre);
  named_bar_sync(gbar, GEO_ROWS);
  for (int ch = split; ch < nchunk; ch += GEO_SPLIT) {
    const int j0 = ch * GEO_CHUNK;
    fetch(ch + GEO_SPLIT, pre);                   // the group's next chunk, in flight during this one
    uint32_t allowed = 0xffffffffu;
    if (pmrow) {
      allowed = 0u;
      const unsigned char* p = pmrow + static_cast<int64_t>(j0) * pj;
      if (pj == 1 && j0 + GEO_CHUNK <= N && (reinterpret_cast<uintptr_t>(p) & 15u) == 0) {
        const uint4 u0 = *reinterpret_cast<const uint4*>(p);
        const uint4 u1 = *reinterpret_cast<const uint4*>(p + 16);
        const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
        for (int q = 0; q < 8; ++q) allowed |= nonzero_byte_bits(w[q]) << (4 * q);
      } else {
        for (int k = 0; k < GEO_CHUNK && j0 + k < N; ++k) allowed |= p[k * pj] ? (1u << k) : 0u;
      }
    }
    if (j0 + GEO_CHUNK > N) allowed &= (N - j0 >= 32) ? 0xffffffffu : ((1u << (N - j0)) - 1u);
    if (qdead) allowed = 0u;
    const float* cur = stg0 + buf * CF;
    // pass 1: the chunk's 32 scores (two per packed instruction) and their maximum
    float2 sv2[GEO_CHUNK / 2];
    float cm = -INFINITY;
#pragma unroll
    for (int t = 0; t < GEO_CHUNK / 2; ++t) {
      const float4* kp4 = reinterpret_cast<const float4*>(cur + t * PAIR);
      const float4 w0 = kp4[0], w1 = kp4[1], w2 = kp4[2], w3 = kp4[3];
      const float2 dot = fma_f32x2(qx, make_float2(w0.x, w0.y),
                                   fma_f32x2(qy, make_float2(w0.z, w0.w), mul_f32x2(qz, make_float2(w1.x, w1.y))));
      const float2 dx = sub_f32x2(px, make_float2(w2.x, w2.y));
      const float2 dy = sub_f32x2(py, make_float2(w2.z, w2.w));
      const float2 dz = sub_f32x2(pz, make_float2(w3.x, w3.y));
      const float2 d2 = fma_f32x2(dx, dx, fma_f32x2(dy, dy, mul_f32x2(dz, dz)));
      const float2 dist = make_float2(dist_sqrt(d2.x), dist_sqrt(d2.y));
      float2 sv = add_f32x2(fma_f32x2(A2, dot, mul_f32x2(nB2, dist)), make_float2(w1.z, w1.w));
      if (!((allowed >> (2 * t)) & 1u)) sv.x = -INFINITY;
      if (!((allowed >> (2 * t + 1)) & 1u)) sv.y = -INFINITY;
      sv2[t] = sv;
      cm = fmax3(cm, sv.x, sv.y);
    }
    if (cm > m + a.tau) {                           // lazy rescale: p stays below 2^tau
      if (m != -INFINITY) {
        const float f = ex2(m - cm);
        const float2 f2 = make_float2(f, f);
        l2 = mul_f32x2(l2, f2);
#pragma unroll
        for (int e = 0; e < V; ++e) acc[e] = mul_f32x2(acc[e], f2);
      }
      m = cm;
    }
    if (m != -INFINITY) {
      // pass 2: probabilities and the value aggregation
      const float2 mb = make_float2(m, m);
#pragma unroll
      for (int t = 0; t < GEO_CHUNK / 2; ++t) {
        const float2 y = sub_f32x2(sv2[t], mb);
        const float2 p2 = make_float2(ex2(y.x), ex2(y.y));
        l2 = add_f32x2(l2, p2);
        const float4* vp4 = reinterpret_cast<const float4*>(cur + t * PAIR + 16);
#pragma unroll
        for (int e2 = 0; e2 < V / 2; ++e2) {
          const float4 vv = vp4[e2];
          acc[2 * e2] = fma_f32x2(p2, make_float2(vv.x, vv.y), acc[2 * e2]);
          acc[2 * e2 + 1] = fma_f32x2(p2, make_float2(vv.z, vv.w), acc[2 * e2 + 1]);
        }
        if (V & 1) {
          const float2 vv = reinterpret_cast<const float2*>(cur + t * PAIR + 16)[V - 1];
          acc[V - 1] = fma_f32x2(p2, vv, acc[V - 1]);
        }
      }
    }
    buf ^= 1;
    stage(stg0 + buf * CF, pre);
    named_bar_sync(gbar, GEO_ROWS);               // the next chunk is staged; this one is free
  }
  const float l = l2.x + l2.y;
  float accs[V];
#pragma unroll
  for (int e = 0; e < V; ++e) accs[e] = acc[e].x + acc[e].y;

  // merge the key splits
  auto sm_at = [&](int s2, int e) -> float& { return geo_merge[(s2 * (2 + V) + e) * GEO_ROWS + r]; };
  sm_at(split, 0) = m;
  sm_at(split, 1) = l;
#pragma unroll
  for (int e = 0; e < V; ++e) sm_at(split, 2 + e) = accs[e];
  __syncthreads();
  if (split != 0 || !in_range) return;
  float mf = -INFINITY;
#pragma unroll
  for (int s2 = 0; s2 < GEO_SPLIT; ++s2) mf = fmaxf(mf, sm_at(s2, 0));
  float lf = 0.f, af[V];
#pragma unroll
  for (int e = 0; e < V; ++e) af[e] = 0.f;
  if (mf != -INFINITY) {
#pragma unroll
    for (int s2 = 0; s2 < GEO_SPLIT; ++s2) {
      const float ms = sm_at(s2, 0);
      if (ms == -INFINITY) continue;
      const float f = ex2(ms - mf);
      lf = fmaf(sm_at(s2, 1), f, lf);
#pragma unroll
      for (int e = 0; e < V; ++e) af[e] = fmaf(sm_at(s2, 2 + e), f, af[e]);
    }
  }
  const bool has = lf > 0.f;
  const float inv = has ? 1.f / lf : 0.f;
  const float* R = a.rotf + (static_cast<int64_t>(b) * N + i) * 9;
  const int64_t nbhn = static_cast<int64_t>(a.B) * a.H * N;
  float* dst = IPA_SPAN(a.out_vectors, ((static_cast<int64_t>(b) * N + i) * a.H + h) * V, V, nbhn * V, a.err);
  if (a.agg) {
    float* ag = IPA_SPAN(a.agg, (bh * N + i) * a.VW, V, nbhn * a.VW, a.err);
#pragma unroll
    for (int e = 0; e < V; ++e) ag[e] = has ? af[e] * inv : 0.f;
  }
#pragma unroll
  for (int mm = 0; mm < M; ++mm) {
    const float gx = af[3 * mm] * inv, gy = af[3 * mm + 1] * inv, gz = af[3 * mm + 2] * inv;
#pragma unroll
    for (int x = 0; x < 3; ++x)  // R^T g
      dst[3 * mm + x] = has ? fmaf(R[x], gx, fmaf(R[3 + x], gy, R[6 + x] * gz)) : 0.f;
  }
  *IPA_AT(a.ml, bh * N + i, nbhn, a.err) = make_float2(mf, lf);
  *IPA_AT(a.live, (static_cast<int64_t>(b) * N + i) * a.H + h, nbhn, a.err) = has ? 1 : 0;
}

struct MapArgs {
  int B, N, H;
  const float4* qg;
  const float4* kg;
  const float2* sc;
  const float2* ml;
  const unsigned char* pm;
  int64_t pms[4];
  float* att;   // [B, H, N, N]
  int* err;
};

// One block per (16 query rows, head, batch): each thread owns four
// consecutive keys at a time, loads their terms once and writes the 16 rows'
// probabilities for them as float4 stores (a warp writes 512 contiguous bytes
// of a row).  Key terms are read N / 16 times per (b, h) instead of N times.
// The pair-mask words of all 16 rows are loaded before any score, so their
// latency is paid once per four keys, and the scores are taken two keys per
// packed instruction (each lane rounds as geo_pair does).
constexpr int MAP_ROWS = 16;
constexpr int MAP_KEYS = 4;

__global__ void __launch_bounds__(256, 3) geo_map_kernel(const MapArgs a) {
  const int i0 = blockIdx.x * MAP_ROWS, h = blockIdx.y, b = blockIdx.z;
  const int N = a.N;
  const int64_t bh = static_cast<int64_t>(b) * a.H + h;
  __shared__ float4 qs[MAP_ROWS][2];
  __shared__ float2 rs[MAP_ROWS];            // (running max m, 1 / l), l = 0 -> row of zeros
  if (threadIdx.x < MAP_ROWS) {
    const int i = i0 + threadIdx.x;
    float4 q0 = make_float4(0.f, 0.f, 0.f, 0.f), q1 = q0;
    float2 st = make_float2(0.f, 0.f);
    if (i < N) {
      q0 = a.qg[2 * (bh * N + i)];
      q1 = a.qg[2 * (bh * N + i) + 1];
      const float2 ml = a.ml[bh * N + i];
      st = make_float2(ml.x, ml.y > 0.f ? 1.f / ml.y : 0.f);
    }
    qs[threadIdx.x][0] = q0;
    qs[threadIdx.x][1] = q1;
    rs[threadIdx.x] = st;
  }
  __syncthreads();
  const float2 sc = a.sc[h];
  const float2 A2 = make_float2(sc.x, sc.x), nB2 = make_float2(-sc.y, -sc.y);
  const int nrows = N - i0 < MAP_ROWS ? N - i0 : MAP_ROWS;
  const bool vec_store = (N & 3) == 0;
  const unsigned char* pmb = a.pm ? a.pm + b * a.pms[0] + h * a.pms[1] : nullptr;
  const bool vec_mask = pmb != nullptr && a.pms[3] == 1 && (a.pms[2] & 3) == 0 &&
                        (reinterpret_cast<uintptr_t>(pmb) & 3u) == 0;
  for (int j0 = MAP_KEYS * threadIdx.x; j0 < N; j0 += MAP_KEYS * blockDim.x) {
    float4 k0[MAP_KEYS], k1[MAP_KEYS];
#pragma unroll
    for (int t = 0; t < MAP_KEYS; ++t) {
      const int j = j0 + t < N ? j0 + t : N - 1;
      k0[t] = a.kg[2 * (bh * N + j)];
      k1[t] = a.kg[2 * (bh * N + j) + 1];
    }
    const bool full = j0 + MAP_KEYS <= N;
    // the four keys' mask bytes of every row, loaded together, kept as 4
    // bits per row (bit 4 rr + t: key j0 + t allowed for row i0 + rr)
    uint32_t wv[MAP_ROWS];
#pragma unroll
    for (int rr = 0; rr < MAP_ROWS; ++rr) {
      wv[rr] = 0x01010101u;
      if (pmb != nullptr && rr < nrows) {
        const unsigned char* pr = pmb + static_cast<int64_t>(i0 + rr) * a.pms[2];
        if (vec_mask && full) {
          wv[rr] = *reinterpret_cast<const uint32_t*>(pr + j0);
        } else {
          uint32_t w = 0u;
#pragma unroll
          for (int t = 0; t < MAP_KEYS; ++t)
            if (j0 + t < N && pr[static_cast<int64_t>(j0 + t) * a.pms[3]]) w |= 1u << (8 * t);
          wv[rr] = w;
        }
      }
    }
    uint64_t allow = 0u;
#pragma unroll
    for (int rr = 0; rr < MAP_ROWS; ++rr) {
      allow |= static_cast<uint64_t>(nonzero_byte_bits(wv[rr])) << (4 * rr);
    }
    // key terms in lane pairs: keys (0, 1) and (2, 3)
    float2 kx[2], ky[2], kz[2], px[2], py[2], pz[2], kb[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const float4 a0 = k0[2 * u], a1 = k0[2 * u + 1], c0 = k1[2 * u], c1 = k1[2 * u + 1];
      kx[u] = make_float2(a0.x, a1.x);
      ky[u] = make_float2(a0.y, a1.y);
      kz[u] = make_float2(a0.z, a1.z);
      kb[u] = make_float2(a0.w, a1.w);
      px[u] = make_float2(c0.x, c1.x);
      py[u] = make_float2(c0.y, c1.y);
      pz[u] = make_float2(c0.z, c1.z);
    }
#pragma unroll
    for (int rr = 0; rr < MAP_ROWS; ++rr) {
      if (rr >= nrows) break;
      const int i = i0 + rr;
      const float4 q0 = qs[rr][0], q1 = qs[rr][1];
      const float2 st = rs[rr];
      const uint32_t al = static_cast<uint32_t>(allow >> (4 * rr));
      float v[MAP_KEYS];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        // the operation sequence of geo_pair, two keys per instruction
        const float2 dot = fma_f32x2(make_float2(q0.x, q0.x), kx[u],
                                     fma_f32x2(make_float2(q0.y, q0.y), ky[u],
                                               mul_f32x2(make_float2(q0.z, q0.z), kz[u])));
        const float2 dx = sub_f32x2(make_float2(q1.x, q1.x), px[u]);
        const float2 dy = sub_f32x2(make_float2(q1.y, q1.y), py[u]);
        const float2 dz = sub_f32x2(make_float2(q1.z, q1.z), pz[u]);
        const float2 d2 = fma_f32x2(dx, dx, fma_f32x2(dy, dy, mul_f32x2(dz, dz)));
        const float2 dist = make_float2(dist_sqrt(d2.x), dist_sqrt(d2.y));
        const float2 s = add_f32x2(add_f32x2(fma_f32x2(A2, dot, mul_f32x2(nB2, dist)), make_float2(q0.w, q0.w)), kb[u]);
        const float2 y = sub_f32x2(s, make_float2(st.x, st.x));
        const bool ok0 = st.y > 0.f && ((al >> (2 * u)) & 1u) != 0;
        const bool ok1 = st.y > 0.f && ((al >> (2 * u + 1)) & 1u) != 0;
        v[2 * u] = ok0 ? ex2(y.x) * st.y : 0.f;
        v[2 * u + 1] = ok1 ? ex2(y.y) * st.y : 0.f;
      }
      const int64_t nw = full ? MAP_KEYS : (N - j0 < MAP_KEYS ? N - j0 : MAP_KEYS);
      float* dst = IPA_SPAN(a.att, (bh * N + i) * static_cast<int64_t>(N) + j0, nw,
                            static_cast<int64_t>(a.B) * a.H * N * static_cast<int64_t>(N), a.err);
      if (vec_store && full) {
        *reinterpret_cast<float4*>(dst) = make_float4(v[0], v[1], v[2], v[3]);
      } else {
#pragma unroll
        for (int t = 0; t < MAP_KEYS; ++t)
          if (j0 + t < N) dst[t] = v[t];
      }
    }
  }
}

struct ReadArgs {
  int B, N, H, HM3, Cout;
  const float* vec;   // [B*N, HM3]
  const unsigned char* live;
  const float* wf;
  const float* bf;
  float* out;         // [B*N, Cout]
  int* err;
};

constexpr int RD_TM = 64, RD_TN = 64;

// out[row, :] = vec[row, :] W + b over a 64 x 64 tile per block; rows whose
// heads all lacked an allowed key are forced to 0.
__global__ void __launch_bounds__(256) geo_readout_kernel(const ReadArgs a) {
  __shared__ int any_live[RD_TM];
  const int64_t nrows = static_cast<int64_t>(a.B) * a.N;
  const int r0 = blockIdx.x * RD_TM, c0 = blockIdx.y * RD_TN;
  if (threadIdx.x < RD_TM) {
    int anyl = 0;
    const int64_t row = r0 + static_cast<int>(threadIdx.x);
    if (row < nrows)
      for (int h = 0; h < a.H; ++h) anyl |= a.live[row * a.H + h];
    any_live[threadIdx.x] = anyl;
  }
  float acc[RD_TM / 16][RD_TN / 16];
  tile_product<RD_TM, RD_TN>(
      r0, c0, a.HM3,
      [&](int r, int k) { return (r < nrows && k < a.HM3) ? a.vec[static_cast<int64_t>(r) * a.HM3 + k] : 0.f; },
      [&](int k, int c) { return (k < a.HM3 && c < a.Cout) ? a.wf[static_cast<int64_t>(k) * a.Cout + c] : 0.f; },
      acc);
  const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
#pragma unroll
  for (int i = 0; i < RD_TM / 16; ++i) {
    const int64_t row = r0 + ty + 16 * i;
    if (row >= nrows) continue;
#pragma unroll
    for (int j = 0; j < RD_TN / 16; ++j) {
      const int col = c0 + tx + 16 * j;
      if (col < a.Cout)
        *IPA_AT(a.out, row * a.Cout + col, nrows * a.Cout, a.err) =
            any_live[ty + 16 * i] ? acc[i][j] + a.bf[col] : 0.f;
    }
  }
}

template <int M>
cudaError_t launch_attn(const AttnArgs& t, int B, int N, int H, cudaStream_t st) {
  dim3 grid((N + GEO_ROWS - 1) / GEO_ROWS, H, B);
  const size_t smem = sizeof(float) * GEO_SPLIT * ((2 + 3 * M) * GEO_ROWS + 2 * GeoChunk<3 * M>::FLOATS);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(geo_attn_kernel<M>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  geo_attn_kernel<M><<<grid, GEO_ROWS * GEO_SPLIT, smem, st>>>(t);
  return cudaSuccess;
}

}  // namespace

GeoWorkspace geo_workspace_layout(int B, int N, int H, int M, int Cout) {
  auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  GeoWorkspace w{};
  size_t o = 0;
  const size_t bhn = static_cast<size_t>(B) * H * N;
  const int VW = 3 * M;
  const int HM3 = H * M * 3;
  w.qg = o; o = up(o + bhn * 32);
  w.kg = o; o = up(o + bhn * 32);
  w.vg = o; o = up(o + bhn * VW * 4);
  w.rotf = o; o = up(o + static_cast<size_t>(B) * N * 36);
  w.ml = o; o = up(o + bhn * 8);
  w.live = o; o = up(o + bhn);
  w.wf = o; o = up(o + static_cast<size_t>(HM3) * Cout * 4);
  w.bf = o; o = up(o + static_cast<size_t>(Cout) * 4);
  w.sc = o; o = up(o + static_cast<size_t>(H) * 8);
  w.err = o; o = up(o + 16);
  w.total = o;
  return w;
}

cudaError_t geo_launch_all(const GeoLaunch& a, cudaStream_t st) {
  unsigned char* ws = a.ws;
  const GeoWorkspace& w = a.lay;
  const int VW = 3 * a.M;

  WArgs wa{};
  wa.H = a.H; wa.HM3 = a.HM3; wa.Cout = a.Cout; wa.has_bias = a.has_bias;
  wa.dscale = a.direction_scale; wa.xscale = a.distance_scale; wa.w = a.output_weight; wa.bias = a.output_bias;
  wa.sc = reinterpret_cast<float2*>(ws + w.sc);
  wa.wf = reinterpret_cast<float*>(ws + w.wf);
  wa.bf = reinterpret_cast<float*>(ws + w.bf);
  wa.err = a.err;
  {
    int64_t n = static_cast<int64_t>(a.HM3) * a.Cout;
    if (n < a.Cout) n = a.Cout;
    if (n < a.H) n = a.H;
    geo_weights_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, st>>>(wa);
  }

  PrepArgs pa{};
  pa.B = a.B; pa.N = a.N; pa.H = a.H; pa.M = a.M; pa.VW = VW;
  pa.qd = a.q_direction; pa.kd = a.k_direction; pa.qp = a.q_point; pa.kp = a.k_point;
  pa.val = a.values; pa.rot = a.rotation; pa.trans = a.translation; pa.fmask = a.frame_mask;
  pa.qg = reinterpret_cast<float4*>(ws + w.qg);
  pa.kg = reinterpret_cast<float4*>(ws + w.kg);
  pa.vg = reinterpret_cast<float*>(ws + w.vg);
  pa.rotf = reinterpret_cast<float*>(ws + w.rotf);
  pa.err = a.err;
  {
    const int64_t n = static_cast<int64_t>(a.B) * a.N * a.H;
    geo_prep_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, st>>>(pa);
  }

  AttnArgs t{};
  t.B = a.B; t.N = a.N; t.H = a.H; t.VW = VW; t.tau = 8.f;
  t.qg = pa.qg; t.kg = pa.kg; t.vg = pa.vg; t.sc = wa.sc; t.rotf = pa.rotf;
  t.pm = a.has_pair_mask ? reinterpret_cast<const unsigned char*>(a.pair_mask.p) : nullptr;
  for (int d = 0; d < 4; ++d) t.pms[d] = a.has_pair_mask ? a.pair_mask.s[d] : 0;
  t.out_vectors = a.out_vectors;
  t.ml = reinterpret_cast<float2*>(ws + w.ml);
  t.live = ws + w.live;
  t.agg = a.out_agg;
  t.err = a.err;
  cudaError_t le = cudaErrorInvalidValue;
  switch (a.M) {
    case 1: le = launch_attn<1>(t, a.B, a.N, a.H, st); break;
    case 2: le = launch_attn<2>(t, a.B, a.N, a.H, st); break;
    case 3: le = launch_attn<3>(t, a.B, a.N, a.H, st); break;
    case 4: le = launch_attn<4>(t, a.B, a.N, a.H, st); break;
    case 5: le = launch_attn<5>(t, a.B, a.N, a.H, st); break;
    case 6: le = launch_attn<6>(t, a.B, a.N, a.H, st); break;
    case 7: le = launch_attn<7>(t, a.B, a.N, a.H, st); break;
    case 8: le = launch_attn<8>(t, a.B, a.N, a.H, st); break;
    default: break;
  }
  if (le != cudaSuccess) return le;

  if (a.out_attention) {
    MapArgs ma{};
    ma.B = a.B; ma.N = a.N; ma.H = a.H;
    ma.qg = pa.qg; ma.kg = pa.kg; ma.sc = wa.sc; ma.ml = t.ml;
    ma.pm = t.pm;
    for (int d = 0; d < 4; ++d) ma.pms[d] = t.pms[d];
    ma.att = a.out_attention;
    ma.err = a.err;
    geo_map_kernel<<<dim3((a.N + MAP_ROWS - 1) / MAP_ROWS, a.H, a.B), 256, 0, st>>>(ma);
  }

  if (a.skip_readout) return cudaGetLastError();

  ReadArgs ra{};
  ra.B = a.B; ra.N = a.N; ra.H = a.H; ra.HM3 = a.HM3; ra.Cout = a.Cout;
  ra.vec = a.out_vectors; ra.live = t.live; ra.wf = wa.wf; ra.bf = wa.bf; ra.out = a.out_output;
  ra.err = a.err;
  {
    const int64_t rows = static_cast<int64_t>(a.B) * a.N;
    dim3 grid(static_cast<unsigned>((rows + RD_TM - 1) / RD_TM), static_cast<unsigned>((a.Cout + RD_TN - 1) / RD_TN));
    geo_readout_kernel<<<grid, 256, 0, st>>>(ra);
  }
  return cudaGetLastError();
}

}  // namespace fipa
