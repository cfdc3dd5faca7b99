// Output pass of the fused IPA core, shared by the single-CTA and the
// CTA-pair attention kernels.
//
// The softmax threads stage, per query row of a 128-row tile, the normalised
// accumulators and the row's frame in shared memory:
//
//   [ O_v (64) | O_pair (DZ) | R (9, row-major) | t - centroid (3) | dead (1) | pad ]
//
// with O_v = [o (C) | gv hi (3 Pv) | gv lo (3 Pv)] (value points relative to
// the centroid) and O_pair = sum_j a_ij z2_j.  Eight warps then write the
// rows of the tile, one row per warp at a time, consecutive lanes on
// consecutive output features (coalesced stores):
//
//   out[b, i, h, :] = [ o (C) | R_i^T (gv - t_i) (3 Pv) | |.| per point (Pv) |
//                       sum_r z1_i[r] (.) O_pair[r] (Cz) ]
//
// (Flash Invariant Point Attention, TL;DR: the factorised pair output; the
// point output is mapped back into the residue's local frame as in the IPA
// formulation.)  A row with no allowed key is written as zeros.
#pragma once

#include <cstdint>

#include "bounds.cuh"
#include "sm100.cuh"

#pragma push_macro("IPA_FILE_TAG")
#undef IPA_FILE_TAG
#define IPA_FILE_TAG 4

namespace fipa {

// Frame columns of a staged row start at 64 + DZ; the pitch is 4 x odd floats
// so that per-thread float4 stores of consecutive rows are conflict-free.
__host__ __device__ constexpr int stage_pitch(int DZ) { return 64 + DZ + 20; }

__device__ __forceinline__ void stage_frame(float* orow_frame, float4 g0, float4 g1, float4 g2, float4 cn,
                                            bool dead) {
  *reinterpret_cast<float4*>(orow_frame) = g0;
  *reinterpret_cast<float4*>(orow_frame + 4) = g1;
  *reinterpret_cast<float4*>(orow_frame + 8) = make_float4(g2.x, g2.y - cn.x, g2.z - cn.y, g2.w - cn.z);
  orow_frame[12] = dead ? 1.f : 0.f;
}

struct EpilogueArgs {
  float* stage;          // 128 staged rows
  int DZ, Cz, RCz, F, H, L;
  int b, h, row0;        // first query row of the tile
  const float* z1f;      // [B, L, DZ] fp32, zero-padded
  float* out;            // [B, L, H, F]
  float* uagg = nullptr; // training forward only: [B, L, H, R Cz] pair aggregate U (else null)
  int64_t rows = 0;      // B L H: output rows (extent of out and uagg in rows; bounds-checked build)
  int* err = nullptr;    // error word of the bounds-checked build
#ifdef IPA_TRACE
  unsigned long long* trace = nullptr;   // phase clocks of warp 0 (tracing build only)
#endif
};

// One output row, written by one warp from its staged row O (the pair sums
// sum_r z1 (.) O_pair already reduced into O[64 .. 64 + Cz)):
//   * point p, coordinate x on lane 3p + x: g = gv - t' (hi + lo), the three
//     coordinates of a point meet by shuffles, R^T g, then the norm on lane p;
//   * pair feature cc on the lane of its output position.
// The lane-to-feature map below is written for C = 16, PV = 8: output chunk 0
// is [o (16) | coordinates 0..15], chunk 1 is [coordinates 16..23 | norms (8) |
// pair 0..15], later chunks are pair features.  No loop here has a runtime
// trip count, so the loads of a row issue together.
template <int C, int PV>
__device__ __forceinline__ void write_row(const float* O, float* dst, int lane, int DZ, int F) {
  static_assert(C == 16 && PV == 8, "output lane map assumes the (16, 8) head shape");
  const int FR = 64 + DZ;
  const int l = lane < 3 * PV ? lane : 0;
  const int x = l % 3, p3 = l - x;
  const float gd = O[C + l] + O[C + 3 * PV + l] - O[FR + 9 + x];
  const float r0 = O[FR + x], r1 = O[FR + 3 + x], r2 = O[FR + 6 + x];
  const float own = O[lane];
  const bool rdead = O[FR + 12] != 0.f;
  float pv[9];                          // pair features of output chunks 1..9 (F = 48 + Cz <= 304)
#pragma unroll
  for (int k = 1; k < 10; ++k) {
    const int f = 32 * k + lane;
    const int cc = f - C - 4 * PV;
    pv[k - 1] = (cc >= 0 && f < F) ? O[64 + cc] : 0.f;
  }
  const float g0 = __shfl_sync(0xffffffffu, gd, p3);
  const float g1 = __shfl_sync(0xffffffffu, gd, p3 + 1);
  const float g2 = __shfl_sync(0xffffffffu, gd, p3 + 2);
  const float op = fmaf(r0, g0, fmaf(r1, g1, r2 * g2));   // (R^T g)_x
  const float sq = op * op;
  const int pp = (lane < PV ? lane : 0) * 3;
  const float nrm = sqrtf(__shfl_sync(0xffffffffu, sq, pp) + __shfl_sync(0xffffffffu, sq, pp + 1) +
                          __shfl_sync(0xffffffffu, sq, pp + 2));
  const float c_lo = __shfl_sync(0xffffffffu, op, (lane - 16) & 31);   // coordinates 0..15 on lanes 16..31
  const float c_hi = __shfl_sync(0xffffffffu, op, (lane + 16) & 31);   // coordinates 16..23 on lanes 0..7
  const float n_p = __shfl_sync(0xffffffffu, nrm, (lane - 8) & 31);    // norms on lanes 8..15
#pragma unroll
  for (int k = 0; k < 10; ++k) {
    const int f = 32 * k + lane;
    float val;
    if (k == 0) val = lane < C ? own : c_lo;
    else if (k == 1 && lane < 8) val = c_hi;
    else if (k == 1 && lane < 16) val = n_p;
    else val = pv[k - 1];
    if (f < F) dst[f] = rdead ? 0.f : val;
  }
}

// Phase A for the 16 rows of one warp: z1 (.) O_pair summed over the R
// factors into O_pair[0 .. Cz) of each staged row.  z1 rows are read as
// float4 (lane q holds columns 4q .. 4q + 3 and 128 + 4q ..), four rows ahead
// of the row being folded: wide loads keep the number of outstanding L1 requests
// low, which is what bounds this phase.  When Cz % 128 == 0 all R factors of
// a pair feature sit on one lane and fold in registers; otherwise the
// products are written in place and reduced in a second, float4 pass.
static __device__ __noinline__ void fold_pairs_rows(const EpilogueArgs& e, int warp, int lane) {
  if (e.RCz == 0) return;                     // no pair block (distance-aware attention)
  const int pitch = stage_pitch(e.DZ);
  const int nq = e.RCz >> 2;                  // float4 columns holding pair factors (RCz % 16 == 0)
  const int R = e.RCz / e.Cz, cq = e.Cz >> 2;
  const bool lane_local = (e.Cz & 127) == 0;
  const float4 zero4 = make_float4(0.f, 0.f, 0.f, 0.f);
  constexpr int AHEAD = 4;                    // rows of z1 in flight ahead of the row being folded
  float4 zb[AHEAD + 1][2];
  auto load_row = [&](int rr, float4 (&z)[2]) {
    const int grow = e.row0 + warp * 16 + rr;
    const bool in = rr < 16 && grow < e.L;
    const float4* zr =
        reinterpret_cast<const float4*>(e.z1f + (static_cast<int64_t>(e.b) * e.L + (in ? grow : 0)) * e.DZ);
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int q = lane + 32 * u;
      z[u] = (in && q < nq) ? __ldg(zr + q) : zero4;
    }
  };
  auto mul4 = [](float4 a, float4 b) { return make_float4(a.x * b.x, a.y * b.y, a.z * b.z, a.w * b.w); };
#pragma unroll
  for (int rr = 0; rr < AHEAD; ++rr) load_row(rr, zb[rr]);
#pragma unroll
  for (int rr = 0; rr < 16; ++rr) {
    load_row(rr + AHEAD, zb[(rr + AHEAD) % (AHEAD + 1)]);
    float4* P = reinterpret_cast<float4*>(e.stage + (warp * 16 + rr) * pitch + 64);
    const float4 z0 = zb[rr % (AHEAD + 1)][0], z1 = zb[rr % (AHEAD + 1)][1];
    if (lane_local && R == 2) {              // Cz = 128: columns lane and 32 + lane hold factors 0 and 1
      const float4 o0 = P[lane], o1 = P[32 + lane];
      P[lane] = make_float4(fmaf(z1.x, o1.x, z0.x * o0.x), fmaf(z1.y, o1.y, z0.y * o0.y),
                            fmaf(z1.z, o1.z, z0.z * o0.z), fmaf(z1.w, o1.w, z0.w * o0.w));
    } else {                                 // R == 1, or products in place before the reduction
      if (lane < nq) P[lane] = mul4(P[lane], z0);
      if (32 + lane < nq) P[32 + lane] = mul4(P[32 + lane], z1);
    }
  }
  __syncwarp();
  if (!lane_local && R > 1) {
    for (int rr = 0; rr < 16; ++rr) {
      float4* P = reinterpret_cast<float4*>(e.stage + (warp * 16 + rr) * pitch + 64);
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int c4 = lane + 32 * u;
        if (c4 < cq) {
          float4 acc = P[c4];
          for (int r2 = 1; r2 < R; ++r2) {
            const float4 v = P[r2 * cq + c4];
            acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
          }
          P[c4] = acc;
        }
      }
    }
    __syncwarp();
  }
}

// Training forward: the normalised pair aggregate U_i = sum_j a_ij z2_j of
// the warp's 16 rows, R Cz floats per row, copied out of the stage before
// phase A folds it with z1 (rows without an allowed key hold zeros).
static __device__ __noinline__ void store_pair_aggregate(const EpilogueArgs& e, int warp, int lane) {
  const int pitch = stage_pitch(e.DZ);
  const int nq = e.RCz >> 2;                  // float4 per row (RCz % 16 == 0)
  for (int rr = 0; rr < 16; ++rr) {
    const int grow = e.row0 + warp * 16 + rr;
    if (grow >= e.L) break;
    const float4* src = reinterpret_cast<const float4*>(e.stage + (warp * 16 + rr) * pitch + 64);
    float4* dst = reinterpret_cast<float4*>(IPA_SPAN(e.uagg, ((static_cast<int64_t>(e.b) * e.L + grow) * e.H + e.h) * e.RCz,
                                                     e.RCz, e.rows * e.RCz, e.err));
    for (int q = lane; q < nq; q += 32) dst[q] = src[q];
  }
  __syncwarp();
}

// Called by all 8 warps (warp = 0..7) after the staged rows are complete;
// warp w handles rows 16 w .. 16 w + 15 of the tile: phase A (above), then
// phase B: the output rows with coalesced stores.  No global load is issued after a global store.
template <int C, int PV>
__device__ __forceinline__ void write_rows(const EpilogueArgs& e, int warp, int lane) {
  const int pitch = stage_pitch(e.DZ);
#ifdef IPA_TRACE
#define EPI_TR(k)                                                  \
  do {                                                             \
    if (e.trace != nullptr && lane == 0) e.trace[(k)] = clock64(); \
  } while (0)
#else
#define EPI_TR(k) \
  do {            \
  } while (0)
#endif
  EPI_TR(0);
  if (e.uagg != nullptr) store_pair_aggregate(e, warp, lane);
  fold_pairs_rows(e, warp, lane);
  EPI_TR(1);
#pragma unroll 2
  for (int rr = 0; rr < 16; ++rr) {
    const int rloc = warp * 16 + rr;
    const int grow = e.row0 + rloc;
    if (grow < e.L)
      write_row<C, PV>(e.stage + rloc * pitch,
                       IPA_SPAN(e.out, ((static_cast<int64_t>(e.b) * e.L + grow) * e.H + e.h) * e.F, e.F, e.rows * e.F,
                                e.err),
                       lane, e.DZ, e.F);
    EPI_TR(3 + rr);
  }
  EPI_TR(2);
}

#undef EPI_TR

// Direct output pass for the CTA-pair kernel, whose tensor memory holds
// [O_pair (DZ) | O_v (64)] per row, when the pair block has no padding
// (R Cz == DZ) and Cz is a multiple of 64.  Thread (row, half) folds z1
// into the pair features c in [half Cz/2, (half + 1) Cz/2), 32 at a time,
// straight from tensor memory (for each factor r: O_pair[r Cz + c] / l
// times z1_i[r, c], summed over r in the order of the staged pass), and
// writes them as 16-byte stores; half 0 also writes the scalar outputs, the
// value points mapped back with R_i^T and their norms.  No shared-memory
// stage and no per-warp pass over rows: the z1 loads of all rows are in
// flight together.  tcgen05.ld is warp-collective, so every lane loads
// and only the stores depend on the row being in range.
template <int C, int PV>
__device__ __forceinline__ void write_row_points(uint32_t tmem_v, float inv, bool dead, bool in_range, float* outr,
                                                 float4 g0, float4 g1, float4 g2, float4 cn);

template <int C, int PV>
__device__ __forceinline__ void write_row_direct(uint32_t tmem_row, int half, int DZ, int Cz, int R, float inv,
                                                 bool dead, bool in_range, const float* z1r, float* outr, float* ur,
                                                 float4 g0, float4 g1, float4 g2, float4 cn,
                                                 unsigned long long* trace = nullptr) {
  static_assert(C == 16 && PV == 8, "feature map written for the (16, 8) head shape");
  for (int c0 = half * (Cz / 2); c0 < (half + 1) * (Cz / 2); c0 += 32) {
    float acc[32];
    for (int rf = 0; rf < R; ++rf) {
      uint32_t o[32];
      sm100::tmem_ld32(tmem_row + rf * Cz + c0, o);
      float4 z[8];
      const float4* zp = reinterpret_cast<const float4*>(z1r + rf * Cz + c0);
#pragma unroll
      for (int e = 0; e < 8; ++e) z[e] = __ldg(zp + e);
      sm100::tmem_ld_wait();
      float u[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) u[e] = __uint_as_float(o[e]) * inv;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float zz[4] = {z[e].x, z[e].y, z[e].z, z[e].w};
#pragma unroll
        for (int k = 0; k < 4; ++k) acc[4 * e + k] = rf == 0 ? zz[k] * u[4 * e + k] : fmaf(zz[k], u[4 * e + k], acc[4 * e + k]);
      }
      if (ur != nullptr && in_range) {
        float4* up = reinterpret_cast<float4*>(ur + rf * Cz + c0);
#pragma unroll
        for (int e = 0; e < 8; ++e) up[e] = make_float4(u[4 * e], u[4 * e + 1], u[4 * e + 2], u[4 * e + 3]);
      }
    }
    if (in_range) {
      float4* op = reinterpret_cast<float4*>(outr + C + 4 * PV + c0);
#pragma unroll
      for (int e = 0; e < 8; ++e) op[e] = make_float4(acc[4 * e], acc[4 * e + 1], acc[4 * e + 2], acc[4 * e + 3]);
    }
  }
  if (trace != nullptr) trace[0] = clock64();   // tracing build: end of the pair part
  if (half == 0) write_row_points<C, PV>(tmem_row + DZ, inv, dead, in_range, outr, g0, g1, g2, cn);
}

// Pair features of the CTA's rows through shared memory, for the layouts
// the tensor-memory copy supports (R Cz = DZ, Cz a multiple of 32): z1 rows
// come from TMA-loaded boxes and the folded features go to staging boxes
// that one thread then stores with TMA.  Both are 128-row x 32-float boxes
// with the 128-byte swizzle (16-byte chunk e of row r at byte 16 (e ^ (r & 7))
// of the row), so thread-per-row float4 accesses are free of bank conflicts.
// z1box(k): box k of the z1 row (columns 32 k ..); obox(k): staging box of
// output pair features 32 k ..
template <typename ZBox, typename OBox>
__device__ __forceinline__ void stage_row_pair(uint32_t tmem_row, int half, int Cz, int R, float inv, int r,
                                               float* ur, bool in_range, ZBox z1box, OBox obox) {
  const int sw = r & 7;
  for (int c0 = half * (Cz / 2); c0 < (half + 1) * (Cz / 2); c0 += 32) {
    float acc[32];
    for (int rf = 0; rf < R; ++rf) {
      uint32_t o[32];
      sm100::tmem_ld32(tmem_row + rf * Cz + c0, o);
      const unsigned char* zrow = z1box((rf * Cz + c0) >> 5) + r * 128;
      float4 z[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) z[e] = *reinterpret_cast<const float4*>(zrow + 16 * (e ^ sw));
      sm100::tmem_ld_wait();
      float u[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) u[e] = __uint_as_float(o[e]) * inv;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float zz[4] = {z[e].x, z[e].y, z[e].z, z[e].w};
#pragma unroll
        for (int k = 0; k < 4; ++k) acc[4 * e + k] = rf == 0 ? zz[k] * u[4 * e + k] : fmaf(zz[k], u[4 * e + k], acc[4 * e + k]);
      }
      if (ur != nullptr && in_range) {
        float4* up = reinterpret_cast<float4*>(ur + rf * Cz + c0);
#pragma unroll
        for (int e = 0; e < 8; ++e) up[e] = make_float4(u[4 * e], u[4 * e + 1], u[4 * e + 2], u[4 * e + 3]);
      }
    }
    unsigned char* orow = obox(c0 >> 5) + r * 128;
#pragma unroll
    for (int e = 0; e < 8; ++e)
      *reinterpret_cast<float4*>(orow + 16 * (e ^ sw)) = make_float4(acc[4 * e], acc[4 * e + 1], acc[4 * e + 2], acc[4 * e + 3]);
  }
}

// Scalar and point features of one row (the value aggregate O_v in tensor
// memory at tmem_v): v / l, the value points mapped back with R^T, their norms.
template <int C, int PV>
__device__ __forceinline__ void write_row_points(uint32_t tmem_v, float inv, bool dead, bool in_range, float* outr,
                                                 float4 g0, float4 g1, float4 g2, float4 cn) {
  {
    uint32_t v0[32], v1[32];
    sm100::tmem_ld32(tmem_v, v0);
    sm100::tmem_ld32(tmem_v + 32, v1);
    sm100::tmem_ld_wait();
    if (!in_range) return;
    float4* op = reinterpret_cast<float4*>(outr);
    if (dead) {
#pragma unroll
      for (int e = 0; e < (C + 4 * PV) / 4; ++e) op[e] = make_float4(0.f, 0.f, 0.f, 0.f);
      return;
    }
    // O_v = [v (C) | gv hi (3 PV) | gv lo (3 PV)] relative to the centroid
    float f[C + 4 * PV];
#pragma unroll
    for (int e = 0; e < C; ++e) f[e] = __uint_as_float(v0[e]) * inv;
    const float Rm[9] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w, g2.x};
    const float tp[3] = {g2.y - cn.x, g2.z - cn.y, g2.w - cn.z};
#pragma unroll
    for (int p = 0; p < PV; ++p) {
      float g[3];
#pragma unroll
      for (int x = 0; x < 3; ++x) {
        const int hi = C + 3 * p + x, lo = C + 3 * PV + 3 * p + x;
        const float a = __uint_as_float(hi < 32 ? v0[hi & 31] : v1[hi & 31]) * inv;
        const float bb = __uint_as_float(lo < 32 ? v0[lo & 31] : v1[lo & 31]) * inv;
        g[x] = a + bb - tp[x];
      }
      float sqs = 0.f;
#pragma unroll
      for (int x = 0; x < 3; ++x) {
        const float o = fmaf(Rm[x], g[0], fmaf(Rm[3 + x], g[1], Rm[6 + x] * g[2]));   // (R^T g)_x
        f[C + 3 * p + x] = o;
        sqs = x == 0 ? o * o : sqs + o * o;
      }
      f[C + 3 * PV + p] = sqrtf(sqs);
    }
#pragma unroll
    for (int e = 0; e < (C + 4 * PV) / 4; ++e) op[e] = make_float4(f[4 * e], f[4 * e + 1], f[4 * e + 2], f[4 * e + 3]);
  }
}

}  // namespace fipa

#pragma pop_macro("IPA_FILE_TAG")
