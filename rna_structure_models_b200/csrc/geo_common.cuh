// Helpers shared by the forward and backward kernels of the geometric
// direction-and-distance attention variant.
#pragma once

#include <cmath>
#include <cstdint>

#include "internal.h"
#include "sm100.cuh"

namespace fipa {
namespace geo {

constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ float ldf(const View& v, int64_t off) {
  if (v.dtype == 1) return static_cast<float>(reinterpret_cast<const double*>(v.p)[off]);
  return reinterpret_cast<const float*>(v.p)[off];
}
__device__ __forceinline__ bool ldb(const View& v, int64_t off) {
  return reinterpret_cast<const unsigned char*>(v.p)[off] != 0;
}

// log(1 + exp(x)) without overflow: max(x, 0) + log1p(exp(-|x|))
__device__ __forceinline__ float softplus_stable(float x) {
  return fmaxf(x, 0.f) + log1pf(expf(-fabsf(x)));
}

// Score in the log2 domain and its parts.  The same operation sequence is
// used by the aggregation kernel (in packed pairs: fma.rn.f32x2 etc. round
// each lane exactly like the scalar operation), the attention-map kernel and
// the gradient kernels, so all of them see identical values.  The distance
// is the hardware square-root approximation with subnormals flushed
// (sqrt.approx.ftz.f32: exact at 0; a squared distance below the smallest
// normal float, |d| < 1.1e-19, counts as 0).
__device__ __forceinline__ float dist_sqrt(float d2) {
  float y;
  asm("sqrt.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(d2));
  return y;
}

// Bit t (t < 4) set iff byte t of w is nonzero.  ((b & 0x7f) + 0x7f) | b has
// its top bit set iff the byte b is nonzero, with no carry into the next byte
// ((b & 0x7f) + 0x7f <= 0xfe); shifted to bit 8 t, the four flags are
// gathered into bits 24 .. 27 by one multiplication by 2^24 + 2^17 + 2^10 +
// 2^3, whose sixteen partial products land on distinct bits.
__device__ __forceinline__ uint32_t nonzero_byte_bits(uint32_t w) {
  const uint32_t h = ((((w & 0x7f7f7f7fu) + 0x7f7f7f7fu) | w) & 0x80808080u) >> 7;
  return ((h * 0x01020408u) >> 24) & 0xfu;
}

struct GeoPair {
  float s;            // log2(e) (A dot - B dist) / sqrt(3) + frame biases
  float dot, dist;    // <qd, kd>, |qp - kp|
  float dx, dy, dz;   // qp - kp
};

__device__ __forceinline__ GeoPair geo_pair(const float4 q0, const float4 q1, const float4 k0,
                                            const float4 k1, float A, float Bd) {
  GeoPair g;
  g.dot = fmaf(q0.x, k0.x, fmaf(q0.y, k0.y, __fmul_rn(q0.z, k0.z)));
  g.dx = __fsub_rn(q1.x, k1.x);
  g.dy = __fsub_rn(q1.y, k1.y);
  g.dz = __fsub_rn(q1.z, k1.z);
  const float d2 = fmaf(g.dx, g.dx, fmaf(g.dy, g.dy, __fmul_rn(g.dz, g.dz)));
  g.dist = dist_sqrt(d2);
  g.s = __fadd_rn(__fadd_rn(fmaf(A, g.dot, -__fmul_rn(Bd, g.dist)), q0.w), k0.w);
  return g;
}

__device__ __forceinline__ float geo_score(const float4 q0, const float4 q1, const float4 k0,
                                           const float4 k1, float A, float Bd) {
  return geo_pair(q0, q1, k0, k1, A, Bd).s;
}

// Register-tiled fp32 product on the CUDA cores for the small dense products
// of the variant (the readout, and the two products of its gradient): a
// 256-thread block computes the TM x TN tile at (r0, c0) of C = A B.  Thread
// (ty, tx) = (tid / 16, tid % 16) owns rows r0 + ty + 16 i and columns
// c0 + tx + 16 j.  K is staged 32 at a time in shared memory (A transposed,
// so that a k-column of the tile is contiguous); the next 32 are loaded into
// registers while the current ones are multiplied.  Every output accumulates
// fmaf(a_k, b_k, acc) in increasing k, the order of a plain loop over k.
// load_a(r, k) and load_b(k, c) return the operands, 0 outside the matrices.
template <int TM, int TN, class LoadA, class LoadB>
__device__ __forceinline__ void tile_product(int r0, int c0, int K, LoadA load_a, LoadB load_b,
                                             float (&acc)[TM / 16][TN / 16]) {
  static_assert(TM % 16 == 0 && TN % 16 == 0 && TM <= 64 && TN <= 64, "tile of 16-multiples up to 64");
  constexpr int NA = 32 * TM / 256, NB = 32 * TN / 256;   // staged values per thread
  __shared__ float As[32][TM + 1];
  __shared__ float Bs[32][TN + 1];
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
#pragma unroll
  for (int i = 0; i < TM / 16; ++i)
#pragma unroll
    for (int j = 0; j < TN / 16; ++j) acc[i][j] = 0.f;
  float ra[NA], rb[NB];
  auto fetch = [&](int k0) {
#pragma unroll
    for (int u = 0; u < NA; ++u) {   // A[r0 + r][k0 + k], k fastest across threads
      const int e = tid + 256 * u, r = e >> 5, k = e & 31;
      ra[u] = load_a(r0 + r, k0 + k);
    }
#pragma unroll
    for (int u = 0; u < NB; ++u) {   // B[k0 + k][c0 + c], c fastest
      const int e = tid + 256 * u, k = e / TN, c = e % TN;
      rb[u] = load_b(k0 + k, c0 + c);
    }
  };
  fetch(0);
  for (int k0 = 0; k0 < K; k0 += 32) {
#pragma unroll
    for (int u = 0; u < NA; ++u) {
      const int e = tid + 256 * u;
      As[e & 31][e >> 5] = ra[u];
    }
#pragma unroll
    for (int u = 0; u < NB; ++u) {
      const int e = tid + 256 * u;
      Bs[e / TN][e % TN] = rb[u];
    }
    __syncthreads();
    if (k0 + 32 < K) fetch(k0 + 32);
    const int kn = K - k0 < 32 ? K - k0 : 32;
    for (int k = 0; k < kn; ++k) {
      float av[TM / 16], bv[TN / 16];
#pragma unroll
      for (int i = 0; i < TM / 16; ++i) av[i] = As[k][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < TN / 16; ++j) bv[j] = Bs[k][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < TM / 16; ++i)
#pragma unroll
        for (int j = 0; j < TN / 16; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
}

}  // namespace geo
}  // namespace fipa
