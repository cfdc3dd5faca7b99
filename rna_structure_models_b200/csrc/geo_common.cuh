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
// is the hardware square-root approximation (sqrt.approx.f32, exact at 0).
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
  g.dist = sm100::sqrt_approx(d2);
  g.s = __fadd_rn(__fadd_rn(fmaf(A, g.dot, -__fmul_rn(Bd, g.dist)), q0.w), k0.w);
  return g;
}

__device__ __forceinline__ float geo_score(const float4 q0, const float4 q1, const float4 k0,
                                           const float4 k1, float A, float Bd) {
  return geo_pair(q0, q1, k0, k1, A, Bd).s;
}

}  // namespace geo
}  // namespace fipa
