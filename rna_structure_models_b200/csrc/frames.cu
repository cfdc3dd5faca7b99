// Residue frames from backbone atoms (Flash Invariant Point Attention,
// Figure 1: the frame sits on C_alpha and C_alpha -> C, C_alpha -> N span it
// by Gram-Schmidt):
//   e1 = (C - CA) / |C - CA|,  e2 = normalise((N - CA) - (e1 . (N - CA)) e1),
//   e3 = e1 x e2,  R = [e1 | e2 | e3] (columns),  t = CA.
#include <cstdint>

#include "bounds.cuh"
#include "internal.h"

#define IPA_FILE_TAG 9

namespace fipa {

namespace {

__global__ void __launch_bounds__(256) frames_kernel(const FramesArgs a) {
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= static_cast<int64_t>(a.B) * a.L) return;
  const int i = static_cast<int>(t % a.L), b = static_cast<int>(t / a.L);
  auto atom = [&](const View& v, float (&x)[3]) {
    const float* p = static_cast<const float*>(v.p) + b * v.s[0] + i * v.s[1];
#pragma unroll
    for (int d = 0; d < 3; ++d) x[d] = p[d * v.s[2]];
  };
  float n[3], ca[3], c[3];
  atom(a.n, n);
  atom(a.ca, ca);
  atom(a.c, c);
  float v1[3], v2[3];
#pragma unroll
  for (int d = 0; d < 3; ++d) {
    v1[d] = c[d] - ca[d];
    v2[d] = n[d] - ca[d];
  }
  const float r1 = rsqrtf(fmaf(v1[0], v1[0], fmaf(v1[1], v1[1], v1[2] * v1[2])));
  float e1[3] = {v1[0] * r1, v1[1] * r1, v1[2] * r1};
  const float p = fmaf(e1[0], v2[0], fmaf(e1[1], v2[1], e1[2] * v2[2]));
  float u2[3] = {v2[0] - p * e1[0], v2[1] - p * e1[1], v2[2] - p * e1[2]};
  const float r2 = rsqrtf(fmaf(u2[0], u2[0], fmaf(u2[1], u2[1], u2[2] * u2[2])));
  float e2[3] = {u2[0] * r2, u2[1] * r2, u2[2] * r2};
  float e3[3] = {e1[1] * e2[2] - e1[2] * e2[1], e1[2] * e2[0] - e1[0] * e2[2], e1[0] * e2[1] - e1[1] * e2[0]};
  const int64_t n_res = static_cast<int64_t>(a.B) * a.L;
  float* R = IPA_SPAN(a.rot, t * 9, 9, n_res * 9, a.err);
#pragma unroll
  for (int x = 0; x < 3; ++x) {   // row x of R: (e1_x, e2_x, e3_x)
    R[3 * x] = e1[x];
    R[3 * x + 1] = e2[x];
    R[3 * x + 2] = e3[x];
  }
  float* tr = IPA_SPAN(a.trans, t * 3, 3, n_res * 3, a.err);
  tr[0] = ca[0];
  tr[1] = ca[1];
  tr[2] = ca[2];
}

}  // namespace

cudaError_t frames_launch(const FramesArgs& a, cudaStream_t stream) {
  const int64_t n = static_cast<int64_t>(a.B) * a.L;
  frames_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace fipa
