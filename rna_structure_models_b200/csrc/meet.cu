// Distance-aware attention (MEET §2.2, eq. (6)-(8)) on the fused IPA core.
//
// A_ij = rho_h (<q_i, k_j> - s_h^2 ||x_i - x_j||^2) is an IPA logit with
//   * the scalar term w_L * scalar_scale * q'.k, with w_L = scalar_scale = 1
//     and q' = rho_h q (per-head scale applied here);
//   * the point term -w_L gamma_h w_C / 2 * sum_p ||gq_p - gk_p||^2 over the
//     core's 4 query points, with identity rotations, frame origins t_i = x_i
//     and all local points 0, so every global point is x_i and the sum is
//     4 ||x_i - x_j||^2; w_C = 1/2 and gamma_h = rho_h s_h^2 give
//     -rho_h s_h^2 ||x_i - x_j||^2;
//   * no pair term (w_bias = 0, one 16-channel factor of zeros).
// The outputs o = sum_j a_ij v_j are the first 16 features of the core's
// output row.  The zero / identity operands are stride-0 views of a small
// constant block in the workspace.
#include <cstdint>

#include "bounds.cuh"
#include "internal.h"

#define IPA_FILE_TAG 8

namespace fipa {

namespace {

__global__ void __launch_bounds__(256) meet_prep_kernel(const MeetPrep m) {
  const int64_t n = static_cast<int64_t>(m.B) * m.L * m.H * MEET_C;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t < n) {
    const int c = static_cast<int>(t % MEET_C);
    const int64_t r = t / MEET_C;
    const int h = static_cast<int>(r % m.H);
    const int64_t bi = r / m.H;
    const int i = static_cast<int>(bi % m.L), b = static_cast<int>(bi / m.L);
    const float* q = static_cast<const float*>(m.q.p);
    const float rho = static_cast<const float*>(m.rho.p)[h * m.rho.s[0]];
    *IPA_AT(m.qs, t, n, m.err) = rho * q[b * m.q.s[0] + i * m.q.s[1] + h * m.q.s[2] + c * m.q.s[3]];
  }
  if (blockIdx.x == 0) {
    for (int h = threadIdx.x; h < m.H; h += blockDim.x) {
      const float rho = static_cast<const float*>(m.rho.p)[h * m.rho.s[0]];
      const float s = static_cast<const float*>(m.s.p)[h * m.s.s[0]];
      *IPA_AT(m.gamma, h, m.H, m.err) = rho * s * s;
    }
    // constant block: MEET_ZEROS zeros, then the 3x3 identity
    for (int e = threadIdx.x; e < MEET_ZEROS + 9; e += blockDim.x)
      *IPA_AT(m.consts, e, MEET_ZEROS + 9, m.err) = e < MEET_ZEROS ? 0.f : ((e - MEET_ZEROS) % 4 == 0 ? 1.f : 0.f);
  }
}

// out[r, 0:16] = core_out[r, 0:16] for every (b, i, h) row r
__global__ void __launch_bounds__(256) meet_extract_kernel(const float4* __restrict__ src, float4* __restrict__ dst,
                                                           int64_t rows, int src_row_f4, int* err) {
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= rows * (MEET_C / 4)) return;
  const int64_t r = t / (MEET_C / 4);
  const int q = static_cast<int>(t % (MEET_C / 4));
  *IPA_AT(dst, t, rows * (MEET_C / 4), err) = src[r * src_row_f4 + q];
}

}  // namespace

MeetWorkspace meet_workspace_layout(int B, int L, int H) {
  auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  MeetWorkspace w{};
  const IpaWorkspace core = ipa_workspace_layout(B, L, H, MEET_DZ, MEET_RCZ);
  const size_t rows = static_cast<size_t>(B) * L * H;
  size_t o = 0;
  w.ipa = o; o = up(o + core.total);
  w.qs = o; o = up(o + rows * MEET_C * 4);
  w.gamma = o; o = up(o + static_cast<size_t>(H) * 4);
  w.consts = o; o = up(o + (MEET_ZEROS + 9) * 4);
  w.out = o; o = up(o + rows * MEET_F * 4);
  w.total = o;
  return w;
}

cudaError_t meet_launch_prep(const MeetPrep& m, cudaStream_t stream) {
  const int64_t n = static_cast<int64_t>(m.B) * m.L * m.H * MEET_C;
  const unsigned blocks = static_cast<unsigned>((n + 255) / 256);
  meet_prep_kernel<<<blocks, 256, 0, stream>>>(m);
  return cudaGetLastError();
}

cudaError_t meet_launch_extract(const float* core_out, float* out, int64_t rows, int* err, cudaStream_t stream) {
  const int64_t n = rows * (MEET_C / 4);
  meet_extract_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, stream>>>(
      reinterpret_cast<const float4*>(core_out), reinterpret_cast<float4*>(out), rows, MEET_F / 4, err);
  return cudaGetLastError();
}

}  // namespace fipa
