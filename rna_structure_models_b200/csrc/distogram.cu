// Local nearest-neighbour distogram of residue positions (Flash Invariant
// Point Attention, TL;DR: pair information from "a local nearest-neighbor
// distogram"; the page gives no neighbour count, bins or factor map, so the
// count and the bin edges are parameters of the call).
//
// One warp per residue i: every lane scans the keys j = lane, lane + 32, ...
// and keeps its KM nearest valid j != i in a sorted register list keyed by
// (float32 squared distance, j) packed into one 64-bit integer (non-negative
// floats order like their bit patterns), so lexicographic order -- nearest
// first, equal distances in increasing j -- is integer order.  The warp then
// merges the 32 lists k times by a butterfly minimum.  Lane s keeps result s:
// neighbour index, its bin against the squared edges, and the warp counts
// the bins with ballots for the histogram.  Squared distances are evaluated
// as (dx*dx + dy*dy) + dz*dz with round-to-nearest operations and no
// contraction, so that every integer result is fixed by float32 arithmetic.
#include <cuda_runtime.h>

#include <cstdint>

#include "bounds.cuh"
#include "internal.h"

#define IPA_FILE_TAG 12

namespace fipa {

namespace {

__device__ __forceinline__ uint64_t umin64(uint64_t a, uint64_t b) { return a < b ? a : b; }
__device__ __forceinline__ uint64_t umax64(uint64_t a, uint64_t b) { return a < b ? b : a; }

template <int KM>
__global__ void __launch_bounds__(256) knn_distogram_kernel(const DistogramArgs a) {
  const int64_t wid = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (wid >= static_cast<int64_t>(a.B) * a.L) return;
  const int i = static_cast<int>(wid % a.L), b = static_cast<int>(wid / a.L);
  const float* xp = static_cast<const float*>(a.x.p);
  const unsigned char* mp = static_cast<const unsigned char*>(a.mask.p);
  const int64_t xb = b * a.x.s[0], mbase = b * a.mask.s[0];
  auto X = [&](int r, int c) { return xp[xb + r * a.x.s[1] + c * a.x.s[2]]; };
  auto valid_at = [&](int r) { return mp[mbase + r * a.mask.s[1]] != 0; };
  const int64_t nres = static_cast<int64_t>(a.B) * a.L;
  int32_t* idx = IPA_SPAN(a.idx, wid * a.k, a.k, nres * a.k, a.err);
  int32_t* bins = IPA_SPAN(a.bins, wid * a.k, a.k, nres * a.k, a.err);
  float* hist = IPA_SPAN(a.hist, wid * a.nb, a.nb, nres * a.nb, a.err);
  const bool valid = valid_at(i);

  uint64_t keys[KM];
#pragma unroll
  for (int s = 0; s < KM; ++s) keys[s] = ~0ull;
  if (valid) {
    const float xi = X(i, 0), yi = X(i, 1), zi = X(i, 2);
    for (int j = lane; j < a.L; j += 32) {
      if (j == i || !valid_at(j)) continue;
      const float dx = __fsub_rn(X(j, 0), xi), dy = __fsub_rn(X(j, 1), yi), dz = __fsub_rn(X(j, 2), zi);
      const float d2 = __fadd_rn(__fadd_rn(__fmul_rn(dx, dx), __fmul_rn(dy, dy)), __fmul_rn(dz, dz));
      const uint64_t key = (static_cast<uint64_t>(__float_as_uint(d2)) << 32) | static_cast<uint32_t>(j);
      if (key < keys[KM - 1]) {
        uint64_t cur = key;                     // carry the larger value up the sorted list
#pragma unroll
        for (int s = 0; s < KM; ++s) {
          const uint64_t lo = umin64(keys[s], cur);
          cur = umax64(keys[s], cur);
          keys[s] = lo;
        }
      }
    }
  }
  // k rounds of a warp-wide minimum over the lanes' list heads
  uint64_t mine = ~0ull;
  for (int s = 0; s < a.k; ++s) {
    uint64_t m = keys[0];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = umin64(m, __shfl_xor_sync(0xffffffffu, m, off));
    if (m != ~0ull && keys[0] == m) {           // the owning lane pops its head
#pragma unroll
      for (int t = 0; t + 1 < KM; ++t) keys[t] = keys[t + 1];
      keys[KM - 1] = ~0ull;
    }
    if (lane == s) mine = m;
  }
  int bin = -1, nbr = -1;
  if (lane < a.k && mine != ~0ull) {
    nbr = static_cast<int>(mine & 0xffffffffu);
    const float d2 = __uint_as_float(static_cast<uint32_t>(mine >> 32));
    bin = 0;
    for (int m = 0; m < a.nb - 1; ++m) bin += d2 >= a.edge2[m] ? 1 : 0;
  }
  if (lane < a.k) {
    idx[lane] = nbr;
    bins[lane] = bin;
  }
  for (int c0 = 0; c0 < a.nb; c0 += 32) {
    int cnt = 0;
    for (int c = c0; c < c0 + 32 && c < a.nb; ++c) {
      const int n = __popc(__ballot_sync(0xffffffffu, bin == c));
      if (lane == c - c0) cnt = n;
    }
    if (c0 + lane < a.nb) hist[c0 + lane] = static_cast<float>(cnt);
  }
}

}  // namespace

cudaError_t distogram_launch(const DistogramArgs& a, cudaStream_t stream) {
  const int64_t warps = static_cast<int64_t>(a.B) * a.L;
  const unsigned blocks = static_cast<unsigned>((warps + 7) / 8);
  if (a.k <= 8)
    knn_distogram_kernel<8><<<blocks, 256, 0, stream>>>(a);
  else if (a.k <= 16)
    knn_distogram_kernel<16><<<blocks, 256, 0, stream>>>(a);
  else
    knn_distogram_kernel<32><<<blocks, 256, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace fipa
