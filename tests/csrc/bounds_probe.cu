// Test probe of the bounds-checked build's store check (compiled with
// -DIPA_BOUNDS_CHECK): one thread stores 1.0 through IPA_AT(buf, idx, n, err).
// An index inside [0, n) writes buf[idx]; any other index must leave buf
// untouched, land in the library's scratch area and record
// 0x10000 | (file tag << 12) | line in *err.  Every access stays in bounds by
// construction: the check redirects the out-of-range ones.
#include <cuda_runtime.h>

#include <cstdint>

#include "bounds.cuh"

#define IPA_FILE_TAG 15

namespace {

constexpr int kStoreSite = (IPA_FILE_TAG << 12) | (__LINE__ + 2);   // the checked store two lines below
__global__ void bounds_probe_kernel(float* buf, int64_t n, int64_t idx, int* err) {
  *IPA_AT(buf, idx, n, err) = 1.f;
}

}  // namespace

extern "C" __attribute__((visibility("default"))) int probe_bounds_store(void* buf, long long n, long long idx,
                                                                         void* err, void* stream) {
  bounds_probe_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<float*>(buf), n, idx,
                                                                      static_cast<int*>(err));
  return cudaGetLastError() == cudaSuccess ? 0 : 1;
}

// Source line of the checked store above (the code the probe must record).
extern "C" __attribute__((visibility("default"))) int probe_bounds_site(void) { return kStoreSite; }
