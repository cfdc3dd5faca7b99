// Bounds-checked build of the kernels (compiled with -DIPA_BOUNDS_CHECK; off
// in the product build).
//
// Every pointer a kernel stores through to global memory is formed by
// IPA_SPAN(base, idx, n, extent, err): the elements [idx, idx + n) that the
// store (or the run of stores through the returned pointer) covers are
// checked against the extent of the destination buffer, which the kernel
// computes from the call's shapes.  A span outside [0, extent) records
//   DEV_BOUNDS | (file tag << 12) | source line
// in the caller's error word (first error wins) and the pointer is redirected
// to a per-module scratch area, so the kernel runs on without touching memory
// outside its buffers and the host reads back where the bad index was formed.
// Spans are at most kSinkBytes long.  IPA_CHECK(cond, err) records the same
// code for a condition that must hold before an access the hardware performs
// (a TMA store coordinate) and returns it, so that the access is skipped.  In
// the product build IPA_SPAN is the plain pointer arithmetic and IPA_CHECK
// is true.
#pragma once

#include <cstdint>

namespace fipa_bounds {

constexpr int kDevBounds = 0x10000;   // bit 16 of the error word: a span outside its buffer
constexpr int64_t kSinkBytes = 16384;

#ifdef IPA_BOUNDS_CHECK
static __device__ __align__(128) unsigned char g_sink[kSinkBytes];

__device__ __forceinline__ void record(int* err, int site) {
  if (err != nullptr) atomicCAS(err, 0, kDevBounds | site);
}

template <class T>
__device__ __forceinline__ T* span(T* base, int64_t idx, int64_t n, int64_t extent, int* err, int site) {
  const bool ok = idx >= 0 && n >= 0 && idx + n <= extent && n * static_cast<int64_t>(sizeof(T)) <= kSinkBytes;
  if (ok) return base + idx;
  record(err, site);
  return reinterpret_cast<T*>(g_sink);
}

__device__ __forceinline__ bool check(bool cond, int* err, int site) {
  if (!cond) record(err, site);
  return cond;
}
#else
template <class T>
__device__ __forceinline__ T* span(T* base, int64_t idx, int64_t, int64_t, int*, int) {
  return base + idx;
}
__device__ __forceinline__ bool check(bool, int*, int) { return true; }
#endif

}  // namespace fipa_bounds

// Source tag of a check: each translation unit (and each header with stores)
// defines IPA_FILE_TAG (0..15) before its first IPA_SPAN.
#define IPA_SITE ((IPA_FILE_TAG << 12) | (__LINE__ & 0xfff))
#define IPA_SPAN(base, idx, n, extent, err)                                                          \
  ::fipa_bounds::span((base), static_cast<int64_t>(idx), static_cast<int64_t>(n),                    \
                      static_cast<int64_t>(extent), (err), IPA_SITE)
#define IPA_AT(base, idx, extent, err) IPA_SPAN(base, idx, 1, extent, err)
#define IPA_CHECK(cond, err) ::fipa_bounds::check((cond), (err), IPA_SITE)
