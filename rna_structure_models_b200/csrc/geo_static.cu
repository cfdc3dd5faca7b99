// geo_attn_fwd_static: the geometric direction/distance attention with its
// scratch memory in a fixed device array owned by this library instead of a
// caller-provided workspace.
//
// Who needs it: callers that are not allowed to allocate device memory at
// the point where they run the operator -- for example an operator hook
// invoked by a host framework that hands out no scratch buffer and forbids
// cudaMalloc on that path (a device allocation can synchronise the device
// and disturb a pre-planned memory pool), or a C program that links this
// library without any allocator of its own.
//
// What it costs: the array below (GEO_STATIC_SCRATCH_BYTES) is reserved on
// every GPU that loads this library, until the process exits.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "flashipa_b200.h"
#include "internal.h"

namespace {

// Scratch shared by every geo_attn_fwd_static call on a device.  In host code
// this name is only a host-side stand-in: its device address must be looked
// up with cudaGetSymbolAddress on each device before a kernel may use it.
static __device__ __align__(256) unsigned char g_geo_scratch[GEO_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
// Per device ordinal: the context the address was looked up in, and the address.
void* g_scratch_ctx[kMaxDevices] = {};
void* g_scratch_addr[kMaxDevices] = {};

using CtxGetCurrentFn = CUresult (*)(CUcontext*);

CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(f);
  });
  return fn;
}

// Device address of the scratch array on the current device.  It is looked
// up (cudaGetSymbolAddress) on the first call in a device's context and again
// whenever that context has changed since (after cudaDeviceReset the module
// is loaded anew and the array may sit elsewhere).
ipa_status_t scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return IPA_ERR_CUDA;
  const CtxGetCurrentFn get_ctx = ctx_get_current();
  if (get_ctx == nullptr) return IPA_ERR_CUDA;
  CUcontext ctx = nullptr;   // null until the runtime has set this device up in this thread
  if (get_ctx(&ctx) != CUDA_SUCCESS) return IPA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (ctx == nullptr || g_scratch_addr[dev] == nullptr || g_scratch_ctx[dev] != static_cast<void*>(ctx)) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_geo_scratch) != cudaSuccess || p == nullptr) return IPA_ERR_CUDA;
    if (get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr) return IPA_ERR_CUDA;
    g_scratch_addr[dev] = p;
    g_scratch_ctx[dev] = static_cast<void*>(ctx);
  }
  *out = g_scratch_addr[dev];
  return IPA_OK;
}

}  // namespace

extern "C" ipa_status_t geo_attn_fwd_static(
    const geo_params_t* p, const ipa_tensor_t* q_direction, const ipa_tensor_t* k_direction,
    const ipa_tensor_t* q_point, const ipa_tensor_t* k_point, const ipa_tensor_t* values,
    const ipa_tensor_t* direction_scale, const ipa_tensor_t* distance_scale,
    const ipa_tensor_t* output_weight, const ipa_tensor_t* output_bias, const ipa_tensor_t* rotation,
    const ipa_tensor_t* translation, const ipa_tensor_t* frame_mask, const ipa_tensor_t* pair_mask,
    const ipa_tensor_t* out_vectors, const ipa_tensor_t* out_output, const ipa_tensor_t* out_attention,
    void* stream, int32_t* dev_err) {
  if (p == nullptr) return IPA_ERR_NULL;
  const size_t need = geo_attn_workspace_size(p);
  if (need == 0) {
    // invalid or unsupported dimensions: let the regular entry point name the reason
    return geo_attn_fwd(p, q_direction, k_direction, q_point, k_point, values, direction_scale,
                        distance_scale, output_weight, output_bias, rotation, translation, frame_mask,
                        pair_mask, out_vectors, out_output, out_attention, nullptr, 0, stream, dev_err);
  }
  if (need > GEO_STATIC_SCRATCH_BYTES) return IPA_ERR_WORKSPACE;
  void* scratch = nullptr;
  const ipa_status_t st = scratch_address(&scratch);
  if (st != IPA_OK) return st;
  // Every region the kernels read is written earlier in the same call, except
  // the error word, which geo_attn_fwd clears itself when dev_err is NULL.
  return geo_attn_fwd(p, q_direction, k_direction, q_point, k_point, values, direction_scale,
                      distance_scale, output_weight, output_bias, rotation, translation, frame_mask,
                      pair_mask, out_vectors, out_output, out_attention, scratch, GEO_STATIC_SCRATCH_BYTES,
                      stream, dev_err);
}
