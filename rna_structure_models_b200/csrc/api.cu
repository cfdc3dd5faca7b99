// Host side of the C ABI declared in include/flashipa_b200.h: argument
// validation, workspace carving, tensor-map encoding and launches.  No device
// memory is allocated here.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <initializer_list>
#include <mutex>

#include "flashipa_b200.h"
#include "internal.h"

namespace fipa {

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                   CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

bool check_tensor(const ipa_tensor_t* t, int dtype, int ndim, const int64_t* sizes, ipa_status_t* st,
                  bool allow_f64 = false) {
  if (t == nullptr || t->data == nullptr) { *st = IPA_ERR_NULL; return false; }
  if (!(t->dtype == dtype || (allow_f64 && t->dtype == IPA_DTYPE_F64))) { *st = IPA_ERR_DTYPE; return false; }
  if (t->ndim != ndim) { *st = IPA_ERR_SHAPE; return false; }
  for (int d = 0; d < ndim; ++d) {
    if (t->size[d] != sizes[d] || sizes[d] < 1) { *st = IPA_ERR_SHAPE; return false; }
    if (t->stride[d] < 0) { *st = IPA_ERR_STRIDE_ALIGN; return false; }
  }
  const int esz = t->dtype == IPA_DTYPE_F64 ? 8 : t->dtype == IPA_DTYPE_BOOL ? 1 : t->dtype == IPA_DTYPE_F16 ? 2 : 4;
  if (reinterpret_cast<uintptr_t>(t->data) % esz != 0) { *st = IPA_ERR_STRIDE_ALIGN; return false; }
  return true;
}

bool check_contiguous_out(const ipa_tensor_t* t, int ndim, const int64_t* sizes, ipa_status_t* st) {
  if (!check_tensor(t, IPA_DTYPE_F32, ndim, sizes, st)) return false;
  int64_t expect = 1;
  for (int d = ndim - 1; d >= 0; --d) {
    if (sizes[d] > 1 && t->stride[d] != expect) { *st = IPA_ERR_STRIDE_ALIGN; return false; }
    expect *= sizes[d];
  }
  if (reinterpret_cast<uintptr_t>(t->data) % 16 != 0) { *st = IPA_ERR_STRIDE_ALIGN; return false; }
  return true;
}

View view_of(const ipa_tensor_t* t) {
  View v{};
  v.p = t ? t->data : nullptr;
  for (int d = 0; d < 6; ++d) v.s[d] = (t && d < t->ndim) ? t->stride[d] : 0;
  v.dtype = !t ? 0 : t->dtype == IPA_DTYPE_F64 ? 1 : t->dtype == IPA_DTYPE_BOOL ? 2 : 0;
  return v;
}

bool ipa_dims_ok(const ipa_params_t* p, ipa_status_t* st) {
  if (p == nullptr) { *st = IPA_ERR_NULL; return false; }
  if (p->B < 1 || p->L < 1 || p->H < 1 || p->C < 1 || p->Pq < 1 || p->Pv < 1 || p->R < 1 || p->Cz < 1) {
    *st = IPA_ERR_SHAPE;
    return false;
  }
  if (p->C != IPA_C || p->Pq != IPA_PQ || p->Pv != IPA_PV || p->Cz % 16 != 0 || p->H > 128 ||
      static_cast<int64_t>(p->R) * p->Cz > MAX_DZ || p->L > (1 << 20) ||
      static_cast<int64_t>(p->B) * p->H * p->L > (int64_t{1} << 31) / 64) {
    *st = IPA_ERR_UNSUPPORTED;
    return false;
  }
  return true;
}

int pair_width(const ipa_params_t* p) { return ((p->R * p->Cz + 63) / 64) * 64; }

bool geo_dims_ok(const geo_params_t* p, ipa_status_t* st) {
  if (p == nullptr) { *st = IPA_ERR_NULL; return false; }
  if (p->B < 1 || p->N < 1 || p->H < 1 || p->M < 1 || p->Cout < 1) { *st = IPA_ERR_SHAPE; return false; }
  if (p->M > 8 || p->H * p->M * 3 > 384 || p->N > (1 << 20) || p->H > 65535 || p->B > 65535) {
    *st = IPA_ERR_UNSUPPORTED;
    return false;
  }
  return true;
}

}  // namespace

bool encode_tmap_f16_3d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                        uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t box0, uint32_t box1,
                        int swizzle_bytes) {
  EncodeTiledFn fn = get_encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {stride1_bytes, stride2_bytes};
  const cuuint32_t box[3] = {box0, box1, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void*>(base), dims, strides, box,
                        estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// [B, L, DZ] fp16 seen as 64-column panels: dims (64 columns, L rows, DZ/64
// panels, B) with strides (DZ*2, 128, L*DZ*2) bytes.  One box of
// (64, box_rows, box_panels) lands in shared memory as box_panels consecutive
// 128-byte swizzled K-major panels of box_rows rows, the layout the MMA
// descriptors read, so a whole multi-panel tile is one copy.
bool encode_tmap_f16_panels(CUtensorMap* map, const void* base, uint64_t DZ, uint64_t L, uint64_t B,
                            uint32_t box_rows, uint32_t box_panels) {
  EncodeTiledFn fn = get_encode_fn();
  if (fn == nullptr || DZ % 64 != 0) return false;
  const cuuint64_t dims[4] = {64, L, DZ / 64, B};
  const cuuint64_t strides[3] = {DZ * 2, 128, L * DZ * 2};
  const cuuint32_t box[4] = {64, box_rows, box_panels, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// fp32 tensor of rank 3 or 4 (dims innermost first, byte strides of dims 1..)
// read or written in boxes whose inner extent is 32 elements (128 bytes) with
// the 128-byte swizzle; out-of-range elements of a load are filled with zeros
// and those of a store are dropped.
bool encode_tmap_f32_sw128(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                           const uint64_t* strides_bytes, const uint32_t* box) {
  EncodeTiledFn fn = get_encode_fn();
  if (fn == nullptr || rank < 3 || rank > 4 || box[0] != 32) return false;
  if ((reinterpret_cast<uintptr_t>(base) & 15u) != 0) return false;
  cuuint64_t d[4];
  cuuint64_t st[3];
  cuuint32_t bx[4], estr[4] = {1, 1, 1, 1};
  for (int k = 0; k < rank; ++k) {
    d[k] = dims[k];
    bx[k] = box[k];
    if (k + 1 < rank) {
      st[k] = strides_bytes[k];
      if (st[k] % 16 != 0) return false;
    }
  }
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, static_cast<cuuint32_t>(rank), const_cast<void*>(base),
                        d, st, bx, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace fipa

using namespace fipa;

extern "C" {

const char* ipa_status_string(ipa_status_t s) {
  switch (s) {
    case IPA_OK: return "ok";
    case IPA_ERR_NULL: return "null pointer";
    case IPA_ERR_SHAPE: return "shape mismatch";
    case IPA_ERR_STRIDE_ALIGN: return "bad stride or alignment";
    case IPA_ERR_DTYPE: return "bad dtype";
    case IPA_ERR_WORKSPACE: return "workspace too small or misaligned";
    case IPA_ERR_UNSUPPORTED: return "dimensions outside the supported envelope";
    case IPA_ERR_CUDA: return "CUDA runtime error";
    case IPA_ERR_TIMEOUT: return "device wait timed out";
    case IPA_ERR_BOUNDS: return "device store index outside its buffer (bounds-checked build)";
  }
  return "unknown status";
}

ipa_status_t ipa_device_error_status(int32_t v) {
  if (v == 0) return IPA_OK;
  if (v >= 1 && v <= 5) return IPA_ERR_TIMEOUT;
  if (v & 0x10000) return IPA_ERR_BOUNDS;
  return IPA_ERR_CUDA;
}

#ifdef IPA_BOUNDS_CHECK
const char* ipa_version(void) { return "flashipa_b200 sm_100a 0.1 bounds-checked"; }
#else
const char* ipa_version(void) { return "flashipa_b200 sm_100a 0.1"; }
#endif

size_t ipa_attn_workspace_size(const ipa_params_t* p) {
  ipa_status_t st;
  if (!ipa_dims_ok(p, &st)) return 0;
  return ipa_workspace_layout(p->B, p->L, p->H, pair_width(p), p->R * p->Cz, true).total;
}

}  // extern "C"

namespace {

// Validation + launch description shared by the three IPA entry points.
// inputs == false: only the params, `out` and the workspace are checked.
// with_split == false: the layout without the core's key-split reserve (the
// gradient call's recomputed prologue).
ipa_status_t ipa_prepare(const ipa_params_t* p, const ipa_tensor_t* const* in, const ipa_tensor_t* out,
                         void* workspace, size_t workspace_bytes, void* stream, int32_t* dev_err,
                         bool inputs, bool reset_err, IpaLaunch* a, bool with_split = true) {
  ipa_status_t st = IPA_OK;
  if (!ipa_dims_ok(p, &st)) return st;
  const int64_t B = p->B, L = p->L, H = p->H, C = p->C, Pq = p->Pq, Pv = p->Pv, R = p->R, Cz = p->Cz;
  const int64_t F = C + 4 * Pv + Cz;
  if (inputs) {
    const int64_t s_qkv[4] = {B, L, H, C};
    const int64_t s_qp[5] = {B, L, H, Pq, 3};
    const int64_t s_vp[5] = {B, L, H, Pv, 3};
    const int64_t s_rot[4] = {B, L, 3, 3};
    const int64_t s_tr[3] = {B, L, 3};
    const int64_t s_z[4] = {B, L, R, Cz};
    const int64_t s_w[2] = {Cz, H};
    const int64_t s_g[1] = {H};
    const int64_t s_m[2] = {B, L};
    const int64_t* shp[13] = {s_qkv, s_qkv, s_qkv, s_qp, s_qp, s_vp, s_rot, s_tr, s_z, s_z, s_w, s_g, s_m};
    const int nd[13] = {4, 4, 4, 5, 5, 5, 4, 3, 4, 4, 2, 1, 2};
    for (int t = 0; t < 13; ++t)
      if (!check_tensor(in[t], t == 12 ? IPA_DTYPE_BOOL : IPA_DTYPE_F32, nd[t], shp[t], &st)) return st;
  }
  if (out != nullptr || !inputs) {
    const int64_t s_o[4] = {B, L, H, F};
    if (!check_contiguous_out(out, 4, s_o, &st)) return st;
  }
  const int DZ = pair_width(p);
  const IpaWorkspace lay = ipa_workspace_layout(p->B, p->L, p->H, DZ, p->R * p->Cz, with_split);
  if (workspace == nullptr) return IPA_ERR_NULL;
  if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0 || workspace_bytes < lay.total) return IPA_ERR_WORKSPACE;

  *a = IpaLaunch{};
  a->B = p->B; a->L = p->L; a->H = p->H; a->C = p->C; a->Pq = p->Pq; a->Pv = p->Pv; a->R = p->R; a->Cz = p->Cz;
  a->DZ = DZ; a->RCz = p->R * p->Cz; a->F = static_cast<int>(F);
  a->nqt = (p->L + QT - 1) / QT; a->nkt = (p->L + KT - 1) / KT;
  a->w_L = p->w_L; a->w_C = p->w_C; a->scalar_scale = p->scalar_scale;
  if (inputs) {
    View* vs[13] = {&a->q, &a->k, &a->v, &a->q_pts, &a->k_pts, &a->v_pts, &a->rot, &a->trans,
                    &a->z1, &a->z2, &a->w_bias, &a->gamma, &a->mask};
    for (int t = 0; t < 13; ++t) *vs[t] = view_of(in[t]);
  }
  a->out = out ? static_cast<float*>(const_cast<void*>(out->data)) : nullptr;
  a->ws = static_cast<unsigned char*>(workspace);
  a->lay = lay;
  if (dev_err != nullptr) {
    a->err = dev_err;
  } else {
    a->err = reinterpret_cast<int*>(a->ws + lay.err);
    if (reset_err && cudaMemsetAsync(a->err, 0, sizeof(int), static_cast<cudaStream_t>(stream)) != cudaSuccess)
      return IPA_ERR_CUDA;
  }
  return IPA_OK;
}

}  // namespace

extern "C" {

ipa_status_t ipa_attn_prologue(const ipa_params_t* p, const ipa_tensor_t* q, const ipa_tensor_t* k,
                               const ipa_tensor_t* v, const ipa_tensor_t* q_pts, const ipa_tensor_t* k_pts,
                               const ipa_tensor_t* v_pts, const ipa_tensor_t* rot, const ipa_tensor_t* trans,
                               const ipa_tensor_t* z1, const ipa_tensor_t* z2, const ipa_tensor_t* w_bias,
                               const ipa_tensor_t* gamma, const ipa_tensor_t* mask, void* workspace,
                               size_t workspace_bytes, void* stream, int32_t* dev_err) {
  const ipa_tensor_t* in[13] = {q, k, v, q_pts, k_pts, v_pts, rot, trans, z1, z2, w_bias, gamma, mask};
  IpaLaunch a;
  const ipa_status_t st = ipa_prepare(p, in, nullptr, workspace, workspace_bytes, stream, dev_err, true, true, &a);
  if (st != IPA_OK) return st;
  return ipa_launch_prologue(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? IPA_OK : IPA_ERR_CUDA;
}

ipa_status_t ipa_attn_core(const ipa_params_t* p, const ipa_tensor_t* out, void* workspace,
                           size_t workspace_bytes, void* stream, int32_t* dev_err) {
  IpaLaunch a;
  const ipa_status_t st = ipa_prepare(p, nullptr, out, workspace, workspace_bytes, stream, dev_err, false, false, &a);
  if (st != IPA_OK) return st;
  return ipa_launch_core(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? IPA_OK : IPA_ERR_CUDA;
}

ipa_status_t ipa_attn_fwd(const ipa_params_t* p, const ipa_tensor_t* q, const ipa_tensor_t* k,
                          const ipa_tensor_t* v, const ipa_tensor_t* q_pts, const ipa_tensor_t* k_pts,
                          const ipa_tensor_t* v_pts, const ipa_tensor_t* rot, const ipa_tensor_t* trans,
                          const ipa_tensor_t* z1, const ipa_tensor_t* z2, const ipa_tensor_t* w_bias,
                          const ipa_tensor_t* gamma, const ipa_tensor_t* mask, const ipa_tensor_t* out,
                          void* workspace, size_t workspace_bytes, void* stream, int32_t* dev_err) {
  const ipa_tensor_t* in[13] = {q, k, v, q_pts, k_pts, v_pts, rot, trans, z1, z2, w_bias, gamma, mask};
  IpaLaunch a;
  if (out == nullptr) return IPA_ERR_NULL;
  const ipa_status_t st = ipa_prepare(p, in, out, workspace, workspace_bytes, stream, dev_err, true, true, &a);
  if (st != IPA_OK) return st;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (ipa_launch_prologue(a, s) != cudaSuccess) return IPA_ERR_CUDA;
  if (ipa_launch_core(a, s) != cudaSuccess) return IPA_ERR_CUDA;
  return IPA_OK;
}

}  // extern "C"

namespace {

// Byte sizes of the 13 inputs and the output, in the order of ipa_attn_fwd.
void ipa_host_sizes(const ipa_params_t* p, size_t sz[14]) {
  const size_t B = p->B, L = p->L, H = p->H, C = p->C, Pq = p->Pq, Pv = p->Pv, R = p->R, Cz = p->Cz;
  const size_t f = 4;
  const size_t v[14] = {B * L * H * C * f, B * L * H * C * f, B * L * H * C * f, B * L * H * Pq * 3 * f,
                        B * L * H * Pq * 3 * f, B * L * H * Pv * 3 * f, B * L * 9 * f, B * L * 3 * f,
                        B * L * R * Cz * f, B * L * R * Cz * f, Cz * H * f, H * f, B * L,
                        B * L * H * (C + 4 * Pv + Cz) * f};
  for (int t = 0; t < 14; ++t) sz[t] = v[t];
}

size_t up256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

bool dense(const ipa_tensor_t* t) {
  int64_t expect = 1;
  for (int d = t->ndim - 1; d >= 0; --d) {
    if (t->size[d] > 1 && t->stride[d] != expect) return false;
    expect *= t->size[d];
  }
  return true;
}

}  // namespace

extern "C" {

size_t ipa_attn_host_staging_size(const ipa_params_t* p) {
  ipa_status_t st;
  if (!ipa_dims_ok(p, &st)) return 0;
  size_t sz[14], total = 0;
  ipa_host_sizes(p, sz);
  for (int t = 0; t < 14; ++t) total += up256(sz[t]);
  return total;
}

}  // extern "C"

namespace {

// Host-buffer call: the inputs up into `staging` (one copy per input, or,
// when packed_bytes > 0, one copy of the packed buffer that starts at q's
// data and holds the inputs at the staging offsets), the kernels, the result
// down.
ipa_status_t host_call(const ipa_params_t* p, const ipa_tensor_t* const in13[13], const ipa_tensor_t* out,
                       void* staging, size_t staging_bytes, void* workspace, size_t workspace_bytes, void* stream,
                       int32_t* dev_err, size_t packed_bytes) {
  if (out == nullptr) return IPA_ERR_NULL;
  for (int t = 0; t < 13; ++t)
    if (in13[t] == nullptr) return IPA_ERR_NULL;
  const ipa_tensor_t* in[14];
  for (int t = 0; t < 13; ++t) in[t] = in13[t];
  in[13] = out;
  // shapes, dtypes and the workspace through the device entry point's checks
  // (host pointers are only compared, never dereferenced, there)
  IpaLaunch a;
  ipa_status_t st = ipa_prepare(p, in, out, workspace, workspace_bytes, stream, dev_err, true, true, &a);
  if (st != IPA_OK) return st;
  for (int t = 0; t < 14; ++t)
    if (!dense(in[t])) return IPA_ERR_STRIDE_ALIGN;
  if (staging == nullptr) return IPA_ERR_NULL;
  if (reinterpret_cast<uintptr_t>(staging) % 256 != 0 || staging_bytes < ipa_attn_host_staging_size(p))
    return IPA_ERR_WORKSPACE;
  size_t sz[14];
  ipa_host_sizes(p, sz);
  unsigned char* sbase = static_cast<unsigned char*>(staging);
  ipa_tensor_t dev[14];
  size_t off = 0;
  const cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (packed_bytes > 0 && cudaMemcpyAsync(sbase, in[0]->data, packed_bytes, cudaMemcpyHostToDevice, cs) != cudaSuccess)
    return IPA_ERR_CUDA;
  for (int t = 0; t < 14; ++t) {
    dev[t] = *in[t];
    dev[t].data = sbase + off;
    if (packed_bytes == 0 && t < 13 &&
        cudaMemcpyAsync(sbase + off, in[t]->data, sz[t], cudaMemcpyHostToDevice, cs) != cudaSuccess)
      return IPA_ERR_CUDA;
    off += up256(sz[t]);
  }
  const ipa_tensor_t* din[13] = {&dev[0], &dev[1], &dev[2], &dev[3], &dev[4], &dev[5], &dev[6],
                                 &dev[7], &dev[8], &dev[9], &dev[10], &dev[11], &dev[12]};
  st = ipa_prepare(p, din, &dev[13], workspace, workspace_bytes, stream, dev_err, true, false, &a);
  if (st != IPA_OK) return st;
  if (ipa_launch_prologue(a, cs) != cudaSuccess || ipa_launch_core(a, cs) != cudaSuccess) return IPA_ERR_CUDA;
  if (cudaMemcpyAsync(const_cast<void*>(out->data), dev[13].data, sz[13], cudaMemcpyDeviceToHost, cs) != cudaSuccess)
    return IPA_ERR_CUDA;
  return IPA_OK;
}

}  // namespace

extern "C" {

ipa_status_t ipa_attn_fwd_host(const ipa_params_t* p, const ipa_tensor_t* q, const ipa_tensor_t* k,
                               const ipa_tensor_t* v, const ipa_tensor_t* q_pts, const ipa_tensor_t* k_pts,
                               const ipa_tensor_t* v_pts, const ipa_tensor_t* rot, const ipa_tensor_t* trans,
                               const ipa_tensor_t* z1, const ipa_tensor_t* z2, const ipa_tensor_t* w_bias,
                               const ipa_tensor_t* gamma, const ipa_tensor_t* mask, const ipa_tensor_t* out,
                               void* staging, size_t staging_bytes, void* workspace, size_t workspace_bytes,
                               void* stream, int32_t* dev_err) {
  const ipa_tensor_t* in[13] = {q, k, v, q_pts, k_pts, v_pts, rot, trans, z1, z2, w_bias, gamma, mask};
  return host_call(p, in, out, staging, staging_bytes, workspace, workspace_bytes, stream, dev_err, 0);
}

size_t ipa_attn_host_packed_layout(const ipa_params_t* p, size_t offsets[13]) {
  ipa_status_t st;
  if (offsets == nullptr || !ipa_dims_ok(p, &st)) return 0;
  size_t sz[14], off = 0;
  ipa_host_sizes(p, sz);
  for (int t = 0; t < 13; ++t) {
    offsets[t] = off;
    off += up256(sz[t]);
  }
  return off;
}

ipa_status_t ipa_attn_fwd_host_packed(const ipa_params_t* p, const void* host_inputs, size_t host_bytes,
                                      const ipa_tensor_t* out, void* staging, size_t staging_bytes,
                                      void* workspace, size_t workspace_bytes, void* stream, int32_t* dev_err) {
  if (host_inputs == nullptr || out == nullptr) return IPA_ERR_NULL;
  size_t offs[13];
  const size_t in_bytes = ipa_attn_host_packed_layout(p, offs);
  if (in_bytes == 0) return IPA_ERR_SHAPE;
  if (host_bytes < in_bytes) return IPA_ERR_SHAPE;
  const int64_t B = p->B, L = p->L, H = p->H, C = p->C, Pq = p->Pq, Pv = p->Pv, R = p->R, Cz = p->Cz;
  // the 13 inputs, dense, in argument order (the layout ipa_attn_host_packed_layout describes)
  struct Shape {
    int nd;
    int64_t s[5];
    int32_t dt;
  };
  const Shape shp[13] = {{4, {B, L, H, C}, IPA_DTYPE_F32},      {4, {B, L, H, C}, IPA_DTYPE_F32},
                         {4, {B, L, H, C}, IPA_DTYPE_F32},      {5, {B, L, H, Pq, 3}, IPA_DTYPE_F32},
                         {5, {B, L, H, Pq, 3}, IPA_DTYPE_F32},  {5, {B, L, H, Pv, 3}, IPA_DTYPE_F32},
                         {4, {B, L, 3, 3}, IPA_DTYPE_F32},      {3, {B, L, 3}, IPA_DTYPE_F32},
                         {4, {B, L, R, Cz}, IPA_DTYPE_F32},     {4, {B, L, R, Cz}, IPA_DTYPE_F32},
                         {2, {Cz, H}, IPA_DTYPE_F32},           {1, {H}, IPA_DTYPE_F32},
                         {2, {B, L}, IPA_DTYPE_BOOL}};
  ipa_tensor_t host[13];
  const ipa_tensor_t* hin[13];
  for (int t = 0; t < 13; ++t) {
    ipa_tensor_t& d = host[t];
    d = ipa_tensor_t{};
    d.data = static_cast<const unsigned char*>(host_inputs) + offs[t];
    d.dtype = shp[t].dt;
    d.ndim = shp[t].nd;
    int64_t st = 1;
    for (int k = shp[t].nd - 1; k >= 0; --k) {
      d.size[k] = shp[t].s[k];
      d.stride[k] = st;
      st *= shp[t].s[k];
    }
    hin[t] = &host[t];
  }
  return host_call(p, hin, out, staging, staging_bytes, workspace, workspace_bytes, stream, dev_err, in_bytes);
}

ipa_status_t ipa_attn_fwd_train(const ipa_params_t* p, const ipa_tensor_t* q, const ipa_tensor_t* k,
                                const ipa_tensor_t* v, const ipa_tensor_t* q_pts, const ipa_tensor_t* k_pts,
                                const ipa_tensor_t* v_pts, const ipa_tensor_t* rot, const ipa_tensor_t* trans,
                                const ipa_tensor_t* z1, const ipa_tensor_t* z2, const ipa_tensor_t* w_bias,
                                const ipa_tensor_t* gamma, const ipa_tensor_t* mask, const ipa_tensor_t* out,
                                const ipa_tensor_t* lse, const ipa_tensor_t* u_agg, void* workspace,
                                size_t workspace_bytes, void* stream, int32_t* dev_err) {
  const ipa_tensor_t* in[13] = {q, k, v, q_pts, k_pts, v_pts, rot, trans, z1, z2, w_bias, gamma, mask};
  IpaLaunch a;
  if (out == nullptr) return IPA_ERR_NULL;
  ipa_status_t st = ipa_prepare(p, in, out, workspace, workspace_bytes, stream, dev_err, true, true, &a);
  if (st != IPA_OK) return st;
  const int64_t s_l[3] = {p->B, p->H, p->L};
  const int64_t s_u[5] = {p->B, p->L, p->H, p->R, p->Cz};
  if (!check_contiguous_out(lse, 3, s_l, &st) || !check_contiguous_out(u_agg, 5, s_u, &st)) return st;
  a.lse = static_cast<float*>(const_cast<void*>(lse->data));
  a.uagg = static_cast<float*>(const_cast<void*>(u_agg->data));
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (ipa_launch_prologue(a, s) != cudaSuccess) return IPA_ERR_CUDA;
  if (ipa_launch_core(a, s) != cudaSuccess) return IPA_ERR_CUDA;
  return IPA_OK;
}

size_t ipa_attn_bwd_workspace_size(const ipa_params_t* p) {
  ipa_status_t st;
  if (!ipa_dims_ok(p, &st)) return 0;
  return ipa_bwd_workspace_layout(p->B, p->L, p->H, pair_width(p), p->R * p->Cz).total;
}

ipa_status_t ipa_attn_bwd(const ipa_params_t* p, const ipa_tensor_t* q, const ipa_tensor_t* k,
                          const ipa_tensor_t* v, const ipa_tensor_t* q_pts, const ipa_tensor_t* k_pts,
                          const ipa_tensor_t* v_pts, const ipa_tensor_t* rot, const ipa_tensor_t* trans,
                          const ipa_tensor_t* z1, const ipa_tensor_t* z2, const ipa_tensor_t* w_bias,
                          const ipa_tensor_t* gamma, const ipa_tensor_t* mask, const ipa_tensor_t* out,
                          const ipa_tensor_t* lse, const ipa_tensor_t* u_agg, const ipa_tensor_t* g_out,
                          const ipa_grads_t* grads, void* workspace, size_t workspace_bytes, void* stream,
                          int32_t* dev_err) {
  const ipa_tensor_t* in[13] = {q, k, v, q_pts, k_pts, v_pts, rot, trans, z1, z2, w_bias, gamma, mask};
  if (grads == nullptr) return IPA_ERR_NULL;
  ipa_status_t st = IPA_OK;
  if (!ipa_dims_ok(p, &st)) return st;
  const int64_t B = p->B, L = p->L, H = p->H, C = p->C, Pq = p->Pq, Pv = p->Pv, R = p->R, Cz = p->Cz;
  const int64_t F = C + 4 * Pv + Cz;
  const int64_t s_o[4] = {B, L, H, F};
  const int64_t s_l[3] = {B, H, L};
  const int64_t s_u[5] = {B, L, H, R, Cz};
  if (!check_tensor(out, IPA_DTYPE_F32, 4, s_o, &st) || !check_tensor(lse, IPA_DTYPE_F32, 3, s_l, &st) ||
      !check_tensor(u_agg, IPA_DTYPE_F32, 5, s_u, &st) || !check_tensor(g_out, IPA_DTYPE_F32, 4, s_o, &st))
    return st;
  const int64_t s_qkv[4] = {B, L, H, C}, s_qp[5] = {B, L, H, Pq, 3}, s_vp[5] = {B, L, H, Pv, 3};
  const int64_t s_rot[4] = {B, L, 3, 3}, s_tr[3] = {B, L, 3}, s_z[4] = {B, L, R, Cz}, s_w[2] = {Cz, H};
  const int64_t s_g[1] = {H};
  if (!check_contiguous_out(&grads->q, 4, s_qkv, &st) || !check_contiguous_out(&grads->k, 4, s_qkv, &st) ||
      !check_contiguous_out(&grads->v, 4, s_qkv, &st) || !check_contiguous_out(&grads->q_pts, 5, s_qp, &st) ||
      !check_contiguous_out(&grads->k_pts, 5, s_qp, &st) || !check_contiguous_out(&grads->v_pts, 5, s_vp, &st) ||
      !check_contiguous_out(&grads->rot, 4, s_rot, &st) || !check_contiguous_out(&grads->trans, 3, s_tr, &st) ||
      !check_contiguous_out(&grads->z1, 4, s_z, &st) || !check_contiguous_out(&grads->z2, 4, s_z, &st) ||
      !check_contiguous_out(&grads->w_bias, 2, s_w, &st) || !check_contiguous_out(&grads->gamma, 1, s_g, &st))
    return st;
  const int DZ = pair_width(p);
  const IpaBwdWorkspace lay = ipa_bwd_workspace_layout(p->B, p->L, p->H, DZ, p->R * p->Cz);
  if (workspace == nullptr) return IPA_ERR_NULL;
  if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0 || workspace_bytes < lay.total) return IPA_ERR_WORKSPACE;
  IpaBwdLaunch b{};
  // inputs and the forward part of the workspace (prologue outputs) through the forward's checks
  st = ipa_prepare(p, in, nullptr, workspace, lay.fwd.total, stream, dev_err, true, true, &b.f, false);
  if (st != IPA_OK) return st;
  b.out = view_of(out);
  b.lse = view_of(lse);
  b.uagg = view_of(u_agg);
  b.g_out = view_of(g_out);
  auto outp = [](const ipa_tensor_t& t) { return static_cast<float*>(const_cast<void*>(t.data)); };
  b.d_q = outp(grads->q); b.d_k = outp(grads->k); b.d_v = outp(grads->v);
  b.d_q_pts = outp(grads->q_pts); b.d_k_pts = outp(grads->k_pts); b.d_v_pts = outp(grads->v_pts);
  b.d_rot = outp(grads->rot); b.d_trans = outp(grads->trans); b.d_z1 = outp(grads->z1); b.d_z2 = outp(grads->z2);
  b.d_w_bias = outp(grads->w_bias); b.d_gamma = outp(grads->gamma);
  b.lay = lay;
  if (ipa_launch_bwd(b, static_cast<cudaStream_t>(stream)) != cudaSuccess) return IPA_ERR_CUDA;
  return IPA_OK;
}

ipa_status_t ipa_knn_distogram(int32_t B, int32_t L, int32_t k, int32_t n_edges, const ipa_tensor_t* x,
                               const ipa_tensor_t* mask, const float* edges, const ipa_tensor_t* idx,
                               const ipa_tensor_t* bins, const ipa_tensor_t* hist, void* stream) {
  if (B < 1 || L < 1 || k < 1 || n_edges < 0) return IPA_ERR_SHAPE;
  if (k > DIST_MAX_K || n_edges > DIST_MAX_EDGES || L > (1 << 24) || static_cast<int64_t>(B) * L > (int64_t{1} << 31))
    return IPA_ERR_UNSUPPORTED;
  if (n_edges > 0 && edges == nullptr) return IPA_ERR_NULL;
  for (int m = 0; m < n_edges; ++m)
    if (!(edges[m] >= 0.f) || (m > 0 && !(edges[m] > edges[m - 1]))) return IPA_ERR_SHAPE;
  ipa_status_t st = IPA_OK;
  const int64_t s_x[3] = {B, L, 3}, s_m[2] = {B, L}, s_k[3] = {B, L, k}, s_h[3] = {B, L, n_edges + 1};
  if (!check_tensor(x, IPA_DTYPE_F32, 3, s_x, &st) || !check_tensor(mask, IPA_DTYPE_BOOL, 2, s_m, &st)) return st;
  auto check_i32_out = [&](const ipa_tensor_t* t) {
    if (t == nullptr || t->data == nullptr) { st = IPA_ERR_NULL; return false; }
    if (t->dtype != IPA_DTYPE_I32) { st = IPA_ERR_DTYPE; return false; }
    ipa_tensor_t f = *t;
    f.dtype = IPA_DTYPE_F32;                 // same size and alignment rules as an fp32 output
    return check_contiguous_out(&f, 3, s_k, &st);
  };
  if (!check_i32_out(idx) || !check_i32_out(bins) || !check_contiguous_out(hist, 3, s_h, &st)) return st;
  DistogramArgs a{};
  a.B = B; a.L = L; a.k = k; a.nb = n_edges + 1;
  a.x = view_of(x);
  a.mask = view_of(mask);
  for (int m = 0; m < n_edges; ++m) a.edge2[m] = edges[m] * edges[m];
  a.idx = static_cast<int32_t*>(const_cast<void*>(idx->data));
  a.bins = static_cast<int32_t*>(const_cast<void*>(bins->data));
  a.hist = static_cast<float*>(const_cast<void*>(hist->data));
  return distogram_launch(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? IPA_OK : IPA_ERR_CUDA;
}

size_t meet_attn_workspace_size(const meet_params_t* p) {
  if (p == nullptr || p->B < 1 || p->L < 1 || p->H < 1 || p->C != MEET_C || p->H > 128 || p->L > (1 << 20) ||
      static_cast<int64_t>(p->B) * p->H * p->L > (int64_t{1} << 31) / 64)
    return 0;
  return meet_workspace_layout(p->B, p->L, p->H).total;
}

ipa_status_t meet_attn_fwd(const meet_params_t* p, const ipa_tensor_t* q, const ipa_tensor_t* k,
                           const ipa_tensor_t* v, const ipa_tensor_t* x, const ipa_tensor_t* rho,
                           const ipa_tensor_t* s, const ipa_tensor_t* mask, const ipa_tensor_t* out,
                           void* workspace, size_t workspace_bytes, void* stream, int32_t* dev_err) {
  if (p == nullptr) return IPA_ERR_NULL;
  if (p->B < 1 || p->L < 1 || p->H < 1 || p->C < 1) return IPA_ERR_SHAPE;
  if (p->C != MEET_C || p->H > 128 || p->L > (1 << 20) ||
      static_cast<int64_t>(p->B) * p->H * p->L > (int64_t{1} << 31) / 64)
    return IPA_ERR_UNSUPPORTED;
  const int64_t B = p->B, L = p->L, H = p->H, C = p->C;
  ipa_status_t st = IPA_OK;
  const int64_t s_qkv[4] = {B, L, H, C}, s_x[3] = {B, L, 3}, s_h[1] = {H}, s_m[2] = {B, L};
  if (!check_tensor(q, IPA_DTYPE_F32, 4, s_qkv, &st) || !check_tensor(k, IPA_DTYPE_F32, 4, s_qkv, &st) ||
      !check_tensor(v, IPA_DTYPE_F32, 4, s_qkv, &st) || !check_tensor(x, IPA_DTYPE_F32, 3, s_x, &st) ||
      !check_tensor(rho, IPA_DTYPE_F32, 1, s_h, &st) || !check_tensor(s, IPA_DTYPE_F32, 1, s_h, &st) ||
      !check_tensor(mask, IPA_DTYPE_BOOL, 2, s_m, &st) || !check_contiguous_out(out, 4, s_qkv, &st))
    return st;
  const MeetWorkspace lay = meet_workspace_layout(p->B, p->L, p->H);
  if (workspace == nullptr) return IPA_ERR_NULL;
  if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0 || workspace_bytes < lay.total) return IPA_ERR_WORKSPACE;
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  const cudaStream_t cs = static_cast<cudaStream_t>(stream);

  MeetPrep m{};
  m.B = p->B; m.L = p->L; m.H = p->H;
  m.q = view_of(q); m.rho = view_of(rho); m.s = view_of(s);
  m.qs = reinterpret_cast<float*>(ws + lay.qs);
  m.gamma = reinterpret_cast<float*>(ws + lay.gamma);
  m.consts = reinterpret_cast<float*>(ws + lay.consts);

  // the IPA problem: C = 16, Pq = 4, Pv = 8, no pair block (R = 0 factors of
  // width 16); w_L = 1, w_C = 1/2, scalar scale 1
  IpaLaunch a{};
  a.B = p->B; a.L = p->L; a.H = p->H; a.C = MEET_C; a.Pq = IPA_PQ; a.Pv = IPA_PV; a.R = 0; a.Cz = 16;
  a.DZ = MEET_DZ; a.RCz = MEET_RCZ; a.F = MEET_F;
  a.nqt = (p->L + QT - 1) / QT; a.nkt = (p->L + KT - 1) / KT;
  a.w_L = 1.f; a.w_C = 0.5f; a.scalar_scale = 1.f;
  auto dense = [](const void* ptr, std::initializer_list<int64_t> strides) {
    View vv{};
    vv.p = ptr;
    int d = 0;
    for (int64_t st2 : strides) vv.s[d++] = st2;
    return vv;
  };
  const float* zeros = m.consts;
  const float* ident = m.consts + MEET_ZEROS;
  a.q = dense(m.qs, {L * H * C, H * C, C, 1});
  a.k = view_of(k);
  a.v = view_of(v);
  a.q_pts = dense(zeros, {0, 0, 0, 0, 0});
  a.k_pts = dense(zeros, {0, 0, 0, 0, 0});
  a.v_pts = dense(zeros, {0, 0, 0, 0, 0});
  a.rot = dense(ident, {0, 0, 3, 1});
  a.trans = view_of(x);
  a.z1 = dense(zeros, {0, 0, 0, 0});
  a.z2 = dense(zeros, {0, 0, 0, 0});
  a.w_bias = dense(zeros, {0, 0});
  a.gamma = dense(m.gamma, {1});
  a.mask = view_of(mask);
  a.mask.dtype = 2;
  a.ws = ws + lay.ipa;
  a.lay = ipa_workspace_layout(p->B, p->L, p->H, MEET_DZ, MEET_RCZ);
  a.out = reinterpret_cast<float*>(ws + lay.out);
  if (dev_err != nullptr) {
    a.err = dev_err;
  } else {
    a.err = reinterpret_cast<int*>(a.ws + a.lay.err);
    if (cudaMemsetAsync(a.err, 0, sizeof(int), cs) != cudaSuccess) return IPA_ERR_CUDA;
  }
  m.err = a.err;
  if (meet_launch_prep(m, cs) != cudaSuccess) return IPA_ERR_CUDA;
  if (ipa_launch_prologue(a, cs) != cudaSuccess) return IPA_ERR_CUDA;
  if (ipa_launch_core(a, cs) != cudaSuccess) return IPA_ERR_CUDA;
  if (meet_launch_extract(a.out, static_cast<float*>(const_cast<void*>(out->data)), B * L * H, a.err, cs) != cudaSuccess)
    return IPA_ERR_CUDA;
  return IPA_OK;
}

ipa_status_t ipa_frames_from_backbone(int32_t B, int32_t L, const ipa_tensor_t* n, const ipa_tensor_t* ca,
                                      const ipa_tensor_t* c, const ipa_tensor_t* rot_out,
                                      const ipa_tensor_t* trans_out, void* stream) {
  if (B < 1 || L < 1) return IPA_ERR_SHAPE;
  if (static_cast<int64_t>(B) * L > (int64_t{1} << 31) / 16) return IPA_ERR_UNSUPPORTED;
  ipa_status_t st = IPA_OK;
  const int64_t s_a[3] = {B, L, 3}, s_r[4] = {B, L, 3, 3};
  if (!check_tensor(n, IPA_DTYPE_F32, 3, s_a, &st) || !check_tensor(ca, IPA_DTYPE_F32, 3, s_a, &st) ||
      !check_tensor(c, IPA_DTYPE_F32, 3, s_a, &st) || !check_tensor(rot_out, IPA_DTYPE_F32, 4, s_r, &st) ||
      !check_tensor(trans_out, IPA_DTYPE_F32, 3, s_a, &st))
    return st;
  for (const ipa_tensor_t* o : {rot_out, trans_out}) {    // outputs dense row-major
    int64_t expect = 1;
    for (int d = o->ndim - 1; d >= 0; --d) {
      if (o->size[d] > 1 && o->stride[d] != expect) return IPA_ERR_STRIDE_ALIGN;
      expect *= o->size[d];
    }
  }
  FramesArgs a{};
  a.B = B; a.L = L;
  a.n = view_of(n); a.ca = view_of(ca); a.c = view_of(c);
  a.rot = static_cast<float*>(const_cast<void*>(rot_out->data));
  a.trans = static_cast<float*>(const_cast<void*>(trans_out->data));
  if (frames_launch(a, static_cast<cudaStream_t>(stream)) != cudaSuccess) return IPA_ERR_CUDA;
  return IPA_OK;
}

size_t geo_attn_workspace_size(const geo_params_t* p) {
  ipa_status_t st;
  if (!geo_dims_ok(p, &st)) return 0;
  return geo_workspace_layout(p->B, p->N, p->H, p->M, p->Cout).total;
}

namespace {

// Checks the variant's inputs (shared by the forward and the gradient) and
// fills the input part of a launch.
ipa_status_t geo_inputs(const geo_params_t* p, const ipa_tensor_t* q_direction,
                        const ipa_tensor_t* k_direction, const ipa_tensor_t* q_point,
                        const ipa_tensor_t* k_point, const ipa_tensor_t* values,
                        const ipa_tensor_t* direction_scale, const ipa_tensor_t* distance_scale,
                        const ipa_tensor_t* output_weight, const ipa_tensor_t* output_bias,
                        const ipa_tensor_t* rotation, const ipa_tensor_t* translation,
                        const ipa_tensor_t* frame_mask, const ipa_tensor_t* pair_mask, fipa::GeoLaunch* a,
                        int* fdt_out) {
  ipa_status_t st = IPA_OK;
  if (!geo_dims_ok(p, &st)) return st;
  const int64_t B = p->B, N = p->N, H = p->H, M = p->M, Cout = p->Cout;
  const int fdt = q_direction ? q_direction->dtype : IPA_DTYPE_F32;
  if (fdt != IPA_DTYPE_F32 && fdt != IPA_DTYPE_F64) return q_direction ? IPA_ERR_DTYPE : IPA_ERR_NULL;
  const bool has_bias = output_bias != nullptr && output_bias->data != nullptr;
  const bool has_pm = pair_mask != nullptr && pair_mask->data != nullptr;
  const int64_t s_v3[4] = {B, N, H, 3};
  const int64_t s_val[5] = {B, N, H, M, 3};
  const int64_t s_h[1] = {H};
  const int64_t s_w[2] = {H * M * 3, Cout};
  const int64_t s_b[1] = {Cout};
  const int64_t s_rot[4] = {B, N, 3, 3};
  const int64_t s_tr[3] = {B, N, 3};
  const int64_t s_fm[2] = {B, N};
  const int64_t s_pm[4] = {B, H, N, N};
  if (!check_tensor(q_direction, fdt, 4, s_v3, &st) || !check_tensor(k_direction, fdt, 4, s_v3, &st) ||
      !check_tensor(q_point, fdt, 4, s_v3, &st) || !check_tensor(k_point, fdt, 4, s_v3, &st) ||
      !check_tensor(values, fdt, 5, s_val, &st) || !check_tensor(direction_scale, fdt, 1, s_h, &st) ||
      !check_tensor(distance_scale, fdt, 1, s_h, &st) || !check_tensor(output_weight, fdt, 2, s_w, &st) ||
      (has_bias && !check_tensor(output_bias, fdt, 1, s_b, &st)) ||
      !check_tensor(rotation, fdt, 4, s_rot, &st) || !check_tensor(translation, fdt, 3, s_tr, &st) ||
      !check_tensor(frame_mask, IPA_DTYPE_BOOL, 2, s_fm, &st))
    return st;
  if (has_pm) {
    // broadcastable to [B, H, N, N]: each size equals the full size or is 1 (stride ignored then)
    if (pair_mask->dtype != IPA_DTYPE_BOOL) return IPA_ERR_DTYPE;
    if (pair_mask->ndim != 4) return IPA_ERR_SHAPE;
    for (int d = 0; d < 4; ++d) {
      if (pair_mask->size[d] != s_pm[d] && pair_mask->size[d] != 1) return IPA_ERR_SHAPE;
      if (pair_mask->stride[d] < 0) return IPA_ERR_STRIDE_ALIGN;
    }
  }
  fipa::GeoLaunch& g = *a;
  g = fipa::GeoLaunch{};
  g.B = p->B; g.N = p->N; g.H = p->H; g.M = p->M; g.Cout = p->Cout; g.HM3 = p->H * p->M * 3;
  g.q_direction = view_of(q_direction); g.k_direction = view_of(k_direction);
  g.q_point = view_of(q_point); g.k_point = view_of(k_point); g.values = view_of(values);
  g.direction_scale = view_of(direction_scale); g.distance_scale = view_of(distance_scale);
  g.output_weight = view_of(output_weight); g.output_bias = view_of(has_bias ? output_bias : nullptr);
  g.output_bias.dtype = has_bias ? g.output_bias.dtype : g.output_weight.dtype;
  g.rotation = view_of(rotation); g.translation = view_of(translation); g.frame_mask = view_of(frame_mask);
  g.pair_mask = view_of(has_pm ? pair_mask : nullptr);
  if (has_pm)
    for (int d = 0; d < 4; ++d)
      if (pair_mask->size[d] == 1) g.pair_mask.s[d] = 0;  // broadcast dimension
  g.has_bias = has_bias; g.has_pair_mask = has_pm;
  *fdt_out = fdt;
  return IPA_OK;
}

}  // namespace

ipa_status_t geo_attn_fwd(const geo_params_t* p, const ipa_tensor_t* q_direction,
                          const ipa_tensor_t* k_direction, const ipa_tensor_t* q_point,
                          const ipa_tensor_t* k_point, const ipa_tensor_t* values,
                          const ipa_tensor_t* direction_scale, const ipa_tensor_t* distance_scale,
                          const ipa_tensor_t* output_weight, const ipa_tensor_t* output_bias,
                          const ipa_tensor_t* rotation, const ipa_tensor_t* translation,
                          const ipa_tensor_t* frame_mask, const ipa_tensor_t* pair_mask,
                          const ipa_tensor_t* out_vectors, const ipa_tensor_t* out_output,
                          const ipa_tensor_t* out_attention, void* workspace, size_t workspace_bytes,
                          void* stream, int32_t* dev_err) {
  GeoLaunch a{};
  int fdt = 0;
  ipa_status_t st = geo_inputs(p, q_direction, k_direction, q_point, k_point, values, direction_scale,
                               distance_scale, output_weight, output_bias, rotation, translation, frame_mask,
                               pair_mask, &a, &fdt);
  if (st != IPA_OK) return st;
  const int64_t B = p->B, N = p->N, H = p->H, M = p->M, Cout = p->Cout;
  const bool has_att = out_attention != nullptr && out_attention->data != nullptr;
  const int64_t s_val[5] = {B, N, H, M, 3};
  const int64_t s_o3[3] = {B, N, Cout};
  const int64_t s_att[4] = {B, H, N, N};
  if (!check_contiguous_out(out_vectors, 5, s_val, &st) || !check_contiguous_out(out_output, 3, s_o3, &st) ||
      (has_att && !check_contiguous_out(out_attention, 4, s_att, &st)))
    return st;
  const GeoWorkspace lay = geo_workspace_layout(p->B, p->N, p->H, p->M, p->Cout);
  if (workspace == nullptr) return IPA_ERR_NULL;
  if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0 || workspace_bytes < lay.total) return IPA_ERR_WORKSPACE;
  a.out_vectors = static_cast<float*>(const_cast<void*>(out_vectors->data));
  a.out_output = static_cast<float*>(const_cast<void*>(out_output->data));
  a.out_attention = has_att ? static_cast<float*>(const_cast<void*>(out_attention->data)) : nullptr;
  a.ws = static_cast<unsigned char*>(workspace);
  a.lay = lay;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dev_err != nullptr) {
    a.err = dev_err;
  } else {
    a.err = reinterpret_cast<int*>(a.ws + lay.err);
    if (cudaMemsetAsync(a.err, 0, sizeof(int), s) != cudaSuccess) return IPA_ERR_CUDA;
  }
  if (geo_launch_all(a, s) != cudaSuccess) return IPA_ERR_CUDA;
  return IPA_OK;
}

size_t ipa_linear_workspace_size(int32_t M, int32_t K, int32_t N) {
  if (M < 1 || K < 1 || N < 1 || K > 65536 || M > (1 << 23)) return 0;
  return linear_workspace_layout(M, K, N).total;
}

ipa_status_t ipa_linear_fwd(int32_t M, int32_t K, int32_t N, const ipa_tensor_t* x, const ipa_tensor_t* w,
                            const ipa_tensor_t* b, const ipa_tensor_t* y, void* workspace,
                            size_t workspace_bytes, void* stream, int32_t* dev_err) {
  if (M < 1 || K < 1 || N < 1) return IPA_ERR_SHAPE;
  if (K > 65536 || M > (1 << 23)) return IPA_ERR_UNSUPPORTED;
  ipa_status_t st = IPA_OK;
  const int64_t s_x[2] = {M, K}, s_w[2] = {K, N}, s_b[1] = {N}, s_y[2] = {M, N};
  const bool has_b = b != nullptr && b->data != nullptr;
  if (!check_tensor(x, IPA_DTYPE_F32, 2, s_x, &st) || !check_tensor(w, IPA_DTYPE_F32, 2, s_w, &st) ||
      (has_b && !check_contiguous_out(b, 1, s_b, &st)) || !check_contiguous_out(y, 2, s_y, &st))
    return st;
  const LinearWorkspace lay = linear_workspace_layout(M, K, N);
  if (workspace == nullptr) return IPA_ERR_NULL;
  if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0 || workspace_bytes < lay.total) return IPA_ERR_WORKSPACE;
  LinearLaunch a{};
  a.M = M; a.K = K; a.N = N;
  a.x = view_of(x); a.w = view_of(w);
  a.bias = has_b ? static_cast<const float*>(b->data) : nullptr;
  a.y = static_cast<float*>(const_cast<void*>(y->data));
  a.ldy = N;
  a.ws = static_cast<unsigned char*>(workspace);
  a.lay = lay;
  a.err = dev_err;
  if (linear_launch(a, static_cast<cudaStream_t>(stream)) != cudaSuccess) return IPA_ERR_CUDA;
  return IPA_OK;
}

namespace {

struct ModuleLayout {
  int64_t M, width, HF;
  size_t y, o, lin, core, total;
};

bool module_layout(const ipa_module_params_t* p, ModuleLayout* m) {
  if (p == nullptr || p->c_s < 1) return false;
  const ipa_params_t& c = p->core;
  const size_t core_ws = ipa_attn_workspace_size(&c);
  if (core_ws == 0) return false;
  auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  m->M = static_cast<int64_t>(c.B) * c.L;
  m->width = static_cast<int64_t>(c.H) * (3 * c.C + 3 * (2 * c.Pq + c.Pv));
  m->HF = static_cast<int64_t>(c.H) * (c.C + 4 * c.Pv + c.Cz);
  if (m->M > (1 << 23) || p->c_s > 65536 || m->width > (1 << 20) || m->HF > 65536) return false;
  const size_t lin_in = ipa_linear_workspace_size(static_cast<int32_t>(m->M), p->c_s, static_cast<int32_t>(m->width));
  const size_t lin_out = ipa_linear_workspace_size(static_cast<int32_t>(m->M), static_cast<int32_t>(m->HF), p->c_s);
  if (lin_in == 0 || lin_out == 0) return false;
  size_t o = 0;
  m->y = o; o = up(o + static_cast<size_t>(m->M) * m->width * 4);
  m->o = o; o = up(o + static_cast<size_t>(m->M) * m->HF * 4);
  m->lin = o; o = up(o + (lin_in > lin_out ? lin_in : lin_out));
  m->core = o; o = up(o + core_ws);
  m->total = o;
  return true;
}

ipa_tensor_t dense_desc(const void* data, int ndim, const int64_t* size, const int64_t* stride) {
  ipa_tensor_t t{};
  t.data = data;
  t.dtype = IPA_DTYPE_F32;
  t.ndim = ndim;
  for (int d = 0; d < ndim; ++d) {
    t.size[d] = size[d];
    t.stride[d] = stride[d];
  }
  return t;
}

}  // namespace

size_t ipa_module_workspace_size(const ipa_module_params_t* p) {
  ModuleLayout m{};
  return module_layout(p, &m) ? m.total : 0;
}

ipa_status_t ipa_module_fwd(const ipa_module_params_t* p, const ipa_tensor_t* s, const ipa_tensor_t* rot,
                            const ipa_tensor_t* trans, const ipa_tensor_t* z1, const ipa_tensor_t* z2,
                            const ipa_tensor_t* w_bias, const ipa_tensor_t* gamma, const ipa_tensor_t* mask,
                            const ipa_tensor_t* w_in, const ipa_tensor_t* b_in, const ipa_tensor_t* w_out,
                            const ipa_tensor_t* b_out, const ipa_tensor_t* out, const ipa_tensor_t* core_out,
                            void* workspace, size_t workspace_bytes, void* stream, int32_t* dev_err) {
  if (p == nullptr) return IPA_ERR_NULL;
  ipa_status_t st = IPA_OK;
  if (!ipa_dims_ok(&p->core, &st)) return st;
  if (p->c_s < 1) return IPA_ERR_SHAPE;
  ModuleLayout m{};
  if (!module_layout(p, &m)) return IPA_ERR_UNSUPPORTED;
  const ipa_params_t& c = p->core;
  const int64_t B = c.B, L = c.L, H = c.H, cs = p->c_s;
  const int64_t F = c.C + 4 * c.Pv + c.Cz;
  const int64_t s_s[3] = {B, L, cs}, s_wi[2] = {cs, m.width}, s_bi[1] = {m.width}, s_wo[2] = {m.HF, cs},
                s_bo[1] = {cs}, s_o[4] = {B, L, H, F};
  const bool has_bi = b_in != nullptr && b_in->data != nullptr;
  const bool has_bo = b_out != nullptr && b_out->data != nullptr;
  const bool has_co = core_out != nullptr && core_out->data != nullptr;
  if (!check_tensor(s, IPA_DTYPE_F32, 3, s_s, &st) || !check_tensor(w_in, IPA_DTYPE_F32, 2, s_wi, &st) ||
      (has_bi && !check_contiguous_out(b_in, 1, s_bi, &st)) || !check_tensor(w_out, IPA_DTYPE_F32, 2, s_wo, &st) ||
      (has_bo && !check_contiguous_out(b_out, 1, s_bo, &st)) || !check_contiguous_out(out, 3, s_s, &st) ||
      (has_co && !check_contiguous_out(core_out, 4, s_o, &st)))
    return st;
  if (B > 1 && s->stride[0] != L * s->stride[1]) return IPA_ERR_STRIDE_ALIGN;   // rows must flatten
  {
    // the core's own arguments, checked here too so that nothing is launched on a bad call
    const int64_t s_rot[4] = {B, L, 3, 3}, s_tr[3] = {B, L, 3}, s_z[4] = {B, L, c.R, c.Cz},
                  s_wb[2] = {c.Cz, H}, s_g[1] = {H}, s_m[2] = {B, L};
    if (!check_tensor(rot, IPA_DTYPE_F32, 4, s_rot, &st) || !check_tensor(trans, IPA_DTYPE_F32, 3, s_tr, &st) ||
        !check_tensor(z1, IPA_DTYPE_F32, 4, s_z, &st) || !check_tensor(z2, IPA_DTYPE_F32, 4, s_z, &st) ||
        !check_tensor(w_bias, IPA_DTYPE_F32, 2, s_wb, &st) || !check_tensor(gamma, IPA_DTYPE_F32, 1, s_g, &st) ||
        !check_tensor(mask, IPA_DTYPE_BOOL, 2, s_m, &st))
      return st;
  }
  if (workspace == nullptr) return IPA_ERR_NULL;
  if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0 || workspace_bytes < m.total) return IPA_ERR_WORKSPACE;
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  cudaStream_t strm = static_cast<cudaStream_t>(stream);
  float* Y = reinterpret_cast<float*>(ws + m.y);
  float* O = has_co ? static_cast<float*>(const_cast<void*>(core_out->data)) : reinterpret_cast<float*>(ws + m.o);

  // 1. Y = s W_in + b_in
  LinearLaunch l1{};
  l1.M = static_cast<int>(m.M); l1.K = p->c_s; l1.N = static_cast<int>(m.width);
  l1.x = view_of(s);
  l1.x.s[0] = s->stride[1];      // [B*L, c_s] rows
  l1.x.s[1] = s->stride[2];
  l1.w = view_of(w_in);
  l1.bias = has_bi ? static_cast<const float*>(b_in->data) : nullptr;
  l1.y = Y; l1.ldy = m.width;
  l1.ws = ws + m.lin; l1.lay = linear_workspace_layout(l1.M, l1.K, l1.N); l1.err = dev_err;
  if (linear_launch(l1, strm) != cudaSuccess) return IPA_ERR_CUDA;

  // 2. the core on strided views of Y
  const int64_t rs = m.width;
  const int64_t HC = H * c.C, HQ = H * c.Pq * 3;
  const int64_t sz_s[4] = {B, L, H, c.C}, st_s[4] = {L * rs, rs, c.C, 1};
  const int64_t sz_q[5] = {B, L, H, c.Pq, 3}, st_q[5] = {L * rs, rs, c.Pq * 3, 3, 1};
  const int64_t sz_v[5] = {B, L, H, c.Pv, 3}, st_v[5] = {L * rs, rs, c.Pv * 3, 3, 1};
  const ipa_tensor_t tq = dense_desc(Y, 4, sz_s, st_s), tk = dense_desc(Y + HC, 4, sz_s, st_s),
                     tv = dense_desc(Y + 2 * HC, 4, sz_s, st_s), tqp = dense_desc(Y + 3 * HC, 5, sz_q, st_q),
                     tkp = dense_desc(Y + 3 * HC + HQ, 5, sz_q, st_q),
                     tvp = dense_desc(Y + 3 * HC + 2 * HQ, 5, sz_v, st_v);
  const int64_t st_o[4] = {L * H * F, H * F, F, 1};
  const ipa_tensor_t to = dense_desc(O, 4, s_o, st_o);
  st = ipa_attn_fwd(&c, &tq, &tk, &tv, &tqp, &tkp, &tvp, rot, trans, z1, z2, w_bias, gamma, mask, &to,
                    ws + m.core, workspace_bytes - m.core, stream, dev_err);
  if (st != IPA_OK) return st;

  // 3. out = flatten(o) W_out + b_out
  LinearLaunch l2{};
  l2.M = static_cast<int>(m.M); l2.K = static_cast<int>(m.HF); l2.N = p->c_s;
  const int64_t sz_o2[2] = {m.M, m.HF}, st_o2[2] = {m.HF, 1};
  const ipa_tensor_t to2 = dense_desc(O, 2, sz_o2, st_o2);
  l2.x = view_of(&to2);
  l2.w = view_of(w_out);
  l2.bias = has_bo ? static_cast<const float*>(b_out->data) : nullptr;
  l2.y = static_cast<float*>(const_cast<void*>(out->data)); l2.ldy = cs;
  l2.ws = ws + m.lin; l2.lay = linear_workspace_layout(l2.M, l2.K, l2.N); l2.err = dev_err;
  if (linear_launch(l2, strm) != cudaSuccess) return IPA_ERR_CUDA;
  return IPA_OK;
}

size_t geo_attn_bwd_workspace_size(const geo_params_t* p) {
  ipa_status_t st = IPA_OK;
  if (!geo_dims_ok(p, &st)) return 0;
  return geo_bwd_workspace_layout(p->B, p->N, p->H, p->M, p->Cout).total;
}

ipa_status_t geo_attn_bwd(const geo_params_t* p, const ipa_tensor_t* q_direction,
                          const ipa_tensor_t* k_direction, const ipa_tensor_t* q_point,
                          const ipa_tensor_t* k_point, const ipa_tensor_t* values,
                          const ipa_tensor_t* direction_scale, const ipa_tensor_t* distance_scale,
                          const ipa_tensor_t* output_weight, const ipa_tensor_t* output_bias,
                          const ipa_tensor_t* rotation, const ipa_tensor_t* translation,
                          const ipa_tensor_t* frame_mask, const ipa_tensor_t* pair_mask,
                          const ipa_tensor_t* g_output, const ipa_tensor_t* g_attention,
                          const ipa_tensor_t* g_vectors, const geo_grads_t* grads, void* workspace,
                          size_t workspace_bytes, void* stream, int32_t* dev_err) {
  GeoBwdLaunch a{};
  int fdt = 0;
  ipa_status_t st = geo_inputs(p, q_direction, k_direction, q_point, k_point, values, direction_scale,
                               distance_scale, output_weight, output_bias, rotation, translation, frame_mask,
                               pair_mask, &a.f, &fdt);
  if (st != IPA_OK) return st;
  if (grads == nullptr) return IPA_ERR_NULL;
  const int64_t B = p->B, N = p->N, H = p->H, M = p->M, Cout = p->Cout;
  const int64_t s_v3[4] = {B, N, H, 3};
  const int64_t s_val[5] = {B, N, H, M, 3};
  const int64_t s_h[1] = {H};
  const int64_t s_w[2] = {H * M * 3, Cout};
  const int64_t s_b[1] = {Cout};
  const int64_t s_rot[4] = {B, N, 3, 3};
  const int64_t s_tr[3] = {B, N, 3};
  const int64_t s_o3[3] = {B, N, Cout};
  const int64_t s_att[4] = {B, H, N, N};
  const bool has_ga = g_attention != nullptr && g_attention->data != nullptr;
  const bool has_gv = g_vectors != nullptr && g_vectors->data != nullptr;
  if (!check_tensor(g_output, fdt, 3, s_o3, &st) || (has_ga && !check_tensor(g_attention, fdt, 4, s_att, &st)) ||
      (has_gv && !check_tensor(g_vectors, fdt, 5, s_val, &st)))
    return st;
  const bool want_bias = a.f.has_bias;
  if (want_bias != (grads->output_bias.data != nullptr)) return grads->output_bias.data ? IPA_ERR_SHAPE : IPA_ERR_NULL;
  if (!check_contiguous_out(&grads->q_direction, 4, s_v3, &st) ||
      !check_contiguous_out(&grads->k_direction, 4, s_v3, &st) ||
      !check_contiguous_out(&grads->q_point, 4, s_v3, &st) || !check_contiguous_out(&grads->k_point, 4, s_v3, &st) ||
      !check_contiguous_out(&grads->values, 5, s_val, &st) ||
      !check_contiguous_out(&grads->direction_scale, 1, s_h, &st) ||
      !check_contiguous_out(&grads->distance_scale, 1, s_h, &st) ||
      !check_contiguous_out(&grads->output_weight, 2, s_w, &st) ||
      (want_bias && !check_contiguous_out(&grads->output_bias, 1, s_b, &st)) ||
      !check_contiguous_out(&grads->rotation, 4, s_rot, &st) ||
      !check_contiguous_out(&grads->translation, 3, s_tr, &st))
    return st;
  const GeoBwdWorkspace lay = geo_bwd_workspace_layout(p->B, p->N, p->H, p->M, p->Cout);
  if (workspace == nullptr) return IPA_ERR_NULL;
  if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0 || workspace_bytes < lay.total) return IPA_ERR_WORKSPACE;
  auto outp = [](const ipa_tensor_t& t) { return static_cast<float*>(const_cast<void*>(t.data)); };
  a.g_output = view_of(g_output);
  a.g_attention = view_of(has_ga ? g_attention : nullptr);
  a.g_vectors = view_of(has_gv ? g_vectors : nullptr);
  a.g_attention.dtype = a.g_vectors.dtype = a.g_output.dtype;
  a.has_g_attention = has_ga;
  a.has_g_vectors = has_gv;
  a.d_q_direction = outp(grads->q_direction); a.d_k_direction = outp(grads->k_direction);
  a.d_q_point = outp(grads->q_point); a.d_k_point = outp(grads->k_point); a.d_values = outp(grads->values);
  a.d_direction_scale = outp(grads->direction_scale); a.d_distance_scale = outp(grads->distance_scale);
  a.d_output_weight = outp(grads->output_weight);
  a.d_output_bias = want_bias ? outp(grads->output_bias) : nullptr;
  a.d_rotation = outp(grads->rotation); a.d_translation = outp(grads->translation);
  a.ws = static_cast<unsigned char*>(workspace);
  a.lay = lay;
  a.f.ws = a.ws;
  a.f.lay = lay.fwd;
  if (dev_err != nullptr) {
    a.f.err = dev_err;
  } else {
    a.f.err = reinterpret_cast<int*>(a.ws + lay.fwd.err);
    if (cudaMemsetAsync(a.f.err, 0, sizeof(int), static_cast<cudaStream_t>(stream)) != cudaSuccess) return IPA_ERR_CUDA;
  }
  if (geo_launch_bwd(a, static_cast<cudaStream_t>(stream)) != cudaSuccess) return IPA_ERR_CUDA;
  return IPA_OK;
}

}  // extern "C"

#ifdef IPA_TRACE
// Tracing build only: copy the per-tile event timestamps to the host.
extern "C" __attribute__((visibility("default"))) int ipa_trace_copy(void* host, size_t bytes) {
  return fipa::ipa_trace_read(host, bytes) ? 0 : 1;
}
extern "C" __attribute__((visibility("default"))) int ipa_pair_trace_copy(void* host, size_t bytes) {
  return fipa::ipa_pair_trace_read(host, bytes) ? 0 : 1;
}
extern "C" __attribute__((visibility("default"))) int ipa_pair_span_copy(void* host, size_t bytes) {
  return fipa::ipa_pair_span_read(host, bytes) ? 0 : 1;
}
extern "C" __attribute__((visibility("default"))) int ipa_bwd_trace_copy(void* host, size_t bytes) {
  return fipa::ipa_bwd_trace_read(host, bytes) ? 0 : 1;
}
extern "C" __attribute__((visibility("default"))) int ipa_pair_max_clusters() { return fipa::ipa_pair_max_clusters(); }
#endif
