/* Host-only check that the C ABI is usable from plain C99: the header
 * compiles without C++, the library links, and the host-side paths (sizes,
 * argument validation, status strings) answer as declared.  Nothing here
 * launches a kernel: every call below is rejected before a launch, or is a
 * pure host function. */
#include <stdio.h>
#include <string.h>

#include "flashipa_b200.h"

static int failures = 0;

#define EXPECT(cond)                                                  \
  do {                                                                \
    if (!(cond)) {                                                    \
      fprintf(stderr, "FAILED line %d: %s\n", __LINE__, #cond);       \
      ++failures;                                                     \
    }                                                                 \
  } while (0)

static ipa_tensor_t tensor(const void* data, int32_t dtype, int ndim, const int64_t* size) {
  ipa_tensor_t t;
  int64_t acc = 1;
  int d;
  memset(&t, 0, sizeof t);
  t.data = data;
  t.dtype = dtype;
  t.ndim = ndim;
  for (d = ndim - 1; d >= 0; --d) {
    t.size[d] = size[d];
    t.stride[d] = acc;
    acc *= size[d];
  }
  return t;
}

int main(void) {
  /* a non-null address that is never dereferenced: every call is rejected first */
  const void* fake = (const void*)(uintptr_t)(1u << 20);
  ipa_params_t p;
  geo_params_t g;
  ipa_module_params_t m;
  size_t ws;

  EXPECT(ipa_version() != NULL && strlen(ipa_version()) > 0);
  EXPECT(strlen(ipa_status_string(IPA_ERR_SHAPE)) > 0);
  EXPECT(ipa_status_string(IPA_OK) != ipa_status_string(IPA_ERR_CUDA));

  p.B = 1; p.L = 4096; p.H = 12; p.C = 16; p.Pq = 4; p.Pv = 8; p.R = 2; p.Cz = 128;
  p.w_L = 0.57735f; p.w_C = 0.2357f; p.scalar_scale = 0.25f;
  ws = ipa_attn_workspace_size(&p);
  EXPECT(ws > 0);
  p.C = 32;
  EXPECT(ipa_attn_workspace_size(&p) == 0);   /* outside the envelope */
  p.C = 16;

  {
    /* q with the wrong head count: IPA_ERR_SHAPE before any launch */
    const int64_t s_bad[4] = {1, 4096, 11, 16}, s_q[4] = {1, 4096, 12, 16};
    const int64_t s_qp[5] = {1, 4096, 12, 4, 3}, s_vp[5] = {1, 4096, 12, 8, 3};
    const int64_t s_r[4] = {1, 4096, 3, 3}, s_t[3] = {1, 4096, 3}, s_z[4] = {1, 4096, 2, 128};
    const int64_t s_wb[2] = {128, 12}, s_g[1] = {12}, s_m[2] = {1, 4096}, s_o[4] = {1, 4096, 12, 176};
    ipa_tensor_t q = tensor(fake, IPA_DTYPE_F32, 4, s_bad), k = tensor(fake, IPA_DTYPE_F32, 4, s_q),
                 v = tensor(fake, IPA_DTYPE_F32, 4, s_q), qp = tensor(fake, IPA_DTYPE_F32, 5, s_qp),
                 kp = tensor(fake, IPA_DTYPE_F32, 5, s_qp), vp = tensor(fake, IPA_DTYPE_F32, 5, s_vp),
                 r = tensor(fake, IPA_DTYPE_F32, 4, s_r), t = tensor(fake, IPA_DTYPE_F32, 3, s_t),
                 z1 = tensor(fake, IPA_DTYPE_F32, 4, s_z), z2 = tensor(fake, IPA_DTYPE_F32, 4, s_z),
                 wb = tensor(fake, IPA_DTYPE_F32, 2, s_wb), gm = tensor(fake, IPA_DTYPE_F32, 1, s_g),
                 mk = tensor(fake, IPA_DTYPE_BOOL, 2, s_m), o = tensor(fake, IPA_DTYPE_F32, 4, s_o);
    EXPECT(ipa_attn_fwd(&p, &q, &k, &v, &qp, &kp, &vp, &r, &t, &z1, &z2, &wb, &gm, &mk, &o, (void*)fake, ws,
                        NULL, NULL) == IPA_ERR_SHAPE);
    q = tensor(fake, IPA_DTYPE_F32, 4, s_q);
    EXPECT(ipa_attn_fwd(&p, &q, &k, &v, &qp, &kp, &vp, &r, &t, &z1, &z2, &wb, &gm, &mk, &o, (void*)fake, 16,
                        NULL, NULL) == IPA_ERR_WORKSPACE);
    EXPECT(ipa_attn_fwd(NULL, &q, &k, &v, &qp, &kp, &vp, &r, &t, &z1, &z2, &wb, &gm, &mk, &o, (void*)fake, ws,
                        NULL, NULL) == IPA_ERR_NULL);
  }

  g.B = 2; g.N = 2048; g.H = 8; g.M = 4; g.Cout = 256;
  EXPECT(geo_attn_workspace_size(&g) > 0);
  EXPECT(geo_attn_bwd_workspace_size(&g) > geo_attn_workspace_size(&g));
  EXPECT(ipa_linear_workspace_size(4096, 384, 1152) > 0);
  EXPECT(ipa_linear_workspace_size(4096, 70000, 16) == 0);
  {
    const int64_t s_x[2] = {64, 32}, s_w[2] = {33, 8}, s_y[2] = {64, 8};
    ipa_tensor_t x = tensor(fake, IPA_DTYPE_F32, 2, s_x), w = tensor(fake, IPA_DTYPE_F32, 2, s_w),
                 y = tensor(fake, IPA_DTYPE_F32, 2, s_y);
    EXPECT(ipa_linear_fwd(64, 32, 8, &x, &w, NULL, &y, (void*)fake, ipa_linear_workspace_size(64, 32, 8), NULL,
                          NULL) == IPA_ERR_SHAPE);
  }
  m.core = p;
  m.c_s = 384;
  EXPECT(ipa_module_workspace_size(&m) > ws);
  m.c_s = 0;
  EXPECT(ipa_module_workspace_size(&m) == 0);
  EXPECT(ipa_device_error_status(0) == IPA_OK);

  if (failures == 0) printf("c abi ok (%s)\n", ipa_version());
  return failures == 0 ? 0 : 1;
}
