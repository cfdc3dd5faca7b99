/* End-to-end use of the C ABI from plain C99 with host buffers: the caller
 * allocates page-locked host inputs and outputs, and device staging and
 * workspace for two in-flight calls, then times `calls` calls of
 * ipa_attn_fwd_host (copies up, prologue and core kernels, copy back, all
 * enqueued by the library) alternating over two streams, with CUDA events,
 * and the same number of ipa_attn_fwd_host_packed calls (the inputs in one
 * page-locked buffer at the offsets ipa_attn_host_packed_layout gives).
 * It also checks that both host results equal, bit for bit, what
 * ipa_attn_fwd gives on the same inputs copied to the device by hand.
 *
 * Usage: e2e_host L [calls]   (B = 1, H = 12, C = 16, Pq = 4, Pv = 8, R = 2,
 * Cz = 128).  Prints "e2e ok ms_per_call=<t> packed_ms_per_call=<t>
 * h2d_bytes=<n> d2h_bytes=<n>". */
#include <cuda_runtime.h>
#include <math.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "flashipa_b200.h"

#define CK(x)                                                                        \
  do {                                                                               \
    cudaError_t e_ = (x);                                                            \
    if (e_ != cudaSuccess) {                                                         \
      fprintf(stderr, "CUDA error %s at line %d\n", cudaGetErrorString(e_), __LINE__); \
      return 1;                                                                      \
    }                                                                                \
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

/* deterministic pseudo-random values in [-1, 1) (a 32-bit LCG) */
static unsigned int lcg = 12345u;
static float urand(void) {
  lcg = lcg * 1664525u + 1013904223u;
  return (float)((lcg >> 8) & 0xFFFFFF) / 8388608.0f - 1.0f;
}

int main(int argc, char** argv) {
  const int L = argc > 1 ? atoi(argv[1]) : 1024;
  const int calls = argc > 2 ? atoi(argv[2]) : 20;
  const int B = 1, H = 12, C = 16, Pq = 4, Pv = 8, R = 2, Cz = 128, F = C + 4 * Pv + Cz;
  ipa_params_t p;
  const int64_t s_qkv[4] = {B, L, H, C}, s_qp[5] = {B, L, H, Pq, 3}, s_vp[5] = {B, L, H, Pv, 3};
  const int64_t s_rot[4] = {B, L, 3, 3}, s_tr[3] = {B, L, 3}, s_z[4] = {B, L, R, Cz}, s_w[2] = {Cz, H};
  const int64_t s_g[1] = {H}, s_m[2] = {B, L}, s_o[4] = {B, L, H, F};
  const int64_t* shp[14] = {s_qkv, s_qkv, s_qkv, s_qp, s_qp, s_vp, s_rot, s_tr, s_z, s_z, s_w, s_g, s_m, s_o};
  const int nd[14] = {4, 4, 4, 5, 5, 5, 4, 3, 4, 4, 2, 1, 2, 4};
  size_t bytes[14], h2d = 0;
  void* host[14];
  void* hout2;
  void* dev[14];
  ipa_tensor_t th[14], td[14];
  int t, d, slot, i;
  size_t stg_bytes, ws_bytes;
  void *stg[2], *ws[2], *ws_dev;
  int32_t* err;
  int32_t herr[3];
  cudaStream_t st[2];
  cudaEvent_t e0, e1;
  float ms = 0.f, ms_packed = 0.f;
  ipa_status_t s;
  size_t offs[13], packed_bytes;
  unsigned char* packed;

  p.B = B; p.L = L; p.H = H; p.C = C; p.Pq = Pq; p.Pv = Pv; p.R = R; p.Cz = Cz;
  p.w_L = (float)sqrt(1.0 / 3.0);
  p.w_C = (float)sqrt(2.0 / (9.0 * Pq));
  p.scalar_scale = 0.25f;
  for (t = 0; t < 14; ++t) {
    size_t n = 1;
    for (d = 0; d < nd[t]; ++d) n *= (size_t)shp[t][d];
    bytes[t] = n * (t == 12 ? 1 : 4);
    if (t < 13) h2d += bytes[t];
    CK(cudaMallocHost(&host[t], bytes[t]));
    CK(cudaMalloc(&dev[t], bytes[t]));
    th[t] = tensor(host[t], t == 12 ? IPA_DTYPE_BOOL : IPA_DTYPE_F32, nd[t], shp[t]);
    td[t] = tensor(dev[t], t == 12 ? IPA_DTYPE_BOOL : IPA_DTYPE_F32, nd[t], shp[t]);
  }
  CK(cudaMallocHost(&hout2, bytes[13]));
  /* inputs: values in [-1, 1), points x 3, frames = identity rotations on a
   * 3.8 A staircase, gamma > 0, every residue valid */
  for (t = 0; t < 12; ++t) {
    float* f = (float*)host[t];
    size_t n = bytes[t] / 4;
    size_t e;
    for (e = 0; e < n; ++e) f[e] = urand() * (t >= 3 && t <= 5 ? 3.0f : 1.0f);
  }
  for (i = 0; i < L; ++i) {
    float* r = (float*)host[6] + 9 * i;
    float* tr = (float*)host[7] + 3 * i;
    memset(r, 0, 9 * sizeof(float));
    r[0] = r[4] = r[8] = 1.0f;
    tr[0] = 2.2f * (float)i; tr[1] = 2.2f * (float)(i % 7); tr[2] = 2.2f * (float)(i % 3);
  }
  for (t = 0; t < H; ++t) ((float*)host[11])[t] = 0.5f + 0.04f * (float)t;
  memset(host[12], 1, bytes[12]);

  stg_bytes = ipa_attn_host_staging_size(&p);
  ws_bytes = ipa_attn_workspace_size(&p);
  if (stg_bytes == 0 || ws_bytes == 0) { fprintf(stderr, "params rejected\n"); return 1; }
  for (slot = 0; slot < 2; ++slot) {
    CK(cudaMalloc(&stg[slot], stg_bytes));
    CK(cudaMalloc(&ws[slot], ws_bytes));
    CK(cudaStreamCreateWithFlags(&st[slot], cudaStreamNonBlocking));
  }
  CK(cudaMalloc(&ws_dev, ws_bytes));
  CK(cudaMalloc((void**)&err, 3 * sizeof(int32_t)));
  CK(cudaMemset(err, 0, 3 * sizeof(int32_t)));

  /* reference: inputs copied by hand, device entry point */
  for (t = 0; t < 13; ++t) CK(cudaMemcpy(dev[t], host[t], bytes[t], cudaMemcpyHostToDevice));
  s = ipa_attn_fwd(&p, &td[0], &td[1], &td[2], &td[3], &td[4], &td[5], &td[6], &td[7], &td[8], &td[9], &td[10],
                   &td[11], &td[12], &td[13], ws_dev, ws_bytes, NULL, err + 2);
  if (s != IPA_OK) { fprintf(stderr, "ipa_attn_fwd: %s\n", ipa_status_string(s)); return 1; }
  CK(cudaDeviceSynchronize());
  CK(cudaMemcpy(hout2, dev[13], bytes[13], cudaMemcpyDeviceToHost));

  /* warm-up and the bitwise check of the host entry point */
  for (slot = 0; slot < 2; ++slot) {
    s = ipa_attn_fwd_host(&p, &th[0], &th[1], &th[2], &th[3], &th[4], &th[5], &th[6], &th[7], &th[8], &th[9],
                          &th[10], &th[11], &th[12], &th[13], stg[slot], stg_bytes, ws[slot], ws_bytes, st[slot],
                          err + slot);
    if (s != IPA_OK) { fprintf(stderr, "ipa_attn_fwd_host: %s\n", ipa_status_string(s)); return 1; }
    CK(cudaStreamSynchronize(st[slot]));
    if (memcmp(host[13], hout2, bytes[13]) != 0) { fprintf(stderr, "host result differs\n"); return 1; }
  }

  /* the packed layout: the same inputs in one page-locked buffer */
  packed_bytes = ipa_attn_host_packed_layout(&p, offs);
  if (packed_bytes == 0) { fprintf(stderr, "packed layout rejected\n"); return 1; }
  CK(cudaMallocHost((void**)&packed, packed_bytes));
  memset(packed, 0, packed_bytes);
  for (t = 0; t < 13; ++t) memcpy(packed + offs[t], host[t], bytes[t]);
  for (slot = 0; slot < 2; ++slot) {
    memset(host[13], 0, bytes[13]);
    s = ipa_attn_fwd_host_packed(&p, packed, packed_bytes, &th[13], stg[slot], stg_bytes, ws[slot], ws_bytes,
                                 st[slot], err + slot);
    if (s != IPA_OK) { fprintf(stderr, "ipa_attn_fwd_host_packed: %s\n", ipa_status_string(s)); return 1; }
    CK(cudaStreamSynchronize(st[slot]));
    if (memcmp(host[13], hout2, bytes[13]) != 0) { fprintf(stderr, "packed host result differs\n"); return 1; }
  }

  /* timed: `calls` calls alternating over the two streams, per-input
   * uploads first, then the packed layout */
  CK(cudaEventCreate(&e0));
  CK(cudaEventCreate(&e1));
  for (d = 0; d < 2; ++d) {
    CK(cudaDeviceSynchronize());
    CK(cudaEventRecord(e0, st[0]));
    CK(cudaStreamWaitEvent(st[1], e0, 0));
    for (i = 0; i < calls; ++i) {
      slot = i & 1;
      if (d == 0)
        s = ipa_attn_fwd_host(&p, &th[0], &th[1], &th[2], &th[3], &th[4], &th[5], &th[6], &th[7], &th[8], &th[9],
                              &th[10], &th[11], &th[12], &th[13], stg[slot], stg_bytes, ws[slot], ws_bytes, st[slot],
                              err + slot);
      else
        s = ipa_attn_fwd_host_packed(&p, packed, packed_bytes, &th[13], stg[slot], stg_bytes, ws[slot], ws_bytes,
                                     st[slot], err + slot);
      if (s != IPA_OK) { fprintf(stderr, "host call: %s\n", ipa_status_string(s)); return 1; }
    }
    {
      cudaEvent_t done;
      CK(cudaEventCreate(&done));
      CK(cudaEventRecord(done, st[1]));
      CK(cudaStreamWaitEvent(st[0], done, 0));
      CK(cudaEventRecord(e1, st[0]));
      CK(cudaEventSynchronize(e1));
      CK(cudaEventDestroy(done));
    }
    CK(cudaEventElapsedTime(d == 0 ? &ms : &ms_packed, e0, e1));
  }
  CK(cudaMemcpy(herr, err, sizeof herr, cudaMemcpyDeviceToHost));
  if (herr[0] || herr[1] || herr[2]) { fprintf(stderr, "device error %d %d %d\n", herr[0], herr[1], herr[2]); return 1; }
  printf("e2e ok ms_per_call=%.4f packed_ms_per_call=%.4f h2d_bytes=%lu d2h_bytes=%lu\n", ms / (float)calls,
         ms_packed / (float)calls, (unsigned long)h2d, (unsigned long)bytes[13]);
  return 0;
}
