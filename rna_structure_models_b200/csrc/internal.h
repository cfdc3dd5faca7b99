// Internal (non-exported) declarations shared by the host API and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

namespace fipa {

// Geometry of the fused IPA kernels.
constexpr int QT = 128;      // query rows per CTA (tcgen05 M)
constexpr int KT = 64;       // keys per tile (N of Q K^T, K of P V)
constexpr int DH = 64;       // width of the per-head augmented rows (fp16)
constexpr int NSTAGE = 3;    // K/V shared-memory stages
constexpr int MAX_DZ = 256;  // widest pair block (R * Cz padded to 64)
constexpr int IPA_C = 16, IPA_PQ = 4, IPA_PV = 8;

// Strided fp32 / byte view of a caller tensor (strides in elements).
struct View {
  const void* p;
  int64_t s[6];
  int dtype;  // 0 f32, 1 f64, 2 u8
};

struct IpaWorkspace {
  size_t qh, kh, vh, z2, z1h, z1f, rowq, colk, frame, part, cen, oq, ok, headc, wqp, err;
  // key-split tail of the CTA-pair core (with_split): partial accumulators
  // of up to split_chunks chunks (two CTAs each, [DZ + 67][128] floats) and
  // a ticket per (tile, CTA) for up to split_tiles tiles; 0 without
  size_t split, ticket;
  int64_t split_tiles, split_chunks;
  size_t total;
};

// Resident CTA pairs of the core on a B200 (148 SMs, one CTA per SM): the
// key-split reserve holds two chunks per pair and a ticket per pair.
constexpr int kSplitPairs = 74;

IpaWorkspace ipa_workspace_layout(int B, int L, int H, int DZ, int RCz, bool with_split = false);

struct SplitPlan {
  int first;   // pair tiles before this run whole
  int S;       // chunks per later tile (1: no split)
};
SplitPlan ipa_split_plan(int T, int nkp, int P, int64_t max_tiles, int64_t max_chunks);

struct IpaLaunch {
  int B, L, H, C, Pq, Pv, R, Cz, DZ, RCz, F, nqt, nkt;
  float w_L, w_C, scalar_scale;
  View q, k, v, q_pts, k_pts, v_pts, rot, trans, z1, z2, w_bias, gamma, mask;
  float* out;
  // training forward only (else null): log-sum-exp of the logits per (b, h, i)
  // in natural-log units (+inf for rows without an allowed key), [B, H, L];
  // pair aggregate U_i = sum_j a_ij z2_j, [B, L, H, R Cz]
  float* lse = nullptr;
  float* uagg = nullptr;
  unsigned char* ws;
  IpaWorkspace lay;
  int* err;
};

// Stage launches; each returns the cudaError_t of its last launch.
cudaError_t ipa_launch_prologue(const IpaLaunch& a, cudaStream_t stream);
cudaError_t ipa_launch_core(const IpaLaunch& a, cudaStream_t stream);

// Gradients of the IPA core (ipa_backward.cu).  The workspace holds the
// forward prologue's outputs (recomputed) followed by the backward's.
struct IpaBwdWorkspace {
  IpaWorkspace fwd;
  size_t doh, du, qp, rowd, dqh, dqp, rsq, dkh, dva, dz2, csk, pts, gsum, wb_part, g_part;
  // query split of the key pass's last wave: partials of up to ksplit_chunks
  // chunks ([DZ + 138][128] floats each) and a ticket per split key tile
  size_t kpart, kticket;
  int64_t ksplit_tiles, ksplit_chunks;
  size_t total;
};

// Resident CTAs of the gradient passes on a B200 (148 SMs, one CTA per SM):
// the key-pass split runs its chunks in one round, at most this many.
constexpr int kBwdSlots = 148;
IpaBwdWorkspace ipa_bwd_workspace_layout(int B, int L, int H, int DZ, int RCz);

struct IpaBwdLaunch {
  IpaLaunch f;                 // forward inputs; f.ws / f.lay point at the backward workspace
  View out, lse, uagg, g_out;  // forward output [B,L,H,F], lse [B,H,L], U [B,L,H,R,Cz], upstream [B,L,H,F]
  // gradients (contiguous fp32, shapes of the inputs)
  float *d_q, *d_k, *d_v, *d_q_pts, *d_k_pts, *d_v_pts, *d_rot, *d_trans, *d_z1, *d_z2, *d_w_bias, *d_gamma;
  IpaBwdWorkspace lay;
};
cudaError_t ipa_launch_bwd(const IpaBwdLaunch& a, cudaStream_t stream);

// Local nearest-neighbour distogram (distogram.cu).
constexpr int DIST_MAX_K = 32, DIST_MAX_EDGES = 63;
struct DistogramArgs {
  int B, L, k, nb;                 // nb = number of edges + 1
  View x, mask;                    // [B, L, 3] f32, [B, L] u8
  float edge2[DIST_MAX_EDGES];     // squared edges (float32 products)
  int32_t* idx;                    // [B, L, k]
  int32_t* bins;                   // [B, L, k]
  float* hist;                     // [B, L, nb]
  int* err;                        // bounds-checked build only; the call has no error word (null)
};
cudaError_t distogram_launch(const DistogramArgs& a, cudaStream_t stream);

// Distance-aware attention (MEET) on the IPA core: C = 16, Pq = 4, Pv = 8 and
// no pair block (pair width 0, which the one-CTA core and the prologue skip),
// output row F = C + 4 Pv.
constexpr int MEET_C = 16, MEET_RCZ = 0, MEET_DZ = 0, MEET_F = 16 + 4 * 8, MEET_ZEROS = 128;

struct MeetWorkspace {
  size_t ipa, qs, gamma, consts, out, total;
};
MeetWorkspace meet_workspace_layout(int B, int L, int H);

struct MeetPrep {
  int B, L, H;
  View q, rho, s;
  float* qs;       // [B, L, H, 16] rho_h q
  float* gamma;    // [H] rho_h s_h^2
  float* consts;   // MEET_ZEROS zeros, then the 3x3 identity
  int* err;
};
cudaError_t meet_launch_prep(const MeetPrep& m, cudaStream_t stream);
cudaError_t meet_launch_extract(const float* core_out, float* out, int64_t rows, int* err, cudaStream_t stream);

// Dense projection y = x W + b (tcgen05, fp16 operands, fp32 accumulation).
struct LinearWorkspace {
  size_t x16, w16, w32, total;
};
LinearWorkspace linear_workspace_layout(int M, int K, int N);

struct LinearLaunch {
  int M, K, N;
  View x, w;            // [M, K], [K, N] fp32
  const float* bias;    // [N] contiguous or null
  float* y;             // [M, ldy] fp32
  int64_t ldy;
  unsigned char* ws;
  LinearWorkspace lay;
  int* err;
};
cudaError_t linear_launch(const LinearLaunch& a, cudaStream_t stream);

// Residue frames from backbone atoms.
struct FramesArgs {
  int B, L;
  View n, ca, c;   // [B, L, 3]
  float* rot;      // [B, L, 3, 3]
  float* trans;    // [B, L, 3]
  int* err;        // bounds-checked build only; the call has no error word (null)
};
cudaError_t frames_launch(const FramesArgs& a, cudaStream_t stream);

struct GeoWorkspace {
  size_t qg, kg, vg, rotf, ml, live, wf, bf, sc, err, total;
};

GeoWorkspace geo_workspace_layout(int B, int N, int H, int M, int Cout);

struct GeoLaunch {
  int B, N, H, M, Cout, HM3;
  View q_direction, k_direction, q_point, k_point, values, direction_scale, distance_scale,
      output_weight, output_bias, rotation, translation, frame_mask, pair_mask;
  bool has_bias, has_pair_mask;
  float* out_vectors;
  float* out_output;
  float* out_attention;  // may be null
  float* out_agg;        // [B*H, N, 3M] global-frame aggregate, or null
  bool skip_readout;     // stop after the vectors (gradient pass)
  unsigned char* ws;
  GeoWorkspace lay;
  int* err;
};

cudaError_t geo_launch_all(const GeoLaunch& a, cudaStream_t stream);

// Gradients of the variant: the forward statistics are recomputed into the
// forward part of the workspace, then the adjoint kernels run.
struct GeoBwdWorkspace {
  GeoWorkspace fwd;   // offsets relative to the start of the gradient workspace
  size_t vec, agg, gvec, rowlive, dagg, rowinfo, dq, dk, dvr, acc, wt, dwpart, dbpart, total;
};
GeoBwdWorkspace geo_bwd_workspace_layout(int B, int N, int H, int M, int Cout);

struct GeoBwdLaunch {
  GeoLaunch f;             // forward inputs; its ws / lay point into the gradient workspace
  View g_output, g_attention, g_vectors;
  bool has_g_attention, has_g_vectors;
  // gradients (contiguous fp32); d_output_bias may be null
  float *d_q_direction, *d_k_direction, *d_q_point, *d_k_point, *d_values, *d_direction_scale,
      *d_distance_scale, *d_output_weight, *d_output_bias, *d_rotation, *d_translation;
  unsigned char* ws;
  GeoBwdWorkspace lay;
};
cudaError_t geo_launch_bwd(const GeoBwdLaunch& a, cudaStream_t stream);

#ifdef IPA_TRACE
bool ipa_trace_read(void* host, size_t bytes);
#endif

// cuTensorMapEncodeTiled obtained through the runtime's driver entry point.
// swizzle_bytes: 128 or 64 (the inner box must then be exactly that many bytes).
bool encode_tmap_f16_3d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1,
                        uint64_t d2, uint64_t stride1_bytes, uint64_t stride2_bytes,
                        uint32_t box0, uint32_t box1, int swizzle_bytes = 128);
bool encode_tmap_f16_panels(CUtensorMap* map, const void* base, uint64_t DZ, uint64_t L, uint64_t B,
                            uint32_t box_rows, uint32_t box_panels);
bool encode_tmap_f32_sw128(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                           const uint64_t* strides_bytes, const uint32_t* box);

// CTA-pair core kernel (cta_group::2): pair-dimension widths it supports and its launch.
bool ipa_pair_supported(int DZ);
cudaError_t ipa_launch_core_pair(const IpaLaunch& a, cudaStream_t stream);
#ifdef IPA_TRACE
bool ipa_pair_trace_read(void* host, size_t bytes);
bool ipa_pair_span_read(void* host, size_t bytes);
bool ipa_bwd_trace_read(void* host, size_t bytes);
int ipa_pair_max_clusters();
#endif

}  // namespace fipa
