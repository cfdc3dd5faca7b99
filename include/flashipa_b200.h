/*
 * flashipa_b200.h -- C ABI of the B200 (sm_100a) fused Invariant Point
 * Attention core, of the geometric direction/distance attention variant and
 * its gradients, of MEET's distance-aware attention, and of the pieces of the
 * IPA layer around the core (residue frames from backbone atoms, tensor-core
 * projections, the whole layer).
 *
 * Every buffer is owned by the caller.  The library never allocates or frees
 * device memory and never writes to an input.  Work is enqueued on the
 * caller's CUDA stream; a return of IPA_OK means "validated and launched".
 * Argument errors are returned before anything is launched; errors that can
 * only be seen on the device (a bounded wait that ran out) are written, first
 * one wins, into the optional device word `dev_err` (0 = no error), which the
 * caller reads after synchronising the stream.  No C++ exception crosses this
 * boundary.
 *
 * Tensors are passed as ipa_tensor_t: a device pointer, a dtype code, and the
 * logical sizes and element strides of every dimension (stride 0 expresses a
 * broadcast where that is allowed).  Inputs may be non-contiguous; outputs
 * must be contiguous.
 */
#ifndef FLASHIPA_B200_H_
#define FLASHIPA_B200_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define IPA_API __attribute__((visibility("default")))
#else
#define IPA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  IPA_OK = 0,
  IPA_ERR_NULL = 1,         /* a required pointer is NULL                       */
  IPA_ERR_SHAPE = 2,        /* sizes disagree with the params or are < 1        */
  IPA_ERR_STRIDE_ALIGN = 3, /* negative stride, non-contiguous output, or a
                               misaligned pointer                               */
  IPA_ERR_DTYPE = 4,        /* wrong element type                               */
  IPA_ERR_WORKSPACE = 5,    /* workspace too small or not 256-byte aligned      */
  IPA_ERR_UNSUPPORTED = 6,  /* dims outside the supported envelope (below)      */
  IPA_ERR_CUDA = 7,         /* a CUDA runtime call failed (launch, attribute)   */
  IPA_ERR_TIMEOUT = 8,      /* device: a bounded wait ran out (in dev_err only) */
  IPA_ERR_BOUNDS = 9        /* device, bounds-checked build only: a store index
                               left its buffer (in dev_err only)                */
} ipa_status_t;

/* Element type codes. */
enum {
  IPA_DTYPE_F32 = 0,
  IPA_DTYPE_F64 = 1,
  IPA_DTYPE_BOOL = 2, /* one byte per element, 0 = false */
  IPA_DTYPE_F16 = 3,
  IPA_DTYPE_I32 = 4
};

#define IPA_MAX_DIMS 6

typedef struct {
  const void* data;              /* device pointer                            */
  int32_t dtype;                 /* IPA_DTYPE_*                               */
  int32_t ndim;                  /* number of dimensions used                 */
  int64_t size[IPA_MAX_DIMS];    /* logical sizes                             */
  int64_t stride[IPA_MAX_DIMS];  /* strides in ELEMENTS (not bytes), >= 0     */
} ipa_tensor_t;

/* --------------------------------------------------------------------------
 * Fused IPA core.
 *
 * Operation (Flash Invariant Point Attention, TL;DR and Abstract: IPA with
 * the factorised pair representation z_ij = sum_r z1_i[r] * z2_j[r]; MEET,
 * section 2.2 eq. (7)-(8) for the squared distance folded into augmented
 * query/key columns).  For batch b, query residue i, key residue j, head h:
 *   gq = R_i q_pts + t_i, gk = R_j k_pts + t_j, gv = R_j v_pts + t_j
 *   logit = w_L * ( scalar_scale * q.k
 *                   + sum_{r,c} w_bias[c,h] z1_i[r,c] z2_j[r,c]
 *                   - gamma_h * w_C / 2 * sum_p |gq_p - gk_p|^2 )
 *   a = softmax over keys j with mask_i && mask_j (no allowed key -> a = 0)
 *   out[b,i,h,:] = [ sum_j a v_j                      (C)
 *                  | R_i^T (sum_j a gv_j - t_i)       (Pv x 3, xyz inner)
 *                  | norms of those Pv points         (Pv)
 *                  | sum_r z1_i[r,:] * sum_j a z2_j[r,:] (Cz) ]
 *   and every feature is 0 for a row with no allowed key.
 * The L x L logits and the pair tensor are never materialised.
 *
 * Shapes (all float inputs IPA_DTYPE_F32, any non-negative strides):
 *   q, k, v          [B, L, H, C]
 *   q_pts, k_pts     [B, L, H, Pq, 3]
 *   v_pts            [B, L, H, Pv, 3]
 *   rot              [B, L, 3, 3]   rot[b,i] maps local column vectors to global
 *   trans            [B, L, 3]
 *   z1, z2           [B, L, R, Cz]
 *   w_bias           [Cz, H]
 *   gamma            [H]            already positive (e.g. softplus of a weight)
 *   mask             [B, L]         IPA_DTYPE_BOOL
 *   out              [B, L, H, C + 4 Pv + Cz], IPA_DTYPE_F32, contiguous
 * Supported envelope: C == 16, Pq == 4, Pv == 8 (the AlphaFold-2 IPA head
 * shape), 1 <= R * Cz <= 256 with Cz a multiple of 16, 1 <= L <= 1048576,
 * 1 <= H <= 128.
 * Arithmetic: fp16 tensor-core operands with fp32 accumulation; point
 * coordinates, key norms and value points carry a second fp16 term for the
 * rounding residue.
 * ------------------------------------------------------------------------ */
typedef struct {
  int32_t B, L, H, C, Pq, Pv, R, Cz;
  float w_L;          /* weight of the whole logit, sqrt(1/3) in AlphaFold-2 */
  float w_C;          /* point weight, sqrt(2 / (9 Pq)) in AlphaFold-2       */
  float scalar_scale; /* 1 / sqrt(C) in AlphaFold-2                          */
} ipa_params_t;

/* Bytes of device workspace ipa_attn_fwd needs for these params (0 if the
 * params are invalid).  Pure host function.  Linear in B L H plus, for pair
 * widths 128 and 256, a bounded reserve for the key-split tail of the core:
 * the last, partial wave of (batch, head, 256-query) tiles may run as
 * chunks of consecutive key tiles whose partial accumulators are stored
 * there and merged by the chunk that finishes last (at most 2 x 74 chunks,
 * 49 MB at a pair width of 256). */
IPA_API size_t ipa_attn_workspace_size(const ipa_params_t* p);

/* Enqueue the fused IPA core on `stream` (a cudaStream_t, NULL = legacy
 * default stream).  workspace: device memory of at least
 * ipa_attn_workspace_size(p) bytes, 256-byte aligned, not shared with a
 * concurrent call.  dev_err: optional device int (NULL allowed). */
IPA_API ipa_status_t ipa_attn_fwd(const ipa_params_t* p,
                          const ipa_tensor_t* q, const ipa_tensor_t* k, const ipa_tensor_t* v,
                          const ipa_tensor_t* q_pts, const ipa_tensor_t* k_pts,
                          const ipa_tensor_t* v_pts,
                          const ipa_tensor_t* rot, const ipa_tensor_t* trans,
                          const ipa_tensor_t* z1, const ipa_tensor_t* z2,
                          const ipa_tensor_t* w_bias, const ipa_tensor_t* gamma,
                          const ipa_tensor_t* mask, const ipa_tensor_t* out,
                          void* workspace, size_t workspace_bytes,
                          void* stream, int32_t* dev_err);

/* The two stages of ipa_attn_fwd, callable separately (same arguments and
 * rules).  ipa_attn_prologue applies the frames and writes the augmented
 * fp16 operands into the workspace; ipa_attn_core runs the fused attention
 * pass from that workspace into `out`.  The core reads only the workspace,
 * so it must follow a prologue with the same params and workspace on the
 * same stream; it may run several times after one prologue.  After a call
 * that reported an error through dev_err, run the prologue again before the
 * next core (the prologue also resets the key-split tickets in the
 * workspace).  ipa_attn_fwd == prologue then core. */
IPA_API ipa_status_t ipa_attn_prologue(const ipa_params_t* p,
                               const ipa_tensor_t* q, const ipa_tensor_t* k, const ipa_tensor_t* v,
                               const ipa_tensor_t* q_pts, const ipa_tensor_t* k_pts,
                               const ipa_tensor_t* v_pts,
                               const ipa_tensor_t* rot, const ipa_tensor_t* trans,
                               const ipa_tensor_t* z1, const ipa_tensor_t* z2,
                               const ipa_tensor_t* w_bias, const ipa_tensor_t* gamma,
                               const ipa_tensor_t* mask,
                               void* workspace, size_t workspace_bytes,
                               void* stream, int32_t* dev_err);
IPA_API ipa_status_t ipa_attn_core(const ipa_params_t* p, const ipa_tensor_t* out,
                           void* workspace, size_t workspace_bytes,
                           void* stream, int32_t* dev_err);

/* --------------------------------------------------------------------------
 * ipa_attn_fwd on HOST buffers (end-to-end call for callers whose inputs and
 * results live in host memory).  Same params and shapes as ipa_attn_fwd;
 * every input and `out` must be a contiguous host buffer (page-locked, e.g.
 * from cudaMallocHost, for the copies to be asynchronous).  On `stream` the
 * call enqueues one cudaMemcpyAsync per input into `staging` (device memory
 * of ipa_attn_host_staging_size(p) bytes, 256-byte aligned, caller-owned),
 * the prologue and core kernels (using `workspace` as ipa_attn_fwd does) and
 * one cudaMemcpyAsync of the result back into `out`.  The caller
 * synchronises the stream before reading `out` or reusing the host inputs.
 * Calls on different streams with their own staging and workspace overlap
 * one call's copies with another's kernels.
 * ------------------------------------------------------------------------ */
IPA_API size_t ipa_attn_host_staging_size(const ipa_params_t* p);

IPA_API ipa_status_t ipa_attn_fwd_host(const ipa_params_t* p,
                          const ipa_tensor_t* q, const ipa_tensor_t* k, const ipa_tensor_t* v,
                          const ipa_tensor_t* q_pts, const ipa_tensor_t* k_pts,
                          const ipa_tensor_t* v_pts,
                          const ipa_tensor_t* rot, const ipa_tensor_t* trans,
                          const ipa_tensor_t* z1, const ipa_tensor_t* z2,
                          const ipa_tensor_t* w_bias, const ipa_tensor_t* gamma,
                          const ipa_tensor_t* mask, const ipa_tensor_t* out,
                          void* staging, size_t staging_bytes,
                          void* workspace, size_t workspace_bytes,
                          void* stream, int32_t* dev_err);

/* Packed host inputs: the 13 inputs of ipa_attn_fwd_host, stored dense
 * (C order, IPA_DTYPE_F32; mask one byte per element) in one host buffer in
 * argument order, input t starting at byte offsets[t] (multiples of 256).
 * ipa_attn_host_packed_layout fills offsets[13] and returns the buffer's
 * size in bytes (0 for invalid params or a null offsets).  Pure host
 * function.
 *
 * ipa_attn_fwd_host_packed is ipa_attn_fwd_host for such a buffer
 * (`host_inputs`, `host_bytes` >= the layout size; page-locked for the copy
 * to be asynchronous): one cudaMemcpyAsync of the whole buffer into
 * `staging` instead of one per input (each copy has a fixed cost on the
 * copy engine; thirteen cost ~0.3 ms per call at L = 4096), then the same
 * kernels and the copy of the result into `out` (host, [B, L, H, C + 4 Pv +
 * Cz] IPA_DTYPE_F32, contiguous).  Same staging, workspace, stream and error
 * rules as ipa_attn_fwd_host; IPA_ERR_SHAPE if host_bytes is too small. */
IPA_API size_t ipa_attn_host_packed_layout(const ipa_params_t* p, size_t offsets[13]);

IPA_API ipa_status_t ipa_attn_fwd_host_packed(const ipa_params_t* p, const void* host_inputs,
                          size_t host_bytes, const ipa_tensor_t* out,
                          void* staging, size_t staging_bytes,
                          void* workspace, size_t workspace_bytes,
                          void* stream, int32_t* dev_err);

/* --------------------------------------------------------------------------
 * Training forward and gradients of the fused IPA core (Flash Invariant
 * Point Attention trains the factorised IPA: TL;DR "drop-in replacement",
 * Abstract "extends training to previously unattainable lengths", Figure 3).
 *
 * ipa_attn_fwd_train: ipa_attn_fwd plus two per-row results the gradient
 * pass needs (same params, inputs, workspace and rules as ipa_attn_fwd):
 *   lse    [B, H, L]        IPA_DTYPE_F32, contiguous: log sum_{allowed j}
 *                           exp(logit_ij) (natural log); +inf for a row with
 *                           no allowed key
 *   u_agg  [B, L, H, R, Cz] IPA_DTYPE_F32, contiguous, 16-byte aligned:
 *                           U_i = sum_j a_ij z2_j (the pair-value aggregate
 *                           before its contraction with z1_i); 0 on rows with
 *                           no allowed key
 *
 * ipa_attn_bwd: gradients of sum(g_out * out) with respect to every float
 * input, for a caller-given upstream gradient g_out of the output layout.
 * Inputs: the 13 forward inputs, the forward's out, lse and u_agg (from
 * ipa_attn_fwd_train on the same inputs), g_out [B, L, H, C + 4 Pv + Cz]
 * (all IPA_DTYPE_F32, any non-negative strides).  Outputs: ipa_grads_t,
 * each IPA_DTYPE_F32, contiguous, with the shape of its input (mask has no
 * gradient).  Readings: rows with no allowed key pass nothing on; the
 * derivative of a point norm |o_pt| at o_pt = 0 is taken as 0.
 * Method: flash-style recomputation on the forward's augmented fp16
 * operands -- a query-side pass (dQ) and a key-side pass (dK, dV, dZ2) on
 * tcgen05 tensor cores with fp32 accumulation, then per-residue kernels that
 * map the augmented gradients back and sum over heads (fixed order, no
 * atomics: bitwise reproducible).  No L x L array is stored; the workspace
 * (ipa_attn_bwd_workspace_size bytes, 256-byte aligned) is linear in L.
 * Same envelope as ipa_attn_fwd.
 * ------------------------------------------------------------------------ */
IPA_API ipa_status_t ipa_attn_fwd_train(const ipa_params_t* p,
                          const ipa_tensor_t* q, const ipa_tensor_t* k, const ipa_tensor_t* v,
                          const ipa_tensor_t* q_pts, const ipa_tensor_t* k_pts,
                          const ipa_tensor_t* v_pts,
                          const ipa_tensor_t* rot, const ipa_tensor_t* trans,
                          const ipa_tensor_t* z1, const ipa_tensor_t* z2,
                          const ipa_tensor_t* w_bias, const ipa_tensor_t* gamma,
                          const ipa_tensor_t* mask, const ipa_tensor_t* out,
                          const ipa_tensor_t* lse, const ipa_tensor_t* u_agg,
                          void* workspace, size_t workspace_bytes,
                          void* stream, int32_t* dev_err);

typedef struct {
  ipa_tensor_t q, k, v, q_pts, k_pts, v_pts, rot, trans, z1, z2, w_bias, gamma;
} ipa_grads_t;

IPA_API size_t ipa_attn_bwd_workspace_size(const ipa_params_t* p);

IPA_API ipa_status_t ipa_attn_bwd(const ipa_params_t* p,
                          const ipa_tensor_t* q, const ipa_tensor_t* k, const ipa_tensor_t* v,
                          const ipa_tensor_t* q_pts, const ipa_tensor_t* k_pts,
                          const ipa_tensor_t* v_pts,
                          const ipa_tensor_t* rot, const ipa_tensor_t* trans,
                          const ipa_tensor_t* z1, const ipa_tensor_t* z2,
                          const ipa_tensor_t* w_bias, const ipa_tensor_t* gamma,
                          const ipa_tensor_t* mask, const ipa_tensor_t* out,
                          const ipa_tensor_t* lse, const ipa_tensor_t* u_agg,
                          const ipa_tensor_t* g_out, const ipa_grads_t* grads,
                          void* workspace, size_t workspace_bytes,
                          void* stream, int32_t* dev_err);

/* --------------------------------------------------------------------------
 * Geometric direction-and-distance attention ("Geometric direction-and-
 * distance attention", Required behavior).  For query i, key j, head h:
 *   qd = R_i q_direction_i, kd = R_j k_direction_j,
 *   qp = R_i q_point_i + t_i, kp = R_j k_point_j + t_j
 *   s = (softplus(direction_scale_h) qd.kd - softplus(distance_scale_h) |qp - kp|) / sqrt(3)
 *   (unsquared distance, no epsilon; softplus evaluated stably)
 *   allowed = frame_mask_i && frame_mask_j && pair_mask[b,h,i,j]
 *   attention = masked softmax over j (a head row with no allowed key is 0)
 *   vectors_i = R_i^T sum_j attention_ij (R_j values_j)   (no translation)
 *   output_i = flatten(vectors_i in H, M, xyz order) . output_weight (+ output_bias),
 *              forced to 0 when no head of query i has an allowed key.
 *
 * Shapes (float inputs IPA_DTYPE_F32 or IPA_DTYPE_F64, all the same; the
 * kernels compute in fp32; any non-negative strides):
 *   q_direction, k_direction, q_point, k_point [B, N, H, 3]
 *   values            [B, N, H, M, 3]
 *   direction_scale, distance_scale [H]   unconstrained logits
 *   output_weight     [H*M*3, Cout]
 *   output_bias       [Cout] or data == NULL (no bias)
 *   rotation          [B, N, 3, 3]; translation [B, N, 3]
 *   frame_mask        [B, N] IPA_DTYPE_BOOL
 *   pair_mask         [B, H, N, N] IPA_DTYPE_BOOL, broadcast by stride 0, or
 *                     NULL / data == NULL (all pairs allowed)
 * Outputs (IPA_DTYPE_F32, contiguous):
 *   out_vectors       [B, N, H, M, 3]
 *   out_output        [B, N, Cout]
 *   out_attention     [B, H, N, N] or NULL / data == NULL (not written)
 * Supported envelope: H*M*3 <= 384, N <= 1048576.
 * ------------------------------------------------------------------------ */
typedef struct {
  int32_t B, N, H, M, Cout;
} geo_params_t;

IPA_API size_t geo_attn_workspace_size(const geo_params_t* p);

IPA_API ipa_status_t geo_attn_fwd(const geo_params_t* p,
                          const ipa_tensor_t* q_direction, const ipa_tensor_t* k_direction,
                          const ipa_tensor_t* q_point, const ipa_tensor_t* k_point,
                          const ipa_tensor_t* values,
                          const ipa_tensor_t* direction_scale,
                          const ipa_tensor_t* distance_scale,
                          const ipa_tensor_t* output_weight, const ipa_tensor_t* output_bias,
                          const ipa_tensor_t* rotation, const ipa_tensor_t* translation,
                          const ipa_tensor_t* frame_mask, const ipa_tensor_t* pair_mask,
                          const ipa_tensor_t* out_vectors, const ipa_tensor_t* out_output,
                          const ipa_tensor_t* out_attention,
                          void* workspace, size_t workspace_bytes,
                          void* stream, int32_t* dev_err);

/* --------------------------------------------------------------------------
 * Gradients of the geometric attention ("Geometric direction-and-distance
 * attention", Required behavior: the operator is differentiated, with the
 * derivative of the distance at a zero displacement defined as the zero
 * vector).  Given the forward's inputs (as for geo_attn_fwd) and upstream
 * gradients of its results, writes the gradients of
 *   sum(g_output * output) + sum(g_attention * attention) + sum(g_vectors * vectors)
 * with respect to every floating input.  The forward statistics are
 * recomputed inside the call; no N x N array is stored.
 *   g_output     [B, N, Cout]        same dtype as the inputs, any strides
 *   g_attention  [B, H, N, N] or NULL / data == NULL (zero)
 *   g_vectors    [B, N, H, M, 3] or NULL / data == NULL (zero)
 *   grads        one IPA_DTYPE_F32 contiguous buffer per floating input, of
 *                the input's shape; grads->output_bias.data may be NULL only
 *                when output_bias is absent.
 * Queries with no allowed key in any head pass no g_output on (their output
 * is forced to zero).  The caller owns every buffer; errors as for
 * geo_attn_fwd.  Workspace: geo_attn_bwd_workspace_size(p) bytes, 256-byte
 * aligned.
 * ------------------------------------------------------------------------ */
typedef struct {
  ipa_tensor_t q_direction, k_direction, q_point, k_point, values;
  ipa_tensor_t direction_scale, distance_scale, output_weight, output_bias;
  ipa_tensor_t rotation, translation;
} geo_grads_t;

IPA_API size_t geo_attn_bwd_workspace_size(const geo_params_t* p);

IPA_API ipa_status_t geo_attn_bwd(const geo_params_t* p,
                          const ipa_tensor_t* q_direction, const ipa_tensor_t* k_direction,
                          const ipa_tensor_t* q_point, const ipa_tensor_t* k_point,
                          const ipa_tensor_t* values,
                          const ipa_tensor_t* direction_scale,
                          const ipa_tensor_t* distance_scale,
                          const ipa_tensor_t* output_weight, const ipa_tensor_t* output_bias,
                          const ipa_tensor_t* rotation, const ipa_tensor_t* translation,
                          const ipa_tensor_t* frame_mask, const ipa_tensor_t* pair_mask,
                          const ipa_tensor_t* g_output, const ipa_tensor_t* g_attention,
                          const ipa_tensor_t* g_vectors, const geo_grads_t* grads,
                          void* workspace, size_t workspace_bytes, void* stream,
                          int32_t* dev_err);

/* --------------------------------------------------------------------------
 * geo_attn_fwd without a workspace argument (no counterpart on the pages:
 * this is an interface convenience of this library, not part of the method).
 *
 * For callers that may not allocate device memory where they run this
 * operator -- e.g. an operator hook inside a host framework that provides no
 * scratch buffer and forbids cudaMalloc on that path, or a plain C program
 * linking this library without an allocator.  It allocates nothing: its
 * scratch is a fixed array of GEO_STATIC_SCRATCH_BYTES inside this library,
 * reserved on every GPU that loads the library until the process exits.
 *   - Same arguments, results and errors as geo_attn_fwd, minus the
 *     workspace; returns IPA_ERR_WORKSPACE when geo_attn_workspace_size(p)
 *     exceeds GEO_STATIC_SCRATCH_BYTES (e.g. B*H*N above roughly 64 K rows
 *     of 128 bytes for M = 4).
 *   - The first call on a device looks the array's device address up
 *     (cudaGetSymbolAddress); make that first call outside any stream
 *     capture.  The address is cached per device and context, and looked up
 *     again when the device's current context differs from the cached one
 *     (after cudaDeviceReset, for example).
 *   - All calls on a device share the one array and it keeps the previous
 *     call's contents: calls whose executions overlap on the GPU (other
 *     streams, other host threads) race on it and must be serialised by the
 *     caller.  Every byte a call reads from it is written earlier in the same
 *     call.
 * ------------------------------------------------------------------------ */
#define GEO_STATIC_SCRATCH_BYTES (8u * 1024u * 1024u)

IPA_API ipa_status_t geo_attn_fwd_static(const geo_params_t* p,
                                 const ipa_tensor_t* q_direction, const ipa_tensor_t* k_direction,
                                 const ipa_tensor_t* q_point, const ipa_tensor_t* k_point,
                                 const ipa_tensor_t* values,
                                 const ipa_tensor_t* direction_scale,
                                 const ipa_tensor_t* distance_scale,
                                 const ipa_tensor_t* output_weight, const ipa_tensor_t* output_bias,
                                 const ipa_tensor_t* rotation, const ipa_tensor_t* translation,
                                 const ipa_tensor_t* frame_mask, const ipa_tensor_t* pair_mask,
                                 const ipa_tensor_t* out_vectors, const ipa_tensor_t* out_output,
                                 const ipa_tensor_t* out_attention,
                                 void* stream, int32_t* dev_err);

/* --------------------------------------------------------------------------
 * Local nearest-neighbour distogram of residue positions (Flash Invariant
 * Point Attention, TL;DR: the pair representation is built from "a local
 * nearest-neighbor distogram").  The page fixes neither the neighbour count
 * nor the distance bins nor the map to pair factors, so the first two are
 * arguments here and the third is left to the caller (e.g. a projection of
 * the histogram with ipa_linear_fwd).  For batch b and valid residue i:
 *   idx[b,i,:]   the k valid residues j != i nearest to i (|x_j - x_i|),
 *                nearest first, equal distances in increasing j; -1 in
 *                slots beyond the number of valid other residues
 *   bins[b,i,:]  bin of each neighbour's distance: #{m : d >= edges[m]},
 *                in [0, n_edges]; -1 in empty slots
 *   hist[b,i,c]  number of neighbours in bin c (n_edges + 1 bins)
 * and all slots -1 / 0 for a masked residue.  Distances are compared as
 * float32 squared distances (dx*dx + dy*dy) + dz*dz against float32 squared
 * edges, so the integer results are those of float32 arithmetic.
 * Inputs: x [B, L, 3] IPA_DTYPE_F32 (C-alpha or frame origins, any strides),
 * mask [B, L] IPA_DTYPE_BOOL, edges: HOST array of n_edges strictly
 * increasing non-negative float32 values (validated on the host).
 * Outputs (contiguous): idx, bins [B, L, k] IPA_DTYPE_I32, hist [B, L,
 * n_edges + 1] IPA_DTYPE_F32.  Envelope: 1 <= k <= 32, 0 <= n_edges <= 63.
 * No workspace.
 * ------------------------------------------------------------------------ */
IPA_API ipa_status_t ipa_knn_distogram(int32_t B, int32_t L, int32_t k, int32_t n_edges,
                               const ipa_tensor_t* x, const ipa_tensor_t* mask,
                               const float* edges, const ipa_tensor_t* idx,
                               const ipa_tensor_t* bins, const ipa_tensor_t* hist, void* stream);

/* --------------------------------------------------------------------------
 * Distance-aware attention (MEET, §2.2 "distance-aware attention",
 * eq. (6)-(8)), run on the fused IPA core:
 *
 *   A_ij^h = rho_h * ( <q_i^h, k_j^h> - s_h^2 * ||x_i - x_j||^2 )
 *   o_i^h  = sum_j softmax_j(A_i.^h) * v_j^h   over keys with mask_i and mask_j
 *
 * rows with no allowed key are 0 (the passage defines the logits; the value
 * aggregation and the masking are this library's reading).  The distance is
 * folded into the augmented query/key columns like the IPA point term
 * (eq. (7)-(8)): each coordinate enters as a frame origin with identity
 * rotation, the pair term is zero.
 *
 * Inputs (element strides, any layout):
 *   q, k, v   [B, L, H, C] IPA_DTYPE_F32, C == 16 (the core's scalar width)
 *   x         [B, L, 3]    IPA_DTYPE_F32 coordinates
 *   rho, s    [H]          IPA_DTYPE_F32 attention and distance scales
 *   mask      [B, L]       IPA_DTYPE_BOOL
 * Output: out [B, L, H, C] IPA_DTYPE_F32, contiguous.
 * Workspace: meet_attn_workspace_size(p) bytes, 256-byte aligned, caller
 * owned; errors as for ipa_attn_fwd.  Supported: C == 16, H <= 128,
 * L <= 1048576.
 * ------------------------------------------------------------------------ */
typedef struct {
  int32_t B, L, H, C;
} meet_params_t;

IPA_API size_t meet_attn_workspace_size(const meet_params_t* p);

IPA_API ipa_status_t meet_attn_fwd(const meet_params_t* p,
                           const ipa_tensor_t* q, const ipa_tensor_t* k, const ipa_tensor_t* v,
                           const ipa_tensor_t* x, const ipa_tensor_t* rho, const ipa_tensor_t* s,
                           const ipa_tensor_t* mask, const ipa_tensor_t* out,
                           void* workspace, size_t workspace_bytes,
                           void* stream, int32_t* dev_err);

/* --------------------------------------------------------------------------
 * Residue frames from backbone atoms (Flash Invariant Point Attention,
 * Figure 1: the frame is centred on C_alpha and spanned by C_alpha -> C and
 * C_alpha -> N through Gram-Schmidt; this library's reading of the order and
 * handedness):
 *   e1 = (C - CA) / |C - CA|
 *   e2 = normalise((N - CA) - (e1 . (N - CA)) e1)
 *   e3 = e1 x e2,  rot = [e1 | e2 | e3] (columns),  trans = CA
 * so that rot maps local column vectors to global ones, as ipa_attn_fwd's
 * `rot` expects.
 * Inputs n, ca, c [B, L, 3] IPA_DTYPE_F32 (any strides); outputs rot
 * [B, L, 3, 3] and trans [B, L, 3] IPA_DTYPE_F32, contiguous.  No workspace.
 * Collinear N, CA, C give non-finite frames (outside the domain, not
 * checked).  Enqueued on `stream`; errors as for ipa_attn_fwd.
 * ------------------------------------------------------------------------ */
IPA_API ipa_status_t ipa_frames_from_backbone(int32_t B, int32_t L,
                                      const ipa_tensor_t* n, const ipa_tensor_t* ca,
                                      const ipa_tensor_t* c,
                                      const ipa_tensor_t* rot_out, const ipa_tensor_t* trans_out,
                                      void* stream);

/* --------------------------------------------------------------------------
 * Dense projection y = x W + b on the tensor cores, the building block of the
 * layer around the core (Flash Invariant Point Attention keeps the IPA layer's
 * query / key / value / point projections of the single representation and
 * its output projection; the factorised core sits between them).
 *   x [M, K] IPA_DTYPE_F32, any strides; W [K, N] IPA_DTYPE_F32, any strides;
 *   b [N] IPA_DTYPE_F32 contiguous, or NULL / data == NULL (no bias);
 *   y [M, N] IPA_DTYPE_F32 contiguous (written).
 * x and W are rounded to fp16 (into the workspace) and multiplied with fp32
 * accumulation; the result is fp32.  Workspace: ipa_linear_workspace_size
 * bytes, 256-byte aligned, caller-owned.  Envelope: 1 <= K <= 65536,
 * M, N >= 1.  Errors as for ipa_attn_fwd; dev_err (optional) receives a
 * device error code if a bounded wait expires.
 * ------------------------------------------------------------------------ */
IPA_API size_t ipa_linear_workspace_size(int32_t M, int32_t K, int32_t N);

IPA_API ipa_status_t ipa_linear_fwd(int32_t M, int32_t K, int32_t N, const ipa_tensor_t* x,
                            const ipa_tensor_t* w, const ipa_tensor_t* b, const ipa_tensor_t* y,
                            void* workspace, size_t workspace_bytes, void* stream, int32_t* dev_err);

/* --------------------------------------------------------------------------
 * The IPA layer around the factorised core (Flash Invariant Point Attention
 * keeps the IPA layer's projections; this library's reading of them):
 *   Y = s W_in + b_in, s the single representation [B, L, c_s];
 *   Y's columns, in order: q (H x C), k (H x C), v (H x C), q_pts (H x Pq x 3),
 *   k_pts (H x Pq x 3), v_pts (H x Pv x 3), head-major, innermost the
 *   channel (or the point, then xyz): width H (3 C + 3 (2 Pq + Pv));
 *   o = ipa_attn_fwd on those (strided views of Y, no copy) with the frames,
 *   z1, z2, w_bias, gamma and mask; F = C + 4 Pv + Cz features per head;
 *   out = flatten(o) W_out + b_out  [B, L, c_s].
 *   s      [B, L, c_s] IPA_DTYPE_F32, rows flattenable: stride(B) = L stride(L)
 *   w_in   [c_s, width] IPA_DTYPE_F32; b_in [width] contiguous or NULL
 *   w_out  [H F, c_s] IPA_DTYPE_F32;   b_out [c_s] contiguous or NULL
 *   rot .. mask as for ipa_attn_fwd
 *   out    [B, L, c_s] IPA_DTYPE_F32 contiguous
 *   core_out [B, L, H, F] IPA_DTYPE_F32 contiguous, or NULL (then held in the
 *          workspace)
 * Projections run in fp16 with fp32 accumulation (ipa_linear_fwd), the core
 * as ipa_attn_fwd.  Workspace: ipa_module_workspace_size bytes, 256-byte
 * aligned.  Errors as for ipa_attn_fwd.
 * ------------------------------------------------------------------------ */
typedef struct {
  ipa_params_t core;
  int32_t c_s;
} ipa_module_params_t;

IPA_API size_t ipa_module_workspace_size(const ipa_module_params_t* p);

IPA_API ipa_status_t ipa_module_fwd(const ipa_module_params_t* p, const ipa_tensor_t* s,
                            const ipa_tensor_t* rot, const ipa_tensor_t* trans,
                            const ipa_tensor_t* z1, const ipa_tensor_t* z2,
                            const ipa_tensor_t* w_bias, const ipa_tensor_t* gamma,
                            const ipa_tensor_t* mask, const ipa_tensor_t* w_in,
                            const ipa_tensor_t* b_in, const ipa_tensor_t* w_out,
                            const ipa_tensor_t* b_out, const ipa_tensor_t* out,
                            const ipa_tensor_t* core_out, void* workspace, size_t workspace_bytes,
                            void* stream, int32_t* dev_err);

/* Static description of a status code (never NULL). */
IPA_API const char* ipa_status_string(ipa_status_t s);

/* Translate a device error word written by the kernels into a status:
 * 0 -> IPA_OK, bounded-wait expiry -> IPA_ERR_TIMEOUT, a word with bit 16
 * set -> IPA_ERR_BOUNDS, else IPA_ERR_CUDA.
 *
 * Bounds-checked build (the library compiled with -DIPA_BOUNDS_CHECK; its
 * ipa_version() ends in "bounds-checked"): every kernel forms each pointer it
 * stores through to global memory from a span [index, index + n) checked
 * against the extent of the destination buffer (from the call's shapes).  A
 * span outside its buffer writes 0x10000 | (source file tag << 12) | source
 * line into dev_err (first error wins) and the stores go to a scratch area
 * inside the library instead.  ipa_frames_from_backbone and ipa_knn_distogram
 * have no error word: their spans are checked and redirected, not reported.
 * The product build has none of these checks. */
IPA_API ipa_status_t ipa_device_error_status(int32_t dev_err_value);

/* Library build identifier, e.g. "flashipa_b200 sm_100a". */
IPA_API const char* ipa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FLASHIPA_B200_H_ */
