/*
 * tpconv.h -- C ABI of the streaming edge-conditioned O(3) tensor-product convolution
 * for NVIDIA B200 (sm_100a).
 *
 * What it computes ("Sobek: Streaming Equivariant Tensor Product Convolutions",
 * arXiv 2607.18074, section 2): for every receiver node i,
 *
 *     m_i = sum_{j in N(i)} sum_{paths pi} sum_a  w_{ij,pi,a} T_{pi,a}(x_j, Y(r_hat_ij))   (eq. 11)
 *     w_{ij,pi,a} = sum_q phi_q(|r_ij|) A_{q,pi,a}                                          (eq. 12)
 *
 * with r_ij = pos[j] - pos[i] (eq. 8; j = source, i = receiver), Y the real spherical
 * harmonics of the edge direction, phi a radial basis, and T the Clebsch-Gordan
 * coupling of one input irrep block with one harmonic order into one output block
 * (selection rule eq. 5), fully connected over channels ("uvw", eq. 6) or
 * channelwise ("uvu", eq. 7).  It is evaluated in the receiver-factorised streaming
 * order of section 4 (eqs. 32-36): no per-edge weight, message or weight-adjoint
 * tensor is ever formed.  Backward returns eqs. 18-22 carried through to positions;
 * double backward returns eqs. 25, 27 and 30.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All floating-point tensors are float32, all indices int32, all device pointers
 *    16-byte aligned (else TPCONV_ERR_MISALIGNED).
 *  - Features use the ir_mul layout: a node row is the concatenation of its irrep
 *    blocks in the order of the irreps string; a block of C channels and order l
 *    holds (2l+1)*C floats stored [2l+1][C] (channels contiguous).  Component index
 *    k = m + l for the real harmonic order m = -l..l.
 *  - Real harmonics: z polar axis, no Condon-Shortley phase, sum_m Y_lm^2 = 2l+1
 *    (so Y_1 = sqrt(3) (y, z, x)).  Coupling c^pi = sqrt(2 l_out + 1) times the
 *    unit-norm real invariant tensor, first nonzero entry (row-major m_in, m_sh,
 *    m_out) positive.
 *  - Graph: receiver-sorted CSR.  Receiver i owns edges row_ptr[i] .. row_ptr[i+1]-1,
 *    src[e] is the source of edge e.  The source view (t_ptr, t_eid, t_dst) lists the
 *    same edges grouped by source, stable in edge id (tpconv_csr_transpose).
 *  - Paths are enumerated for each input block, for each harmonic order
 *    l_sh = 0..sh_lmax, for each output block, keeping every combination that
 *    satisfies eq. 5.  Weights W (the pages' A) are [K][N_w] row-major; path pi owns
 *    columns w_offset .. w_offset + w_count - 1 laid out [C_in][C_out] (uvw, index
 *    u*C_out + w) or [C_in] (uvu).
 *  - Gradient outputs are overwritten, never accumulated.  A NULL tangent is zero.
 *    A NULL gradient output is not computed.
 *  - Every compute call is asynchronous on `stream`, performs no allocation and no
 *    host synchronisation, and uses only the caller's workspace `ws`
 *    (tpconv_workspace_bytes).  Argument errors are reported before anything is
 *    launched; a failed launch returns TPCONV_ERR_CUDA.
 *  - Results are deterministic: no floating-point atomics; every reduction has a
 *    fixed order (Sobek, section 4: receiver and source CSR ownership).
 *  - tpconv_forward, tpconv_backward and tpconv_double_backward may be captured into
 *    a CUDA graph once the same plan has run each captured pass eagerly on the device
 *    (the first launch of a kernel sets its shared-memory attribute, which is not a
 *    stream operation).  Replays read the buffers' current contents.
 */
#ifndef TPCONV_H
#define TPCONV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;                         /* cudaStream_t is struct CUstream_st* */
typedef struct tpconv_plan* tpconv_plan_t;  /* opaque, owned by the library */

typedef enum {
  TPCONV_OK = 0,
  TPCONV_ERR_INVALID_ARG = 1,
  TPCONV_ERR_PARSE = 2,
  TPCONV_ERR_UNSUPPORTED = 3,
  TPCONV_ERR_WORKSPACE_TOO_SMALL = 4,
  TPCONV_ERR_MISALIGNED = 5,
  TPCONV_ERR_CUDA = 6,
  TPCONV_ERR_GRAPH_INVALID = 7
} tpconv_status;

typedef enum { TPCONV_UVW = 0, TPCONV_UVU = 1 } tpconv_mode;
typedef enum { TPCONV_RADIAL_BESSEL = 0, TPCONV_RADIAL_GAUSSIAN = 1 } tpconv_radial_kind;

/* Radial embedding phi(d) in R^K (the pages leave its form open):
 *   BESSEL:   phi_b = sqrt(2/r_cut) sin(b pi d / r_cut) / d * u(d / r_cut), b = 1..K
 *   GAUSSIAN: phi_b = exp(-(d - mu_b)^2 / (2 sigma^2)) * u(d / r_cut),
 *             mu_b = r_min + b (r_max - r_min)/(K-1), sigma = (r_max - r_min)/(K-1)
 *   u(t) = 1 - (p+1)(p+2)/2 t^p + p(p+2) t^(p+1) - p(p+1)/2 t^(p+2) for t < 1, else 0.
 * num_basis K in 1..16; poly_p >= 1 (6 in every shipped workload).               */
typedef struct {
  int32_t kind;       /* tpconv_radial_kind */
  int32_t num_basis;  /* K */
  float r_cut;
  float r_min;        /* GAUSSIAN only */
  float r_max;        /* GAUSSIAN only */
  int32_t poly_p;
} tpconv_radial_spec;

/* Pass bits for tpconv_workspace_bytes. */
#define TPCONV_PASS_FORWARD 1u
#define TPCONV_PASS_BACKWARD 2u
#define TPCONV_PASS_DOUBLE_BACKWARD 4u

/* Status code as a static string (never NULL). */
const char* tpconv_status_string(tpconv_status s);

/* Build a plan from irreps strings such as "64x0e+64x1o+64x2e" (orders l <= 3,
 * parity e/o) and the harmonic order sh_lmax (<= 3).  mode is tpconv_mode; uvu
 * requires C_out == C_in on every path (eq. 7), else TPCONV_ERR_INVALID_ARG.  The
 * plan owns its path and coupling tables (host memory only).  *out is set only on
 * success.  Errors: PARSE (bad string), UNSUPPORTED (l > 3, K > 16, too many paths),
 * INVALID_ARG (NULL pointers, bad radial spec, no valid path).                      */
tpconv_status tpconv_plan_create(tpconv_plan_t* out, const char* irreps_in, int32_t sh_lmax,
                                 const char* irreps_out, int32_t mode,
                                 const tpconv_radial_spec* radial);

/* Release a plan.  NULL is accepted.  Calls in flight that use it must have been
 * enqueued already (the plan is read on the host at enqueue time only).            */
tpconv_status tpconv_plan_destroy(tpconv_plan_t plan);

/* Sizes: number of paths, flattened input width C_x (eq. 4), output width, radial
 * size K and weight columns N_w (eq. 10).  Any output pointer may be NULL.         */
tpconv_status tpconv_plan_info(tpconv_plan_t plan, int64_t* num_paths, int64_t* dim_in,
                               int64_t* dim_out, int64_t* num_basis, int64_t* weight_cols);

/* Path descriptor number `index` (plan order) as 10 int32:
 * l_in, l_sh, l_out, block_in, block_out, C_in, C_out, w_offset, w_count, nnz.     */
tpconv_status tpconv_plan_path(tpconv_plan_t plan, int64_t index, int32_t out[10]);

/* Coupling tensor c^pi of path `index` as nnz triples (m_in, m_sh, m_out) in idx
 * [nnz*3] and values in val [nnz] (host memory, cap = capacity in entries).        */
tpconv_status tpconv_plan_path_coupling(tpconv_plan_t plan, int64_t index, int32_t* idx,
                                        double* val, int64_t cap);

/* Upper bound on the tensor-product scratch used per call (the pages cap it at 128 MiB,
 * which is the default): node states, split-K slices and the position-gradient staging
 * window.  Larger budgets mean fewer receiver ranges and staging windows; results do
 * not depend on it beyond the order of fp32 sums.  At least 4096 bytes.               */
tpconv_status tpconv_set_workspace_budget(tpconv_plan_t plan, size_t bytes);

/* Arithmetic of the channel contractions (the per-node products with the radial
 * parameters A, Sobek section 4, eqs. 34-36 and their mirrored source-side forms).
 *   TPCONV_MATH_FP32 (default): fp32 products from three TF32 tensor-core products
 *     per term (hi*hi + hi*lo + lo*hi); results match fp32 to about 1e-6 relative.
 *   TPCONV_MATH_TF32: one TF32 product per term (operands truncated to 10 mantissa
 *     bits); about 1e-3 relative error, faster contractions.
 *   TPCONV_MATH_BF16: both operands rounded to bf16 (8 mantissa bits), one bf16
 *     tensor-core product per term with fp32 accumulation; about 3e-3 relative error.
 * The streaming (edge) arithmetic is fp32 in every mode.  Any other value returns
 * TPCONV_ERR_UNSUPPORTED and leaves the plan unchanged.                             */
#define TPCONV_MATH_FP32 0
#define TPCONV_MATH_TF32 1
#define TPCONV_MATH_BF16 2
tpconv_status tpconv_plan_set_math(tpconv_plan_t plan, int32_t math);

/* Boundary layout of the node arrays x, out, grad_out, gg_x, grad_x and grad_grad_out
 * (Sobek's wrapper accepts both):
 *   TPCONV_LAYOUT_IR_MUL (default): each irrep block stored [2l+1][C], channels
 *     contiguous, as described at the top of this header;
 *   TPCONV_LAYOUT_MUL_IR: each block stored [C][2l+1] (components contiguous).
 * With MUL_IR the passes convert their node inputs to ir_mul in workspace buffers and
 * their node outputs back (one extra read and write of each node array); the workspace
 * grows accordingly (tpconv_workspace_bytes accounts for it) and results equal the
 * ir_mul results with the same permutation applied.  Edge arrays (Y, phi and their
 * adjoints), W and positions are unaffected.  Any other value: TPCONV_ERR_UNSUPPORTED. */
#define TPCONV_LAYOUT_IR_MUL 0
#define TPCONV_LAYOUT_MUL_IR 1
tpconv_status tpconv_plan_set_layout(tpconv_plan_t plan, int32_t layout);

/* Workspace bytes needed by the passes in pass_mask for a graph of N nodes and E
 * edges.  The result does not depend on E: the node states of a receiver (or source)
 * range, the split-K slices of the channel contractions and, in backward and double
 * backward, a staging window for the per-edge position gradients (an eighth of the
 * budget, at most 16 MiB; the edges are staged window by window) all fit the scratch
 * budget (tpconv_set_workspace_budget), plus 8 bytes per node (receiver order; cursors
 * into the source view for the position sums).                                         */
tpconv_status tpconv_workspace_bytes(tpconv_plan_t plan, int64_t N, int64_t E,
                                     uint32_t pass_mask, size_t* bytes);

/* Source view of a receiver-sorted CSR: t_ptr[N+1], t_eid[E] (edge ids grouped by
 * source, increasing inside each group) and t_dst[E] (receiver of t_eid[k]).
 * Bit-exact and deterministic.  Needs tpconv_csr_transpose_workspace_bytes of ws. */
tpconv_status tpconv_csr_transpose_workspace_bytes(int64_t N, int64_t E, size_t* bytes);
tpconv_status tpconv_csr_transpose(int64_t N, int64_t E, const int32_t* row_ptr,
                                   const int32_t* src, int32_t* t_ptr, int32_t* t_eid,
                                   int32_t* t_dst, void* ws, size_t ws_bytes,
                                   struct CUstream_st* stream);

/* Debug check of a receiver-sorted CSR on the device: row_ptr[0] == 0, non-decreasing,
 * row_ptr[N] == E, 0 <= src[e] < N.  Writes 0 (valid) or a nonzero code (1: row_ptr
 * bounds, 2: not monotone, 3: src out of range) to the device int *d_err.  Never traps. */
tpconv_status tpconv_validate_graph(int64_t N, int64_t E, const int32_t* row_ptr,
                                    const int32_t* src, int32_t* d_err,
                                    struct CUstream_st* stream);

/* Forward, eq. 11 with eq. 12 (Sobek section 2), evaluated as eqs. 32-35.
 * x [N][dim_in], pos [N][3], row_ptr [N+1], src [E], W [K][N_w] -> out [N][dim_out]. */
tpconv_status tpconv_forward(tpconv_plan_t plan, int64_t N, int64_t E, const float* x,
                             const float* pos, const int32_t* row_ptr, const int32_t* src,
                             const float* W, float* out, void* ws, size_t ws_bytes,
                             struct CUstream_st* stream);

/* Backward: given grad_out = dL/dout [N][dim_out], returns grad_x [N][dim_in]
 * (eq. 21), grad_pos [N][3] (eqs. 20 and 22 through Y(r_hat) and phi(|r|)) and
 * grad_W [K][N_w] (eq. 19).  Each output is optional (NULL = skip).  The source view
 * (t_ptr, t_eid, t_dst) is required when grad_x, grad_W or grad_pos is requested.   */
tpconv_status tpconv_backward(tpconv_plan_t plan, int64_t N, int64_t E, const float* x,
                              const float* pos, const int32_t* row_ptr, const int32_t* src,
                              const int32_t* t_ptr, const int32_t* t_eid,
                              const int32_t* t_dst, const float* W, const float* grad_out,
                              float* grad_x, float* grad_pos, float* grad_W, void* ws,
                              size_t ws_bytes, struct CUstream_st* stream);

/* Double backward.  With (x_bar, pos_bar, W_bar) = backward(x, pos, W, grad_out) and
 *   Lambda = <gg_x, x_bar> + <gg_pos, pos_bar> + <gg_W, W_bar>,
 * returns grad_x = dLambda/dx (eq. 30), grad_W = dLambda/dW (eq. 27) and
 * grad_grad_out = dLambda/dgrad_out (eq. 25, the forward tangent) and
 * grad_pos = dLambda/dpos [N][3].  This is what an autograd engine requests after a
 * first backward taken with create_graph.  The pages stop at the first-order terms;
 * grad_pos is the tangent of the backward's per-edge position gradient
 * g_e = (dphi/dr)^T phi_bar + (dY/dr)^T Y_bar along (gg_x, gg_pos, gg_W), which needs
 * the second derivatives of Y(r_hat) and phi(|r|), scattered like g_e.  Tangents gg_*
 * may be NULL (zero); outputs may be NULL (skipped).  The source view is required for
 * grad_x (t_ptr, t_dst) and grad_pos (t_ptr, t_eid).                                 */
tpconv_status tpconv_double_backward(tpconv_plan_t plan, int64_t N, int64_t E, const float* x,
                                     const float* pos, const int32_t* row_ptr,
                                     const int32_t* src, const int32_t* t_ptr,
                                     const int32_t* t_eid, const int32_t* t_dst,
                                     const float* W, const float* grad_out, const float* gg_x,
                                     const float* gg_pos, const float* gg_W, float* grad_x,
                                     float* grad_W, float* grad_grad_out, float* grad_pos,
                                     void* ws, size_t ws_bytes, struct CUstream_st* stream);

/* Sobek's own interface (section 3 and the wrapper it describes): the edge embedding is
 * given per edge instead of computed from positions.  Y [E][(lmax+1)^2] holds the real
 * harmonics (or any per-edge vector in their place, same component order as the plan's
 * sh_lmax) and phi [E][K] any invariant edge embedding (e.g. a learned function of
 * |r_e|), both fp32 in receiver-CSR edge order.  uvw and uvu plans.  Workspace: as
 * tpconv_forward / tpconv_backward.
 *   forward: out as tpconv_forward (eqs. 11-13 with the given phi, Y).
 *   backward: grad_x (eq. 21), grad_W (eq. 19) and the edge-owned adjoints
 *     grad_phi [E][K] (eq. 20) and grad_Y [E][(lmax+1)^2] (eq. 22); each nullable;
 *     t_ptr/t_eid/t_dst (tpconv_csr_transpose) are needed for grad_x and grad_W.      */
tpconv_status tpconv_forward_embedded(tpconv_plan_t plan, int64_t N, int64_t E, const float* x,
                                      const float* Y, const float* phi, const int32_t* row_ptr,
                                      const int32_t* src, const float* W, float* out, void* ws,
                                      size_t ws_bytes, struct CUstream_st* stream);
tpconv_status tpconv_backward_embedded(tpconv_plan_t plan, int64_t N, int64_t E, const float* x,
                                       const float* Y, const float* phi, const int32_t* row_ptr,
                                       const int32_t* src, const int32_t* t_ptr, const int32_t* t_eid,
                                       const int32_t* t_dst, const float* W, const float* grad_out,
                                       float* grad_x, float* grad_W, float* grad_phi, float* grad_Y,
                                       void* ws, size_t ws_bytes, struct CUstream_st* stream);

/* Forward without any allocation by the caller or the library, for callers that
 * cannot obtain device memory themselves: for example a plug-in whose host application
 * owns every device allocation, or code that must not call cudaMalloc because that
 * call can synchronise the device in the middle of latency-critical work.
 *
 * Same inputs, outputs and result as tpconv_forward, but the scratch lives in a fixed
 * array of TPCONV_STATIC_SCRATCH_BYTES compiled into the library, which every GPU that
 * loads the library keeps until the process exits.  The paper has no counterpart to
 * this entry point.
 *  - The first call on a device looks up that array's device address (once per device,
 *    with the device current); make that first call before any stream capture.  The
 *    address is kept for the life of the process, so do not use the library across a
 *    cudaDeviceReset.
 *  - Plans whose per-receiver state does not fit the array even one receiver at a time
 *    are rejected with TPCONV_ERR_WORKSPACE_TOO_SMALL; larger graphs are processed in
 *    receiver ranges that fit.
 *  - All calls share the one array and every call overwrites what it reads, so nothing
 *    needs clearing between calls; calls whose executions overlap on the GPU (several
 *    streams, or several host threads) race on the array and must be serialised by the
 *    caller.                                                                            */
#define TPCONV_STATIC_SCRATCH_BYTES (32u << 20)
tpconv_status tpconv_forward_no_alloc(tpconv_plan_t plan, int64_t N, int64_t E, const float* x,
                                      const float* pos, const int32_t* row_ptr,
                                      const int32_t* src, const float* W, float* out,
                                      struct CUstream_st* stream);

/* Profiling (off by default; host-side bookkeeping only).  While enabled, every kernel
 * the library launches is bracketed by a pair of CUDA events on its stream and
 * attributed to a category (tpconv_profile_category_name).  tpconv_profile_begin
 * clears the records (capacity: max_records launches; later launches are counted but
 * not timed).  tpconv_profile_end waits for the recorded events, writes per-category
 * total device milliseconds and launch counts into ms[n] / launches[n] (either may be
 * NULL; n <= TPCONV_PROF_CATEGORIES) and disables recording.  Not for use during
 * stream capture.                                                                     */
#define TPCONV_PROF_CATEGORIES 13

/* Reads and clears the library's device error word (0 = fine; nonzero = a bounded wait
 * inside a tensor-core kernel gave up, so results of that launch are invalid).
 * Synchronises the current device; for tests and debugging.                        */
tpconv_status tpconv_device_error(int32_t* out);
tpconv_status tpconv_profile_begin(int32_t max_records);
tpconv_status tpconv_profile_end(double* ms, int64_t* launches, int32_t n);
const char* tpconv_profile_category_name(int32_t category);

#ifdef __cplusplus
}
#endif
#endif /* TPCONV_H */
