/*
 * omnimoe.h -- C ABI of the routed atomic-expert branch of an OmniMoE layer,
 * B200 (sm_100a) implementation.
 *
 * The layer (sources are web pages about OmniMoE, cited by title/section):
 *   [NL 2.1]  "OmniMoE: An Efficient MoE by Orchestrating Atomic Experts at
 *             Scale" (gist.science, Dutch), Technisch Overzicht section 2.1:
 *             atomic expert i is a vector pair (w_in, w_out) computing
 *             E_i(x) = sigma(x w_in^T) w_out; all N experts are the rows of
 *             two global matrices W, V (N x d).
 *   [NL 2.2]  same page, section 2.2: the Cartesian Product Router (row and
 *             column logits over an Nr x Nc grid of experts) and
 *             Expert-Centric Scheduling (task collection, grouping and
 *             sorting, grouped execution).
 *   [MS router] OmniMoE explainer (omnimoeexpl, manus.space), Cartesian
 *             product router section: S_ij = pr[i] + pc[j] in log space,
 *             no N-wide score vector.
 *   [MS sched]  same page, Expert-Centric Scheduling steps and the traffic
 *             model D = 2d*L*K (token-centric) vs 2d*|E_active|.
 *   [MS expert] same page, Atomic Expert section: the expert's activation is
 *             named as SwiGLU.
 *
 * Conventions for every call
 *   - All pointers are DEVICE pointers owned by the caller (except `dims`,
 *     `bytes` and the returned strings, which are host memory).  The library
 *     allocates no memory and keeps no state between calls; scratch space is
 *     the caller's workspace `ws` of `ws_bytes` bytes (size from
 *     omni_workspace_size, 256-byte aligned pointer).
 *   - Calls are asynchronous on `stream` (a cudaStream_t passed as void*;
 *     NULL = the legacy default stream).  Nothing synchronises the host;
 *     data-dependent sizes (number of active experts, of groups) stay on the
 *     device in `counts`.
 *   - Row-major layouts.  x [L x d], W, V [N x d], y [L x d] in the storage
 *     type `dims->dtype` (OMNI_F32: float, OMNI_BF16: bfloat16).  The router
 *     keys Wr [Nr x d] and Wc [Nc x d] hold one d-vector per grid row/column
 *     (the d x Nr projection of the pages, stored transposed), so row logit i
 *     of token t is x[t] . Wr[i].  Optional biases are float [Nr], [Nc].
 *     Expert id of grid cell (i, j) is e = i*Nc + j.
 *   - Pointers to x, Wr, Wc, W, V, y and the logits must be 16-byte aligned,
 *     all others 4-byte aligned; `ws` 256-byte aligned.
 *   - Return value: OMNI_OK when the work was enqueued; an error code when
 *     the host-side checks failed (nothing was enqueued) or a CUDA launch
 *     failed.  No exception or exit crosses the ABI.
 *   - counts (int32[4], device): [0] number of active experts, [1] number of
 *     groups (both written by the scheduling step), [2] device status bits,
 *     OR-ed by kernels and never cleared by the library (the caller zeroes
 *     it; see OMNI_DEV_*), [3] reserved.
 */
#ifndef OMNIMOE_H
#define OMNIMOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define OMNI_ABI_VERSION 1

/* host-side status codes (return values) */
#define OMNI_OK 0
#define OMNI_ERR_INVALID_ARG 1  /* null/misaligned pointer, inconsistent sizes */
#define OMNI_ERR_UNSUPPORTED 2  /* valid but outside this build's limits */
#define OMNI_ERR_WORKSPACE 3    /* ws too small or misaligned */
#define OMNI_ERR_CUDA 4         /* a CUDA runtime/driver call failed */

/* device status bits, OR-ed into counts[2] */
#define OMNI_DEV_TIMEOUT 1      /* a bounded device wait gave up (kernel returned early) */
#define OMNI_DEV_BAD_INDEX 2    /* an expert id outside [0, N) was read and ignored */

/* storage types */
#define OMNI_F32 0
#define OMNI_BF16 1

/* dims.flags bits */
#define OMNI_FLAG_ROUTER_SIMT 1 /* diagnostic: router logits on CUDA cores for bf16 too */
#define OMNI_FLAG_STAGED_SMALL 2 /* diagnostic: omni_moe_forward of a batch whose rows
                                    fit in L2 runs the scheduled order (the kernels of
                                    omni_schedule and omni_expert_forward, or the window
                                    order of the sweeps) instead of its two-kernel
                                    routing-order tail */
#define OMNI_FLAG_DENSE_TENSOR_CORES 4 /* grouped execution of bf16 batches without
                                          column sweeps: the activations of dense groups
                                          (>= 384 tasks per 128-token tile of a group's
                                          B <= 128 experts) are formed on the tensor cores;
                                          counts[3] receives how many groups were */

/* Limits of this build (host checks return OMNI_ERR_UNSUPPORTED beyond them). */
#define OMNI_MAX_AXIS 4096      /* Nr, Nc */
#define OMNI_MAX_TOPK 256       /* k, K */

/* Host checks of omni_dims, made by every call that takes dims.
 * A field outside its range returns OMNI_ERR_INVALID_ARG:
 *   L < 0; d, Nr, Nc, k, K or B < 1; k > min(Nr, Nc); K > k*k;
 *   an unknown dtype or flag.
 * A valid field beyond this build's limits returns OMNI_ERR_UNSUPPORTED:
 *   Nr or Nc > OMNI_MAX_AXIS; k or K > OMNI_MAX_TOPK; N >= 2^31;
 *   L*K >= 2^30; d not a multiple of 8, or d > 65536.
 * When both apply, OMNI_ERR_INVALID_ARG is returned.
 * The calls that select experts (omni_route, omni_route_select and
 * omni_moe_forward) also return OMNI_ERR_UNSUPPORTED for K > k: the top-K of the k x k
 * candidate pairs is the top-K over all N joint scores only when k >= K
 * (a grid row outside the per-axis top-k is beaten by at least k others, so
 * none of its pairs can reach the top K).  The other calls, and
 * omni_workspace_size, do not use k and take any K <= k*k. */

typedef struct omni_dims {
  int64_t L;     /* tokens in the batch (>= 0; L*K < 2^30 tasks) */
  int64_t d;     /* model width (a multiple of 8, at most 65536) */
  int64_t Nr;    /* grid rows */
  int64_t Nc;    /* grid columns; N = Nr*Nc atomic experts (< 2^31) */
  int64_t k;     /* per-axis top-k, 1 <= k <= min(Nr, Nc) */
  int64_t K;     /* experts per token, 1 <= K <= k*k; K <= k where experts are selected */
  int64_t B;     /* active experts per scheduling group, >= 1 */
  int32_t dtype; /* OMNI_F32 or OMNI_BF16 */
  int32_t flags; /* OMNI_FLAG_* */
} omni_dims;

/* workspace kinds for omni_workspace_size */
#define OMNI_WS_ROUTE 0
#define OMNI_WS_SCHEDULE 1
#define OMNI_WS_EXPERT 2
#define OMNI_WS_FUSED 3
#define OMNI_WS_TOKEN 4
#define OMNI_WS_SELECT 5
#define OMNI_WS_BACKWARD 6

/* Bytes of workspace the call `which` needs for `dims` (0 is possible). */
int omni_workspace_size(const omni_dims* dims, int which, size_t* bytes);

/*
 * Cartesian Product Router [NL 2.2], [MS router].
 * For every token t: row logits z_r = x[t] Wr^T + bias_r, column logits
 * z_c = x[t] Wc^T + bias_c (fp32 accumulation); per-axis log-softmax
 * lr, lc; top-k rows R and top-k columns C (value desc, index asc); joint
 * scores S = lr[i] + lc[j] over R x C only; the K best by (S desc, e asc).
 * Outputs, K per token in that order:
 *   idx   int32 [L x K]  expert ids e = i*Nc + j
 *   gate  float [L x K]  softmax of the K selected joint scores
 *   score float [L x K]  the joint log-probabilities S (nullable)
 * bias_r / bias_c may be NULL (no bias).
 */
int omni_route(const omni_dims* dims, const void* x, const void* Wr, const void* Wc,
               const float* bias_r, const float* bias_c, int32_t* idx, float* gate,
               float* score, int32_t* counts, void* ws, size_t ws_bytes, void* stream);

/*
 * The projection half of omni_route [NL 2.2]: logits float [L x (Nr + Nc)],
 * row t = (x[t] Wr^T, x[t] Wc^T), fp32 accumulation, no bias.  bf16 storage
 * runs on the tensor cores (tcgen05), fp32 storage on CUDA cores.  Small
 * batches split the reduction over d into partial sums that are added in a
 * fixed order (the result does not depend on timing); ws needs the
 * OMNI_WS_ROUTE size for these dims.
 */
int omni_router_logits(const omni_dims* dims, const void* x, const void* Wr, const void* Wc,
                       float* logits, int32_t* counts, void* ws, size_t ws_bytes, void* stream);

/*
 * The selection half of omni_route, from axis logits the caller computed:
 * logits float [L x (Nr + Nc)] holds z_r then z_c of each token (biases are
 * added here when given).  Same outputs as omni_route.
 */
int omni_route_select(const omni_dims* dims, const float* logits, const float* bias_r,
                      const float* bias_c, int32_t* idx, float* gate, float* score,
                      int32_t* counts, void* ws, size_t ws_bytes, void* stream);

/*
 * Expert-Centric Scheduling [NL 2.2], [MS sched].
 * Tasks are the M = L*K triples (t, idx[t,k], gate[t,k]).  U = the sorted
 * unique active expert ids; the group of expert e is (rank of e in U) / B;
 * tasks are sorted by (group, token, expert).  Outputs:
 *   task_token, task_expert int32 [M], task_gate float [M]  sorted tasks
 *   uniq      int32 [min(N, M)]        U (first counts[0] entries valid)
 *   group_off int32 [G_max + 1]        group g = tasks [group_off[g], group_off[g+1]);
 *                                      G_max = ceil(min(N, M) / B); first
 *                                      counts[1] + 1 entries valid
 *   counts    [0] = |U|, [1] = ceil(|U| / B)
 * An id outside [0, N) sets OMNI_DEV_BAD_INDEX and is treated as expert 0.
 */
int omni_schedule(const omni_dims* dims, const int32_t* idx, const float* gate,
                  int32_t* task_token, int32_t* task_expert, float* task_gate, int32_t* uniq,
                  int32_t* group_off, int32_t* counts, void* ws, size_t ws_bytes, void* stream);

/*
 * Grouped (expert-centric) execution [NL 2.1], [NL 2.2], [MS sched]: group
 * by group, every task (t, e, g) adds g * SiLU(x[t] . W[e]) * V[e] to y[t]
 * (sigma = scalar SiLU).  Inputs are omni_schedule's outputs (counts read on
 * the device).  y [L x d] is overwritten (tokens without tasks get 0);
 * accumulation is fp32, the bf16 result rounded to nearest even.
 */
int omni_expert_forward(const omni_dims* dims, const void* x, const void* W, const void* V,
                        const int32_t* task_token, const int32_t* task_expert,
                        const float* task_gate, const int32_t* uniq, const int32_t* group_off,
                        int32_t* counts, void* y, void* ws, size_t ws_bytes, void* stream);

/*
 * omni_expert_forward for callers that cannot allocate device memory when the
 * layer runs: code running while a CUDA graph is being captured, runtimes that
 * plan every device buffer ahead of time, plugin hosts that own all device
 * memory and pass an operator only its inputs and outputs.  The pages have no
 * counterpart of this call; it is a packaging of the same computation.
 * Arguments and results are those of omni_expert_forward, without ws.  The
 * fp32 accumulator it needs lives in a fixed device array inside the library
 * (16 MiB, held by every GPU that loads the library until the process exits),
 * so L*d must not exceed 4194304 (OMNI_ERR_UNSUPPORTED otherwise).  The array
 * is shared by every call and zeroed by each call before use: calls that can
 * overlap on the GPU (different streams, or several host threads) race on it
 * and must be serialised by the caller.  The array used is the one on the
 * current device, which must be the device of `stream` and of every pointer.
 * The first call on a device looks up the array's device address and keeps
 * it for the life of the process (it is not looked up again after a
 * cudaDeviceReset); make that first call before any stream capture.
 * Allocates nothing.
 */
int omni_expert_forward_noalloc(const omni_dims* dims, const void* x, const void* W,
                                const void* V, const int32_t* task_token,
                                const int32_t* task_expert, const float* task_gate,
                                const int32_t* uniq, const int32_t* group_off, int32_t* counts,
                                void* y, void* stream);

/*
 * The whole routed branch on one stream, intermediates in ws: omni_route,
 * then scheduling, then grouped execution.  idx_out / gate_out (nullable,
 * [L x K]) receive the routing decisions; counts[0], counts[1] are written as
 * by omni_schedule; y as in omni_expert_forward.
 * The execution order depends on the batch's shape (never on its data):
 *  - A batch whose rows fit in L2 runs as two kernels straight from the
 *    routing.  That means at most 64 MiB of the W and V rows it can touch
 *    (min(N, L*K) of each), or at most 1 GiB of rows even if no row were
 *    reused (L*K of each); it also needs N <= 2^20, L <= 65535 and a row
 *    width of 256, 512, 1024 or 2048 bf16 / 128 .. 1024 fp32 elements.
 *    The first kernel computes every task's activation
 *    gate * SiLU(x[t] . W[e]) in routing order, and counts |U| and the
 *    groups from a bitmap of the active ids.  The second forms
 *    y[t] = sum of activation * V[e] over the token's tasks and writes it
 *    once.  The rows stay in L2, so each leaves HBM about once without
 *    sorting the tasks by expert.  No schedule arrays are written
 *    (counts[0], counts[1] are).  OMNI_FLAG_STAGED_SMALL turns this path off.
 *  - Other batches run omni_schedule's order.  If their fp32 accumulator is
 *    executed in column-slice sweeps (L*d*4 above about 40 MiB), they go
 *    from the routing straight to the executor's order: the same groups, in
 *    windows of consecutive groups, each window's tasks ordered by token.
 *    The (group, token, expert) order itself is not formed.
 * Every task is executed once, so y differs from the staged calls only in
 * the order of its fp32 additions.
 */
int omni_moe_forward(const omni_dims* dims, const void* x, const void* Wr, const void* Wc,
                     const float* bias_r, const float* bias_c, const void* W, const void* V,
                     void* y, int32_t* idx_out, float* gate_out, int32_t* counts, void* ws,
                     size_t ws_bytes, void* stream);

/*
 * The shared dense MLP branch [NL 2.1] (an always-on dense MLP beside the
 * routed experts; the pages give neither its width nor its activation, and
 * this library takes one hidden layer of F units with the experts' scalar
 * SiLU):  y (+)= SiLU(x W1^T) W2^T.
 *   W1 [F x d], W2 [d x F]: bf16, row-major, 16-byte aligned.
 *   y  [L x d] bf16: overwritten (accumulate == 0) or added to (accumulate
 *      != 0: y = bf16(y + MLP(x)), one rounding of the sum).
 * Both products run on the tensor cores; the hidden activations are stored
 * in bf16 in ws (omni_mlp_workspace_size with with_routed = 0).
 * F < 1 returns OMNI_ERR_INVALID_ARG; F not a multiple of 8, F > 65536 or
 * fp32 storage return OMNI_ERR_UNSUPPORTED.  counts (nullable) receives
 * device status bits in counts[2].
 */
int omni_shared_mlp(const omni_dims* dims, int64_t F, const void* x, const void* W1,
                    const void* W2, void* y, int accumulate, int32_t* counts, void* ws,
                    size_t ws_bytes, void* stream);

/*
 * The whole OmniMoE layer output of [NL 2.1], y = routed(x) + MLP(x): the
 * routed branch as omni_moe_forward (same arguments and outputs), then the
 * shared MLP of omni_shared_mlp added into y on the same stream.  The routed
 * part is rounded to bf16 in y before the MLP's sum is added and rounded
 * again.  ws: omni_mlp_workspace_size with with_routed = 1.
 */
int omni_moe_mlp_forward(const omni_dims* dims, int64_t F, const void* x, const void* Wr,
                         const void* Wc, const float* bias_r, const float* bias_c, const void* W,
                         const void* V, const void* W1, const void* W2, void* y,
                         int32_t* idx_out, float* gate_out, int32_t* counts, void* ws,
                         size_t ws_bytes, void* stream);

/* Bytes of workspace of omni_shared_mlp (with_routed == 0) or of
 * omni_moe_mlp_forward (with_routed != 0) for these dims and width F; the
 * same dims and F checks as those calls. */
int omni_mlp_workspace_size(const omni_dims* dims, int64_t F, int with_routed, size_t* bytes);

/*
 * Token-centric execution, the order Expert-Centric Scheduling replaces
 * [NL 2.2], [MS sched]: every token gathers the rows of its own K experts,
 * y[t] = sum_k gate[t,k] * SiLU(x[t] . W[idx[t,k]]) * V[idx[t,k]].
 * Kept as the in-library ablation.  idx/gate as produced by omni_route.
 */
int omni_token_centric_forward(const omni_dims* dims, const void* x, const void* W,
                               const void* V, const int32_t* idx, const float* gate, void* y,
                               int32_t* counts, void* ws, size_t ws_bytes, void* stream);

/*
 * Gated atomic experts (SwiGLU, named by [MS expert]; the pages give only the
 * pair (w_in, w_out), and the gated form taken here adds a third global
 * matrix U [N x d], row e the gate vector of expert e):
 *   h = SiLU(x[t] . W[e]) * (x[t] . U[e]),  y[t] = sum gate * h * V[e].
 * Each of the three calls below is its plain counterpart (same arguments,
 * workspace, outputs, orders and error codes) with U added: U is a DEVICE
 * pointer, the dtype of x, row-major [N x d], 16-byte aligned, checked like
 * W and V (OMNI_ERR_INVALID_ARG if NULL or misaligned in a non-empty
 * batch).  Expert-centric order
 * loads each active expert's three rows once; the tensor-core activations of
 * dense groups (OMNI_FLAG_DENSE_TENSOR_CORES) are not used for gated experts.
 */
int omni_moe_forward_glu(const omni_dims* dims, const void* x, const void* Wr, const void* Wc,
                         const float* bias_r, const float* bias_c, const void* W, const void* U,
                         const void* V, void* y, int32_t* idx_out, float* gate_out,
                         int32_t* counts, void* ws, size_t ws_bytes, void* stream);
int omni_expert_forward_glu(const omni_dims* dims, const void* x, const void* W, const void* U,
                            const void* V, const int32_t* task_token, const int32_t* task_expert,
                            const float* task_gate, const int32_t* uniq, const int32_t* group_off,
                            int32_t* counts, void* y, void* ws, size_t ws_bytes, void* stream);
int omni_token_centric_forward_glu(const omni_dims* dims, const void* x, const void* W,
                                   const void* U, const void* V, const int32_t* idx,
                                   const float* gate, void* y, int32_t* counts, void* ws,
                                   size_t ws_bytes, void* stream);

/*
 * Expert-sharded forward, one call per process (GPU) of a group that splits
 * the N experts by contiguous id ranges.  The pages describe no distribution;
 * this follows the natural split of the expert-centric order: routing and
 * scheduling are replicated (Wr, Wc are small), each process executes only
 * the tasks whose expert lies in its ids [e_lo, e_hi), and the partial
 * outputs are summed across processes by the caller (one all-reduce).
 *   W, V (and U, nullable: gated experts as in omni_moe_forward_glu): the
 *      shard's rows only, [(e_hi - e_lo) x d], id e in row e - e_lo.
 *   y_part [L x d] fp32, overwritten with this shard's partial sum
 *      sum over the tasks (t, e, g) with e in [e_lo, e_hi) of g * h * V[e]
 *      (tokens without such a task get 0).  The sum over a partition of
 *      [0, N) of the y_part is y of omni_moe_forward up to the order of fp32
 *      additions; omni_cast_output rounds it to the storage type.
 *   idx_out / gate_out (nullable): the whole batch's routing, as
 *      omni_moe_forward (every process computes the same).
 *   counts[0], counts[1]: the number of active ids in [e_lo, e_hi) and
 *      their group count ceil(counts[0] / B); counts[2] status bits.
 *   ws: omni_workspace_size(dims, OMNI_WS_FUSED).
 * dims describe the whole layer (N = Nr * Nc ids); 0 <= e_lo < e_hi <= N
 * else OMNI_ERR_INVALID_ARG; the other checks as omni_moe_forward.  The
 * tensor-core activations of dense groups are not used.
 */
int omni_moe_forward_shard(const omni_dims* dims, int64_t e_lo, int64_t e_hi, const void* x,
                           const void* Wr, const void* Wc, const float* bias_r,
                           const float* bias_c, const void* W, const void* U, const void* V,
                           float* y_part, int32_t* idx_out, float* gate_out, int32_t* counts,
                           void* ws, size_t ws_bytes, void* stream);

/*
 * omni_moe_forward_shard from a routing computed elsewhere: idx, gate [L x K]
 * (as omni_route writes them, for all L tokens) are read, not computed, so
 * that the processes of a group can each route a share of the tokens and
 * exchange the routing instead of every process routing the whole batch.
 * The other arguments and the results are those of omni_moe_forward_shard;
 * the dims checks are those of omni_schedule (k is not used).  Ids outside
 * [0, N) set OMNI_DEV_BAD_INDEX in counts[2].
 */
int omni_moe_forward_shard_routed(const omni_dims* dims, int64_t e_lo, int64_t e_hi,
                                  const void* x, const void* W, const void* U, const void* V,
                                  const int32_t* idx, const float* gate, float* y_part,
                                  int32_t* counts, void* ws, size_t ws_bytes, void* stream);

/*
 * y [L x d] in the storage type of dims <- src [L x d] fp32 (bf16: rounded
 * to nearest even; fp32: copied unless src == y).  The last step of a
 * sharded forward, after the partial sums are added.  src == y with bf16
 * storage is OMNI_ERR_INVALID_ARG.
 */
int omni_cast_output(const omni_dims* dims, const float* src, void* y, void* stream);

/*
 * Backward of the routed branch: the gradients of the loss sum(dy * y) with
 * the forward's routing fixed (the pages train the model [NL 4]; this is the
 * forward differentiated by the chain rule).  Per task (t, k), e = idx[t,k],
 * a = x[t] . W[e], h = SiLU(a), s = dy[t] . V[e]:
 *   dV[e] += gate h dy[t];  dW[e] += da x[t];  dx[t] += da W[e],
 *   with da = gate s SiLU'(a);
 * through gate = softmax of the selected joint scores S_k = lr[i_k] + lc[j_k]
 * and the per-axis log-softmax: dS_k = gate_k (h_k s_k - sum_q gate_q h_q s_q)
 * added to row logit i_k and column logit j_k; then
 *   dx += dZ [Wr; Wc],  [dWr; dWc] += dZ^T x,  dbias += column sums of dZ.
 * The selection of the experts is piecewise constant: no gradient flows
 * through it.
 *   x, Wr, Wc, W, V: the forward's inputs; idx, gate: its routing outputs
 *     ([L x K], as omni_moe_forward's idx_out / gate_out); dy [L x d] in the
 *     storage type.
 *   dx [L x d] fp32: overwritten.
 *   dW, dV [N x d], dWr [Nr x d], dWc [Nc x d], dbias_r [Nr], dbias_c [Nc]
 *     (the two biases nullable) fp32: added to when accumulate != 0, so that
 *     gradients accumulate across calls; overwritten when accumulate == 0
 *     (without reading them: the first micro-batch).  Either way the rows
 *     of dW and dV of experts no token chose are not touched.
 *   counts[0], counts[1]: the active experts; counts[2]: status bits.
 *   ws: omni_workspace_size(dims, OMNI_WS_BACKWARD).
 * All arrays 16-byte aligned.  Router gradients go through tensor-core
 * products of bf16 operands (dZ rounded to bf16, fp32 accumulation); the
 * experts' gradients are fp32 throughout.  bf16 storage only (fp32 storage
 * returns OMNI_ERR_UNSUPPORTED); the other checks as omni_expert_forward.
 */
int omni_moe_backward(const omni_dims* dims, const void* x, const void* Wr, const void* Wc,
                      const void* W, const void* V, const int32_t* idx, const float* gate,
                      const void* dy, float* dx, float* dW, float* dV, float* dWr, float* dWc,
                      float* dbias_r, float* dbias_c, int accumulate, int32_t* counts, void* ws,
                      size_t ws_bytes, void* stream);

/* Static description of a status code (never NULL). */
const char* omni_status_string(int status);

/* Name of the CUDA error behind the last OMNI_ERR_CUDA returned on this host
 * thread ("cudaSuccess" if none); a static string. */
const char* omni_last_cuda_error_name(void);

/* OMNI_ABI_VERSION of the loaded library. */
int omni_abi_version(void);

/* Diagnostic of the library's failure reporting, not an operation of the
 * layer.  Every spin wait inside the kernels is bounded: after about 1 s (or
 * a fixed number of failed polls) it gives up, ORs OMNI_DEV_TIMEOUT into
 * counts[2] and its kernel returns, so that the context stays usable.  This
 * call makes one such wait run out: one thread waits on a shared-memory
 * barrier that nothing completes.
 * counts: device int32[4], 4-byte aligned, caller-owned; only counts[2] is
 * written (OR).  Asynchronous on the stream; the wait takes about 1 s of one
 * thread.  Returns OMNI_ERR_INVALID_ARG for a null or misaligned counts,
 * OMNI_ERR_CUDA if the launch fails. */
int omni_wait_selftest(int32_t* counts, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* OMNIMOE_H */
