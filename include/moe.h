/*
 * moe.h — C ABI of a B200 (sm_100a) library for the forward pass of one
 * Mixture-of-Experts layer.
 *
 * The layer (Step3 推論最適化 (MI308X vs H20), §背景: "3-in-48" expert
 * selection; §最適化技術: one-stage MoE kernel tuned along inter_dim, shared
 * expert MLP fused into the layer, mixed BF16 / FP8 block-scale GEMMs;
 * [SGLang] MoE 모델을 위한 Single Batch Overlap 기법, §들어가며: dispatch,
 * down projection GEMM, combine) computes, for every valid row t of x:
 *
 *   l[t,e]   = sum_h x[t,h] Wr[e,h] (+ b[e])                 router logits (fp32)
 *   ids[t,:] = the k largest l[t,e], descending, ties to the lower e
 *   w[t,j]   = exp(l[t,ids_j] - l[t,ids_0]) / sum_j' exp(...)   (renormalised)
 *              or the full-softmax probability of ids_j (renormalize = 0)
 *   y_e(x)   = Wd[e] (silu(Wg[e] x) * (Wu[e] x)),  silu(z) = z / (1 + e^-z)
 *   out[t]   = bf16( sum_j w[t,j] y_{ids_j}(x[t]) + y_shared(x[t]) )
 *
 * and writes +0.0 to every row whose valid flag is 0 (padding rows of a
 * data-parallel all_gather, DP Attention and TBO for DeepSeek-V4 on MI355X,
 * §PrefillDelayer): such rows are not routed and not computed, and their
 * contents never matter.
 *
 * Conventions for every entry point:
 *  - All tensors are dense and row-major.  Device pointers are addresses in
 *    the current CUDA device's memory, owned by the caller; the library never
 *    allocates, frees or retains device memory.  Host pointers are read only
 *    during the call.
 *  - Device pointers to tensors must be 16-byte aligned; the workspace must be
 *    256-byte aligned.
 *  - Work is enqueued on the given cudaStream_t (passed as void*, NULL = the
 *    legacy default stream) without host synchronisation, device-to-host
 *    copies or allocation, so moe_forward can be captured in a CUDA graph once
 *    it has been called on the device outside capture (the first call sets
 *    kernel attributes).
 *  - Argument errors are detected on the host before anything is enqueued and
 *    return a negative moe_status; nothing is launched in that case.
 *  - Failures detected on the device (a bounded wait that expired, an expert
 *    index out of range) set bits in a status word inside the workspace; read
 *    them with moe_check_device_status.  The library never aborts the process
 *    and never traps on the device.
 *  - One workspace may serve one forward at a time: calls that share a
 *    workspace must be ordered on one stream.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = -1,   /* a null pointer, a size out of range, misalignment */
    MOE_ERR_UNSUPPORTED = -2,   /* a shape or type the library does not implement */
    MOE_ERR_WORKSPACE = -3,     /* workspace smaller than moe_plan_create reported */
    MOE_ERR_CUDA = -4,          /* a CUDA runtime call failed (launch, attribute, sync) */
    MOE_ERR_DEVICE = -5         /* moe_check_device_status found a device-side failure */
} moe_status;

typedef enum {
    MOE_W_BF16 = 0,             /* bf16 expert weights */
    MOE_W_FP8_E4M3_B128 = 1     /* OCP e4m3 weights with one fp32 scale per 128x128 block;
                                   activations quantised e4m3 per 1x128 group inside the call */
} moe_wtype;

/* Device status bits (moe_check_device_status). */
#define MOE_DEV_WAIT_TIMEOUT_GATE_UP 0x1u   /* a bounded wait expired in the gate/up GEMM */
#define MOE_DEV_WAIT_TIMEOUT_DOWN    0x2u   /* a bounded wait expired in the down GEMM */
#define MOE_DEV_BAD_EXPERT_ID        0x4u   /* a routed expert index outside [0, E) */
#define MOE_DEV_WAIT_TIMEOUT_ROUTER  0x8u   /* a bounded wait expired in the router GEMM */
#define MOE_DEV_WAIT_TIMEOUT_SEND    0x10u  /* a sender gave up waiting for a group's tiles */

/* Shape of the layer; fixed for the lifetime of a plan. */
typedef struct {
    int max_tokens;     /* largest T a forward will be given (rows, valid + padding), >= 1 */
    int hidden;         /* H: multiple of 128 */
    int num_experts;    /* E: 1..256 routed experts */
    int top_k_max;      /* largest k a forward will be given: 1..min(8, E) */
    int inter;          /* I: routed expert intermediate size, multiple of 128 */
    int num_shared;     /* S: 0 or 1 always-on shared expert */
    int shared_inter;   /* Is: shared expert intermediate size, multiple of 128 (S = 1) */
    int renormalize;    /* 1: softmax over the selected k; 0: full softmax over E */
    moe_wtype wtype;
} moe_config;

typedef struct moe_plan_s *moe_plan_t;

/* Validates the shape and sizes the workspace.  Host only: touches no device.
 * *plan receives a new plan (free with moe_plan_destroy), *workspace_bytes the
 * device workspace size every forward with this plan needs. */
moe_status moe_plan_create(const moe_config *cfg, moe_plan_t *plan, size_t *workspace_bytes);
void moe_plan_destroy(moe_plan_t plan);

/* Upper bound on every device-side wait, in nanoseconds (default 2e9).  A
 * wait that runs out sets a MOE_DEV_WAIT_TIMEOUT_* bit and its kernel returns
 * early with its output incomplete.  0 makes every wait that is not already
 * satisfied give up at once; it exists to exercise that path. */
moe_status moe_plan_set_wait_limit(moe_plan_t plan, uint64_t limit_ns);

/* Weights (device pointers).
 *  router_w   fp32 [E, H];  router_b fp32 [E] or NULL (added to the logits)
 *  w_gate_up  [E, 2I, H]: rows 0..I-1 of each expert are the gate projection,
 *             rows I..2I-1 the up projection (bf16, or e4m3 codes as bytes)
 *  w_down     [E, H, I]
 *  s_gate_up  fp32 [E, 2I/128, H/128], s_down fp32 [E, H/128, I/128] (FP8 only)
 *  ws_gate_up [2Is, H], ws_down [H, Is], ss_* likewise: the shared expert
 *             (NULL when num_shared = 0).
 *  router_split  the bf16 split of router_w that moe_split_router_weights
 *             wrote, or NULL: then every forward splits router_w again (into
 *             the workspace) before the router GEMM. */
typedef struct {
    const float *router_w;
    const float *router_b;
    const void *w_gate_up;
    const void *w_down;
    const float *s_gate_up;
    const float *s_down;
    const void *ws_gate_up;
    const void *ws_down;
    const float *ss_gate_up;
    const float *ss_down;
    const void *router_split;
} moe_weights;

/* The router GEMM runs on the tensor cores (which multiply bf16, not fp32,
 * operands) with the fp32 router weights split exactly into three bf16 parts,
 * Wr = W1 + W2 + W3, each part the round-to-nearest bf16 of what the parts
 * before it left; every product of a bf16 hidden value with a part is exact in
 * fp32, so the logits are the fp32-accumulated products with the full fp32
 * weights.  The split depends on the weights only: make it once when the
 * weights are loaded (and again whenever router_w changes) and pass it as
 * moe_weights.router_split, and no forward repeats it.
 *
 * moe_router_split_bytes: bytes of the split, 3 * E16 * H * 2 with E16 = E
 *   rounded up to a multiple of 16 (0 for a NULL plan).
 * moe_split_router_weights: writes the split of router_w (fp32 [E, H], device)
 *   into split (device, 16-byte aligned, split_bytes at least the size above:
 *   else MOE_ERR_WORKSPACE), bf16 [3][E16][H], rows past E zero; enqueued on
 *   the stream. */
size_t moe_router_split_bytes(moe_plan_t plan);
moe_status moe_split_router_weights(moe_plan_t plan, const float *router_w, void *split,
                                    size_t split_bytes, void *stream);

/* Optional copies of intermediate results (device pointers, each may be NULL):
 *  logits    fp32 [T, E]   (0 in padding rows)
 *  topk_ids  int32 [T, k]  (-1 in padding rows)
 *  topk_w    fp32 [T, k]   (0 in padding rows)
 *  perm      int32 [T*k]   first Tv*k entries: pair index t*k+j, grouped by
 *                          expert, ascending t inside an expert
 *  offsets   int32 [E+1]   exclusive prefix sum of the per-expert pair counts
 *  events    cudaEvent_t handles (as void*) recorded on the stream before the
 *            first stage and after each of the MOE_NUM_STAGES stages
 *            (router, top-k, permute, gather, gate/up GEMM, down GEMM,
 *            combine); NULL entries are skipped. */
#define MOE_NUM_STAGES 7
typedef struct {
    float *logits;
    int *topk_ids;
    float *topk_w;
    int *perm;
    int *offsets;
    void *events[MOE_NUM_STAGES + 1];
} moe_debug;

/* The forward pass.
 *  hidden  bf16 [T, H] (device);  valid uint8 [T] (device; NULL = all rows valid)
 *  T       0..max_tokens rows;  k  1..top_k_max experts per token
 *  out     bf16 [T, H] (device), fully written (padding rows get +0.0)
 *  workspace / ws_bytes: device scratch of at least the size moe_plan_create gave
 *  stream  cudaStream_t;  dbg  optional, may be NULL. */
moe_status moe_forward(moe_plan_t plan, const moe_weights *weights, const void *hidden,
                       const uint8_t *valid, int T, int k, void *out, void *workspace,
                       size_t ws_bytes, void *stream, moe_debug *dbg);

/* Tensor-parallel MoE (DP Attention and TBO for DeepSeek-V4 on MI355X,
 * introduction: DP attention in front of a TP MoE joined by all_gather /
 * reduce_scatter).  Each of n ranks holds a 1/n share of every expert's
 * intermediate dimension (a plan with inter = I/n, shared_inter = Is/n, and
 * the matching rows of w_gate_up and columns of w_down), runs the layer on the
 * all-gathered rows T = n * rows_per_rank, and its contributions are summed.
 *
 * moe_forward_scatter is the forward pass whose combine writes each token's
 * fp32 sum (this rank's share, routed + shared, not rounded; padding rows
 * +0.0) directly into the receive slab of the rank that owns the token:
 *   token t -> dst[t / rows_per_rank] + (slot * rows_per_rank + t % rows_per_rank) * H
 * so the slab of owner r is [n_dst][rows_per_rank][H] fp32 with one row block
 * per contributing rank, and `slot` is this rank's index.  dst is a host
 * array of n_dst (1..8) device pointers, 16-byte aligned; they may point into
 * other GPUs' memory (peer-mapped: the kernel only stores to them), which
 * makes the combine carry the reduce-scatter's data movement.  With n_dst = 1,
 * rows_per_rank = T, slot = 0 it writes the plain fp32 partial [T, H].
 * Requires n_dst * rows_per_rank == T and 0 <= slot < n_dst.  Completion on
 * this stream says nothing about the other ranks: the owner must know that
 * every contributor's forward has finished (a barrier) before reducing.
 *
 * moe_reduce_partials is the owner's half: out[t] = bf16(sum over g = 0..n_slots-1
 * of slots[g][t]), in that order, rounded once; rows with valid[t] == 0 get
 * +0.0.  slots: fp32 [n_slots][rows][H] (device), valid: uint8 [rows] or NULL,
 * out: bf16 [rows][H]; H a multiple of 8, pointers 16-byte aligned. */
moe_status moe_forward_scatter(moe_plan_t plan, const moe_weights *weights, const void *hidden,
                               const uint8_t *valid, int T, int k, float *const *dst, int n_dst,
                               int rows_per_rank, int slot, void *workspace, size_t ws_bytes,
                               void *stream, moe_debug *dbg);
moe_status moe_reduce_partials(const float *slots, int n_slots, int rows, int H,
                               const uint8_t *valid, void *out, void *stream);

/* Expert-parallel rank: moe_forward_scatter restricted to the routed experts
 * [expert_begin, expert_end) of the plan's num_experts.  Routing (logits, top-k,
 * weights) is computed over all experts from the router weights as usual; pairs
 * routed to other experts are left out of this rank's permutation (their groups
 * stay empty and cost nothing) and out of its combine, so each token's fp32 sum
 * is its share over this rank's experts (plus the shared expert's, when the
 * plan has one: split its intermediate dimension over the ranks as in the
 * tensor-parallel layout).  The routed weights given hold only these experts:
 * w_gate_up [expert_end - expert_begin, 2I, H], w_down [.., H, I] and, for FP8,
 * their scales; expert e's rows are at index e - expert_begin.  Summed over
 * the ranks (moe_reduce_partials), the partials give the layer.  Requires
 * 0 <= expert_begin < expert_end <= num_experts; other arguments as
 * moe_forward_scatter, which is this call with the full range. */
moe_status moe_forward_scatter_experts(moe_plan_t plan, const moe_weights *weights,
                                       const void *hidden, const uint8_t *valid, int T, int k,
                                       float *const *dst, int n_dst, int rows_per_rank, int slot,
                                       int expert_begin, int expert_end, void *workspace,
                                       size_t ws_bytes, void *stream, moe_debug *dbg);

/* Expert-parallel rank with the per-pair return, sends overlapping the down GEMM
 * ([SGLang] MoE 모델을 위한 Single Batch Overlap 기법, §핵심 코드 분석: a per-expert
 * completion signal between the down projection GEMM and the combine's sends, and
 * a set number of SMs for the sends).
 *
 * moe_forward_scatter_pairs computes, like moe_forward_scatter_experts, the
 * routed experts [expert_begin, expert_end) of the plan (their weights given) for
 * the gathered rows, but instead of a combine it returns every routed pair's
 * expert output row unweighted, so each owner can sum a token's k rows in the
 * one-GPU order.  The down GEMM's launch is cooperative: send_ctas of its CTAs
 * (1 .. SMs - 1) do no tiles; each waits on a per-group counter that the other
 * CTAs' epilogue warps raise after storing each tile, and as soon as an expert's
 * tiles are all stored, copies its rows to the owners' slabs while later experts
 * are still being multiplied.  The receive slab of owner r is fp32
 * [n_slots][rows_per_rank][H], slot-major:
 *   pair (t, j) of a routed expert -> dst[t / rows_per_rank] + (j * rows_per_rank
 *                                     + t % rows_per_rank) * H,          j < k
 *   the shared expert's row of t   -> slot shared_slot (>= k) likewise (plans with
 *                                     num_shared = 1 only; ignored otherwise).
 * dst: n_dst (1..8) device pointers, 16-byte aligned, possibly peer memory (the
 * kernel only stores to them); n_dst * rows_per_rank == T.  Nothing but those
 * rows is written to the slabs.  A sender that waits longer than the plan's wait
 * limit sets MOE_DEV_WAIT_TIMEOUT_SEND and stops (its rows stay unsent).
 *
 * moe_reduce_pairs is the owner's half: out[t] = bf16(sum_{j<k} w[t,j] *
 * slab[j][t] (fused multiply-adds, j ascending) + sum_{s<n_extra} slab[k+s][t]
 * (s ascending)), padding rows +0.0; slab fp32 [k + n_extra][rows][H], w fp32
 * [rows, k] (this owner's rows' routing weights), valid uint8 [rows] or NULL,
 * out bf16 [rows, H]; H a multiple of 8, slab and out 16-byte aligned.  On one
 * rank with every expert local this is the plain forward's combine, bit for bit. */
moe_status moe_forward_scatter_pairs(moe_plan_t plan, const moe_weights *weights,
                                     const void *hidden, const uint8_t *valid, int T, int k,
                                     float *const *dst, int n_dst, int rows_per_rank,
                                     int shared_slot, int expert_begin, int expert_end,
                                     int send_ctas, void *workspace, size_t ws_bytes,
                                     void *stream, moe_debug *dbg);
moe_status moe_reduce_pairs(const float *slab, int k, int n_extra, int rows, int H,
                            const float *w, const uint8_t *valid, void *out, void *stream);

/* Routing only, from given fp32 logits [T, E] (device): the top-k selection,
 * weights, per-expert offsets and permutation exactly as moe_forward computes
 * them.  Outputs as in moe_debug (topk_ids, topk_w [T,k]; perm [T*k];
 * offsets [E+1]); none may be NULL. */
moe_status moe_route_from_logits(moe_plan_t plan, const float *logits, const uint8_t *valid,
                                 int T, int k, int *topk_ids, float *topk_w, int *perm,
                                 int *offsets, void *workspace, size_t ws_bytes, void *stream);

/* moe_route_from_logits without a caller workspace.  The pages have no
 * counterpart to this entry point; it exists for callers that cannot allocate
 * device memory: code running inside a framework whose memory pool owns the
 * whole device and forbids further cudaMalloc, plain-C hosts handed only
 * device pointers, or code that must not allocate because a CUDA graph is
 * being captured on its stream.
 *
 * Results are identical to moe_route_from_logits, bit for bit: the same top-k
 * kernel, and the single-block routing kernel that moe_route_from_logits also
 * runs up to 1024 tokens (above 1024 the workspace path spreads the counting
 * over three kernels; the result, a stable counting sort, is the same).  Its
 * scratch (status word, group offsets, the inverse permutation and the
 * row -> token map; the logits are not copied) lives in one file-scope
 * __device__ array of MOE_STATIC_SCRATCH_BYTES that every GPU which loads the
 * library holds until the process exits.  A call needs
 *   256 + a(4 (E + 2)) + 2 a(4 T (k + S))  bytes,  a(n) = n rounded up to 256,
 * (S = num_shared) and returns MOE_ERR_UNSUPPORTED, launching nothing, when
 * that exceeds MOE_STATIC_SCRATCH_BYTES (E = 256, k = 8, S = 1: up to 58,232
 * tokens).
 *  - It allocates nothing: no cudaMalloc, no cudaFree, no allocating library call.
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call
 *    before capturing the stream into a graph.
 *  - Every call on a device shares the one array, which keeps the previous
 *    call's contents (each call clears what it needs cleared).  Calls whose
 *    work overlaps on the GPU — on two streams, or from two threads — race on
 *    it: order them on one stream.
 *  - Its device status word is inside the array too, and nothing can set it:
 *    the top-k kernel emits only ids in [0, E) for valid rows and -1 for
 *    padding rows, which routing skips, so the out-of-range check of the
 *    routing kernel never fires.
 * Arguments as in moe_route_from_logits; none of the output pointers may be NULL. */
#define MOE_STATIC_SCRATCH_BYTES (4u << 20)
moe_status moe_route_from_logits_noalloc(moe_plan_t plan, const float *logits,
                                         const uint8_t *valid, int T, int k, int *topk_ids,
                                         float *topk_w, int *perm, int *offsets, void *stream);

/* Synchronises the stream, reads and clears the device status word of this
 * workspace.  *bits (may be NULL) receives the MOE_DEV_* bits that were set.
 * Returns MOE_OK if none, MOE_ERR_DEVICE otherwise. */
moe_status moe_check_device_status(moe_plan_t plan, void *workspace, void *stream,
                                   uint32_t *bits);

/* Device addresses of the intermediate buffers inside a workspace, for
 * inspection after a forward (host arithmetic only; nothing is launched):
 *  row_token  int32 [R]     token index of each permuted row (R = Tv*(k+S))
 *  x_perm     [R, H]        permuted activations (bf16; e4m3 codes for FP8)
 *  h          SwiGLU output rows: bf16 weights: [2R, Imax], row 2r = bf16(h_r) and
 *                           row 2r + 1 = bf16(h_r - that) (two parts, multiplied both
 *                           by the down GEMM); FP8: [R, Imax] e4m3 codes
 *  y          [R, H]        expert output rows before the weighted combine
 *                           (fp32 for bf16 weights, bf16 for FP8 weights)
 *  group_offsets int32 [E+S+1]: rows of expert e are [go[e], go[e+1]); the
 *             shared expert is group E.
 *  x_scale, h_scale  FP8 only (else NULL): fp32 scales of x_perm and h, one per
 *             1x128 group, row-major: [R][H/128] and [R][Imax/128]. */
typedef struct {
    int *row_token;
    void *x_perm;
    void *h;
    void *y;
    int *group_offsets;
    int h_stride;       /* Imax = max(I, Is) elements per h row */
    float *x_scale;
    float *h_scale;
} moe_workspace_views;
moe_status moe_get_workspace_views(moe_plan_t plan, void *workspace, moe_workspace_views *views);

/* Host-to-host forwards whose copies overlap the neighbouring batches' compute.
 *
 * A caller whose hidden states live in host memory pays, per batch, an upload of
 * x and the mask and a download of out.  A pipeline runs them on two copy
 * streams of its own beside a compute stream: the upload of batch i+1 and the
 * download of batch i-1 proceed on the copy engines while batch i computes.
 * Each of `depth` slots owns device buffers for one batch (x, mask, out, in
 * caller-provided device memory); a slot is refilled only after its previous
 * download has finished, and the forwards run one after another on the compute
 * stream, so they share one workspace.  With three slots a step costs the
 * longest of the forward, the upload and the download.
 *
 * moe_pipeline_slot_bytes: device bytes the slots of (plan, rows, depth) need.
 * moe_pipeline_create: rows 1..max_tokens rows a batch, depth 1..8 slots, k as
 *   for moe_forward; `weights` (the structure is copied; the tensors it points
 *   to must stay valid and unchanged), `slots` (device, 256-byte aligned, at
 *   least moe_pipeline_slot_bytes) and `workspace` are owned by the caller and
 *   used by no one else while the pipeline lives.  With use_graph != 0 each
 *   slot's forward is captured once as a CUDA graph and replayed.  Creation
 *   synchronises the device (the weights the caller prepared are then ready) and
 *   runs one forward per slot on all-padding rows.
 * moe_pipeline_submit: enqueues one batch and returns: hidden bf16 [rows, H]
 *   and valid uint8 [rows] (NULL = all valid) are read from host memory, out
 *   bf16 [rows, H] is written to host memory; the caller keeps the inputs
 *   unchanged and does not read out until the batch is done (for example after
 *   moe_pipeline_synchronize).  Page-locked host memory lets the copies overlap;
 *   pageable memory works but copies synchronously.
 * moe_pipeline_synchronize: waits until every submitted batch's output is in
 *   host memory.
 * moe_pipeline_streams: the pipeline's upload, compute and download streams
 *   (cudaStream_t as void*), for callers that order or time work against them.
 * moe_pipeline_destroy: waits for the batches in flight, releases the streams,
 *   events and graphs (not the caller's memory). */
typedef struct moe_pipeline_s *moe_pipeline_t;
moe_status moe_pipeline_slot_bytes(moe_plan_t plan, int rows, int depth, size_t *bytes);
moe_status moe_pipeline_create(moe_plan_t plan, const moe_weights *weights, int k, int rows,
                               int depth, int use_graph, void *slots, size_t slots_bytes,
                               void *workspace, size_t ws_bytes, moe_pipeline_t *pipeline);
moe_status moe_pipeline_submit(moe_pipeline_t pipeline, const void *hidden_host,
                               const uint8_t *valid_host, void *out_host);
moe_status moe_pipeline_synchronize(moe_pipeline_t pipeline);
moe_status moe_pipeline_streams(moe_pipeline_t pipeline, void **upload, void **compute,
                                void **download);
void moe_pipeline_destroy(moe_pipeline_t pipeline);

const char *moe_status_string(moe_status s);

/* Text of the last CUDA runtime error behind an MOE_ERR_CUDA returned to this
 * thread ("no error" if none). */
const char *moe_last_cuda_error_string(void);

#ifdef __cplusplus
}
#endif
#endif /* MOE_B200_H */
