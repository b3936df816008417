/*
 * hstu_attn.h — C ABI of libhstu_attn.so: forward pass of jagged, target-aware
 * HSTU pointwise (SiLU) attention on NVIDIA B200 (sm_100a).
 *
 * What is computed (per user b, head h, query position i of user b's segment):
 *
 *     out[i,h,:] = (1/N) * sum_{j in A(i)} silu(alpha * <q[i,h,:], k[j,h,:]>) * v[j,h,:]
 *
 *     silu(x) = x / (1 + exp(-x))
 *     A(i)    = { j : j <= i }            if i <  U_b   (history token: causal over history)
 *             = { j : j <  U_b } + { i }  if i >= U_b   (candidate: all history, then itself)
 *
 * Sources (page title, then section):
 *   - "DLRMv3: MLPerf Inference generative recommendation benchmark" (winzheng.jp review),
 *     section "model selection", time/position-encoding paragraph: DLRMv3 drops the
 *     relative bias, so attention is Mask(SiLU(Q K^T)) V.
 *   - same page, same section, FLOP-formula paragraph: one history (UIH) encoding is shared
 *     by all ~2K candidates of a request, and UIH-related K/V state is reused across a
 *     user's consecutive timestamps (the cached variant below).
 *   - infolabhq.com "multi-stage sequence model" page, section on the offline user model:
 *     the user-side representation never depends on an ad candidate (history tokens never
 *     see candidates); section "Target-Aware Multi-Head Attention": every layer re-weights
 *     past actions against the candidate being scored (candidates see all history).
 *   - voagi.com DLRM/TorchRec tutorial, section 2.1: jagged data = concatenated values plus
 *     a lengths vector; a zero length is legal.  Here seq_offsets is the exclusive prefix
 *     sum of the lengths.
 *   The scale alpha and the normaliser 1/N are not printed on the pages; they are explicit
 *   scalar arguments (one value per call).
 *
 * Layout.  All token tensors are jagged [total, H, d] bf16, row-major, heads interleaved:
 * element (t, h, c) sits at ((size_t)t * H + h) * d + c.  User b owns rows
 * [seq_offsets[b], seq_offsets[b+1]).  Its last num_targets[b] rows are the candidates
 * (targets); the first U_b = L_b - T_b rows are its history.
 *
 * Ownership.  The caller owns every buffer.  Pointers must stay valid until the work
 * queued on `stream` has completed; the library keeps none of them after it returns.
 * hstu_attn_fwd / hstu_attn_fwd_cached take a small stream-ordered plan buffer (work list,
 * work counter) from the library's own per-device memory pool and return it on the same
 * stream; hstu_attn_plan / hstu_attn_fwd_planned use a plan buffer the caller owns.
 * When total_q (or total_tokens) is 0 nothing is read or written and the token pointers may
 * be NULL.
 *
 * Errors.  Bad scalars or NULL pointers return HSTU_ERR_INVALID_ARGUMENT synchronously and
 * launch nothing; an unsupported head size or a misaligned pointer returns
 * HSTU_ERR_UNSUPPORTED; a failed launch returns HSTU_ERR_CUDA.  Problems that only the
 * device can see (inconsistent seq_offsets / num_targets / cached_len, a pipeline wait
 * that ran past its time limit) are recorded in a per-device error word and reported by
 * hstu_attn_get_error().  Users whose offsets are inconsistent are skipped (their output
 * rows are not written).  Nothing in the library traps or aborts.
 *
 * Streams.  `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 * Every call is asynchronous on that stream; calls are re-entrant and thread-safe.
 *
 * Inputs must be finite: rows past a user's end that share a tile with its last rows are
 * read (and masked to an exact zero weight), so a NaN/Inf in a neighbouring user's V row
 * could leak through 0 * Inf.
 */
#ifndef HSTU_ATTN_H_
#define HSTU_ATTN_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum hstu_status {
  HSTU_OK = 0,
  HSTU_ERR_INVALID_ARGUMENT = 1, /* NULL pointer, negative size, N <= 0, non-finite alpha/N */
  HSTU_ERR_UNSUPPORTED = 2,      /* d not in {32, 64, 128}, H*d*2 not a multiple of 16 bytes, misaligned base */
  HSTU_ERR_CUDA = 3,             /* a CUDA runtime/driver call failed */
  HSTU_ERR_BAD_OFFSETS = 4,      /* device-detected: offsets not monotone / out of range, T_b > L_b, cached_len_b > U_b */
  HSTU_ERR_TIMEOUT = 5           /* device-detected: a pipeline wait exceeded its time limit */
} hstu_status_t;

/*
 * hstu_attn_fwd — full forward pass over a jagged batch.
 *
 *   q, k, v       device, bf16 [total_tokens, H, d], 16-byte aligned base addresses.
 *   seq_offsets   device, int32 [B+1]: seq_offsets[0] = 0, non-decreasing,
 *                 seq_offsets[B] = total_tokens.  L_b = seq_offsets[b+1] - seq_offsets[b].
 *   num_targets   device, int32 [B], 0 <= T_b <= L_b; NULL means every T_b = 0 (plain causal).
 *   B             number of users (>= 0; B = 0 or total_tokens = 0 launches nothing).
 *   H, d          heads and head size; d in {32, 64, 128}; H >= 1.
 *   total_tokens  rows of q, k, v and out.
 *   max_seq_len   an upper bound on every L_b (sizes the schedule; a user longer than this
 *                 is reported as HSTU_ERR_BAD_OFFSETS and skipped).
 *   alpha         score scale inside the SiLU (finite).
 *   N             output normaliser, one scalar for the whole call (finite, > 0).
 *   out           device, bf16 [total_tokens, H, d]; must not overlap q, k or v.
 *   stream        cudaStream_t as void*.
 */
hstu_status_t hstu_attn_fwd(const void* q, const void* k, const void* v,
                            const int32_t* seq_offsets, const int32_t* num_targets,
                            int32_t B, int32_t H, int32_t d,
                            int32_t total_tokens, int32_t max_seq_len,
                            float alpha, float N,
                            void* out, void* stream);

/*
 * hstu_attn_fwd_cached — streaming variant: only the new tokens of each user are queried;
 * keys and values cover the cached history prefix plus the new tokens (the K/V reuse across
 * consecutive timestamps of the DLRMv3 review, section "model selection").
 *
 *   q             device, bf16 [total_q, H, d]: for each user, its new rows only, users
 *                 packed in order (user b's new rows start at
 *                 seq_offsets[b] - sum_{b' < b} cached_len[b']).
 *   k, v          device, bf16 [total_kv, H, d]: full segments (cached prefix + new rows),
 *                 jagged by seq_offsets exactly as in hstu_attn_fwd.
 *   num_targets   as in hstu_attn_fwd (targets are the last T_b rows of the full segment).
 *   cached_len    device, int32 [B]: 0 <= cached_len[b] <= U_b (the prefix is history only).
 *                 NULL means all zero, which makes the call identical to hstu_attn_fwd.
 *   total_q       must equal total_kv - sum_b cached_len[b] (checked on the device).
 *   out           device, bf16 [total_q, H, d]: row r of user b is the output of position
 *                 cached_len[b] + r, identical to that row of a full recomputation.
 *   Other arguments as in hstu_attn_fwd.
 */
hstu_status_t hstu_attn_fwd_cached(const void* q, const void* k, const void* v,
                                   const int32_t* seq_offsets, const int32_t* num_targets,
                                   const int32_t* cached_len,
                                   int32_t B, int32_t H, int32_t d,
                                   int32_t total_kv, int32_t total_q, int32_t max_seq_len,
                                   float alpha, float N,
                                   void* out, void* stream);

/*
 * hstu_attn_fwd_rab — the relative-attention-bias variant that the DLRMv3 review (section
 * "model selection", time/position-encoding paragraph) prints for the original HSTU,
 * Mask(SiLU(Q K^T) + bias) V, and that DLRMv3 drops because it slows attention.  Reading taken:
 * every visible pair (i, j) gets silu(alpha * <q_i, k_j>) + rab[h * rab_len + min(i - j,
 * rab_len - 1)], a bias that depends only on the query-key distance, clipped at the table's
 * last entry; masked pairs contribute nothing.  Positions i, j count from the start of the
 * user's segment (cached prefix included), so the bias of a pair is the same in the full and
 * the cached form.
 *   rab      device float [H, rab_len], 4-byte aligned, read only; owned by the caller.
 *   rab_len  1 .. 2^24 entries per head.
 *   Other arguments as hstu_attn_fwd_cached; cached_len may be NULL (full sequences, q holds
 *   every token).
 * Errors: HSTU_ERR_INVALID_ARGUMENT for rab == NULL (with rows to compute) or rab_len out of
 * range, HSTU_ERR_UNSUPPORTED for a misaligned table; otherwise as hstu_attn_fwd_cached.
 */
hstu_status_t hstu_attn_fwd_rab(const void* q, const void* k, const void* v,
                                const int32_t* seq_offsets, const int32_t* num_targets,
                                const int32_t* cached_len, const float* rab, int32_t rab_len,
                                int32_t B, int32_t H, int32_t d,
                                int32_t total_kv, int32_t total_q, int32_t max_seq_len,
                                float alpha, float N,
                                void* out, void* stream);

/*
 * Two-step form.  hstu_attn_fwd / hstu_attn_fwd_cached are hstu_attn_plan followed by
 * hstu_attn_fwd_planned on a buffer the library takes from its own pool.  Callers that run the
 * attention several times over the same jagged structure (several layers, heads groups or
 * repeated requests) can build the plan once and replay it; the plan is also what a caller
 * inspects to see the work list.
 *
 * hstu_attn_plan_bytes — bytes of a plan buffer for (B, H, total_q) (0 for invalid sizes).
 *   Layout (all int32, little endian):
 *     header[4]          {work counter, num_items, finished-CTA counter, 0}
 *     q_start[B]         first query row of each user (-1: user skipped), padded to 16 bytes
 *     block_start[B+1]   index of each user's first 128-row block, padded to 16 bytes
 *     items[cap][4]      {b, block, h, cost}, cap = H * (total_q / 128 + B); the first
 *                        num_items entries are valid.  `block` is a block of 128 query rows of
 *                        user b; `cost` is the number of 128x128 score tiles the block computes
 *                        (fully masked tiles are not counted).  Order: users are taken in waves
 *                        by their first key row, floor(seq_offsets[b] / W) with
 *                        W = 32 MiB / (512 * H) rows (the rows whose K and V fill about a quarter
 *                        of L2 at d = 128), and items go by wave, then by non-increasing cost; a
 *                        batch of fewer than W rows is in non-increasing cost order.
 *
 * hstu_attn_plan — validates the offsets on the device and writes the plan.
 *   seq_offsets, num_targets, cached_len, B, H, total_kv, total_q, max_seq_len: as in
 *   hstu_attn_fwd_cached (cached_len NULL and total_q = total_kv for a full pass).
 *   plan         device, 16-byte aligned, plan_bytes >= hstu_attn_plan_bytes(B, H, total_q).
 *
 * hstu_attn_fwd_planned — the attention kernel over a plan built by hstu_attn_plan from the
 *   same seq_offsets / num_targets / cached_len / B / H / total_q.  Arguments as in
 *   hstu_attn_fwd_cached.  The kernel re-arms the plan's work counter when it finishes, so a
 *   plan may be replayed any number of times on one stream; two calls that share a plan must
 *   not overlap in time.
 */
int64_t hstu_attn_plan_bytes(int32_t B, int32_t H, int32_t total_q);

hstu_status_t hstu_attn_plan(const int32_t* seq_offsets, const int32_t* num_targets,
                             const int32_t* cached_len,
                             int32_t B, int32_t H, int32_t total_kv, int32_t total_q,
                             int32_t max_seq_len,
                             void* plan, int64_t plan_bytes, void* stream);

hstu_status_t hstu_attn_fwd_planned(const void* q, const void* k, const void* v,
                                    const int32_t* seq_offsets, const int32_t* num_targets,
                                    const int32_t* cached_len,
                                    int32_t B, int32_t H, int32_t d,
                                    int32_t total_kv, int32_t total_q,
                                    float alpha, float N,
                                    void* plan, void* out, void* stream);

/*
 * hstu_attn_fwd_noalloc — hstu_attn_fwd_cached without any device-memory allocation.  (An
 * addition of this library for its callers; the pages describe no such call.)
 *
 * Why: some callers cannot allocate device memory while they run a batch — serving processes
 * that reserve all of the GPU's memory up front for their own caching allocator, or code on a
 * latency-critical path where an allocator call may block or synchronise.  Every other entry
 * point either takes its plan buffer from the library's memory pool or wants the caller to
 * provide one; this one keeps the plan in a fixed array of HSTU_ATTN_NOALLOC_PLAN_BYTES bytes
 * that is part of the library's device image.
 *
 *   Arguments are those of hstu_attn_fwd_cached (cached_len = NULL and total_q = total_kv for a
 *   full pass).  The caller still provides q, k, v and out.
 *   Limit: hstu_attn_plan_bytes(B, H, total_q) must not exceed HSTU_ATTN_NOALLOC_PLAN_BYTES
 *   (1 MiB: about 65,000 work items of 128 query rows x 1 head, e.g. H = 8 and 1 million query
 *   rows); larger batches return HSTU_ERR_UNSUPPORTED before anything is launched.
 *   Memory: every GPU that loads the library holds the 1 MiB array until the process exits.
 *   First call: the first call on each device (with that device current) looks up the array's
 *   device address once; make that first call before any stream capture.
 *   Sharing: all calls on a device use the same array.  Calls whose GPU work overlaps in time
 *   (different streams, or different host threads without ordering) race on it and may produce
 *   wrong outputs; order them on one stream or with events.  Each call rewrites the part of the
 *   array it reads, so leftovers from earlier calls are harmless.
 *   Returns, besides the statuses of hstu_attn_fwd_cached, HSTU_ERR_UNSUPPORTED for a batch over
 *   the limit.  It calls no cudaMalloc, cudaFree or other allocating routine.
 */
#define HSTU_ATTN_NOALLOC_PLAN_BYTES (1u << 20)

hstu_status_t hstu_attn_fwd_noalloc(const void* q, const void* k, const void* v,
                                    const int32_t* seq_offsets, const int32_t* num_targets,
                                    const int32_t* cached_len,
                                    int32_t B, int32_t H, int32_t d,
                                    int32_t total_kv, int32_t total_q, int32_t max_seq_len,
                                    float alpha, float N,
                                    void* out, void* stream);

/*
 * hstu_attn_bwd — backward pass of hstu_attn_fwd for training: the gradients of a scalar loss
 * with respect to q, k and v, given its gradient dout with respect to out.  The pages print no
 * backward pass; the infolabhq.com multi-stage page (scaling section) is about training such
 * models, and the forward definition above fixes the gradients by the chain rule.  For every
 * user, head and visible pair (i, j), with x = alpha <q_i, k_j>:
 *
 *     dv[j] += silu(x) * dout[i] / N
 *     ds     = (<dout[i], v[j]> / N) * silu'(x) * alpha,   silu'(x) = sigma(x) (1 + x (1 - sigma(x)))
 *     dq[i] += ds * k[j],      dk[j] += ds * q[i]
 *
 * Masked pairs contribute nothing.  Products accumulate in fp32 on the tensor cores; silu(x) and
 * ds are rounded to bf16 before their matrix products, and the gradients to bf16 once.
 *
 *   q, k, v, dout   device, bf16 [total_tokens, H, d], 16-byte aligned (the forward's inputs and
 *                   the loss gradient of its output).
 *   seq_offsets, num_targets, B, H, d, total_tokens, max_seq_len, alpha, N: as in hstu_attn_fwd
 *                   (full sequences; there is no cached form).
 *   dq, dk, dv      device, bf16 [total_tokens, H, d], written; none may overlap an input or
 *                   another gradient.  Rows of users skipped for inconsistent offsets are not
 *                   written.
 *   stream          cudaStream_t as void*.
 * A stream-ordered plan buffer is taken from the library's pool and returned, as in
 * hstu_attn_fwd.  Errors as in hstu_attn_fwd; inputs must be finite (as there).
 * Workspace: the dK/dV kernel forms every bf16 dS tile; when a workspace for them fits the limit
 * set by hstu_attn_bwd_workspace_limit (2 bytes per visible pair and head, sized on the host from
 * an upper bound in total_tokens, B, H and max_seq_len), it keeps them there, stream-ordered from
 * the pool, and dq is a plain product of them with k.  Otherwise the dQ kernel recomputes them.
 * Both ways give the same gradients.
 */
hstu_status_t hstu_attn_bwd(const void* q, const void* k, const void* v, const void* dout,
                            const int32_t* seq_offsets, const int32_t* num_targets,
                            int32_t B, int32_t H, int32_t d,
                            int32_t total_tokens, int32_t max_seq_len,
                            float alpha, float N,
                            void* dq, void* dk, void* dv, void* stream);

/*
 * hstu_attn_bwd_workspace_limit — sets the largest dS workspace (bytes) hstu_attn_bwd may take
 * from the pool for one call, and returns the previous limit.  Default 16 GiB; 0 makes every call
 * recompute dS in its dQ kernel.  Process-wide; takes effect for calls made after it returns.
 */
uint64_t hstu_attn_bwd_workspace_limit(uint64_t max_bytes);

/*
 * hstu_attn_partition — splits one jagged batch across `parts` GPUs (host function, no GPU work).
 * Users are independent: no row of one user reads another user's K/V (the mask of hstu_attn_fwd),
 * so a batch shards by user with no exchange between GPUs.  Following the jagged layout of the
 * TorchRec tutorial (voagi.com, section 2.1: concatenated values plus lengths), each GPU takes a
 * contiguous run of users, users [user_start[p], user_start[p+1]) for GPU p, so that its rows are
 * one contiguous block of q, k, v and out; its seq_offsets are the batch's, rebased to 0.
 * The runs minimise the largest per-GPU cost, the cost of a user being its number of visible
 * (query, key) pairs (the algorithmic work of its attention); trailing runs may be empty.
 *   seq_offsets   HOST int32 [B+1];  num_targets, cached_len: HOST int32 [B] or NULL (all 0).
 *   user_start    HOST int32 [parts+1], written.
 * Returns HSTU_ERR_INVALID_ARGUMENT for B < 0, parts < 1 or NULL pointers, HSTU_ERR_BAD_OFFSETS for
 * inconsistent lengths, else HSTU_OK.  The pages have no multi-GPU scheme for this step; this is
 * the plain sharding that the layout allows.
 */
hstu_status_t hstu_attn_partition(const int32_t* seq_offsets, const int32_t* num_targets,
                                  const int32_t* cached_len, int32_t B, int32_t parts,
                                  int32_t* user_start);

/*
 * hstu_attn_get_error — synchronises `stream`, returns the device error word of the current
 * device as a status (HSTU_OK if clean) and clears it.  The word is shared by all calls on
 * the device, so a nonzero status may come from any call completed since the last read.
 */
hstu_status_t hstu_attn_get_error(void* stream);

/* Static, human-readable name of a status. */
const char* hstu_attn_status_string(hstu_status_t s);

/*
 * hstu_attn_gemm_bf16 — C = A · Wᵀ on the tensor cores: A bf16 [M, K], W bf16 [N, K] (a linear
 * layer's weight, out-features × in-features), C bf16 [M, N], all row-major on the device;
 * products accumulate in fp32 and are rounded to bf16 once.  These are the dense projections
 * of the HSTU layer around the attention, whose flops the DLRMv3 review counts as 4·L·D² and
 * 3·L·D² per layer (section "model selection", FLOP-formula paragraph); the pages do not give
 * the layer's other steps.
 *   M, N >= 0 (M or N == 0: nothing is done), K >= 1; K and N multiples of 8 (16-byte rows);
 *   pointers 16-byte aligned; C must not overlap A or W.  Asynchronous on `stream`.
 * Errors: HSTU_ERR_INVALID_ARGUMENT (NULL pointers, negative sizes, overlap),
 * HSTU_ERR_UNSUPPORTED (alignment, K or N not a multiple of 8), HSTU_ERR_CUDA (launch); a
 * device-side timeout is reported by hstu_attn_get_error.
 */
hstu_status_t hstu_attn_gemm_bf16(const void* a, const void* w, void* c, int32_t M, int32_t N, int32_t K,
                             void* stream);

/*
 * HSTU layer: the attention step between the two dense projections whose flops the DLRMv3 review
 * counts per layer as 4*L*D^2 and 3*L*D^2 (section "model selection", FLOP-formula paragraph:
 * 2 * layers * (L*L*D/2 + 4*L*D^2 + 3*L*D^2)), with layers stacked as the infolabhq.com multi-stage
 * page describes (section "Target-Aware Multi-Head Attention").  The pages give only the flop
 * terms; the layer built here is the plainest composition with exactly those terms (D = H * d):
 *
 *     UVQK = X W_uvqk^T        X [total, D], W_uvqk [4D, D]  -> [total, 4D] = [U | V | Q | K]
 *     A    = hstu_attn_fwd(Q, K, V)                         (each a [total, H, d] view of UVQK)
 *     Y    = [U | A | U*A] W_out^T                           W_out [D, 3D] -> Y [total, D]
 *
 * U*A is elementwise.  No normalisation, activation or residual is added: the pages name none.
 * All tensors are bf16, row-major, on the device; products accumulate in fp32 and every stored
 * tensor (UVQK, A, U*A, Y) is rounded to bf16 once.  The attention reads Q, K, V in place and its
 * epilogue writes U, A and U*A straight into the second projection's input, so the layer is
 * three kernels over one work plan.
 *
 * hstu_layer_workspace_bytes — device bytes of the workspace for num_layers stacked layers
 *   (UVQK, the [U | A | U*A] buffer and, for more than one layer, the hidden activations):
 *   total * D * 2 * (7 + (num_layers > 1)); 0 for invalid sizes.
 *
 * hstu_layer_fwd — one layer over a plan built by hstu_attn_plan(seq_offsets, num_targets, NULL,
 *   B, H, total, total, ...) (the plan may be reused by every layer of the batch).
 *   x, y          device bf16 [total, D]; y must not overlap the workspace; x may equal y.
 *   w_uvqk, w_out device bf16 [4D, D] and [D, 3D] (out-features x in-features), 16-byte aligned.
 *   seq_offsets, num_targets, B, H, d, total, alpha, N: as in hstu_attn_fwd.
 *   workspace     device, >= hstu_layer_workspace_bytes(H, d, total, 1) bytes, 16-byte aligned.
 *
 * hstu_layers_fwd — num_layers layers, layer l using w_uvqk[l] and w_out[l] (HOST arrays of
 *   device pointers); builds one plan (from the library's pool, like hstu_attn_fwd) and reuses it
 *   for every layer.  x is the first layer's input, y the last layer's output.
 *
 * Errors as in hstu_attn_fwd and hstu_attn_gemm_bf16 (HSTU_ERR_INVALID_ARGUMENT for a short
 * workspace or one that overlaps x or y); asynchronous on `stream`.
 */
int64_t hstu_layer_workspace_bytes(int32_t H, int32_t d, int32_t total, int32_t num_layers);

hstu_status_t hstu_layer_fwd(const void* x, const void* w_uvqk, const void* w_out,
                             const int32_t* seq_offsets, const int32_t* num_targets,
                             int32_t B, int32_t H, int32_t d, int32_t total,
                             float alpha, float N, void* plan,
                             void* workspace, int64_t workspace_bytes, void* y, void* stream);

hstu_status_t hstu_layers_fwd(int32_t num_layers, const void* x,
                              const void* const* w_uvqk, const void* const* w_out,
                              const int32_t* seq_offsets, const int32_t* num_targets,
                              int32_t B, int32_t H, int32_t d, int32_t total, int32_t max_seq_len,
                              float alpha, float N,
                              void* workspace, int64_t workspace_bytes, void* y, void* stream);

/*
 * hstu_attn_selfcheck_wait_timeout — exercises the failure-detection path on `stream`: one
 * thread of a one-warp kernel waits, through the same bounded mbarrier wait every role of the
 * attention kernel uses, on a barrier that nothing arrives on.  After limit_ns nanoseconds
 * (1 .. 1e9) the wait gives up, sets the timeout bit of the device error word and the kernel
 * returns; the next hstu_attn_get_error on the device reports HSTU_ERR_TIMEOUT and clears it.
 * Nothing traps or hangs and the context stays usable.  Returns HSTU_ERR_INVALID_ARGUMENT for
 * a limit outside the range, HSTU_ERR_CUDA if the launch fails, else HSTU_OK.  The pages have
 * no counterpart: this is a test hook of the library's own failure handling.
 */
hstu_status_t hstu_attn_selfcheck_wait_timeout(uint64_t limit_ns, void* stream);

/*
 * hstu_attn_selfcheck_fwd_timeout — exercises the attention kernel's own abort path: the same work
 * as hstu_attn_fwd, but every pipeline wait of the attention kernel gives up after limit_ns
 * nanoseconds (1 .. 1e9) instead of the normal 4 s.  A wait that runs out sets the timeout bit of
 * the device error word and raises the CTA's abort flag; every role then leaves its loop, waits
 * (each wait at most 0.2 s) for the copies and MMAs it issued, TMEM is freed and the kernel
 * returns, so the next hstu_attn_get_error reports HSTU_ERR_TIMEOUT and the context stays usable.
 * `out` is left partly written.  Arguments and errors as in hstu_attn_fwd, plus
 * HSTU_ERR_INVALID_ARGUMENT for a limit outside the range.  The pages have no counterpart: this is
 * a test hook of the library's own failure handling.
 */
hstu_status_t hstu_attn_selfcheck_fwd_timeout(const void* q, const void* k, const void* v,
                                              const int32_t* seq_offsets, const int32_t* num_targets,
                                              int32_t B, int32_t H, int32_t d,
                                              int32_t total_tokens, int32_t max_seq_len,
                                              float alpha, float N, void* out,
                                              uint64_t limit_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* HSTU_ATTN_H_ */
