/*
 * moe.h -- C ABI of libmoe.so: a routed-expert Mixture-of-Experts layer with
 * decoupled top-k1 / top-k2 renormalisation, for NVIDIA B200 (sm_100a).
 *
 * The method ("Paper of the Week #3 -- Half the FLOPs Is Not Half the Time",
 * sotaaz.com, section "The Receipt", Eq. 2):
 *
 *     z = x W_r^T (+ b)                         router logits
 *     p = softmax(z)  in float32                over the E experts
 *     w_i = p_i / sum_{j in Top-k2} p_j         for i in Top-k1
 *           (k2 = k1: standard renormalisation; k2 >= E: no renormalisation)
 *     y = sum_{i in Top-k1} w_i * FFN_i(x)      FFN_i a SwiGLU gated MLP
 *
 * Each routed expert is a gated MLP whose channel c owns gate row c, up row c
 * and down column c ("Channel Selection for Mixture-of-Experts Decoding Needs
 * No Calibration Data", paperlayer.ai, section 2 "Background"):
 *     h_c = silu(W_gate[c,:] . x) * (W_up[c,:] . x),  o = W_down h.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Pointers named *_bf16 point to bfloat16 data, *_f32/float* to float32,
 *    int32_t* to 32-bit integers.  All tensors are dense row-major.
 *  - All data pointers are DEVICE pointers, owned by the caller, 16-byte
 *    aligned; they must stay valid until the work queued on `stream` ends.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Every call only enqueues work: none synchronises, none
 *    allocates or frees device memory (moe_read_device_status is the one
 *    call that synchronises).
 *  - Shapes: T tokens (T >= 0; T = 0 is a no-op), hidden size d, E experts,
 *    expert intermediate size I (channels), k1 experts run per token, k2
 *    experts in the reference mass.  Requirements: 1 <= k1 <= k2,
 *    k1 <= min(E, 32), 1 <= E <= 1024, d % 64 == 0, I % 16 == 0,
 *    64 <= d <= 8192, 16 <= I <= 8192.  k2 > E is accepted and means
 *    k2 = E (no renormalisation), as the page's min(k2, E) does.
 *  - Routing is deterministic: probabilities are ranked by (p descending,
 *    expert index ascending); the float32 softmax and the top-k2 mass follow
 *    one fixed sequence of float32 operations, so indices and weights are
 *    bit-identical to the CPU oracle that follows the same sequence.
 *  - Weight layouts (per expert e): w_gate, w_up [E x I x d] (row c of
 *    expert e = channel c), w_down [E x d x I] (column c = channel c),
 *    w_router [E x d], bias [E] float32 (nullable).
 *  - Return value: MOE_OK or a negative moe_status.  Argument checks happen
 *    on the host before anything is enqueued; on an error nothing is
 *    enqueued.  MOE_ERR_CUDA means a launch failed (the CUDA error is left
 *    for cudaGetLastError).  Problems found on the device (a bounded wait
 *    that gave up, an index out of range) are recorded in the workspace's
 *    status word; read it with moe_read_device_status.
 *  - Workspace: `ws` is caller-owned device memory of at least
 *    moe_workspace_size(...) bytes, 256-byte aligned, initialised once with
 *    moe_workspace_init before its first use.  Calls leave it initialised.
 *    Calls that share one workspace must be ordered on one stream.
 */
#ifndef MOE_H
#define MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = -1,         /* null pointer, k1/k2 out of range, misaligned pointer   */
    MOE_ERR_UNSUPPORTED_SHAPE = -2,   /* d, I, E, T outside the supported limits                */
    MOE_ERR_WORKSPACE_TOO_SMALL = -3, /* ws_bytes < moe_workspace_size(...)                     */
    MOE_ERR_CUDA = -4,                /* a CUDA runtime call failed                             */
    MOE_ERR_TIMEOUT = -5,             /* device status: a bounded wait gave up                  */
    MOE_ERR_DEVICE_CHECK = -6,        /* device status: an index check failed on the device     */
    MOE_ERR_SCRATCH_LIMIT = -7        /* moe_expert_ffn_noalloc: shapes exceed its fixed scratch */
} moe_status;

/* Output element types for moe_combine / moe_layer. */
#define MOE_DTYPE_F32 0
#define MOE_DTYPE_BF16 1

/* An unused slot of a variable-k (cascade) route: its topk_idx entry; its
 * weight is 0.  The permutation skips such slots without a device check. */
#define MOE_EMPTY_SLOT 0x7fffffff

/* moe_layer / moe_expert_ffn flags: which expert-FFN path runs.
 * AUTO: up to eight tokens with the channel-major down matrix -> DECODE; two or more
 * tokens with d and I multiples of 128 -> GROUPED; otherwise STREAM. */
#define MOE_PATH_AUTO 0
#define MOE_PATH_STREAM 1  /* two-phase weight streaming on CUDA cores, deterministic
                              output                                                  */
#define MOE_PATH_GROUPED 2 /* grouped GEMMs on the tcgen05 tensor cores (d, I multiples
                              of 128); h rounded to bf16 before the down projection;
                              the float32 combine runs in a timing-dependent order, so
                              y may differ between runs in the last bits              */
#define MOE_PATH_DECODE 3  /* 1 <= T <= 8 tokens: a single pass over the union of the
                              routed experts with the down matrix channel-major (needs
                              MOE_WDOWN_CHANNEL_MAJOR);
                              the float32 sum into y runs in a timing-dependent order,
                              so y may differ between runs in the last bits           */
#define MOE_PATH_MASK 0xff
/* moe_layer flag bit: w_down points to the channel-major copy [E x I x d] made
 * by moe_pack_w_down (down column c of expert e is then contiguous). */
#define MOE_WDOWN_CHANNEL_MAJOR 0x100

/* Human-readable text for a moe_status value.  Never NULL. */
const char *moe_status_string(int status);

/* Library version, major*10000 + minor*100 + patch. */
int moe_version(void);

/* Bytes of workspace the calls below need for these shapes (the maximum over
 * moe_route, moe_permute, moe_expert_ffn and moe_layer, on either path).
 * Returns 0 when the shapes are invalid. */
size_t moe_workspace_size(int T, int d, int E, int I, int k1);

/* Zero the whole workspace: the header (status word, the counters and flags
 * the kernels use for cross-block hand-off) and the accumulators the kernels
 * keep zero between calls.  Enqueued on `stream`.  Call it once before the
 * first use, and again after a call recorded MOE_ERR_TIMEOUT. */
int moe_workspace_init(void *ws, size_t ws_bytes, void *stream);

/* Copy the workspace's device status word into *status_out (MOE_OK or a
 * device-side moe_status) and clear it.  Synchronises `stream`. */
int moe_read_device_status(void *ws, int *status_out, void *stream);

/* Router: logits, float32 softmax, top-k1 of the ranking, Eq. 2 weights.
 * ("Paper of the Week #3", sections "The Receipt" (Eq. 2) and "Ship It /
 * Code of the Week": logits = linear(x, W_r); probs = softmax in float32;
 * topk(probs, min(k2, E)); first k1; divided by the sum of all min(k2, E)
 * taken probabilities unless k2 >= E.)
 *
 *  x_bf16 == NULL : `logits` is an INPUT [T x E] float32; w_router_bf16 and
 *                   bias are ignored (this is the entry that routes given
 *                   logits, used for bit-exact comparison).
 *  x_bf16 != NULL : x [T x d] bf16, w_router [E x d] bf16, bias [E] float32
 *                   or NULL; `logits` (nullable) receives x W_r^T + b as
 *                   float32 [T x E] (float32 accumulation).
 *  topk_idx [T x k1] int32: expert ids in rank order.
 *  topk_w   [T x k1] float32: Eq. 2 weights aligned with topk_idx.
 *  ws: workspace (needed only when x_bf16 != NULL and logits == NULL; may be
 *      NULL otherwise). */
int moe_route(const void *x_bf16, const void *w_router_bf16, const float *bias, float *logits,
              int T, int d, int E, int k1, int k2, int32_t *topk_idx, float *topk_w, void *ws,
              size_t ws_bytes, void *stream);

/* Stable counting sort of the T*k1 routed slots by expert (slot i = t*k1+s,
 * the s-th expert of token t).  The grouping the expert FFN needs: every
 * expert's tokens become one contiguous run.
 *  expert_offsets [E+1]: exclusive scan of the per-expert slot counts;
 *  sorted_slot [T*k1]: slots ordered by (expert, slot index);
 *  slot_pos    [T*k1]: inverse, sorted_slot[slot_pos[i]] == i.
 *  An expert id outside [0, E) sets MOE_ERR_DEVICE_CHECK in the device status
 *  word when ws is given (the slot is then dropped).  Slots holding
 *  MOE_EMPTY_SLOT (variable-k routes) are skipped without a check; their
 *  slot_pos entries are left as they were.  ws may be NULL. */
int moe_permute(const int32_t *topk_idx, int T, int k1, int E, int32_t *expert_offsets,
                int32_t *sorted_slot, int32_t *slot_pos, void *ws, size_t ws_bytes, void *stream);

/* Expert FFN for every routed slot (unweighted):
 *  out[p, :] = W_down[e] (silu(W_gate[e] x_t) * (W_up[e] x_t))  (float32)
 * for sorted position p in [expert_offsets[e], expert_offsets[e+1]), where
 * t = sorted_slot[p] / k1.  out is [T*k1 x d] float32 in sorted order.
 * ("Channel Selection ...", section 2: channel c = gate row c, up row c,
 * down column c.)  Accumulation is float32; x and the weights are bf16.
 * flags: MOE_PATH_*.  ws: workspace. */
int moe_expert_ffn(const void *x_bf16, const int32_t *expert_offsets, const int32_t *sorted_slot,
                   const void *w_gate_bf16, const void *w_up_bf16, const void *w_down_bf16, int T,
                   int d, int E, int I, int k1, float *out, int flags, void *ws, size_t ws_bytes,
                   void *stream);

/* Weighted combine (Eq. 2 weights):
 *  y[t, :] = sum_{s=0}^{k1-1} topk_w[t, s] * expert_out[slot_pos[t*k1+s], :]
 * summed in s order in float32; y is [T x d] of y_dtype (MOE_DTYPE_*). */
int moe_combine(const float *expert_out, const int32_t *slot_pos, const float *topk_w, int T,
                int d, int k1, void *y, int y_dtype, void *stream);

/* The whole layer: router (as moe_route), permutation, expert FFN and
 * combine.  y [T x d] of y_dtype.  Optional outputs (each nullable):
 * topk_idx_out / topk_w_out [T x k1], logits_out [T x E] float32.
 * flags: MOE_PATH_* | MOE_WDOWN_CHANNEL_MAJOR.  With the HF down layout
 * [E x d x I] the two-phase streaming path runs (deterministic).  With
 * MOE_WDOWN_CHANNEL_MAJOR (w_down from moe_pack_w_down) and 1 <= T <= 8 the
 * single-pass decode path runs, each routed expert's weights read once for
 * all the tokens routed to it (2 <= T <= 4: d <= 5632; 5 <= T <= 8:
 * d <= 2816; T * k1 <= 64); other shapes return MOE_ERR_UNSUPPORTED_SHAPE.
 * ws: workspace. */
int moe_layer(const void *x_bf16, const void *w_router_bf16, const float *bias,
              const void *w_gate_bf16, const void *w_up_bf16, const void *w_down_bf16, int T, int d,
              int E, int I, int k1, int k2, void *y, int y_dtype, int32_t *topk_idx_out,
              float *topk_w_out, float *logits_out, int flags, void *ws, size_t ws_bytes,
              void *stream);

/* Variable number of experts per token (the "cascade ... cover" arm of
 * "Reading the MoE measurement defects", kozo-lab, sections 4 and 6.2-6.3:
 * each token runs experts in rank order until they cover a share tau of its
 * probability mass).  Reading taken here: the mass after k experts is the
 * float32 sum of the first k ranked probabilities in rank order (the same
 * partial sums as the top-k2 mass of Eq. 2); token t takes k_t = the smallest
 * k <= k1 whose mass is >= tau, else k1 (so 1 <= k_t <= k1).  Its weights are
 * Eq. 2 with the fixed k2.  Routing outputs keep k1 slots per token; slots
 * s >= k_t hold MOE_EMPTY_SLOT with weight 0.  topk_count [T] int32
 * (nullable) receives k_t.  tau NaN: MOE_ERR_INVALID_ARG.  Other arguments
 * as for moe_route. */
int moe_route_cascade(const void *x_bf16, const void *w_router_bf16, const float *bias,
                      float *logits, int T, int d, int E, int k1, int k2, float tau,
                      int32_t *topk_idx, float *topk_w, int32_t *topk_count, void *ws,
                      size_t ws_bytes, void *stream);

/* moe_layer with the variable-k route of moe_route_cascade: y[t] sums only
 * the token's k_t experts.  Runs on the decode path (down matrix
 * channel-major, up to eight tokens) and on the tensor-core grouped path (d, I multiples of 128);
 * other shapes return MOE_ERR_UNSUPPORTED_SHAPE.  topk_count_out [T] int32
 * (nullable) receives k_t.  Other arguments as for moe_layer. */
int moe_layer_cascade(const void *x_bf16, const void *w_router_bf16, const float *bias,
                      const void *w_gate_bf16, const void *w_up_bf16, const void *w_down_bf16,
                      int T, int d, int E, int I, int k1, int k2, float tau, void *y, int y_dtype,
                      int32_t *topk_idx_out, float *topk_w_out, int32_t *topk_count_out,
                      float *logits_out, int flags, void *ws, size_t ws_bytes, void *stream);

/* Expert skipping with the top-1 expert always kept (the shell of "ACE",
 * aimodeling.com, section "How ACE decides what to skip: GSP + RCR": a slot
 * is skipped only when two views both call it low, and the top-1 expert is
 * never skipped).  Reading taken here: the first view is a per-expert scalar
 * table looked up at inference (expert_score [E] float32, device, 16-byte
 * aligned; the page's offline statistic, supplied by the caller), the second
 * is the slot's own Eq. 2 weight (the token's router-conditioned view).  Slot
 * s >= 1 of token t is skipped when expert_score[e] < theta_expert AND
 * topk_w[t, s] < theta_weight; skipped slots hold MOE_EMPTY_SLOT with weight
 * 0, kept slots keep their Eq. 2 weights (no renormalisation over the kept
 * set), and topk_count [T] (nullable) receives the kept count.  A NaN
 * threshold or a null table: MOE_ERR_INVALID_ARG.  moe_layer_skip runs on the
 * same paths as moe_layer_cascade.  Other arguments as for moe_route /
 * moe_layer. */
int moe_route_skip(const void *x_bf16, const void *w_router_bf16, const float *bias,
                   float *logits, int T, int d, int E, int k1, int k2, const float *expert_score,
                   float theta_expert, float theta_weight, int32_t *topk_idx, float *topk_w,
                   int32_t *topk_count, void *ws, size_t ws_bytes, void *stream);
int moe_layer_skip(const void *x_bf16, const void *w_router_bf16, const float *bias,
                   const void *w_gate_bf16, const void *w_up_bf16, const void *w_down_bf16, int T,
                   int d, int E, int I, int k1, int k2, const float *expert_score,
                   float theta_expert, float theta_weight, void *y, int y_dtype,
                   int32_t *topk_idx_out, float *topk_w_out, int32_t *topk_count_out,
                   float *logits_out, int flags, void *ws, size_t ws_bytes, void *stream);

/* Channel top-k inside the activated experts ("Channel Selection for
 * Mixture-of-Experts Decoding Needs No Calibration Data", paperlayer.ai,
 * sections 2, 5.2 and 5.3).  Per token, every channel (s, c) of its k1 routed
 * experts (slot s in rank order, channel c < I; flat index q = s*I + c) gets
 * the output-scaled score
 *     score[q] = (w_s * n[e_s][c]) * |h_c|     (two float32 products),
 * the norm of that channel's contribution to y; the token keeps the `keep`
 * channels with the largest scores over all its slots (equal scores go to
 * the lower q) and
 *     y[t, :] = sum over kept q of w_s * h_q * W_down[e_s][:, c]
 * (kept channels exact; skipped channels add nothing: the pages' ternary
 * sketch and low-rank recovery are not part of this call).  h is computed
 * exactly for every channel, so every gate and up row of the routed experts
 * is read; only the kept channels' down columns are.
 *
 * moe_channel_norms: n[e][c] = ||W_down[e][:, c]||_2 in float32 (float32
 *   sum of squares, IEEE square root), norms [E x I] float32, from w_down in
 *   the HF layout [E x d x I] (flags 0) or channel-major [E x I x d]
 *   (flags MOE_WDOWN_CHANNEL_MAJOR, from moe_pack_w_down).  Computed once
 *   when the weights are loaded.
 * moe_layer_channel_topk: the layer with channel top-k.  w_down_cm is the
 *   channel-major down matrix (moe_pack_w_down), norms from
 *   moe_channel_norms.  1 <= keep <= k1*I <= 16384.  Tokens run one after
 *   another (two kernels each).  Optional outputs (each nullable):
 *   topk_idx_out / topk_w_out [T x k1], logits_out [T x E], h_out and
 *   scores_out [T x k1 x I] float32, kept_out [T x keep] int32 (the kept
 *   flat indices q, ascending).  Scores, h and the kept set are
 *   deterministic; y sums the kept channels in a timing-dependent order (last
 *   bits may differ between runs).  Non-finite activations leave the kept set
 *   unspecified.  Other arguments and the workspace as for moe_layer. */
int moe_channel_norms(const void *w_down_bf16, int E, int d, int I, int flags, float *norms,
                      void *stream);
int moe_layer_channel_topk(const void *x_bf16, const void *w_router_bf16, const float *bias,
                           const void *w_gate_bf16, const void *w_up_bf16, const void *w_down_cm_bf16,
                           const float *norms, int T, int d, int E, int I, int k1, int k2, int keep,
                           void *y, int y_dtype, int32_t *topk_idx_out, float *topk_w_out,
                           float *logits_out, float *h_out, float *scores_out, int32_t *kept_out,
                           void *ws, size_t ws_bytes, void *stream);

/* Channel-major copy of a down matrix, made once when the weights are
 * loaded: w_down_cm[e][c][r] = w_down[e][r][c] (w_down [E x d x I] bf16 ->
 * w_down_cm [E x I x d] bf16, separate buffers).  The channel decomposition
 * of a routed expert ("Channel Selection for Mixture-of-Experts Decoding
 * Needs No Calibration Data", section 2: channel c owns down column c) then
 * reads each channel's down column as one contiguous row.  Enqueued on
 * `stream`. */
int moe_pack_w_down(const void *w_down_bf16, void *w_down_cm_bf16, int E, int d, int I,
                    void *stream);

/* moe_expert_ffn without a caller workspace.  The paper has no counterpart;
 * this entry exists for callers that cannot hand the library device memory
 * for scratch: plugins running inside an engine that owns the whole device
 * memory pool, services that fix their memory footprint at start-up and treat
 * any later allocation as a fault, and bindings that can pass pointers they
 * were given but have no way to allocate device memory themselves.
 *
 * Same inputs, output and result as moe_expert_ffn (flags are not taken: it
 * always uses the weight-streaming path).  Its scratch is a fixed array
 * compiled into libmoe.so (a little over 4 MiB per GPU that loads the library,
 * held until the process exits); the call itself allocates and frees nothing.
 *  - Limit: T * k1 * I <= 1047424 (the float32 channel activations of all
 *    routed slots must fit the array), and the usual shape limits; larger
 *    shapes return MOE_ERR_SCRATCH_LIMIT and enqueue nothing.
 *  - The first call on a device looks up the array's device address (once
 *    per device, with that device current) and keeps it for the life of the
 *    process; make that first call outside any stream capture.  The address
 *    is not looked up again, so calls after cudaDeviceReset on that device
 *    are not supported.
 *  - Every call on a device shares the one array, and each call clears the
 *    part that must start at zero.  Calls whose work overlaps on the GPU
 *    (e.g. on two streams at once) race on the array; order them on one
 *    stream.
 *  - Device-side problems (a bounded wait that gave up, an index check)
 *    leave out unspecified and are recorded in the array's status word,
 *    which calls do not clear: read it with moe_noalloc_read_status. */
int moe_expert_ffn_noalloc(const void *x_bf16, const int32_t *expert_offsets,
                           const int32_t *sorted_slot, const void *w_gate_bf16,
                           const void *w_up_bf16, const void *w_down_bf16, int T, int d, int E,
                           int I, int k1, float *out, void *stream);

/* The device status word of moe_expert_ffn_noalloc on the current device:
 * copied into *status_out (host memory; MOE_OK or the first device-side
 * moe_status any call recorded since the last read) and cleared.  Enqueued on
 * `stream` after the calls to check, then synchronises `stream`.  Allocates
 * nothing.  The paper has no counterpart. */
int moe_noalloc_read_status(int *status_out, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H */
