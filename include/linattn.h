/*
 * linattn.h — C ABI of the B200 (sm_100a) kernelized linear-attention library
 * (liblinattn.so).  Feature map phi(x) = elu(x) + 1, alpha = 1.
 *
 * The operations follow:
 *   - "Linear Attention" knowledge-base page (lizeman.github.io/llm-arch-kb),
 *     section 2 "Derivation" (state S = sum phi(k) v^T, normaliser
 *     z = sum phi(k), read-out phi(q)^T S / phi(q)^T z; the causal recurrence)
 *     and section 3 "Reference implementation" (non-causal sums, the per-token
 *     causal loop, eps = 1e-6 added to the denominator);
 *   - the linear-attention concept card (wikillm.com), "Implementation sketch"
 *     (optional per-token scalar decay: state = a*state + outer(phi(k), v),
 *     norm = a*norm + phi(k)) and its "Decaying linear attention with a scalar
 *     state (SSD)" variant (decay 1 is the plain form; chunked algorithm with
 *     exact products inside each chunk and a recurrence between chunks);
 *   - the linear-attention lesson (learn.pranaymahendrakar.com), Researcher
 *     level "Derivation" (o_i over j <= i) and "Implementation reality"
 *     (chunks of 64 or 128, state propagated across chunks).
 *
 * Conventions common to every entry point
 *   - All tensor pointers are DEVICE pointers to contiguous row-major arrays,
 *     16-byte aligned.  The caller owns every buffer, including the workspace;
 *     the library never allocates device memory and never synchronises
 *     (except la_workspace_status and la_noalloc_status, which read a status
 *     word back to the host).
 *   - Calls are asynchronous on `stream` (a cudaStream_t passed as void*;
 *     NULL = the legacy default stream).  Every argument error detectable on
 *     the host is reported before anything is launched, and nothing is then
 *     written.  A failed launch returns LA_ERR_CUDA.
 *   - Every wait inside the tensor-core kernels (on a copy, a tensor-core
 *     product or another warp of the same block) is bounded (~2 s, see
 *     la_set_wait_limit_ns).  A wait that runs out ends its block early and
 *     leaves LA_ERR_TIMEOUT in the call's status word, at the start of the
 *     workspace; the output and state of that call are then incomplete.  The
 *     entry point itself has already returned LA_OK by then (calls are
 *     asynchronous): read the status with la_workspace_status.
 *   - Heads are independent: q, k [B, H, T, d_k], v [B, H, T, d_v],
 *     out [B, H, T, d_v]; state S [B, H, d_k, d_v] and z [B, H, d_k], fp32.
 *   - Supported: d_k == d_v in {32, 64, 128}; in_dtype in {F32, BF16, F16};
 *     out_dtype == in_dtype or LA_F32; B*H <= 65535.  Anything else:
 *     LA_ERR_UNSUPPORTED.
 *   - eps must be finite and >= 0 (it is added to the denominator).
 *   - decay values must lie in (0, 1]; this is a precondition, not checked
 *     on the device.  decay == NULL means no decay (a = 1 everywhere).
 *   - Results are deterministic run to run (no floating-point atomics).
 */
#ifndef LINATTN_H
#define LINATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { LA_F32 = 0, LA_BF16 = 1, LA_F16 = 2 } la_dtype;

typedef enum {
    LA_OK = 0,
    LA_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, negative size, bad eps, short workspace */
    LA_ERR_UNSUPPORTED = 2,  /* valid but not implemented: head dim, chunk, dtype combination */
    LA_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed */
    LA_ERR_TIMEOUT = 4       /* a bounded device-side wait gave up (status word set) */
} la_status;

/* State handling of the prefill / non-causal calls.
 *   NONE : start from zeros; state_S/state_z are not read or written (may be NULL).
 *   OUT  : start from zeros; the final state is written to state_S/state_z.
 *   INOUT: state_S/state_z hold the initial state and receive the final one
 *          (in place). */
typedef enum { LA_STATE_NONE = 0, LA_STATE_OUT = 1, LA_STATE_INOUT = 2 } la_state_mode;

/*
 * Causal prefill (chunked).  For every head and every token t:
 *   S_t = a_t S_{t-1} + phi(k_t) v_t^T,   z_t = a_t z_{t-1} + phi(k_t),
 *   out_t = phi(q_t)^T S_t / (phi(q_t)^T z_t + eps)
 * computed chunk by chunk: exact masked products inside each chunk of `chunk`
 * tokens, the (S, z) state carried between chunks (segments of chunks run in
 * parallel and are joined by a decayed prefix scan over their states).
 *   q, k       [B, H, T, d_k] in_dtype        v [B, H, T, d_v] in_dtype
 *   decay      [B, H, T] fp32 in (0, 1], or NULL
 *   chunk      64 or 128
 *   out        [B, H, T, d_v] out_dtype
 *   workspace  device scratch of at least la_prefill_workspace_size(...)
 *              bytes, 256-byte aligned; contents on entry are ignored.
 * T == 0 (or B*H == 0) is valid: nothing is computed; with LA_STATE_OUT the
 * state is set to zero, with LA_STATE_INOUT it is left unchanged.
 */
la_status la_prefill_causal(const void *q, const void *k, const void *v, la_dtype in_dtype,
                            const float *decay, int B, int H, int T, int d_k, int d_v,
                            float eps, int chunk, float *state_S, float *state_z,
                            la_state_mode mode, void *out, la_dtype out_dtype,
                            void *workspace, size_t workspace_bytes, void *stream);

/*
 * la_prefill_causal_ev — la_prefill_causal that also records caller-owned
 * CUDA events on `stream` at the boundaries of the kernels it launches, so a
 * caller can time each pass on the device without synchronising:
 *   events[0] before the state pass (K1), events[1] before the segment scan,
 *   events[2] before the output pass, events[3] after it.
 * `events` is NULL (then this is la_prefill_causal) or an array of 4
 * cudaEvent_t created by the caller (a NULL entry is skipped); the library
 * records them and never creates, waits on or destroys them.  A failed record
 * returns LA_ERR_CUDA.  On the T == 0 / B*H == 0 paths nothing is recorded.
 */
la_status la_prefill_causal_ev(const void *q, const void *k, const void *v, la_dtype in_dtype,
                               const float *decay, int B, int H, int T, int d_k, int d_v,
                               float eps, int chunk, float *state_S, float *state_z,
                               la_state_mode mode, void *out, la_dtype out_dtype,
                               void *workspace, size_t workspace_bytes, void *stream,
                               void *const *events);

/*
 * la_prefill_causal_gated — the causal prefill with a per-token gain b_t on
 * the new term (the gated form):
 *   S_t = a_t S_{t-1} + b_t phi(k_t) v_t^T,   z_t = a_t z_{t-1} + b_t phi(k_t),
 *   out_t = phi(q_t)^T S_t / (phi(q_t)^T z_t + eps).
 * Random Feature Attention's sigmoid gate g_t (concept card "Linear
 * attention", RFA variant and the closing paragraph of its implementation
 * sketch; RFA eq. 7) is decay = g, gain = 1 - g; NodeFormer's per-key
 * multiplier is a gain without decay.
 *   gain   [B, H, T] fp32, finite and >= 0 (a documented precondition, not
 *          checked on the device), 16-byte aligned, or NULL (b = 1: this is
 *          la_prefill_causal).
 * Every other argument, the workspace size and the error behaviour are those
 * of la_prefill_causal.
 */
la_status la_prefill_causal_gated(const void *q, const void *k, const void *v, la_dtype in_dtype,
                                  const float *decay, const float *gain, int B, int H, int T,
                                  int d_k, int d_v, float eps, int chunk, float *state_S,
                                  float *state_z, la_state_mode mode, void *out, la_dtype out_dtype,
                                  void *workspace, size_t workspace_bytes, void *stream);

/*
 * la_prefill_causal_mlstm — the causal prefill with the mLSTM read-out
 * (concept card "Linear attention", "Matrix memory with exponential gates
 * (mLSTM)": C_t = f_t C_{t-1} + i_t v_t k_t^T, n_t = f_t n_{t-1} + i_t k_t,
 * h_t = C_t q_t / max(|n_t^T q_t|, 1); the card's implementation sketch fits
 * it to the running-sum loop with the identity as the feature map).  In this
 * library's terms, with S = C^T and z = n:
 *   S_t = f_t S_{t-1} + i_t k_t v_t^T,   z_t = f_t z_{t-1} + i_t k_t,
 *   out_t = q_t^T S_t / max(|q_t^T z_t|, 1)          (no feature map, no eps)
 *   forget      [B, H, T] fp32 in (0, 1], or NULL (f = 1)
 *   input_gate  [B, H, T] fp32, finite and >= 0 (an exponential gate's value;
 *               the stabiliser state of exponential gating is the caller's),
 *               or NULL (i = 1)
 * Both are 16-byte aligned; the state carries the raw keys.  Other arguments,
 * the workspace size and the error behaviour are those of la_prefill_causal.
 */
la_status la_prefill_causal_mlstm(const void *q, const void *k, const void *v, la_dtype in_dtype,
                                  const float *forget, const float *input_gate, int B, int H, int T,
                                  int d_k, int d_v, int chunk, float *state_S, float *state_z,
                                  la_state_mode mode, void *out, la_dtype out_dtype, void *workspace,
                                  size_t workspace_bytes, void *stream);

/*
 * la_prefill_causal_flash — the FLASH chunk form (concept card "Linear
 * attention", "Chunked attention: exact inside blocks, linear across them
 * (FLASH)", and the closing paragraph of its implementation sketch): the
 * sequence is cut into chunks of `chunk` tokens; inside a chunk, exact
 * squared-ReLU attention over the chunk's earlier tokens; across chunks, a
 * linear term read from the summaries of the earlier chunks.  For token t in
 * chunk g, with s = 1 (scaled = 0: the card's equations) or s = chunk
 * (scaled = 1: its listings, also for a shorter last chunk):
 *   out_t = sum_{j <= t, j in g} relu(q_t . k_j / s)^2 v_j
 *         + q_t^T (sum_{j in chunks before g} k_j v_j^T) / s
 * No feature map and no normaliser (softmax-free); the chunk is part of the
 * definition here, not only a blocking choice.  The state is the raw running
 * sum over every token processed:
 *   state_S = sum_j k_j v_j^T   [B, H, d_k, d_v],   state_z = sum_j k_j   [B, H, d_k]
 * (the read-out divides it by s), so a hand-off through the state continues
 * the same chunking when the earlier part's length is a multiple of `chunk`.
 * Tensor-core path only: in_dtype BF16 or F16, d_k = d_v in {64, 128},
 * chunk 64 or 128; otherwise LA_ERR_UNSUPPORTED.  scaled not 0 or 1:
 * LA_ERR_INVALID_ARG.  The workspace size and every other argument and error
 * are those of la_prefill_causal.
 */
la_status la_prefill_causal_flash(const void *q, const void *k, const void *v, la_dtype in_dtype,
                                  int B, int H, int T, int d_k, int d_v, int chunk, int scaled,
                                  float *state_S, float *state_z, la_state_mode mode, void *out,
                                  la_dtype out_dtype, void *workspace, size_t workspace_bytes,
                                  void *stream);

/*
 * Sequence sharding (one sequence's tokens split over several GPUs, in
 * order).  The causal recurrence is affine in the state: a shard maps an
 * entry state X to A X + dX, with
 *   dS = sum_j w_j b_j phi(k_j) v_j^T,  dz = sum_j w_j b_j phi(k_j),
 *   A = prod_t a_t over the shard,  w_j = prod_{t > j in the shard} a_t
 * (concept card "Linear attention", SSD variant: the chunked algorithm's
 * recurrence between blocks, here between shards).  Each rank summarises
 * its shard (la_prefill_causal_summary), the ranks exchange the summaries
 * (an all-gather, done by the caller, e.g. NCCL), each rank folds the
 * summaries of the shards before its own into its entry state
 * (la_state_combine), and runs la_prefill_causal on its shard with that
 * state as LA_STATE_INOUT.
 *
 * la_prefill_causal_summary: dS -> sum_S [B, H, d_k, d_v], dz -> sum_z
 * [B, H, d_k], A -> sum_A [B, H] (fp32, 16-byte aligned, required) for the
 * elu+1 forms (decay and gain optional, as in la_prefill_causal_gated).
 * Takes no queries and writes no output; the workspace is
 * la_prefill_workspace_size(B, H, T, d_k, d_v, chunk) bytes (T == 0 gives
 * (0, 0, 1) and needs 256 bytes).  Other arguments and errors as
 * la_prefill_causal.
 */
la_status la_prefill_causal_summary(const void *k, const void *v, la_dtype in_dtype, const float *decay,
                                    const float *gain, int B, int H, int T, int d_k, int d_v, int chunk,
                                    float *sum_S, float *sum_z, float *sum_A, void *workspace,
                                    size_t workspace_bytes, void *stream);

/*
 * la_state_combine: the entry state of shard r of R from the gathered
 * summaries, X_0 = (S_in, z_in) or zeros (both NULL), X_{i+1} = A_i X_i + dX_i,
 * written to (S_out, z_out) = X_r.
 *   S_all [R, B, H, d_k, d_v], z_all [R, B, H, d_k], A_all [R, B, H]: fp32,
 *   the shards' la_prefill_causal_summary outputs in shard order (may be NULL
 *   when r == 0).  S_out [B, H, d_k, d_v], z_out [B, H, d_k] must not overlap
 *   the inputs.  Errors: LA_ERR_INVALID_ARG for r outside [0, R) or missing
 *   buffers, LA_ERR_UNSUPPORTED for head dims other than 32, 64, 128.
 */
la_status la_state_combine(const float *S_all, const float *z_all, const float *A_all, int R, int r, int B,
                           int H, int d_k, int d_v, const float *S_in, const float *z_in, float *S_out,
                           float *z_out, void *stream);

/* Bytes of workspace la_prefill_causal needs for these sizes (0 if none). */
size_t la_prefill_workspace_size(int B, int H, int T, int d_k, int d_v, int chunk);

/* Size of the device scratch array behind la_prefill_causal_noalloc. */
#define LA_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)

/*
 * la_prefill_causal_noalloc — la_prefill_causal without a workspace argument.
 * The pages have no counterpart: this exists for callers that cannot allocate
 * device memory at all, such as a plugin hosted by a runtime that owns every
 * device allocation, or a process that forbids allocation after start-up
 * (fixed-budget serving, real-time deployments).
 *
 * The scratch (per-segment states) lives in a fixed array of
 * LA_NOALLOC_SCRATCH_BYTES inside the library's device memory; every GPU that
 * loads the library holds it until the process exits.  The caller still
 * passes inputs, outputs and state exactly as for la_prefill_causal, and gets
 * the same results.  The call allocates nothing (no cudaMalloc, cudaFree or
 * allocating library routine).
 *   - Sizes whose la_prefill_workspace_size exceeds LA_NOALLOC_SCRATCH_BYTES
 *     return LA_ERR_UNSUPPORTED before anything is launched.
 *   - Every call looks up the array's device address (cudaGetSymbolAddress,
 *     which allocates nothing) with the call's device current, so the address
 *     stays right across a teardown of the primary context.  The first call on
 *     a device may load the library's device code; make it before any stream
 *     capture.  LA_ERR_CUDA if the lookup fails.
 *   - The call's status word is in the array: read it with la_noalloc_status.
 *   - All calls share the one array, which keeps the last call's contents;
 *     nothing in it needs to start at zero (every entry is written before it
 *     is read).  Calls that overlap on the GPU (e.g. on two streams at once)
 *     race on the array and corrupt each other's results: serialise them.
 */
la_status la_prefill_causal_noalloc(const void *q, const void *k, const void *v,
                                    la_dtype in_dtype, const float *decay, int B, int H, int T,
                                    int d_k, int d_v, float eps, int chunk, float *state_S,
                                    float *state_z, la_state_mode mode, void *out,
                                    la_dtype out_dtype, void *stream);

/*
 * Non-causal form: every query attends to all Lk keys of its head.
 *   S = S_in + sum_j phi(k_j) v_j^T,  z = z_in + sum_j phi(k_j)
 *   out_i = phi(q_i)^T S / (phi(q_i)^T z + eps)
 * S_in/z_in are zero unless mode == LA_STATE_INOUT.  With OUT or INOUT the
 * totals S, z are written to state_S/state_z.
 *   q [B, H, Lq, d_k]; k [B, H, Lk, d_k]; v [B, H, Lk, d_v]; out [B, H, Lq, d_v]
 *   decay must be NULL (no decayed non-causal form is defined): otherwise
 *   LA_ERR_UNSUPPORTED.
 */
la_status la_forward_noncausal(const void *q, const void *k, const void *v, la_dtype in_dtype,
                               const float *decay, int B, int H, int Lq, int Lk, int d_k,
                               int d_v, float eps, float *state_S, float *state_z,
                               la_state_mode mode, void *out, la_dtype out_dtype,
                               void *workspace, size_t workspace_bytes, void *stream);

/* Bytes of workspace la_forward_noncausal needs for these sizes. */
size_t la_noncausal_workspace_size(int B, int H, int Lk, int d_k, int d_v);

/*
 * One constant-state decode step per head (the causal loop body once):
 *   S <- a S + phi(k) v^T,  z <- a z + phi(k),  out = phi(q)^T S / (phi(q)^T z + eps)
 *   q, k [B, H, d_k] in_dtype; v [B, H, d_v] in_dtype; decay [B, H] fp32 or NULL
 *   state_S [B, H, d_k, d_v], state_z [B, H, d_k]: fp32, required, updated in place
 *   out [B, H, d_v] out_dtype
 */
la_status la_decode_step(const void *q, const void *k, const void *v, la_dtype in_dtype,
                         const float *decay, int B, int H, int d_k, int d_v, float eps,
                         float *state_S, float *state_z, void *out, la_dtype out_dtype,
                         void *stream);

/*
 * One gated decode step: S <- a S + b phi(k) v^T, z <- a z + b phi(k), then
 * the read-out of la_decode_step.  gain [B, H] fp32 (b >= 0, 16-byte aligned)
 * or NULL (b = 1: this is la_decode_step); the RFA gate is decay = g,
 * gain = 1 - g.  Other arguments as la_decode_step.
 */
la_status la_decode_step_gated(const void *q, const void *k, const void *v, la_dtype in_dtype,
                               const float *decay, const float *gain, int B, int H, int d_k,
                               int d_v, float eps, float *state_S, float *state_z, void *out,
                               la_dtype out_dtype, void *stream);

/*
 * One mLSTM decode step (see la_prefill_causal_mlstm):
 *   S <- f S + i k v^T, z <- f z + i k, out = q^T S / max(|q^T z|, 1)
 * forget, input_gate: [B, H] fp32 or NULL (1).  Other arguments as
 * la_decode_step.
 */
la_status la_decode_step_mlstm(const void *q, const void *k, const void *v, la_dtype in_dtype,
                               const float *forget, const float *input_gate, int B, int H, int d_k,
                               int d_v, float *state_S, float *state_z, void *out, la_dtype out_dtype,
                               void *stream);

/*
 * Status of the last call that used `workspace` (a workspace passed to
 * la_prefill_causal*, la_forward_noncausal or la_prefill_causal_noalloc's
 * array): LA_OK, or LA_ERR_TIMEOUT if a bounded device-side wait of that call
 * gave up (its output and state are then incomplete).  *waiter (if non-NULL)
 * receives the id of the first wait that gave up (0 if none), for diagnosis.
 * Unlike every other entry point this one synchronises `stream`: it copies
 * the 8-byte status word to the host on `stream` and waits for it.  Call it on
 * the stream of the call it checks.  LA_ERR_INVALID_ARG for a null or
 * misaligned workspace, LA_ERR_CUDA if the copy fails.  Each call clears the
 * status word of its own workspace before launching anything.
 */
la_status la_workspace_status(const void *workspace, int *waiter, void *stream);

/* la_workspace_status for la_prefill_causal_noalloc, whose status word lives
 * in the library's scratch array (this device's copy). */
la_status la_noalloc_status(int *waiter, void *stream);

/*
 * Sets the limit, in nanoseconds, of every bounded device-side wait of the
 * calls launched after it, process-wide, and returns the previous limit.  The
 * default is 2e9 (2 s).  0 makes every wait that is not already satisfied at
 * its first poll give up at once: a test of the timeout path, not a setting
 * for production.  The drain waits through which a block lets its copies and
 * products in flight complete before it exits keep their own fixed bound.
 */
uint64_t la_set_wait_limit_ns(uint64_t ns);

/* Static description of a status code (never NULL). */
const char *la_status_string(la_status s);

/* Text of the last failure that made an entry point return LA_ERR_CUDA on
 * the calling thread ("<step>: <CUDA error>"), or "" if none.  The pointer
 * stays valid until the thread's next failing call. */
const char *la_last_error_string(void);

/* Which kernel family la_prefill_causal would run for these arguments
 * (has_decay: whether a decay array is passed): 0 = fp32 CUDA-core (SIMT)
 * kernels, 1 = tcgen05 tensor-core kernels, -1 = unsupported.  Host-only,
 * launches nothing.  Tensor cores take 16-bit inputs with d in {64, 128}
 * (either chunk, with or without decay); fp32 inputs and d = 32 run on the
 * CUDA cores. */
int la_prefill_path(la_dtype in_dtype, int d_k, int d_v, int chunk, int has_decay);

/* The segment plan la_prefill_causal uses for these sizes: each head's T
 * tokens are cut into *n_seg segments of *seg_len tokens (the last may be
 * shorter), one CTA per segment.  Host-only, launches nothing.  Returns
 * LA_ERR_INVALID_ARG for negative sizes, null outputs or chunk not in
 * {64, 128}. */
la_status la_prefill_plan(int B, int H, int T, int d_k, int chunk, int *n_seg, int *seg_len);

/* Number of kernels this library has launched in this process so far, over
 * all entry points and devices (kernels later replayed from a captured CUDA
 * graph are counted once, at capture).  Host-only bookkeeping. */
uint64_t la_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* LINATTN_H */
