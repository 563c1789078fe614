/*
 * la2.h -- C ABI of libla2: tiled causal linear attention with per-head decay
 * (the Lightning Attention-2 schedule) for NVIDIA B200 (sm_100a).
 *
 * The operation, per batch b and head h (rows t, j = 0..L-1):
 *
 *     o_t = sum_{j <= t} lambda_h^(t-j) (q_t . k_j) v_j  +  lambda_h^(t+1) q_t kv0
 *
 * i.e. O = (Q K^T (.) M) V with M_tj = lambda_h^(t-j) for j <= t and 0 above
 * the diagonal; lambda_h = 1 is plain causal linear attention.  The
 * Lightning Attention-2 notes page (phantomic12.github.io, "Lightning
 * Attention-2: A Free Lunch for Handling Unlimited Sequence Lengths in Large
 * Language Models", "Tiling." paragraph) describes the schedule used here: an
 * intra-block part done as ordinary dense masked attention and an inter-block
 * part done through the linear-attention state, in forward and backward.  The
 * Lightning Attention glossary page (jisaku.com, section "主な特徴・仕組み")
 * gives the two equivalent forms -- parallel for training, recurrent with a
 * fixed-size state for inference -- that la2_forward/la2_backward and
 * la2_decode_step implement.  The decay lambda_h, the fp32 state and the
 * argument conventions below are this library's definition; the pages give
 * none of them.
 *
 * Conventions common to every call
 *   - All tensor pointers are DEVICE pointers, contiguous row-major:
 *       q, k, dq, dk      [B, H, L, d]
 *       v, o, dO, dv      [B, H, L, e]
 *       states            [B, H, d, e]  fp32 (kv0, kv_out, dkv0, decode kv)
 *       lambda            [H]           fp32, one decay per head
 *     `dt` (LA2_F32 or LA2_BF16) is the element type of q, k, v, o, dO, dq,
 *     dk, dv.  Arithmetic is fp32 (bf16 tensor-core products with fp32
 *     accumulation for LA2_BF16; fp32 FMA for LA2_F32).
 *   - Supported head sizes: d, e in {64, 128}.  With LA2_BF16, la2_forward
 *     and la2_backward run every size on the tensor cores (a 64-column
 *     tensor is read with zero columns up to 128, its states padded to
 *     128 x 128 in workspace scratch, which la2_workspace_size includes);
 *     the other entry points do so for d = e = 128 and use fp32 FMA
 *     kernels for 64.
 *   - Every pointer must be 16-byte aligned.
 *   - The caller owns all memory.  The library allocates nothing on the
 *     device: scratch memory comes from the caller as `workspace`, sized by
 *     la2_workspace_size() for the same arguments.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and never synchronised: results are ready when the stream is.
 *   - Arguments are validated before anything is launched.  A call that
 *     returns an error has enqueued nothing.
 *   - lambda values are read on the device; any finite value is accepted,
 *     values in [0, 1] are the meaningful range (0^0 is taken as 1).
 *   - L, B or H equal to 0 is an empty problem: nothing is computed except
 *     that state outputs are still written (kv_out = kv0 or 0; dkv0 = 0).
 *   - The elementwise feature-map calls (la2_feature_map,
 *     la2_feature_map_backward) take a count of values instead of shapes and
 *     may write in place; their declarations state these exceptions.
 *
 * Errors: LA2_ERR_INVALID for bad arguments (null required pointer, negative
 * size, unaligned pointer, an output overlapping an input, kv_out == kv0,
 * workspace too small); LA2_ERR_UNSUPPORTED for (d, e, dt) outside the
 * supported set; LA2_ERR_CUDA when a launch fails; device-side watchdog
 * expiries are reported later by la2_last_device_error().
 */
#ifndef LA2_H
#define LA2_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#ifndef __CUDA_RUNTIME_API_H__
typedef struct CUstream_st *cudaStream_t;
#endif

typedef enum {
    LA2_OK = 0,
    LA2_ERR_INVALID = 1,
    LA2_ERR_UNSUPPORTED = 2,
    LA2_ERR_CUDA = 3,
    LA2_ERR_TIMEOUT = 4
} la2_status;

typedef enum { LA2_F32 = 0, LA2_BF16 = 1 } la2_dtype;

/* Operation codes for la2_workspace_size(). */
enum { LA2_OP_FORWARD = 0, LA2_OP_BACKWARD = 1, LA2_OP_SHARD_STATE = 2, LA2_OP_DLAMBDA = 3 };

/*
 * Bytes of device scratch that la2_forward (op = LA2_OP_FORWARD),
 * la2_backward (op = LA2_OP_BACKWARD), la2_shard_state (op =
 * LA2_OP_SHARD_STATE) or la2_backward_dlambda_ex (op = LA2_OP_DLAMBDA)
 * needs for these sizes on the CURRENT device.  The scratch holds the fp32
 * d x e states at the boundaries of the
 * sequence chunks that run in parallel (the split of one long sequence over
 * several CTAs); it may be 0 when the sequence is not split.  Returns 0 for
 * unsupported arguments as well; the call then reports the error.
 */
size_t la2_workspace_size(int op, int B, int H, int64_t L, int d, int e,
                          la2_dtype dt);

/*
 * Forward pass.  Writes o [B,H,L,e] and, when kv_out is not NULL, the state
 * after the last row, kv_out = lambda^L kv0 + sum_j lambda^(L-1-j) k_j^T v_j
 * (fp32 [B,H,d,e]), which la2_decode_step or a later la2_forward (as kv0) can
 * continue from.  kv0 may be NULL (zero initial state).
 * Source: Lightning Attention-2 notes page, "Tiling." paragraph (intra-block
 * dense part + inter-block state part); glossary page, FAQ Q1 (aggregate
 * K^T V first, then multiply by Q).
 */
la2_status la2_forward(const void *q, const void *k, const void *v,
                       const float *lambda, const float *kv0,
                       void *o, float *kv_out,
                       int B, int H, int64_t L, int d, int e, la2_dtype dt,
                       void *workspace, size_t workspace_bytes,
                       cudaStream_t stream);

/*
 * Forward pass that allocates nothing and takes no workspace, for callers
 * that cannot call cudaMalloc or any allocating routine (plug-ins whose host
 * framework owns all device memory, latency-critical paths that cannot
 * afford cudaMalloc's device synchronisation, callbacks that only receive
 * device pointers).  The pages have no counterpart of this entry point; it
 * is a convenience of this library.  Arguments, results and errors are those
 * of la2_forward; the chunk-boundary states live instead in a fixed 32 MiB
 * device array that every GPU loading the library holds until the process
 * exits.  Calls whose plan needs more than 32 MiB of states (B*H*S*d*e*4
 * bytes, S = chunks per sequence) return LA2_ERR_UNSUPPORTED before
 * launching anything.  Arguments are checked exactly as la2_forward checks
 * them, before the array is touched.  The first valid call on a device looks
 * up the array's device address (once per device, with that device current)
 * and should come before any stream capture.  The address is kept for the
 * life of the process and belongs to the device's current context: after a
 * cudaDeviceReset() of that device the kept address is stale, so a process
 * that resets a device must not call this entry point on it again.  All
 * calls share the array and it keeps the last call's contents
 * (every state it holds is written before it is read, so nothing needs
 * clearing); calls that overlap on the same GPU -- from concurrent streams
 * or host threads -- race on it, so serialise them.  Each GPU has its own
 * copy of the array.
 */
la2_status la2_forward_noalloc(const void *q, const void *k, const void *v,
                               const float *lambda, const float *kv0,
                               void *o, float *kv_out,
                               int B, int H, int64_t L, int d, int e, la2_dtype dt,
                               cudaStream_t stream);

/*
 * Backward pass for an upstream gradient dO [B,H,L,e]: writes dq, dk [B,H,L,d],
 * dv [B,H,L,e] -- the gradients of sum(o * dO) -- and, when dkv0 is not NULL,
 * the gradient with respect to the initial state (fp32 [B,H,d,e]).  Inputs
 * are those of the forward call (kv0 may be NULL).  dq is found by a forward
 * scan that rebuilds the state; dk and dv by a reverse scan over a second
 * d x e state.
 * Source: Lightning Attention-2 notes page, "Tiling." paragraph (the same
 * tiling applied in the backward pass).
 */
la2_status la2_backward(const void *q, const void *k, const void *v,
                        const float *lambda, const float *kv0, const void *dO,
                        void *dq, void *dk, void *dv, float *dkv0,
                        int B, int H, int64_t L, int d, int e, la2_dtype dt,
                        void *workspace, size_t workspace_bytes,
                        cudaStream_t stream);

/*
 * la2_backward with flags.  LA2_BWD_REUSE_FORWARD_STATES: `workspace`
 * already holds the chunk entry states that la2_forward wrote for the same
 * q, k, v, lambda, kv0 and sizes -- the caller gave la2_forward this same
 * workspace (sized for LA2_OP_BACKWARD) and has not touched it since, with
 * the same split option in force -- so the backward skips recomputing them
 * (one pass over k and v fewer for long sequences).  With stale or foreign
 * contents the gradients are wrong; the library cannot check this.  Unknown
 * flag bits return LA2_ERR_INVALID.  flags = 0 is la2_backward.
 */
enum { LA2_BWD_REUSE_FORWARD_STATES = 1 };
la2_status la2_backward_ex(const void *q, const void *k, const void *v,
                           const float *lambda, const float *kv0, const void *dO,
                           void *dq, void *dk, void *dv, float *dkv0,
                           int B, int H, int64_t L, int d, int e, la2_dtype dt,
                           void *workspace, size_t workspace_bytes, unsigned flags,
                           cudaStream_t stream);

/*
 * Packed variable-length batches: N sequences of different lengths stored
 * back to back.  q, k [H, T, d] and v, o [H, T, e] (row-major; the slab of
 * head h holds all sequences' rows for that head), cu_seqlens device int64
 * [N+1] (8-byte aligned) with 0 = cu[0] <= cu[1] <= ... <= cu[N] = T:
 * sequence n owns rows [cu[n], cu[n+1]) of every head's slab.  Each
 * sequence is an independent problem with its own decay state, reset at its
 * first row: kv0 / kv_out (and dkv0 in the backward) are fp32 [N, H, d, e],
 * kv0 may be NULL (zero), kv_out / dkv0 may be NULL (not written); an empty
 * sequence passes kv0 through to kv_out (its dkv0 is 0).  lambda [H] as for
 * la2_forward.  The forward computes, per sequence, what la2_forward does
 * for B = 1, L = its length; the backward, what la2_backward does.  One CTA
 * per (sequence, head) walks the whole sequence (no chunk split, so no
 * workspace): a batch with a few very long sequences runs at the speed of
 * its longest one.  No synchronisation.
 * Errors: LA2_ERR_INVALID for negative sizes, a NULL lambda or cu_seqlens,
 * NULL tensors with T > 0, misaligned pointers, an output overlapping any
 * argument, kv_out == kv0; LA2_ERR_UNSUPPORTED for an unknown dtype or a
 * (d, e) outside the supported set.  Offsets outside [0, T] or decreasing
 * are not checked on the host (that would synchronise): the kernel treats
 * such a sequence as empty and sets the bounds bit (2) of the device error
 * word, which la2_last_device_error() reports as LA2_ERR_INVALID.
 * Source: the Lightning Attention-2 notes page, "Tiling." paragraph, applied
 * to each sequence of the batch; the pages describe no packed form (it is
 * the batching the parallel training form needs).
 */
la2_status la2_forward_varlen(const void *q, const void *k, const void *v,
                              const float *lambda, const int64_t *cu_seqlens,
                              const float *kv0, void *o, float *kv_out,
                              int N, int H, int64_t T, int d, int e, la2_dtype dt,
                              cudaStream_t stream);
la2_status la2_backward_varlen(const void *q, const void *k, const void *v,
                               const float *lambda, const int64_t *cu_seqlens,
                               const float *kv0, const void *dO,
                               void *dq, void *dk, void *dv, float *dkv0,
                               int N, int H, int64_t T, int d, int e, la2_dtype dt,
                               cudaStream_t stream);

/*
 * One recurrent decode step for one new token per (b,h):
 *     kv <- lambda kv + k^T v,    o = q kv
 * q, k [B,H,d], v, o [B,H,e] of type dt; kv fp32 [B,H,d,e] updated IN PLACE
 * (the constant-size state; it does not grow with the number of steps).  The
 * updated state includes the current token, matching M_tt = 1.
 * Source: glossary page, section "主な特徴・仕組み" (recurrent inference with
 * a fixed-size state; KV cache constant regardless of length).
 */
la2_status la2_decode_step(const void *q, const void *k, const void *v,
                           const float *lambda, float *kv, void *o,
                           int B, int H, int d, int e, la2_dtype dt,
                           cudaStream_t stream);

/*
 * Gradient of sum(o * dO) with respect to each head's decay: dlambda fp32
 * [H] (written), summed over the batch -- for training a learnable decay.
 * Inputs as for la2_backward (kv0 may be NULL).  Per head
 *   dlambda_h = sum_b sum_t dO_t . ( sum_{j<t} (t-j) lambda^(t-j-1)
 *               (q_t . k_j) v_j + (t+1) lambda^t q_t kv0 ),
 * computed block by block with a second carried state (the position-
 * weighted sum of k^T v) next to the usual one; exact at lambda = 0.  It
 * runs on the fp32-FMA path (no tensor cores), one CTA per (b,h) over the
 * whole sequence; the batch sum is made with atomics, so it is not bitwise
 * reproducible across runs.  Errors as for la2_backward (dlambda
 * overlapping an input: LA2_ERR_INVALID).  The pages do not treat the decay
 * as learnable; the derivative is the chain rule through the recurrence of
 * the Lightning Attention-2 notes page (opening paragraph's running state,
 * with decay).
 */
la2_status la2_backward_dlambda(const void *q, const void *k, const void *v,
                                const float *lambda, const float *kv0, const void *dO,
                                float *dlambda, int B, int H, int64_t L, int d, int e,
                                la2_dtype dt, cudaStream_t stream);

/*
 * la2_backward_dlambda with a workspace of la2_workspace_size(
 * LA2_OP_DLAMBDA, ...) bytes (16-byte aligned; caller-owned; it may not
 * overlap an input): when B*H is below the number of SMs each sequence is
 * split into chunks that run in parallel, their entry states (KV, W) coming
 * from a chunk-state pre-pass and a scan over the chunks (the pair composes
 * as W' = lambda^Lc (Lc KV + W) + dW, KV' = lambda^Lc KV + dKV).  A size of
 * 0 means no split; workspace may then be NULL.  A workspace smaller than
 * needed: LA2_ERR_INVALID.
 */
la2_status la2_backward_dlambda_ex(const void *q, const void *k, const void *v,
                                   const float *lambda, const float *kv0, const void *dO,
                                   float *dlambda, int B, int H, int64_t L, int d, int e,
                                   la2_dtype dt, void *workspace, size_t workspace_bytes,
                                   cudaStream_t stream);

/*
 * Feature map phi(x) = elu(x) + 1, applied to q and k before the attention
 * calls (which take their q and k as already mapped):
 *     phi(x) = x + 1 for x > 0,  e^x for x <= 0      (elementwise)
 * The Lightning Attention glossary page (section "主な特徴・仕組み") has
 * linear attention replace softmax by a kernel feature map so that K^T V can
 * be aggregated first, but names no map; elu + 1 is the positive map of
 * "Transformers are RNNs", one of the works the Luna page lists as its basis
 * next to the ELU paper.  Callers using another map, or none, skip this call.
 *
 * la2_feature_map: phi_q = phi(q), phi_k = phi(k); q, k, phi_q, phi_k hold n
 * values each of type dt (any layout: the map is elementwise; n >= 0, any
 * value).  k and phi_k may both be NULL (q alone is mapped).  An output may be
 * the very buffer of its own input (in place: phi_q == q, phi_k == k); any
 * other shared byte between arguments is LA2_ERR_INVALID.
 *
 * la2_feature_map_backward: the chain rule through the map,
 *     dq = dphi_q * phi'(q),  dk = dphi_k * phi'(k),
 *     phi'(x) = 1 for x > 0,  e^x for x <= 0,
 * where dphi_q, dphi_k are the attention's gradients with respect to its
 * mapped inputs (la2_backward's dq, dk on phi_q, phi_k) and q, k the
 * unmapped inputs.  k, dphi_k and dk are all NULL or all given.  dq may be
 * the very buffer of dphi_q (in place), likewise dk of dphi_k.
 *
 * Both: one HBM-bound streaming launch over q and k together; arithmetic in
 * fp32 (e^x: CUDA's expf), results rounded to dt (bf16: to nearest even).
 * Pointers 16-byte aligned, device memory, caller-owned; asynchronous on
 * `stream`.  Errors: LA2_ERR_INVALID for n < 0, a NULL required pointer,
 * misalignment or an overlap other than the in-place ones;
 * LA2_ERR_UNSUPPORTED for another dt; LA2_ERR_CUDA for a failed launch.
 * n = 0: nothing is launched.
 */
la2_status la2_feature_map(const void *q, const void *k, void *phi_q, void *phi_k, int64_t n,
                           la2_dtype dt, cudaStream_t stream);
la2_status la2_feature_map_backward(const void *q, const void *k, const void *dphi_q,
                                    const void *dphi_k, void *dq, void *dk, int64_t n,
                                    la2_dtype dt, cudaStream_t stream);

/*
 * State pool for serving: the recurrent states of many requests live in one
 * fp32 array kv_pool [pool_size, H, d, e]; request b of a call uses state
 * slots[b] (device int32 [B], 4-byte aligned).  A negative slot marks an
 * inactive request: its state is neither read nor written and its outputs
 * are left untouched.  A slot >= pool_size is not checked on the host (that
 * would synchronise): the kernel skips that request the same way and sets
 * the bounds bit of the device error word (la2_last_device_error ->
 * LA2_ERR_INVALID).  Two active requests of one call sharing a slot race:
 * the caller keeps the active slots of a call distinct.
 *
 * la2_forward_pool: prefill straight into the pool.  As la2_forward for q,
 * k, v [B,H,L,d|e] (L >= 1), o [B,H,L,e] and the workspace (sized by
 * la2_workspace_size(LA2_OP_FORWARD, ...)), with the initial state zero, or
 * with flags = LA2_POOL_CONTINUE the slot's current state (a chunked
 * prefill continuing a request, or several tokens decoded at once through
 * the block schedule); the final state is written back to the slot.  Reading
 * and writing one slot in one call is safe: a split sequence reads its
 * entry states from the workspace, never from the pool.
 *
 * la2_decode_tokens: T >= 0 new tokens per request at once, q, k [B,H,T,d],
 * v, o [B,H,T,e]: for t = 0..T-1, kv <- lambda kv + k_t^T v_t, o_t = q_t kv
 * (the la2_decode_step recurrence applied T times), reading and writing the
 * slot's state once per call instead of once per token.  slots may be NULL:
 * request b then uses state b (pool_size >= B).  From 17 tokens per request
 * on (bf16, d = e = 128; LA2_OPT_DECODE_BLOCK_TOKENS overrides) the call runs
 * each request's tokens as one block of the chunk schedule on the tensor
 * cores: up to 128 tokens, one CTA per SM walks a contiguous range of the
 * (head, request) units back to back, each unit's state read from and
 * written back to its slot; beyond 128, la2_forward_pool's path (one chunk
 * per request).  Below that, or for other shapes, token by token in
 * registers.  la2_decode_step is this with T = 1, slots NULL.
 *
 * Errors as for la2_forward / la2_decode_step (LA2_ERR_INVALID also for
 * unknown flag bits, L < 1 in la2_forward_pool, a NULL slot table in
 * la2_forward_pool).  The pages describe the recurrent form and the hand-off
 * from the parallel (training / prefill) form only in words; the pool, its
 * slot table and the multi-token call are this library's serving interface.
 * Source: glossary page, section "主な特徴・仕組み" (parallel form for
 * training, recurrent form with a constant-size state for inference).
 */
enum { LA2_POOL_CONTINUE = 1 };
la2_status la2_forward_pool(const void *q, const void *k, const void *v,
                            const float *lambda, float *kv_pool, const int32_t *slots,
                            int pool_size, void *o, unsigned flags,
                            int B, int H, int64_t L, int d, int e, la2_dtype dt,
                            void *workspace, size_t workspace_bytes, cudaStream_t stream);
la2_status la2_decode_tokens(const void *q, const void *k, const void *v,
                             const float *lambda, float *kv_pool, const int32_t *slots,
                             int pool_size, void *o, int B, int H, int T, int d, int e,
                             la2_dtype dt, cudaStream_t stream);

/*
 * Sequence sharding: a sequence of R * L rows cut into R shards of L rows
 * (one per GPU, in order) needs, per shard, only two d x e summaries of the
 * other shards -- an exact reassociation of the block recurrence.
 *
 * la2_shard_state: one shard's summary, fp32 out [B,H,d,e]: reverse = 0
 * (a = k [B,H,L,d], b = v [B,H,L,e]) the forward delta sum_t
 * lambda^(L-1-t) k_t^T v_t (the shard's final state from a zero start);
 * reverse = 1 (a = q, b = dO) the reverse delta sum_t lambda^t q_t^T dO_t.
 * Workspace: la2_workspace_size(LA2_OP_SHARD_STATE, ...) bytes (required).
 *
 * la2_state_prefix: from the R shards' deltas delta [R,B,H,d,e] (gathered
 * from every rank), every shard's boundary state, out [R,B,H,d,e]: forward
 * out[0] = kv0 (NULL: zero), out[r] = lambda^L out[r-1] + delta[r-1] (the
 * state entering shard r); reverse out[R-1] = 0, out[r] = lambda^L out[r+1]
 * + delta[r+1] (the reverse state flowing into shard r from the rows after
 * it; kv0 ignored).  fp32 throughout; d, e as elsewhere.
 *
 * la2_backward_shard: la2_backward_ex for one shard, with dstate_end [B,H,d,e]
 * (NULL: zero) the reverse state flowing in from the rows after it, i.e. its
 * out[r] of the reverse prefix; kv0 is the shard's entry state (the forward
 * prefix's out[r]).  Its dq, dk, dv are those rows' slices of the gradients
 * of the whole sequence; on the first shard dkv0 is the whole sequence's.
 *
 * A rank then computes its shard's outputs with la2_forward(kv0 = entry
 * state) and its gradients with la2_backward_shard, after one all-gather of
 * the R deltas per direction (the only exchange; see the package's
 * seqpar module).  Errors as for la2_forward / la2_backward.  The pages do
 * not discuss sharding a sequence across devices; the reassociation is the
 * tiling one (Lightning Attention-2 notes page, "Tiling." paragraph) applied
 * to shards.
 */
la2_status la2_shard_state(const void *a, const void *b, const float *lambda, float *out,
                           int B, int H, int64_t L, int d, int e, la2_dtype dt, int reverse,
                           void *workspace, size_t workspace_bytes, cudaStream_t stream);
la2_status la2_state_prefix(const float *delta, const float *kv0, const float *lambda,
                            float *out, int R, int B, int H, int64_t L_shard, int d, int e,
                            int reverse, cudaStream_t stream);
la2_status la2_backward_shard(const void *q, const void *k, const void *v,
                              const float *lambda, const float *kv0, const void *dO,
                              const float *dstate_end, void *dq, void *dk, void *dv,
                              float *dkv0, int B, int H, int64_t L, int d, int e,
                              la2_dtype dt, void *workspace, size_t workspace_bytes,
                              unsigned flags, cudaStream_t stream);

/*
 * Synchronises `stream`, then reports and clears the device error word that
 * the kernels set: LA2_ERR_TIMEOUT when a bounded wait gave up,
 * LA2_ERR_INVALID when a kernel met out-of-range data it could not use (a
 * packed-batch offset outside [0, T]); LA2_ERR_CUDA if the synchronisation
 * itself fails.  LA2_OK otherwise.
 */
la2_status la2_last_device_error(cudaStream_t stream);

/* Human-readable name of a status code (static string). */
const char *la2_status_string(la2_status s);

/*
 * Process-wide tuning overrides (for tests and sweeps; not thread-safe with
 * concurrent calls).  LA2_OPT_SPLIT: number of chunks each (b,h) sequence is
 * split into (0 = automatic).  LA2_OPT_PATH: 0 = automatic, 1 = force the
 * portable fp32-FMA kernels, 2 = require the tensor-core kernels (calls whose
 * shape they do not cover return LA2_ERR_UNSUPPORTED).
 * LA2_OPT_INJECT_TIMEOUT (test hook): when nonzero, the next tensor-core
 * la2_forward withholds one internal completion signal in its first CTA, so
 * that CTA's bounded wait gives up (about 2 s) and la2_last_device_error()
 * then reports LA2_ERR_TIMEOUT; the option resets itself.
 * LA2_OPT_VARIANT: form of the tensor-core kernel (0 = warp-specialised,
 * the default; 1 = the simpler phase-serial form, kept for comparison).
 * LA2_OPT_TRACE: 0 = off; p + 1 = while set, the first CTA of every launch
 * of tensor-core pass p (0 forward, 1 dQ, 2 forward chunk state, 3 dV,
 * 4 dK, 5 reverse chunk state) of the warp-specialised kernel stamps the
 * device clock at fixed points of each block into the trace buffer (see
 * la2_trace_read).  LA2_OPT_VARLEN_ORDER: 0 (default) = the tensor-core
 * passes of a packed batch of at most 64 sequences start the longest
 * sequences first (each CTA ranks the lengths from cu_seqlens on the device),
 * so that short ones fill the last wave; 1 = in the given order.
 * LA2_OPT_DECODE_BLOCK_TOKENS: 0 (default) = la2_decode_tokens runs the
 * tensor-core block form from the library's crossover number of tokens per
 * request on, the token-by-token kernel below it; n > 0 = from n tokens on.
 * LA2_OPT_BWD_FORM: 0 (default) = the tensor-core backward computes dV and
 * dK in one paired launch (two CTAs per chunk, clusters of two, the pair
 * reading Q and dO from HBM once); 1 = two separate passes (for comparison).
 * Under the same chunk split the results are bitwise the same; under the
 * automatic split the paired form may cut a long sequence into fewer chunks
 * (each chunk occupies two SMs), which changes only the rounding.  The
 * workspace size of a backward
 * depends on this option, so query la2_workspace_size with the option that
 * the call will run under.
 * Returns the previous value, or -1 for an unknown option.
 */
enum {
    LA2_OPT_SPLIT = 0, LA2_OPT_PATH = 1, LA2_OPT_INJECT_TIMEOUT = 2, LA2_OPT_VARIANT = 3,
    LA2_OPT_TRACE = 4, LA2_OPT_VARLEN_ORDER = 5, LA2_OPT_DECODE_BLOCK_TOKENS = 6,
    LA2_OPT_BWD_FORM = 7
};

/*
 * Synchronises the device and copies the trace buffer (uint64 nanosecond
 * stamps, laid out [event][block] with 16 events x 512 blocks; 0 = not
 * recorded) into host memory `out` (n entries at most), then clears it.
 * Events: 0 loads issued, 1 S = A0 B1^T issued, 2 P.B2 / state term / state
 * update issued, 3 mask start, 4 mask done, 5 epilogue start, 6 state handed
 * back to the MMA issuer, 7 output tile read by the store, 8 kernel entry,
 * 9 set-up done (all of CTA 0, indexed by block); 10 entry and 11 exit of
 * every CTA (indexed by CTA, first 512).  With out == NULL returns the
 * buffer's entry count.
 */
size_t la2_trace_read(uint64_t *out, size_t n);
int la2_set_option(int option, int value);

/*
 * Per-kernel device timing.  While enabled, every kernel the library
 * launches is bracketed by a pair of CUDA events on its stream.
 * la2_profile_report() synchronises on those events and writes a JSON object
 * {"<kernel>": {"launches": n, "ms": total}, ...} into buf (truncated to
 * buf_bytes), clears the records and returns the number of bytes needed.
 */
void la2_profile_enable(int on);
size_t la2_profile_report(char *buf, size_t buf_bytes);

/* Library version string, e.g. "la2 0.1 sm_100a". */
const char *la2_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LA2_H */
