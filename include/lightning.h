/*
 * lightning.h — C ABI of liblightning.so, MiniMax-M1 Lightning Attention on
 * NVIDIA B200 (sm_100a).
 *
 * The operation ("MINIMAX SIGNAL LAB · M1", §03 Lightning Attention): causal
 * linear attention with a per-head exponential decay, computed in blocks of B
 * tokens. For block t of one (batch, head) with slope s:
 *
 *   intra  O_intra = [(Q_t K_t^T) ⊙ D] V_t,   D_ij = e^{-s(i-j)} 1[i >= j]
 *   inter  O_inter = (Q_t ⊙ d_q) S_{t-1},     d_q[i] = e^{-s(i+1)}
 *   state  S_t     = e^{-s m} S_{t-1} + (K_t ⊙ d_k)^T V_t,  d_k[j] = e^{-s(m-1-j)}
 *   out    O_t     = O_intra + O_inter
 *
 * where m is the block's length (B, or fewer for the last block, as the same
 * section states) and S_{-1} is the carried-in state. Equivalently, token by
 * token: o_i = sum_{j<=i} e^{-s(i-j)} (q_i . k_j) v_j + e^{-s(i+1)} q_i S_in.
 * The pages print no d_q / d_k exponents; the ones above are the readings for
 * which the block form equals the token form.
 *
 * Decode (same section: the recursive, fixed-size KV state; §04: the state
 * does not grow with context): for one new token,
 *   S <- e^{-s} S + k^T v,   o = q S.
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller; the
 *     library never allocates, frees or retains them.
 *   - q, k, v, o are contiguous [batch][heads][seq][dim] (decode: seq = 1,
 *     i.e. [batch][heads][dim]); element type given by `dtype`; o has the
 *     input dtype. Pointers must be 16-byte aligned.
 *   - States are float32, contiguous [batch][heads][dim][dim], row index =
 *     key dimension, column index = value dimension.
 *   - slopes is a device float32 array of `heads` decay slopes s_h >= 0.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream). Every call is asynchronous on that stream.
 *   - Argument errors are detected on the host and returned before anything
 *     is launched; launch failures return LA_ERR_CUDA. No device-side trap
 *     or abort is ever used: a device-side wait that runs out of its
 *     iteration budget records LA_ERR_TIMEOUT in a status word; so does
 *     LA_ERR_INVALID_ARG for a device-side argument the host cannot see (a
 *     decode position outside its cache), whose work is then skipped. The
 *     next launching call returns that status instead of launching, and
 *     lightning_last_device_status() returns it on demand (see there).
 *   - A human-readable reason for the last failure on the calling thread is
 *     returned by lightning_last_error_message().
 *   - lightning_prefill, lightning_prefill_ex, lightning_decode and
 *     lightning_prefill_backward may be recorded into a CUDA graph by stream
 *     capture. Their launches use only `stream` (the backward also uses the
 *     library's side streams, forked from and joined to it with events), so
 *     replaying the graph repeats the call. The host-side argument checks and
 *     the status-word check run once, when the call is recorded.
 */
#ifndef LIGHTNING_H
#define LIGHTNING_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum la_status {
    LA_OK = 0,
    LA_ERR_INVALID_ARG = 1,   /* bad pointer, shape, alignment or aliasing        */
    LA_ERR_UNSUPPORTED = 2,   /* valid request the library has no kernel for      */
    LA_ERR_CUDA = 3,          /* CUDA runtime error while launching               */
    LA_ERR_TIMEOUT = 4        /* a device-side bounded wait gave up               */
} la_status;

typedef enum la_dtype {
    LA_DTYPE_F32 = 0,
    LA_DTYPE_BF16 = 1
} la_dtype;

/* Kernel selection for lightning_prefill_ex. AUTO picks the CTA-pair kernel
 * for bf16, dim 128, block 256; the single-CTA tensor-core kernel for bf16,
 * dim 128, block 128; and the CUDA-core kernel otherwise. */
typedef enum la_variant {
    LA_VARIANT_AUTO = 0,
    LA_VARIANT_SIMT = 1,          /* CUDA-core kernel, fp32 arithmetic, any dtype          */
    LA_VARIANT_TCGEN05 = 2,       /* tcgen05/TMEM/TMA, one CTA per (head, value half),
                                     bf16, dim 128, block 128 or 256                      */
    LA_VARIANT_TCGEN05_PAIR = 3   /* tcgen05 on a CTA pair (cta_group::2) per head,
                                     bf16, dim 128, block 256                             */
} la_variant;

/* Version of this ABI; bumps on any incompatible change. */
int lightning_abi_version(void);

/*
 * Blockwise prefill of `seq` tokens for every (batch, head).
 * Source: "MINIMAX SIGNAL LAB · M1", §03 Lightning Attention (intra-block,
 * inter-block and state-update formulas; last short block uses its length).
 *
 *   q, k, v    [batch][heads][seq][dim], dtype; read only.
 *   dtype      LA_DTYPE_F32 or LA_DTYPE_BF16.
 *   slopes     [heads] float32.
 *   batch      >= 0 (0: nothing to do).  heads >= 1.  seq >= 0.
 *   dim        64 or 128.
 *   block      block length B >= 1 (tensor-core kernels: 128 or 256).
 *   state_in   [batch][heads][dim][dim] float32 carried-in state, or NULL for
 *              zeros.
 *   o          [batch][heads][seq][dim], dtype; written. Must not overlap
 *              q, k, v, slopes or either state.
 *   state_out  [batch][heads][dim][dim] float32 state after the last token, or
 *              NULL to skip. May be the same pointer as state_in (in-place
 *              carry); any other overlap is rejected.
 *   workspace, workspace_bytes
 *              device scratch, caller-owned, 16-byte aligned, overlapping no
 *              other buffer, of at least lightning_prefill_workspace_size
 *              bytes: 48 bytes per (batch, head) for either tensor-core
 *              kernel (its range guard, below), none for the CUDA-core kernel
 *              (NULL/0 is fine there). Too little returns LA_ERR_INVALID_ARG.
 *              Its contents need no initialisation; calls that share one
 *              workspace must not run at the same time.
 *   stream     cudaStream_t as void*.
 * seq == 0 writes state_out = state_in (or zeros) and nothing else.
 *
 * Input range of the tensor-core kernels. They round the operands they form
 * (P ⊙ D, Q ⊙ d_q, K ⊙ d_k, V and the carried state) to fp16, whose range is
 * narrower than bf16's. Both tensor-core kernels guard against that: while
 * they run they take, per (batch, head), the largest |q|, |k|, |v| and |state_in|
 * element, which bound every such operand; a head whose operands could pass
 * 2^15, or whose maxima fall below 2^-9, is recomputed by a second launch with
 * q, k and v scaled by powers of two (exact) chosen from the head's largest
 * row norms of q and k, so that the operands sit in fp16's normal range, and
 * the results scaled back. The results then meet the error bound for any
 * scale of q, k, v and state_in whose row norms lie within about
 * 2^-36 .. 2^44, provided the values inside one (batch, head) span less than
 * about 2^14 (for example a few rows 2^8 above the rest, with |q.k| above
 * 65504, are covered). Inputs holding inf or NaN give non-finite results.
 * Every call of a tensor-core kernel is two launches on `stream`: the kernel,
 * then the guard's second pass, which returns at once for heads it need not
 * redo. With state_out == state_in, the single-CTA kernel runs each head's
 * two CTAs as a thread-block cluster of two.
 */
la_status lightning_prefill(const void *q, const void *k, const void *v, la_dtype dtype,
                            const float *slopes, int batch, int heads, int seq, int dim,
                            int block, const float *state_in, void *o, float *state_out,
                            void *workspace, size_t workspace_bytes, void *stream);

/* Same as lightning_prefill with an explicit kernel choice (la_variant).
 * Requesting a tensor-core variant for a shape it does not take returns
 * LA_ERR_UNSUPPORTED. */
la_status lightning_prefill_ex(const void *q, const void *k, const void *v, la_dtype dtype,
                               const float *slopes, int batch, int heads, int seq, int dim,
                               int block, const float *state_in, void *o, float *state_out,
                               void *workspace, size_t workspace_bytes, void *stream,
                               int variant);

/* Kernel lightning_prefill_ex would run for these arguments (la_variant, never
 * AUTO), or -1 if the request is invalid or unsupported. Host only. */
int lightning_prefill_selected_variant(la_dtype dtype, int batch, int heads, int seq, int dim,
                                       int block, int variant);

/* Bytes of workspace lightning_prefill (with AUTO, bf16 inputs) needs for these
 * sizes: 48 * batch * heads for the CTA-pair kernel (dim 128, block 256), 0
 * otherwise. Enough for every variant and dtype. Host only. */
size_t lightning_prefill_workspace_size(int batch, int heads, int seq, int dim, int block);

/*
 * Prefill that also keeps prefix-cache snapshots of the state. Source:
 * "MINIMAX SIGNAL LAB · M1", §03 Lightning Attention (the recursive fixed-size
 * state S_t; the page's note that prefix caching and speculative decoding are
 * where such states are hard to serve) and §04 (the fp32 state per head).
 *
 * Same arguments and results as lightning_prefill_ex (workspace included), plus
 *   interval   snapshot spacing in tokens: a positive multiple of `block`.
 *   snapshots  [batch][heads][n][dim][dim] float32, n = seq / interval
 *              (lightning_prefill_snapshot_count); snapshot i is the state after
 *              the first (i+1)*interval tokens, i.e. what lightning_prefill on
 *              that prefix returns as state_out (it includes state_in, decayed).
 *              Device pointer, caller-owned, 16-byte aligned, overlapping nothing
 *              else; may be NULL when n == 0.
 * `o` and `state_out` are bit-identical to lightning_prefill_ex's for the same
 * variant. A bad interval or snapshot buffer returns LA_ERR_INVALID_ARG before
 * any launch.
 */
la_status lightning_prefill_snapshots(const void *q, const void *k, const void *v, la_dtype dtype,
                                      const float *slopes, int batch, int heads, int seq, int dim,
                                      int block, const float *state_in, void *o, float *state_out,
                                      int interval, float *snapshots, void *workspace, size_t workspace_bytes,
                                      void *stream, int variant);

/*
 * Gradients of one prefill, for training through the layer. The pages print
 * no backward pass; this is the derivative of the operation defined in
 * "MINIMAX SIGNAL LAB · M1", §03 Lightning Attention (the token-level result
 * above). For the loss  sum_i dO_i . o_i + sum dS_out * S_out, with S_i the
 * state after token i (o_i = q_i S_i):
 *   dq_i  = dO_i S_i^T
 *   R_j   = sum_{i>=j} e^{-s(i-j)} q_i^T dO_i + e^{-s(L-1-j)} dS_out
 *   dk_j  = R_j v_j,   dv_j = R_j^T k_j,   dS_in = e^{-s} R_0 (dS_out if L = 0)
 * computed blockwise as three passes of the prefill recurrence on permuted
 * operands: dQ forward in time on (dO, V, K) with state S^T; dV and dK
 * backward in time on (K, Q, dO) and (V, dO, Q) with state R.
 * Kernels (variant): LA_VARIANT_TCGEN05_PAIR runs the passes on the CTA-pair
 * tensor-core kernel (bf16, dim 128, block 256; the backward-in-time passes
 * run it anti-causally, blocks from last to first; the three passes run side
 * by side: dV and dK on two library-owned streams per device, forked from and
 * joined back into `stream` with events, so the call keeps `stream`'s order);
 * LA_VARIANT_SIMT runs them on CUDA cores in fp32 (any dtype, dim 64 or 128,
 * any block, no workspace); LA_VARIANT_AUTO takes the tensor-core kernels
 * where they apply. LA_VARIANT_TCGEN05 is not a backward variant.
 *
 *   q, k, v, d_o  [batch][heads][seq][dim], dtype; read only.
 *   state_in      as for lightning_prefill (NULL: zeros).
 *   d_state_out   [batch][heads][dim][dim] float32 gradient of state_out, or
 *                 NULL for zeros.
 *   dq, dk, dv    [batch][heads][seq][dim], dtype; written.
 *   d_state_in    [batch][heads][dim][dim] float32, or NULL to skip.
 *   workspace, workspace_bytes
 *                 scratch of at least lightning_prefill_backward_workspace_size
 *                 bytes: the range guard's records of the three tensor-core
 *                 passes (144 bytes per (batch, head); see lightning_prefill),
 *                 none on CUDA cores (NULL/0 is fine there); 16-byte aligned,
 *                 overlapping nothing else, no initialisation needed.
 * All device pointers, caller-owned, 16-byte aligned. No output may overlap
 * an input or another output; a short or overlapping workspace is rejected
 * (all LA_ERR_INVALID_ARG). Shape rules as for lightning_prefill.
 */
la_status lightning_prefill_backward(const void *q, const void *k, const void *v, const void *d_o,
                                     la_dtype dtype, const float *slopes, int batch, int heads, int seq,
                                     int dim, int block, const float *state_in, const float *d_state_out,
                                     void *dq, void *dk, void *dv, float *d_state_in, void *workspace,
                                     size_t workspace_bytes, void *stream, int variant);

/*
 * lightning_prefill_backward for callers that cannot allocate device memory
 * themselves: a runtime whose allocator owns all of the device's memory and
 * hands out none at the point of the call, or a plugin inside another
 * framework that may not call cudaMalloc. The pages have no counterpart to
 * this entry point. It allocates nothing: the scratch the tensor-core passes
 * need (the range guard's records, 144 bytes per (batch, head)) comes from a
 * fixed array inside the library, 4 MiB on every device that loads it, kept
 * until the process exits (lightning_prefill_backward_noalloc_capacity()).
 * Arguments and results are those of lightning_prefill_backward; argument
 * errors come in the same order, then a request that needs more scratch than
 * the array holds (more than 29127 batch x heads) returns LA_ERR_UNSUPPORTED,
 * all before any launch.
 * The first call on a device looks up the array's address on that device
 * (with that device current): make that first call before any stream capture.
 * Every call on a device shares the array, which keeps the last call's
 * contents (nothing in it needs to start at zero): calls that overlap in time
 * on the GPU (on different streams) race on it, so such callers must use
 * lightning_prefill_backward with a workspace of their own.
 */
la_status lightning_prefill_backward_noalloc(const void *q, const void *k, const void *v, const void *d_o,
                                             la_dtype dtype, const float *slopes, int batch, int heads,
                                             int seq, int dim, int block, const float *state_in,
                                             const float *d_state_out, void *dq, void *dk, void *dv,
                                             float *d_state_in, void *stream, int variant);

/* Bytes of scratch lightning_prefill_backward_noalloc has. Host only. */
size_t lightning_prefill_backward_noalloc_capacity(void);

/* Bytes of workspace lightning_prefill_backward needs for these arguments
 * (0 for every current kernel and for an invalid request). Host only. */
size_t lightning_prefill_backward_workspace_size(la_dtype dtype, int batch, int heads, int seq, int dim,
                                                 int block, int variant);

/*
 * Normalisation and gating of the attention output. Source: "MINIMAX SIGNAL
 * LAB · M1", §03 Lightning Attention: the figure sums the intra- and
 * inter-block outputs, then normalises and gates them; the pages print no
 * formula. The reading implemented: RMS normalisation with a learned
 * per-channel weight, then an elementwise sigmoid gate,
 *   y[b][l][n] = gamma[n] x[n] / sqrt(mean_{group} x^2 + eps) * 1 / (1 + e^{-gate[b][l][n]})
 * over the token's channels n = h*dim + c, x[n] = o[b][h][l][c]. The mean
 * runs over the head's dim channels (per_head != 0) or over all heads*dim
 * channels of the token (per_head == 0).
 *
 *   o      [batch][heads][seq][dim], dtype (lightning_prefill's output).
 *   gate   [batch][seq][heads*dim], dtype (the gate projection's output).
 *   gamma  [heads*dim] float32.   eps: finite, >= 0.
 *   y      [batch][seq][heads*dim], dtype; written; must not overlap o, gate
 *          or gamma.
 * dim 64 or 128; heads*dim at most 16384 (bf16) or 8192 (f32) channels, else
 * LA_ERR_UNSUPPORTED. Device pointers, caller-owned, 16-byte aligned.
 */
la_status lightning_norm_gate(const void *o, const void *gate, la_dtype dtype, const float *gamma, float eps,
                              int batch, int heads, int seq, int dim, int per_head, void *y, void *stream);

/*
 * A prefill whose output goes through the normalisation and gating above with
 * the per-head mean (per_head != 0), fused into the prefill's output epilogue:
 * o is never written to memory. Source: "MINIMAX SIGNAL LAB · M1", §03
 * Lightning Attention (the figure's sum of the intra- and inter-block outputs,
 * then normalisation and gate; the same reading as lightning_norm_gate).
 *   y[b][l][h*128 + c] = gamma[h*128 + c] o[b][h][l][c]
 *                        / sqrt(mean_c o[b][h][l][c]^2 + eps) * sigmoid(gate[b][l][h*128 + c])
 * with o the result lightning_prefill defines (before its rounding to bf16;
 * the normalised value is formed from o rounded to bf16 and the fp32 mean).
 *
 *   q, k, v, slopes, state_in, state_out: as for lightning_prefill.
 *   gate   [batch][seq][heads*128] bf16; read only.
 *   gamma  [heads*128] float32.   eps: finite, >= 0.
 *   y      [batch][seq][heads*128] bf16; written; must not overlap any input,
 *          the states, gate or gamma.
 *   workspace, workspace_bytes: as for lightning_prefill (the CTA-pair
 *          kernel's range guard: 48 bytes per (batch, head)).
 * Runs on the CTA-pair tensor-core kernel only: bf16, dim 128, block 256;
 * other shapes or dtypes return LA_ERR_UNSUPPORTED before any launch (the
 * whole-token mean needs every head of a token, which one head's kernel does
 * not see: use lightning_prefill then lightning_norm_gate). Device pointers,
 * caller-owned, 16-byte aligned; asynchronous on `stream`.
 */
la_status lightning_prefill_norm_gate(const void *q, const void *k, const void *v, la_dtype dtype,
                                      const float *slopes, int batch, int heads, int seq, int dim, int block,
                                      const float *state_in, const void *gate, const float *gamma, float eps,
                                      void *y, float *state_out, void *workspace, size_t workspace_bytes,
                                      void *stream);

/* Number of snapshots lightning_prefill_snapshots writes per (batch, head):
 * seq / interval, or -1 if seq < 0 or interval < 1. Host only. */
int lightning_prefill_snapshot_count(int seq, int interval);

/*
 * One decode step for a single new token of every (batch, head), updating the
 * state in place. Source: "MINIMAX SIGNAL LAB · M1", §03 (recursive KV state)
 * and §04 (fixed-size FP32 state per head).
 *
 *   q, k, v  [batch][heads][dim], dtype; read only.
 *   slopes   [heads] float32.
 *   dim      64 or 128.
 *   state    [batch][heads][dim][dim] float32; read and overwritten with
 *            e^{-s} state + k^T v.
 *   o        [batch][heads][dim], dtype; written: q (updated state).
 *            Must not overlap any input or the state.
 */
la_status lightning_decode(const void *q, const void *k, const void *v, la_dtype dtype,
                           const float *slopes, int batch, int heads, int dim, float *state,
                           void *o, void *stream);

/*
 * Failures that kernels record on the device. Source: none in the pages; this
 * is the library's own failure reporting. A kernel whose bounded wait runs out
 * records LA_ERR_TIMEOUT, and one that meets an out-of-range device-side
 * argument records LA_ERR_INVALID_ARG, in a status word; no kernel traps.
 *
 * The word is one per process (managed memory), shared by every device,
 * stream and thread. It is reported in two ways:
 *   - on the next launching call: every entry point that launches work looks
 *     at the word, without synchronising anything, just before its first
 *     launch; if an earlier kernel recorded a failure, the call clears the
 *     word, launches nothing and returns that status (lightning_last_error_message
 *     says so). Calls that launch nothing (argument errors, empty problems,
 *     host-only queries) do not look.
 *   - on demand: lightning_last_device_status synchronises `stream`, then
 *     returns the recorded status (LA_OK if none) and clears the word.
 * Because the word is shared, a failure recorded by a kernel on one stream or
 * device is returned by whichever call looks first, from any thread, and a
 * kernel still running when a call looks may record a failure that only the
 * call after it sees.
 */
la_status lightning_last_device_status(void *stream);

/* The same as lightning_last_device_status (kept under its earlier name). */
la_status lightning_device_status(void *stream);

/*
 * Test hook for the failure-detection path (the pages have no counterpart):
 * enqueues on `stream` one CTA whose bounded mbarrier wait, the one every
 * kernel of the library uses, is never satisfied. The wait runs out, the
 * kernel records LA_ERR_TIMEOUT in the device status word and returns; the
 * context stays usable. Returns LA_OK once the kernel is enqueued (or
 * LA_ERR_CUDA if the launch fails).
 */
la_status lightning_selftest_wait_timeout(void *stream);

/*
 * One decode step of the softmax attention layer that M1 places after every
 * seven Lightning layers. Source: "MINIMAX SIGNAL LAB · M1", §02 (64 query
 * heads x 128; softmax K/V 8 x 128; RoPE on 64 of the 128 dims, in the
 * softmax layers only) and §04 (those layers keep a KV cache that grows with
 * the context). The pages print no formula; the readings: grouped-query
 * attention (query head h reads KV head h / (heads / kv_heads)), scores
 * scaled by `scale` (1/sqrt(dim) in the model), rotate-half RoPE on the first
 * `rot` dims with theta_i = rope_base^{-2i/rot}, a cache of rotated keys.
 * For sequence b the new token sits at position pos[b]: its rotated key and
 * its value are written into the caches there, and
 *   o[b][h] = sum_{p <= pos[b]} softmax_p(scale * rope(q[b][h], pos[b]) . k_p) v_p.
 *
 *   q                [batch][heads][dim], dtype.
 *   k_new, v_new     [batch][kv_heads][dim], dtype.
 *   k_cache, v_cache [batch][kv_heads][cap][dim], dtype; positions < pos[b]
 *                    read, position pos[b] written.
 *   pos              DEVICE int32 [batch], 0 <= pos[b] < cap; an out-of-range
 *                    position skips that sequence (o = 0) and is reported as
 *                    LA_ERR_INVALID_ARG by lightning_device_status().
 *   dim 128; heads / kv_heads at most 32 (bf16) or 8 (float32); rot even,
 *   0 <= rot <= dim.
 *   o                [batch][heads][dim], dtype; written.
 *   workspace        lightning_gqa_decode_workspace_size(batch, heads, cap)
 *                    bytes, 16-byte aligned.
 * Device pointers, caller-owned, 16-byte aligned; the caches, o and the
 * workspace must not overlap any other buffer. Three launches (cache append
 * and query rotation, chunk partials, merge). bf16: the chunk partials on the
 * tensor cores (tcgen05; the rotated queries and the weights rounded to bf16,
 * fp32 softmax and accumulation); float32: CUDA cores, fp32 arithmetic.
 */
la_status lightning_gqa_decode(const void *q, const void *k_new, const void *v_new, void *k_cache, void *v_cache,
                               la_dtype dtype, const int *pos, int batch, int heads, int kv_heads, int dim, int cap,
                               int rot, double rope_base, float scale, void *o, void *workspace,
                               size_t workspace_bytes, void *stream);

/* Workspace bytes of lightning_gqa_decode (0 for an invalid request). Host only. */
size_t lightning_gqa_decode_workspace_size(int batch, int heads, int cap);

/*
 * Prefill of the same softmax attention layer: `seq` new tokens per sequence,
 * sequence b's at positions start[b] .. start[b]+seq-1 (each sequence with a
 * cached prefix of its own length). Source and readings as for
 * lightning_gqa_decode (and §04: the KV cache grows per sequence); the causal
 * order is that of the decode step applied to each new token in turn. The new
 * tokens' rotated keys and their values are written into the caches at
 * positions start[b]+i, and
 *   o[b][h][i] = sum_{p <= start[b]+i} softmax_p(scale * rope(q[b][h][i], start[b]+i) . k_p) v_p,
 * k_p, v_p the cache rows (positions < start[b] as given, the rest as written).
 *
 *   q                [batch][heads][seq][dim], dtype.
 *   k_new, v_new     [batch][kv_heads][seq][dim], dtype.
 *   k_cache, v_cache [batch][kv_heads][cap][dim], dtype; positions < start[b]
 *                    read, positions start[b] .. start[b]+seq-1 written, the
 *                    rest never written (the last key tile a query reads may
 *                    reach past start[b]+seq-1; those rows enter no result,
 *                    whatever they hold).
 *   start            DEVICE int32 [batch], 0 <= start[b] <= cap - seq. A
 *                    start[b] outside that range skips sequence b (its caches
 *                    and o are not written) and is reported as
 *                    LA_ERR_INVALID_ARG through the status word (see
 *                    lightning_last_device_status); the other sequences run.
 *   dtype            LA_DTYPE_BF16 (tensor cores) or LA_DTYPE_F32 (CUDA cores).
 *   dim 128; rot a multiple of 4, 0 <= rot <= dim; scale finite and > 0;
 *   seq <= cap; batch <= 65535.
 *   o                [batch][heads][seq][dim], dtype; written.
 *   workspace        lightning_gqa_prefill_workspace_size(dtype, batch, heads,
 *                    seq, dim) bytes (the rotated queries), 16-byte aligned.
 * Device pointers, caller-owned, 16-byte aligned; the caches, o and the
 * workspace must not overlap any other buffer (start included). seq == 0 or
 * batch == 0 launches nothing. Two launches: the rotation, then the attention:
 * bf16 on the tensor cores (tcgen05; bf16 operands, fp32 accumulation and
 * softmax, P rounded to bf16); float32 on CUDA cores (fp32 throughout, exact
 * online softmax).
 */
la_status lightning_gqa_prefill(const void *q, const void *k_new, const void *v_new, void *k_cache, void *v_cache,
                                la_dtype dtype, const int *start, int batch, int heads, int kv_heads, int seq, int dim,
                                int cap, int rot, double rope_base, float scale, void *o, void *workspace,
                                size_t workspace_bytes, void *stream);

/* Workspace bytes of lightning_gqa_prefill (0 for an invalid request). Host only. */
size_t lightning_gqa_prefill_workspace_size(la_dtype dtype, int batch, int heads, int seq, int dim);

/* Static description of a status code. */
const char *lightning_status_string(int status);

/* Reason for the most recent failure returned on the calling thread ("" if
 * none). The pointer stays valid until the next call on that thread. */
const char *lightning_last_error_message(void);

#ifdef __cplusplus
}
#endif

#endif /* LIGHTNING_H */
