/*
 * race_attn.h -- C ABI of the RACE Attention library for NVIDIA B200 (sm_100a).
 *
 * RACE Attention ("RACE Attention: A Strictly Linear-Time Attention for Long-Sequence
 * Training", arXiv 2510.04008; sections cited below are those of its gist.science
 * summaries: zh = Chinese page, es = Spanish page) replaces softmax attention by a
 * sketch of the sharpened angular kernel (1 - arccos(q.k / |q||k|)/pi)^P (es §2.1,
 * zh §2.1).  Per head, with x^ = x/|x|, L tables of P Gaussian hyperplanes W[L,P,d],
 * u_l = tanh(W_l x^) and R = 2^P hypercube corners (zh §2.2):
 *
 *     phi_l(x)[r] = softmax_r( beta * c_r . u_l ),  c_rp = +1 if bit p of r is set else -1,
 *     Y_i   = sum_l sum_{j in M(i)} (phi_l(q_i) . phi_l(k_j)) [v_j, 1],
 *     out_i = Y_i[0:d] / Y_i[d],   den_i = Y_i[d],
 *
 * with M(i) = every key (Algorithm 1, zh §2.2) or keys j <= i (Algorithm 2, causal
 * streaming statistics, zh §2.3).  beta = 1/tau; tau = 0 selects hard sign hashing
 * (phi_l one-hot at r* = sum_p [W_lp . x > 0] 2^p).
 *
 * Conventions shared by every entry point
 *   - Layout: q, k, v, out, dout, dq, dk, dv are [B, H, N, d] row-major (d fastest),
 *     contiguous; den is [B, H, N]; W is [L, P, d] fp32 and is shared by every (b, h).
 *   - Every pointer named "device" must point to memory of the current CUDA device,
 *     16-byte aligned.  The tensor-core paths move rows in 32-byte accesses and run only
 *     when the buffers of the call are 32-byte aligned (every cudaMalloc or torch
 *     allocation is); with buffers that are only 16-byte aligned the general path gives the
 *     same results, more slowly.  The caller owns all buffers, workspaces included; no entry point
 *     allocates memory.  The library's own state is small and fixed: one device error word
 *     (race_attn_device_error), the kernel timers of race_attn_profile_* (host side, off
 *     unless enabled), and the fixed device buffer of race_attn_forward_noalloc, which is
 *     part of the library's device code and is held by every GPU that loads it.  Apart from
 *     those, nothing persists from one call to the next.
 *   - Execution is asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *     stream).  Nothing synchronises the host.
 *   - Arguments are validated before anything is launched; a rejected call launches
 *     nothing and returns RACE_ERR_INVALID_ARG, RACE_ERR_UNSUPPORTED or
 *     RACE_ERR_WORKSPACE.  A launch failure reported by the CUDA runtime returns
 *     RACE_ERR_CUDA (the runtime's own error stays readable with cudaGetLastError()).
 *   - Supported: B, H >= 1; N >= 0 (N = 0 is a no-op); d a multiple of 8 in [8, 128];
 *     1 <= P <= 5; L >= 1 with L * 2^P <= 1024; tau >= 0 and finite; dtype RACE_F32 or
 *     RACE_BF16.  fp32 inputs are computed in fp32; bf16 inputs of the shape d = 64, L = 16,
 *     P = 4 run on the tensor cores with bf16 operands (features, the staged statistics,
 *     W as a bf16 hi + lo pair) and fp32 accumulation, other bf16 shapes in fp32.
 */
#ifndef RACE_ATTN_H
#define RACE_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t, declared here so the header needs no CUDA include. */
typedef struct CUstream_st *race_stream_t;

typedef enum {
    RACE_OK = 0,
    RACE_ERR_INVALID_ARG = 1, /* null pointer, negative size, misaligned pointer, bad tau */
    RACE_ERR_UNSUPPORTED = 2, /* valid but outside the supported set (d, P, L*2^P, tau=0 backward) */
    RACE_ERR_WORKSPACE = 3,   /* workspace or ctx buffer smaller than the size query says */
    RACE_ERR_CUDA = 4         /* the CUDA runtime reported an error while launching */
} race_status_t;

typedef enum { RACE_F32 = 0, RACE_BF16 = 1 } race_dtype_t;

/* Human-readable name of a status code (static storage, never NULL). */
const char *race_status_string(race_status_t status);

/*
 * Device workspace, in bytes, that race_attn_forward (backward = 0) or
 * race_attn_backward (backward = 1) needs for these sizes, written to *bytes.
 * The workspace holds the per-segment bucket statistics of the chunked scan
 * (fp32, L*2^P x (d+1) per segment and head; the backward needs two such buffers plus
 * 16 KB and one fp32 per token for c_i = -(dO_i . o_i)); it is scratch: its contents on
 * entry are ignored and on exit are unspecified.  For bf16 inputs with d = 128, P = 5,
 * L a multiple of 8 up to 32, causal, the size also covers the per-head arrays of the
 * feature-group tensor-core path (the normalised projections of q and k, one side's
 * dLoss/dp and fp32 sums over the feature groups: about (4 * L * P * 3 + 516) bytes per
 * token of one head in the backward); with a smaller workspace that still holds the
 * statistics, those shapes run on the general path.
 */
race_status_t race_attn_workspace_size(int B, int H, int64_t N, int d, int L, int P, int causal,
                                       int backward, race_dtype_t dtype, size_t *bytes);

/*
 * Size, in bytes, of the optional saved-state buffer `ctx` (fp32 device memory).
 * race_attn_forward can leave in it the key-side bucket statistics of every sequence
 * segment (the running sums A_cum, B_cum of Algorithm 2, zh §2.3, at each segment
 * start; for the bidirectional form, the totals A, B of Algorithm 1); handing the same
 * buffer to race_attn_backward with the same q, k, v, W and sizes saves the backward
 * pass one read of k and v.  For the shapes of the feature-group tensor-core path (d = 128,
 * P = 5, L a multiple of 8, causal) the size leaves room for either path's statistics and a
 * 16-byte tag after them: that path's forward keeps its own layout there and sets the tag,
 * every other forward clears it; the feature-group backward checks the tag on the device
 * and otherwise recomputes, and every other backward recomputes for these shapes.
 */
race_status_t race_attn_ctx_size(int B, int H, int64_t N, int d, int L, int P, int causal,
                                 size_t *bytes);

/*
 * Forward pass (Algorithm 1 when causal = 0, Algorithm 2 when causal = 1; zh §2.2-2.3).
 *   q, k, v    device, [B,H,N,d] of `dtype`, read only.  q and k need not be normalised:
 *              rows are scaled to unit norm inside (|x| floored at 1e-12).
 *   W          device, [L,P,d] fp32, read only: the Gaussian hyperplanes.
 *   out        device, [B,H,N,d] of `dtype`, written.
 *   den        device, [B,H,N] fp32, written: the denominator Y_i[d] (needed by the
 *              backward pass); may be NULL.  Hard hashing can leave a query with no key
 *              in any of its buckets: then den_i = 0 and out_i = 0.
 *   ctx        device or NULL; if not NULL, ctx_bytes >= race_attn_ctx_size(...) and the
 *              saved state is written there.
 *   tau        temperature; beta = 1/tau scales the corner logits; tau = 0 = hard hash.
 *   workspace  device, workspace_bytes >= race_attn_workspace_size(..., backward = 0).
 */
race_status_t race_attn_forward(const void *q, const void *k, const void *v, const float *W,
                                void *out, float *den, float *ctx, size_t ctx_bytes, int B,
                                int H, int64_t N, int d, int L, int P, float tau, int causal,
                                race_dtype_t dtype, void *workspace, size_t workspace_bytes,
                                race_stream_t stream);

/*
 * Backward pass: gradients of sum(out * dout) with respect to q, k and v, by the chain
 * rule through the forward above (the pages state the method is differentiable end to
 * end, es §2.3; they print no gradient formula).  W gets no gradient here: it is a fixed
 * random projection (zh §2.2); race_attn_backward_dw also returns it, for a learned W.
 *   q, k, v, W, out, den   the forward's inputs and outputs (den must not be NULL).
 *   dout       device, [B,H,N,d] of `dtype`.
 *   ctx        NULL, or the buffer a forward call with the same arguments filled.
 *   dq, dk, dv device, [B,H,N,d] of `dtype`, overwritten.
 *   tau        must be > 0 (hard hashing has no gradient: RACE_ERR_UNSUPPORTED).
 *   workspace  device, workspace_bytes >= race_attn_workspace_size(..., backward = 1).
 */
race_status_t race_attn_backward(const void *q, const void *k, const void *v, const float *W,
                                 const void *out, const float *den, const void *dout,
                                 const float *ctx, size_t ctx_bytes, void *dq, void *dk,
                                 void *dv, int B, int H, int64_t N, int d, int L, int P,
                                 float tau, int causal, race_dtype_t dtype, void *workspace,
                                 size_t workspace_bytes, race_stream_t stream);

/*
 * Hard sign-hash bucket of every row in every table (the one-hot assignment the soft
 * hash tends to as beta grows; es §2.3 contrasts the two):
 *   idx[b,h,n,l] = sum_p [W[l,p,:] . x[b,h,n,:] > 0] * 2^p,   int32, device, written.
 *   x          device, [B,H,N,d] of `dtype`.
 */
race_status_t race_attn_hash_indices(const void *x, const float *W, int32_t *idx, int B, int H,
                                     int64_t N, int d, int L, int P, race_dtype_t dtype,
                                     race_stream_t stream);

/*
 * Device-side failure report (a robustness aid; the method has no counterpart).  Every wait
 * of the tensor-core kernels on an MMA or load completion gives up after 2 s; a kernel that
 * gave up skips the rest of its work, waits (again bounded) for its loads in flight, releases
 * its tensor memory, returns, and sets a device error word.  race_attn_device_error waits for `stream`, writes that word to *flag (0 = no wait
 * ever timed out, 1 = one did) and clears it.
 */
race_status_t race_attn_device_error(int *flag, race_stream_t stream);

/*
 * Self-test of that mechanism: launches one CTA that waits on a barrier nothing arrives on,
 * for at most limit_ns nanoseconds (1 <= limit_ns <= 1e9), then records the timeout exactly
 * as a stalled MMA would.  A following race_attn_device_error reports 1.
 */
race_status_t race_attn_selftest_wait_timeout(int64_t limit_ns, race_stream_t stream);

/*
 * Forward pass that allocates nothing and takes no workspace (the method's description has
 * no counterpart to this; it is a deployment convenience).  It is for callers that cannot
 * obtain device memory on their own: code whose device memory is owned by a host
 * framework's allocator that forbids other allocations, or loops that must not pay the
 * device-wide synchronisation a cudaMalloc can cause.  The segment statistics that
 * race_attn_forward keeps in its workspace live instead in one fixed buffer of
 * RACE_NOALLOC_SCRATCH_BYTES that the library defines in device memory; every GPU that
 * loads the library holds that buffer until the process exits.
 *   Arguments as race_attn_forward (ctx is not offered).  Returns RACE_ERR_WORKSPACE, having
 *   launched nothing, when race_attn_workspace_size(..., backward = 0) for these sizes
 *   exceeds RACE_NOALLOC_SCRATCH_BYTES (for d = 64 and 2^P = 16, L = 16, that is B * H * nseg
 *   segment states of 66.5 KB each, nseg being the segments the library plans per sequence:
 *   at most N / 128, usually about (SM count) / (B * H); for bf16, d = 128, P = 5,
 *   causal, it includes the per-head arrays of the feature-group path, about
 *   (4 * L * P * 2 + 516) bytes per token; race_attn_workspace_size gives the exact figure).
 *   The first call on each device looks up the buffer's device address (a runtime call
 *   with that device current).  With CUDA's default lazy module loading, that first call is
 *   also when the library's device code, and with it this buffer, is loaded onto the device,
 *   so it is the one call that can fail for lack of device memory (RACE_ERR_CUDA).  Make one
 *   warm-up call at set-up, on every device, before any stream capture and before a host
 *   framework reserves the device's memory; later calls only reuse the buffer.  The address
 *   is remembered per device together with the ID of the context it belongs to, so after a
 *   cudaDeviceReset the next call looks it up again (and is such a first call again).
 *   All calls share the buffer and it keeps the last call's contents: every element a call
 *   reads is first written by the same call, so nothing needs clearing, but calls whose
 *   executions overlap on the GPU (different streams, or several host threads) race on it
 *   and must be serialised by the caller.
 */
#define RACE_NOALLOC_SCRATCH_BYTES ((size_t)24 << 20)
race_status_t race_attn_forward_noalloc(const void *q, const void *k, const void *v,
                                        const float *W, void *out, float *den, int B, int H,
                                        int64_t N, int d, int L, int P, float tau, int causal,
                                        race_dtype_t dtype, race_stream_t stream);

/*
 * Backward that also returns the gradient with respect to the hyperplanes, for the variant
 * in which W is learned (the pages treat W as fixed Gaussian hyperplanes, zh §2.2; this is
 * the chain rule through p_l = W_l x^ for every q and k row):
 *   dW[l][p][:] = sum over heads and rows of dLoss/dp_lp * x^,   x^ = x / max(|x|, 1e-12).
 *   dW         device fp32 [L,P,d], written (not accumulated; zero when N = 0).
 *   workspace  workspace_bytes >= race_attn_dw_workspace_size(...); scratch.
 * Other arguments, results and errors as race_attn_backward.  dW is summed over rows in a
 * fixed order (per split, then over the splits), so repeated calls give the same bits.
 */
race_status_t race_attn_dw_workspace_size(int B, int H, int64_t N, int d, int L, int P, int causal,
                                          race_dtype_t dtype, size_t *bytes);
race_status_t race_attn_backward_dw(const void *q, const void *k, const void *v, const float *W,
                                    const void *out, const float *den, const void *dout,
                                    const float *ctx, size_t ctx_bytes, void *dq, void *dk,
                                    void *dv, float *dW, int B, int H, int64_t N, int d, int L,
                                    int P, float tau, int causal, race_dtype_t dtype,
                                    void *workspace, size_t workspace_bytes,
                                    race_stream_t stream);

/*
 * ---- one sequence sharded over several devices -------------------------------------------
 * The statistics of Algorithm 2 (zh §2.3) are sums over tokens, so a sequence split into
 * contiguous shards (one per device, shard s holding tokens [s*n, (s+1)*n) of every head)
 * needs from the other shards only their totals: the forward of shard s starts its causal
 * scan from the key-side statistics of shards 0..s-1, and the backward's key side starts
 * from the query-side statistics G of shards s+1.. (bidirectional: every other shard's).
 * Each pass is split in two around that exchange, which the caller performs (an all-gather
 * over the shards, e.g. NCCL, then race_attn_shard_combine).  The two halves of a pass
 * must get the same ctx and workspace; in between, the caller may use the stream freely.
 * A single device is the one-shard case: begin + end with NULL init equals the one-call
 * entry point.
 */

/* Forward, first half: the key-side segment statistics into ctx (or the workspace) and
 * this shard's total, h_total = sum over its keys of phi(k)[v, 1]^T, fp32
 * [B*H][L*2^P][d+1] (required).  Other arguments as race_attn_forward. */
race_status_t race_attn_forward_begin(const void *k, const void *v, const float *W, float *ctx,
                                      size_t ctx_bytes, float *h_total, int B, int H, int64_t N,
                                      int d, int L, int P, float tau, int causal,
                                      race_dtype_t dtype, void *workspace,
                                      size_t workspace_bytes, race_stream_t stream);

/* Forward, second half: the scan starts from h_init ([B*H][L*2^P][d+1] fp32: the keys of
 * the shards before this one, causal; of every other shard, bidirectional; NULL = none),
 * then out, den (and ctx, which then includes h_init) as race_attn_forward. */
race_status_t race_attn_forward_end(const void *q, const void *k, const void *v, const float *W,
                                    const float *h_init, void *out, float *den, float *ctx,
                                    size_t ctx_bytes, int B, int H, int64_t N, int d, int L, int P,
                                    float tau, int causal, race_dtype_t dtype, void *workspace,
                                    size_t workspace_bytes, race_stream_t stream);

/* Backward, first half: dq, and this shard's query-side total g_total = sum over its
 * queries of phi(q_i) dY_i^T, dY_i = [dO_i, c_i] / den_i, fp32 [B*H][L*2^P][d+1]
 * (required).  With ctx from race_attn_forward_end the key-side statistics (h_init
 * included) are read from it; without, they are recomputed starting from h_init. */
race_status_t race_attn_backward_begin(const void *q, const void *k, const void *v,
                                       const float *W, const void *out, const float *den,
                                       const void *dout, const float *ctx, size_t ctx_bytes,
                                       const float *h_init, void *dq, float *g_total, int B,
                                       int H, int64_t N, int d, int L, int P, float tau,
                                       int causal, race_dtype_t dtype, void *workspace,
                                       size_t workspace_bytes, race_stream_t stream);

/* Backward, second half: dk, dv with the key side's suffix statistics starting from g_init
 * (the queries of the shards after this one, causal; of every other shard, bidirectional;
 * NULL = none).  workspace: the one race_attn_backward_begin used, unchanged since. */
race_status_t race_attn_backward_end(const void *q, const void *k, const void *v, const float *W,
                                     const void *out, const float *den, const void *dout,
                                     const float *g_init, void *dk, void *dv, int B, int H,
                                     int64_t N, int d, int L, int P, float tau, int causal,
                                     race_dtype_t dtype, void *workspace,
                                     size_t workspace_bytes, race_stream_t stream);

/* out[e] = sum over the selected shards s of gathered[s][e], in shard order: which = 0 the
 * shards before `shard`, 1 those after it, 2 every other shard.  gathered: device fp32
 * [nshards][elems] (the shards' totals side by side, as an all-gather leaves them). */
race_status_t race_attn_shard_combine(const float *gathered, int nshards, int shard, int which,
                                      int64_t elems, float *out, race_stream_t stream);

/*
 * Bucket statistics of every key of each head: H[m][c] = sum_j phi(k_j)[m] [v_j, 1][c],
 * m = l * 2^P + r, i.e. B_l (columns 0..d-1) and A_l (column d) of zh §2.2 for all tables in
 * one array -- the running statistics of Algorithm 2 (zh §2.3) after the last token, which
 * race_attn_decode_step continues from (a prompt of N tokens, then one token per step).
 *   k, v       device, [B,H,N,d] in dtype, 16-byte aligned.
 *   W          device fp32 [L,P,d], as race_attn_forward.
 *   state      device fp32 [B*H][L*2^P][d+1], written (zero-filled when N = 0).
 *   tau        >= 0 as race_attn_forward (0: hard sign hash).
 *   workspace  device, workspace_bytes >= race_attn_workspace_size(..., backward = 0); scratch.
 * Sizes and errors as race_attn_forward.  Asynchronous on `stream`.
 */
race_status_t race_attn_state(const void *k, const void *v, const float *W, float *state, int B,
                              int H, int64_t N, int d, int L, int P, float tau,
                              race_dtype_t dtype, void *workspace, size_t workspace_bytes,
                              race_stream_t stream);

/* Device workspace, in bytes, that race_attn_decode_step needs for these sizes. */
race_status_t race_attn_decode_workspace_size(int B, int H, int d, int L, int P, size_t *bytes);

/*
 * One streaming (decode-time) step of Algorithm 2 (zh §2.3) for every (b, h): the new
 * token joins the cumulative statistics, then its query is read out of them,
 *   H += phi(k_t) [v_t, 1]^T;   Y = phi(q_t)^T H;   out_t = Y[:d] / Y[d],  den_t = Y[d]
 * with the feature map of race_attn_forward, so that a prompt's race_attn_state followed by
 * steps for tokens N, N+1, ... gives the causal forward's rows N, N+1, ... .
 *   q, k, v    device, [B,H,d] in dtype: the new token of every head.
 *   W          device fp32 [L,P,d].
 *   state      device fp32 [B*H][L*2^P][d+1], read and updated in place.
 *   out        device [B,H,d] in dtype, written; den device fp32 [B,H] or NULL.
 *   tau        >= 0 (0: hard sign hash; a row whose buckets are all empty gets out = 0).
 *   workspace  device, workspace_bytes >= race_attn_decode_workspace_size(...); scratch.
 * Pointers 16-byte aligned.  Sizes as race_attn_forward (N does not apply).  Errors:
 * RACE_ERR_INVALID_ARG (NULL or misaligned pointers, bad sizes or tau),
 * RACE_ERR_UNSUPPORTED, RACE_ERR_WORKSPACE, RACE_ERR_CUDA.  Asynchronous on `stream`;
 * calls on one state must be ordered (same stream).
 */
race_status_t race_attn_decode_step(const void *q, const void *k, const void *v, const float *W,
                                    float *state, void *out, float *den, int B, int H, int d,
                                    int L, int P, float tau, race_dtype_t dtype, void *workspace,
                                    size_t workspace_bytes, race_stream_t stream);

/*
 * Opt-in kernel timing (a measurement aid; the method has no counterpart).  While enabled,
 * every kernel the library launches is bracketed by a pair of CUDA events recorded on the
 * launch stream; race_attn_profile_read waits for the recorded events, adds each
 * kernel's elapsed time to its running total and reports the totals.  Off by default;
 * costs two event records per launch when on.  Not thread-safe.
 */
void race_attn_profile_enable(int on);
void race_attn_profile_reset(void);
/*
 * Writes up to max_kernels entries: names[i] (NUL-terminated, at most 63 chars, in a
 * caller buffer of max_kernels * 64 chars), total milliseconds ms[i] and launch counts
 * launches[i]; returns the number of distinct kernels seen (may exceed max_kernels), or
 * -1 if a recorded event reports an error.
 */
int race_attn_profile_read(char *names, float *ms, int64_t *launches, int max_kernels);

#ifdef __cplusplus
}
#endif

#endif /* RACE_ATTN_H */
