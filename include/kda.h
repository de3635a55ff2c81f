/*
 * kda.h -- C ABI of the B200 (sm_100a) Kimi Delta Attention (KDA) operator.
 *
 * The operator (wiki page "Kimi Linear 高效注意力架构", section "Kimi Delta
 * Attention (KDA)", state-update equation): per head a d_k x d_v state
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,
 *
 * with one decay alpha_t,i in (0, 1] per key channel (same section, channel-wise
 * decay bullet; passed here as log alpha) and a scalar beta_t; the read-out is
 * the delta-rule read-out of the post-update state, o_t = S_t^T q_t.  The pages
 * fix the state at d_k x d_v = 128 x 128 per head (same section, linear
 * complexity bullet).  q and k are used as given: the L2 normalisation and any
 * scaling of q belong to the caller (the KDA layer normalises q and k before the
 * operator, section "模型架构").
 *
 * Conventions shared by every call
 * --------------------------------
 * - All tensor pointers are DEVICE pointers to caller-owned memory, except the
 *   ones named *_host.  The library never allocates or frees device memory.
 * - Layouts are dense row-major, tokens packed over sequences:
 *       q, k       [T_total, H, d_k]   dtype qkv_dtype
 *       v, o       [T_total, H, d_v]   dtype qkv_dtype
 *       log_alpha  [T_total, H, d_k]   float32, every value <= 0
 *       beta       [T_total, H]        float32
 *       S0/S_final [N, H, d_k, d_v]    float32, d_v contiguous
 *   q, k, v, o, log_alpha, S0, S_final must be 16-byte aligned.
 * - Work is queued on `stream` (a cudaStream_t; NULL = legacy default stream)
 *   and runs asynchronously; the call returns once it is queued.
 * - Argument errors are found on the host before anything is queued; they
 *   leave all outputs untouched and return KDA_ERR_INVALID_ARG or
 *   KDA_ERR_UNSUPPORTED.  A failed launch returns KDA_ERR_CUDA.  No call aborts,
 *   throws, or prints.
 */
#ifndef KDA_B200_KDA_H
#define KDA_B200_KDA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Symbols of this header are the library's only exported ones. */
#if defined(__GNUC__)
#define KDA_API __attribute__((visibility("default")))
#else
#define KDA_API
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st *kda_stream_t;

typedef enum {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARG = 1,   /* null pointer, bad size, bad cu_seqlens, misalignment */
    KDA_ERR_UNSUPPORTED = 2,   /* legal arguments no kernel here implements */
    KDA_ERR_WORKSPACE = 3,     /* workspace missing or smaller than required */
    KDA_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed */
    KDA_ERR_DEVICE_FAULT = 5   /* a kernel flagged an internal error (see kda_workspace_status) */
} kda_status_t;

typedef enum {
    KDA_DTYPE_F32 = 0,   /* float32 q/k/v/o */
    KDA_DTYPE_BF16 = 1   /* bfloat16 q/k/v/o (state and gates stay float32) */
} kda_dtype_t;

/* Human-readable name of a status code (static storage, never NULL). */
KDA_API const char *kda_status_string(kda_status_t status);

/* Library ABI version: major * 10000 + minor * 100 + patch. */
KDA_API int kda_version(void);

/*
 * Bytes of device workspace kda_prefill needs for these sizes.  Depends only on
 * its arguments; returns 0 for arguments kda_prefill would reject.  On the
 * tensor-core shapes (bf16, d_k = d_v = 128, chunk 64) with at least 16,384 tokens
 * the size includes room for the start states of a sequence split (up to
 * 3 * P * m * H * 64 KiB, m <= 8 split sequences, P <= 8 segments): a sequence much
 * longer than the rest is cut into as many segments (3 to 8, at least 4096 tokens
 * each) as the device's SMs can run side by side for H heads, with the states between
 * them chained from the segments' transitions.  A workspace of only 256 + 4 num_seqs
 * bytes (rounded up to 256) is still accepted; the call then runs unsplit.
 */
KDA_API size_t kda_prefill_workspace_size(int num_seqs, int64_t total_tokens, int H, int d_k,
                                  int d_v, int chunk, kda_dtype_t qkv_dtype);

/*
 * kda_prefill -- chunked prefill over packed variable-length sequences.
 *
 * Runs the state-update equation over every token of every sequence and head,
 * starting from S0 (NULL = zero state), writes o_t = S_t^T q_t for every token
 * and the state after each sequence's last token to S_final.  The work is
 * organised in chunks of `chunk` tokens (the chunkwise form named in the KDA
 * section's "硬件高效分块算法" bullet); chunks start at each sequence's first token
 * and never cross a sequence boundary.  The result does not depend on `chunk`
 * except through rounding.
 *
 *   q, k, v, qkv_dtype   inputs, layouts above
 *   log_alpha, beta      float32 gates, layouts above
 *   S0                   float32 initial states or NULL; may alias S_final
 *   cu_seqlens_dev       int32 [num_seqs + 1] device copy of the offsets
 *   cu_seqlens_host      int32 [num_seqs + 1] host copy of the same offsets
 *                        (read during the call only; must equal the device copy)
 *                        cu_seqlens[0] = 0, non-decreasing; zero-length
 *                        sequences are allowed and give S_final = S0 (or 0)
 *   num_seqs, H, d_k, d_v  sizes: num_seqs >= 0, H >= 1, 1 <= d_k, d_v <= 128
 *   chunk                16, 32 or 64
 *   o                    [T_total, H, d_v] output, dtype qkv_dtype
 *   S_final              [num_seqs, H, d_k, d_v] float32 output
 *   workspace            device scratch of at least
 *                        kda_prefill_workspace_size(...) bytes, 256-byte aligned;
 *                        contents on entry are ignored; not to be shared by two
 *                        calls that may run at the same time
 *
 * Supported: any 1 <= d_k, d_v <= 128 (float32 CUDA-core path); the tensor-core
 * path is taken for bf16 with d_k = d_v = 128 and chunk = 64.  Anything else
 * returns KDA_ERR_UNSUPPORTED.
 */
KDA_API kda_status_t kda_prefill(const void *q, const void *k, const void *v, kda_dtype_t qkv_dtype,
                         const float *log_alpha, const float *beta, const float *S0,
                         const int32_t *cu_seqlens_dev, const int32_t *cu_seqlens_host,
                         int num_seqs, int H, int d_k, int d_v, int chunk,
                         void *o, float *S_final, void *workspace, size_t workspace_bytes,
                         kda_stream_t stream);

/*
 * kda_prologue -- the KDA layer's input prologue: it makes kda_prefill's inputs from
 * the layer's projections.
 *
 * The wiki page "Kimi Linear 高效注意力架构", section "模型架构", lists ShortConv +
 * Swish + L2Norm (q/k) and a low-rank channel-wise decay gate in the KDA layer,
 * without formulas.  This call computes, per sequence of cu_seqlens, head h and
 * channel c (the plainest reading of that line):
 *
 *   conv(x)[t] = sum_{w < conv_width} conv[h][c][w] * x[t - w]   (x = 0 before the
 *                sequence's first token: the convolution never crosses a sequence)
 *   q = l2norm(swish(conv_q(q_pre))), k = l2norm(swish(conv_k(k_pre))), v = swish(conv_v(v_pre))
 *   swish(z) = z * sigmoid(z),  l2norm(z) = z / sqrt(sum_c z_c^2 + l2_eps) over the head's channels
 *   log_alpha = -rate[h] * softplus(a_gate),  beta = sigmoid(b_gate)
 *
 *   q_pre, k_pre      [T_total, H, d_k] dtype     v_pre   [T_total, H, d_v] dtype
 *   conv_q, conv_k    [H, d_k, conv_width] f32    conv_v  [H, d_v, conv_width] f32
 *   a_gate            [T_total, H, d_k] f32 (the low-rank gate's output)
 *   rate              [H] f32 (> 0 for log_alpha <= 0)     b_gate [T_total, H] f32
 *   q, k, v, log_alpha, beta   outputs in kda_prefill's layouts (q/k/v in dtype)
 * Row pointers (q_pre, k_pre, v_pre, a_gate, q, k, v, log_alpha) are 16-byte aligned.
 * Supported: 1 <= conv_width <= 4, d_k and d_v multiples of 4 up to 128; otherwise
 * KDA_ERR_UNSUPPORTED.  l2_eps >= 0 and finite.  HBM-bound; one launch.
 */
KDA_API kda_status_t kda_prologue(const void *q_pre, const void *k_pre, const void *v_pre, kda_dtype_t dtype,
                          const float *conv_q, const float *conv_k, const float *conv_v, int conv_width,
                          const float *a_gate, const float *rate, const float *b_gate,
                          const int32_t *cu_seqlens_dev, const int32_t *cu_seqlens_host, int num_seqs, int H,
                          int d_k, int d_v, float l2_eps, void *q, void *k, void *v, float *log_alpha,
                          float *beta, kda_stream_t stream);

/*
 * kda_prefill_gated -- kda_prefill with the KDA layer's output epilogue applied to o.
 *
 * The wiki page "Kimi Linear 高效注意力架构", section "模型架构", lists a sigmoid
 * output gate and an RMSNorm as the end of the KDA layer, without a formula.  This
 * call writes, for every token t and head h (the plainest reading of that line),
 *
 *   y[t,h,:] = o[t,h,:] / sqrt(mean_j o[t,h,j]^2 + eps) * norm_weight * sigmoid(gate[t,h,:])
 *
 * where o is what kda_prefill would write, the mean runs over the d_v value channels
 * of one head, and norm_weight is shared by the heads.  On the tensor-core path
 * (bf16, d_k = d_v = 128, chunk = 64) the epilogue is fused into the output store:
 * o never reaches memory.  With float32 inputs (any shape kda_prefill takes) the
 * prefill writes o into y and a second kernel applies the epilogue in place.  Other
 * bf16 shapes return KDA_ERR_UNSUPPORTED (o would be rounded to bf16 twice).
 *
 *   gate         [T_total, H, d_v], dtype qkv_dtype: the gate's pre-activation
 *                (caller-owned, read only; 16-byte aligned)
 *   norm_weight  [d_v] float32 RMSNorm weight (read only)
 *   eps          > 0 and finite, added to the mean square inside the root
 *   y            [T_total, H, d_v] output, dtype qkv_dtype
 * Every other argument, the workspace rule, S_final and the error behaviour are
 * kda_prefill's; a bad eps or a NULL gate / norm_weight (with T_total > 0) returns
 * KDA_ERR_INVALID_ARG.
 */
KDA_API kda_status_t kda_prefill_gated(const void *q, const void *k, const void *v, kda_dtype_t qkv_dtype,
                               const float *log_alpha, const float *beta, const float *S0,
                               const int32_t *cu_seqlens_dev, const int32_t *cu_seqlens_host,
                               int num_seqs, int H, int d_k, int d_v, int chunk,
                               const void *gate, const float *norm_weight, float eps,
                               void *y, float *S_final, void *workspace, size_t workspace_bytes,
                               kda_stream_t stream);

/*
 * kda_decode_step -- one recurrent decode step for B independent sequences.
 *
 * For every (b, h): S <- (I - beta k k^T) Diag(alpha) S + beta k v^T in place,
 * then o = S^T q (the same equation applied to a single token; the fixed-size
 * state is what makes decode cost independent of context length, section
 * "效率" of the same page).
 *
 *   q, k       [B, H, d_k] qkv_dtype      v, o  [B, H, d_v] qkv_dtype
 *   log_alpha  [B, H, d_k] float32        beta  [B, H] float32
 *   S          [B, H, d_k, d_v] float32, read and overwritten in place
 * Supported: 1 <= d_k <= 128, d_v in {4, 8, ..., 128}.  B = 0 is a no-op.
 */
KDA_API kda_status_t kda_decode_step(const void *q, const void *k, const void *v, kda_dtype_t qkv_dtype,
                             const float *log_alpha, const float *beta, float *S,
                             int B, int H, int d_k, int d_v, void *o, kda_stream_t stream);

/*
 * kda_prefill_noalloc -- kda_prefill for callers that cannot allocate device memory.
 *
 * The pages have no counterpart: this is a deployment variant of kda_prefill.
 * Some callers cannot call cudaMalloc where they run the operator (a host
 * framework that owns every allocation, a plug-in handed only its inputs and
 * outputs, a path where allocating would synchronise or fail under memory
 * pressure).  This call takes the same arguments as kda_prefill minus the
 * workspace and allocates nothing, with no library routine that allocates: its
 * scratch (status word and sequence order) is one file-scope device array of
 * 256 + 4 * KDA_NOALLOC_MAX_SEQS bytes that every GPU loading the library holds
 * until the process exits.
 *
 * - num_seqs > KDA_NOALLOC_MAX_SEQS returns KDA_ERR_WORKSPACE before anything is
 *   queued; the other argument checks are kda_prefill's.
 * - It never uses kda_prefill's sequence split (which needs workspace for the
 *   segments' start states): every (sequence, head) runs as one unit.  Where
 *   kda_prefill would split a very long sequence, this call takes longer (the
 *   long sequence's chunks run one after another on one SM per head); elsewhere
 *   it runs the same kernels on the same inputs and gives bit-identical results.
 * - The first call on a device looks up the array's device address for that
 *   device (once per device, with that device current); make that first call
 *   before any stream capture.
 * - All calls share the array and it keeps the last call's contents (the status
 *   word is cleared at the start of each call): calls that may overlap on the GPU,
 *   on any streams, race on it and must be ordered by the caller.
 * - A kernel-side error flag set during this call is not reported back; use
 *   kda_prefill with a workspace and kda_workspace_status to observe it.
 */
#define KDA_NOALLOC_MAX_SEQS 65536
KDA_API kda_status_t kda_prefill_noalloc(const void *q, const void *k, const void *v, kda_dtype_t qkv_dtype,
                                 const float *log_alpha, const float *beta, const float *S0,
                                 const int32_t *cu_seqlens_dev, const int32_t *cu_seqlens_host,
                                 int num_seqs, int H, int d_k, int d_v, int chunk,
                                 void *o, float *S_final, kda_stream_t stream);

/*
 * kda_decode_tokens -- n consecutive tokens for B sequences whose states live in a
 * pool of state slots (serving-style decode, and the multi-token form of the
 * recurrence used to check several drafted tokens at once).
 *
 * For every b with 0 <= slot_idx[b] < num_slots and every head, the state in
 * that slot is advanced through tokens 0 .. n-1 of sequence b by the same
 * equation as kda_decode_step (o written for every token) and written back.  The
 * state crosses HBM once per call instead of once per token.
 *
 *   q, k, log_alpha  [B, n, H, d_k]    v, o  [B, n, H, d_v]    beta  [B, n, H]
 *   S_pool    [num_slots, H, d_k, d_v] float32, 16-byte aligned, read and updated
 *   slot_idx  [B] int32 device array, or NULL for slot b (then num_slots >= B);
 *             a slot outside [0, num_slots) skips sequence b (no output written);
 *             two sequences of one call must not share a slot (their updates race)
 * Supported: 1 <= d_k <= 128, d_v in {4, 8, ..., 128}; B = 0 or n = 0 is a no-op.
 */
KDA_API kda_status_t kda_decode_tokens(const void *q, const void *k, const void *v, kda_dtype_t qkv_dtype,
                               const float *log_alpha, const float *beta, float *S_pool,
                               const int32_t *slot_idx, int num_slots, int B, int n, int H,
                               int d_k, int d_v, void *o, kda_stream_t stream);

/*
 * kda_workspace_status -- waits for `stream`, then reports whether a kernel of
 * the last kda_prefill call that used `workspace` flagged an internal error
 * (KDA_ERR_DEVICE_FAULT, e.g. a bounded wait that ran out) and clears the flag.
 * Returns KDA_OK when none did, KDA_ERR_CUDA when the wait itself failed.
 */
KDA_API kda_status_t kda_workspace_status(const void *workspace, kda_stream_t stream);

/*
 * kda_backward_workspace_size -- bytes of device workspace kda_backward needs for
 * these sizes (0 when they are unsupported).  About
 *   (T/32 + N + 1) * H * ceil(d_v/16) * 8 KiB      state checkpoints
 *   + T * H * 64 * ceil(d_v/16)                    per-token residuals w_t
 * (plus 256 bytes and rounding), e.g. 1.35 GB for T = 16384, H = 32, d = 128.
 */
KDA_API size_t kda_backward_workspace_size(int num_seqs, int64_t total_tokens, int H, int d_k, int d_v);

/*
 * kda_backward -- gradients of the KDA recurrence (training).
 *
 * The forward map is kda_prefill's (the state-update equation of the wiki page
 * "Kimi Linear 高效注意力架构", section "关键技术方法 > Kimi Delta Attention (KDA)",
 * with o_t = S_t^T q_t read from the post-update state).  Given dO = dL/do_t for
 * every token and dS_final = dL/dS_final, this returns the exact gradients of L
 * through the recurrence:
 *
 *   dq, dk       [T, H, d_k] float32      dlog_alpha [T, H, d_k] float32
 *   dv           [T, H, d_v] float32      dbeta      [T, H]      float32
 *   dS0          [N, H, d_k, d_v] float32, or NULL when not wanted
 *
 * Inputs are kda_prefill's (q, k, v of qkv_dtype; log_alpha, beta, S0 float32;
 * S0 NULL = zeros; the same cu_seqlens on the device and the host), plus
 *   dO        [T, H, d_v] of qkv_dtype
 *   dS_final  [N, H, d_k, d_v] float32, or NULL for zeros; may alias dS0
 * All arithmetic is float32 on CUDA cores; the forward states are recomputed
 * inside the call (no forward output is needed).  Every output element is
 * written (gradients of empty sequences' tokens do not exist; dS0 of an empty
 * sequence is dS_final).  dq, dk, dlog_alpha and dbeta are sums over slices of 16
 * value channels, which the kernel adds into the zeroed outputs with float32
 * atomics: the order of those additions is not fixed, so repeated calls can differ
 * in the last bits of these four outputs (dv and dS0 are written once).
 *
 * Supported: 1 <= d_k, d_v <= 128, float32 or bfloat16 q/k/v/dO, num_seqs * H *
 * ceil(d_v / 16) < 2^31 (KDA_ERR_UNSUPPORTED otherwise); no alignment beyond each
 * type's own.  Workspace: kda_backward_workspace_size bytes,
 * 256-byte aligned (KDA_ERR_WORKSPACE otherwise).  Queues four memsets of the
 * outputs and two kernels on `stream`, asynchronously; the workspace and outputs
 * must not be touched until they finish.  Argument errors are reported before anything is queued.
 */
KDA_API kda_status_t kda_backward(const void *q, const void *k, const void *v, kda_dtype_t qkv_dtype,
                                  const float *log_alpha, const float *beta, const float *S0,
                                  const int32_t *cu_seqlens_dev, const int32_t *cu_seqlens_host,
                                  int num_seqs, int H, int d_k, int d_v, const void *dO,
                                  const float *dS_final, float *dq, float *dk, float *dv,
                                  float *dlog_alpha, float *dbeta, float *dS0, void *workspace,
                                  size_t workspace_bytes, kda_stream_t stream);

/*
 * kda_wait_timeout_selftest -- checks, on the caller's device, the error path that
 * every bounded wait inside the prefill kernels takes when the event it waits for
 * never comes.  One small kernel (1 block, 64 threads) waits on an mbarrier phase
 * that no thread completes and on a shared-memory progress counter that no thread
 * advances, each for at most `max_cycles` SM clock cycles; both waits run out, the
 * kernel sets the status word at the start of `workspace` (the same word
 * kda_prefill's kernels set) and exits normally.  Nothing else is touched, so the
 * context stays usable and kda_workspace_status(workspace, stream) then returns
 * KDA_ERR_DEVICE_FAULT (and clears the word).
 *
 *   workspace        device buffer of >= 256 bytes, 256-byte aligned
 *                    (a kda_prefill workspace will do); its first 8 bytes are
 *                    cleared, then written by the kernel
 *   max_cycles       1 .. 4e9 (4e9 is the prefill kernels' own limit, about two
 *                    seconds at the B200's top SM clock)
 *
 * Returns KDA_ERR_WORKSPACE for a missing, short or misaligned workspace,
 * KDA_ERR_INVALID_ARG for max_cycles out of range, KDA_ERR_CUDA if the launch
 * failed; the launch is asynchronous on `stream`.
 */
KDA_API kda_status_t kda_wait_timeout_selftest(void *workspace, size_t workspace_bytes, long long max_cycles,
                                       kda_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* KDA_B200_KDA_H */
