/*
 * kda.h -- C ABI of libkda.so, Kimi Delta Attention (KDA) on NVIDIA B200 (sm_100a).
 *
 * The operator is the per-head gated delta-rule recurrence
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,
 *     o_t = S_t^T q_t,          alpha_t = exp(log_alpha_t) in (0,1]^{d_k},
 *
 * with q_t, k_t L2-normalised and an fp32 d_k x d_v state S per (sequence, head).
 * Sources: "[Kimi-2] Kimi Linear：用 KDA 重写长上下文注意力" (xutianle.me) §3
 * (boxed update, three-step form), §1 (readout o_t = S_t^T q_t), §5 (chunkwise
 * prefill and recurrent decode), §6.2 (L2 norm of q, k; d_k = d_v = 128); and
 * "Kimi Linear — 逐通道的遺忘" (docsaid.org), "KDA：把衰減拆到每個通道".
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Pointers are DEVICE pointers unless stated otherwise. The caller owns every
 *   buffer; the library allocates no device memory and keeps no pointer after
 *   a call returns.
 * - Work is enqueued on `stream` and the call returns without synchronising.
 *   KDA_ERR_CUDA reports a launch error seen at enqueue time; faults during
 *   execution surface at the caller's next synchronisation.
 * - Arguments are validated on the host before anything is enqueued; on any
 *   error nothing is launched and the outputs are untouched.
 * - Every pointer must be 16-byte aligned, except beta and, with
 *   KDA_FLAG_SCALAR_GATE, log_alpha (4-byte aligned); KDA_ERR_MISALIGNED otherwise.
 *   Tensors are dense row-major with the layouts given below.
 * - Not checked (undefined behaviour if violated): cu_seqlens monotone with
 *   cu_seqlens[0] = 0 and cu_seqlens[N] = total_tokens; log_alpha finite and
 *   <= 0; beta in [0, 1]; outputs not overlapping inputs (except S_T == S0).
 * - State layout (one layout for prefill S0/S_T and the decode state):
 *   [N][H][d_k][d_v] fp32, row-major, d_v contiguous (row = key channel).
 */
#ifndef KDA_H_
#define KDA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *kda_stream_t; /* a cudaStream_t; NULL = legacy default stream */

typedef enum {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARG = 1, /* null pointer, bad size or inconsistent sizes */
    KDA_ERR_UNSUPPORTED = 2, /* valid but not implemented (d_k, d_v, chunk, dtype) */
    KDA_ERR_MISALIGNED = 3,  /* a pointer is not 16-byte aligned */
    KDA_ERR_WORKSPACE = 4,   /* workspace NULL or smaller than the minimum */
    KDA_ERR_CUDA = 5,        /* CUDA reported an error while enqueueing */
    KDA_ERR_TIMEOUT = 6      /* reserved: a bounded device-side wait gave up */
} kda_status;

typedef enum {
    KDA_DTYPE_F32 = 0, /* q, k, v and o in fp32 */
    KDA_DTYPE_BF16 = 1 /* q, k, v and o in bf16 (log_alpha, beta, state stay fp32) */
} kda_dtype;

/* flags */
#define KDA_FLAG_NO_L2NORM 0x1 /* q, k are used as given (caller already normalised) */
#define KDA_FLAG_EXACT 0x2     /* fp32 CUDA-core arithmetic even for bf16 inputs */
/* Gated DeltaNet form ("[Kimi-2] Kimi Linear" §3): one forget gate per (token, head),
 * S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T, i.e. the KDA update with
 * alpha_t broadcast over the d_k channels. log_alpha is then [T][H] (prefill) or [N][H]
 * (decode) fp32 instead of [..][H][dk]. */
#define KDA_FLAG_SCALAR_GATE 0x4

/* Human-readable name of a status code (static string, never NULL). */
const char *kda_status_string(kda_status status);

/* Library version as 10000*major + 100*minor + patch. */
int32_t kda_version(void);

/*
 * Workspace bytes kda_prefill performs best with for this problem. Any
 * workspace of at least kda_prefill_workspace_min() bytes also works (the
 * CUDA-core path then runs in more waves; the tensor-core path keeps fewer
 * prepared chunks in flight). Returns 0 if the arguments are invalid.
 * Arguments as for kda_prefill; max_seqlen <= 0 means "unknown"
 * (total_tokens is assumed).
 */
size_t kda_prefill_workspace_size(int32_t num_seqs, int64_t total_tokens, int32_t max_seqlen,
                                  int32_t H, int32_t dk, int32_t dv, kda_dtype dtype,
                                  int32_t chunk, uint32_t flags);
size_t kda_prefill_workspace_min(int32_t num_seqs, int64_t total_tokens, int32_t max_seqlen,
                                 int32_t H, int32_t dk, int32_t dv, kda_dtype dtype,
                                 int32_t chunk, uint32_t flags);

/*
 * Number of kernel launches kda_prefill enqueues for this problem with a
 * workspace of `workspace_bytes` (for sizing CUDA graphs and for accounting).
 * Returns -1 if the arguments are invalid or the workspace is too small.
 */
int64_t kda_prefill_launches(int32_t num_seqs, int64_t total_tokens, int32_t max_seqlen,
                             int32_t H, int32_t dk, int32_t dv, kda_dtype dtype, int32_t chunk,
                             uint32_t flags, size_t workspace_bytes);

/*
 * Chunkwise-parallel prefill over a packed batch of variable-length sequences
 * ("[Kimi-2] Kimi Linear" §5: parallel inside a chunk, recurrent between chunks).
 *
 *   q, k       [T][H][dk]  dtype         (T = total_tokens, all sequences packed)
 *   v          [T][H][dv]  dtype
 *   log_alpha  [T][H][dk]  fp32, <= 0    (per-key-channel log forget gate;
 *                                         [T][H] with KDA_FLAG_SCALAR_GATE)
 *   beta       [T][H]      fp32          (write strength)
 *   S0         [N][H][dk][dv] fp32 entry states, or NULL for zeros
 *   cu_seqlens [N+1] int32 (device) token offsets of the N sequences, or NULL
 *              for one sequence of T tokens (then num_seqs must be 1)
 *   max_seqlen host upper bound on the sequence lengths (<= 0: unknown)
 *   chunk      chunk length; 64 is supported
 *   o          [T][H][dv]  dtype, out: o_t = S_t^T q_t
 *   S_T        [N][H][dk][dv] fp32 exit states, out, or NULL; may alias S0
 *   workspace  device scratch of workspace_bytes (>= kda_prefill_workspace_min)
 *
 * Supported: dk, dv in {64, 128}; chunk = 64; dtype F32 or BF16. bf16 inputs
 * with dk = dv = 128 run on the tensor cores (bf16 operands, fp32 accumulation
 * and state) unless KDA_FLAG_EXACT; every other case uses fp32 CUDA-core
 * arithmetic. Sequences of length 0 are allowed (S_T = S0). max_seqlen must
 * not be smaller than any sequence length.
 */
kda_status kda_prefill(const void *q, const void *k, const void *v, const float *log_alpha,
                       const float *beta, const float *S0, const int32_t *cu_seqlens,
                       int32_t num_seqs, int64_t total_tokens, int32_t max_seqlen, int32_t H,
                       int32_t dk, int32_t dv, kda_dtype dtype, int32_t chunk, uint32_t flags,
                       void *o, float *S_T, void *workspace, size_t workspace_bytes,
                       kda_stream_t stream);

/*
 * Output step of the KDA layer fused into the store of o ("[Kimi-2] Kimi
 * Linear" §6 and §6.3): per (token, head), a head-wise RMSNorm over the d_v
 * channels followed by a sigmoid gate computed from the layer input,
 *
 *     o_t <- o_t / sqrt(mean_j(o_tj^2) + eps) * weight * sigmoid(gate_t).
 *
 *   gate    [T][H][dv] (prefill) / [N][H][dv] (decode), the dtype of q, k, v:
 *           the gate's pre-activation; 16-byte aligned
 *   weight  [dv] fp32, one RMSNorm weight vector shared by the heads; 4-byte aligned
 *   eps     RMSNorm epsilon (> 0)
 * The pages give neither eps nor the weight's shape; both are the caller's.
 */
typedef struct kda_output_gate {
    const void *gate;
    const float *weight;
    float eps;
} kda_output_gate;

/*
 * kda_prefill with the output step fused (out_gate != NULL) or not (NULL, then
 * identical to kda_prefill). Same arguments and rules as kda_prefill otherwise.
 */
kda_status kda_prefill_ex(const void *q, const void *k, const void *v, const float *log_alpha,
                          const float *beta, const float *S0, const int32_t *cu_seqlens,
                          int32_t num_seqs, int64_t total_tokens, int32_t max_seqlen, int32_t H,
                          int32_t dk, int32_t dv, kda_dtype dtype, int32_t chunk, uint32_t flags,
                          const kda_output_gate *out_gate, void *o, float *S_T, void *workspace,
                          size_t workspace_bytes, kda_stream_t stream);

/*
 * kda_prefill without a workspace argument, for callers that cannot allocate
 * device memory where they run the prefill (a runtime that owns all device
 * memory through its own pool and forbids library allocations, a plugin whose
 * host framework hides its allocator, or a serving loop that cannot afford a
 * cudaMalloc, which may synchronise the device). The pages have no
 * counterpart to this entry point; it exists only for such callers.
 *
 * Same arguments, outputs and results as kda_prefill; the workspace is a
 * fixed array of KDA_NOALLOC_SCRATCH_BYTES inside the library's device image,
 * held by every GPU that loads the library until the process exits. Nothing is
 * allocated: no cudaMalloc, cudaFree or allocating library call.
 * - Limit: problems whose kda_prefill_workspace_min() exceeds
 *   KDA_NOALLOC_SCRATCH_BYTES are refused with KDA_ERR_WORKSPACE before
 *   anything is enqueued. On the tensor-core path (bf16, d_k = d_v = 128)
 *   the minimum is about 8.5 MB plus 12 bytes per (sequence, head), so every
 *   practical problem fits; on the CUDA-core path it grows with num_seqs * H.
 * - The first call on a device resolves the array's address on that device
 *   (with that device current); make that first call before any stream
 *   capture begins.
 * - All calls share the one array, which keeps the last call's contents.
 *   Calls that overlap on the GPU (other streams, other host threads) race on
 *   it and give wrong results: order them on one stream or synchronise.
 */
#define KDA_NOALLOC_SCRATCH_BYTES (32u << 20)
kda_status kda_prefill_noalloc(const void *q, const void *k, const void *v, const float *log_alpha,
                               const float *beta, const float *S0, const int32_t *cu_seqlens,
                               int32_t num_seqs, int64_t total_tokens, int32_t max_seqlen,
                               int32_t H, int32_t dk, int32_t dv, kda_dtype dtype, int32_t chunk,
                               uint32_t flags, void *o, float *S_T, kda_stream_t stream);

/*
 * Reads (and with reset != 0 clears) the calling device's error word, which a
 * kernel sets when one of its bounded device-side waits (2 s) ran out; the
 * kernel then abandons its work and the outputs are not valid. Synchronous:
 * it waits for the device. *code = 0 and KDA_OK when no wait failed, else
 * the nonzero code and KDA_ERR_TIMEOUT.
 */
kda_status kda_device_error(int32_t *code, int32_t reset);

/*
 * Bound, in nanoseconds, of the waits between the CTAs of a tensor-core
 * prefill, for every call enqueued after it (any host thread): a scan CTA
 * waiting for a prepared chunk, a preparing CTA waiting for a free ring slot,
 * and the two scan CTAs of a stream exchanging the fused output step's row
 * sums. When one runs out the call abandons its work within microseconds (the
 * kernel returns; its outputs are not valid) and kda_device_error() reports
 * code 1 (KDA_ERR_TIMEOUT). A watchdog setting: the default, 2 s, is far above
 * any normal wait; a bound shorter than the time a prefill takes to prepare
 * its first chunk (tens of microseconds) makes every call fail. The waits for
 * a CTA's own copies and tensor-core products keep the 2 s bound. ns = 0
 * restores the default. Returns the previous bound. Not a per-stream setting:
 * calls already enqueued keep the bound they were enqueued with.
 */
uint64_t kda_set_wait_limit_ns(uint64_t ns);

/*
 * One decode step for N independent sequences, state updated in place
 * ("[Kimi-2] Kimi Linear" §5: S_(t-1) + current token -> S_t + output).
 *
 *   q, k       [N][H][dk]  dtype          v [N][H][dv] dtype
 *   log_alpha  [N][H][dk]  fp32 ([N][H] with KDA_FLAG_SCALAR_GATE)   beta [N][H] fp32
 *   S          [N][H][dk][dv] fp32, read and overwritten with S_t
 *   o          [N][H][dv]  dtype, out
 *
 * Supported: dk, dv in {64, 128}; dtype F32 or BF16. Arithmetic is fp32.
 */
kda_status kda_decode_step(const void *q, const void *k, const void *v, const float *log_alpha,
                           const float *beta, float *S, int32_t N, int32_t H, int32_t dk,
                           int32_t dv, kda_dtype dtype, uint32_t flags, void *o,
                           kda_stream_t stream);

/* kda_decode_step with the output step fused (out_gate != NULL; see kda_output_gate). */
kda_status kda_decode_step_ex(const void *q, const void *k, const void *v, const float *log_alpha,
                              const float *beta, float *S, int32_t N, int32_t H, int32_t dk,
                              int32_t dv, kda_dtype dtype, uint32_t flags,
                              const kda_output_gate *out_gate, void *o, kda_stream_t stream);

/*
 * Causal short convolution followed by Swish, the layer's step before the
 * recurrence ("[Kimi-2] Kimi Linear：用 KDA 重写长上下文注意力" §6 and §6.1;
 * "Kimi Delta Attention：把遗忘门做到每个通道", the pre-processing of q and k):
 * every channel c of a projection x [T][C] is convolved over the tokens of its
 * own sequence with its own W taps, then passed through Swish,
 *
 *     z_t[c] = sum_{j<W} weight[c][j] * x_{t-W+1+j}[c],   y_t[c] = z_t[c] * sigmoid(z_t[c]),
 *
 * positions before a sequence's first token reading that sequence's initial
 * state (or zero). The pages give neither the window nor a bias: the window is
 * the caller's (1 .. KDA_MAX_CONV_WIDTH) and there is no bias. q and k are
 * L2-normalised afterwards by kda_prefill / kda_decode_step (flag default).
 *
 *   width      W
 *   weight     [C][W] fp32, device, 4-byte aligned; weight[c][W-1] weighs the
 *              current token, weight[c][0] the one W-1 tokens earlier
 *   state_in   [N][W-1][C] in the io dtype, device, 16-byte aligned: each
 *              sequence's previous W-1 raw inputs, oldest first; NULL = zeros
 *   state_out  [N][W-1][C], 16-byte aligned: each sequence's last W-1 raw
 *              inputs after the call (reaching into state_in when a sequence is
 *              shorter than W-1); NULL = not written. May alias state_in.
 */
#define KDA_MAX_CONV_WIDTH 8
typedef struct kda_short_conv {
    int32_t width;
    const float *weight;
    const void *state_in;
    void *state_out;
} kda_short_conv;

/*
 * The prefill form: y [T][C] from x [T][C] (the io dtype, device, 16-byte
 * aligned, C a multiple of 8; y must not overlap x). Sequences as in
 * kda_prefill (cu_seqlens device [N+1], or NULL for one sequence). Enqueued on
 * `stream` as kda_short_conv_launches() kernels (the outputs, then state_out
 * when requested). Run it on the q, k and v projections and pass the results
 * to kda_prefill. Errors as kda_prefill's (KDA_ERR_UNSUPPORTED: a width
 * outside 1 .. KDA_MAX_CONV_WIDTH).
 */
kda_status kda_short_conv_swish(const void *x, void *y, const kda_short_conv *conv,
                                const int32_t *cu_seqlens, int32_t num_seqs, int64_t total_tokens,
                                int32_t channels, kda_dtype dtype, kda_stream_t stream);

/* Kernels kda_short_conv_swish launches (writes_state: state_out != NULL); -1 for a bad width. */
int64_t kda_short_conv_launches(int32_t width, int32_t writes_state, int64_t total_tokens);

/*
 * kda_decode_step_ex with the short convolution + Swish fused into the loads of
 * q, k and v: here q, k, v are the step's raw projections ([N][H][d]) and
 * conv_q, conv_k, conv_v (each NULL: that input is used as it is) carry
 * C = H * d channels with states [N][W-1][H * d] (normally state_in ==
 * state_out: updated in place, one token per call). Windows up to
 * KDA_DECODE_MAX_CONV_WIDTH (KDA_ERR_UNSUPPORTED beyond: run
 * kda_short_conv_swish on the step's tokens and kda_decode_step_ex instead).
 */
#define KDA_DECODE_MAX_CONV_WIDTH 4
kda_status kda_decode_step_conv(const void *q, const void *k, const void *v, const float *log_alpha,
                                const float *beta, float *S, int32_t N, int32_t H, int32_t dk,
                                int32_t dv, kda_dtype dtype, uint32_t flags,
                                const kda_short_conv *conv_q, const kda_short_conv *conv_k,
                                const kda_short_conv *conv_v, const kda_output_gate *out_gate, void *o,
                                kda_stream_t stream);

/*
 * kda_prefill_ex with the short convolution + Swish fused into the loads of q,
 * k and v ("[Kimi-2] Kimi Linear" §6 and §6.1): here q, k, v are the raw
 * projections ([T][H][d], as for kda_prefill) and conv_q, conv_k, conv_v (each
 * NULL: that input is used as it is) carry C = H * d channels, weight [C][W],
 * state_in [N][W-1][C] read for each sequence's first W-1 positions (NULL:
 * zeros) and state_out [N][W-1][C] written with each sequence's last W-1 raw
 * inputs after the prefill has read state_in (NULL: not written; may alias
 * state_in). o and S_T equal, bit for bit, those of kda_short_conv_swish on
 * each input followed by kda_prefill_ex on the results; no convolved copy of
 * q, k or v is written to device memory. The tensor-core path only (bf16,
 * d_k = d_v = 128, without KDA_FLAG_EXACT) and windows 1 ..
 * KDA_PREFILL_MAX_CONV_WIDTH: KDA_ERR_UNSUPPORTED otherwise (run
 * kda_short_conv_swish and kda_prefill_ex instead). Workspace as for
 * kda_prefill (kda_prefill_workspace_size). Enqueued as kda_prefill_launches()
 * kernels, then one kernel per written state_out of a width above 1.
 */
#define KDA_PREFILL_MAX_CONV_WIDTH 4
kda_status kda_prefill_conv(const void *q, const void *k, const void *v, const float *log_alpha,
                            const float *beta, const float *S0, const int32_t *cu_seqlens,
                            int32_t num_seqs, int64_t total_tokens, int32_t max_seqlen, int32_t H,
                            int32_t dk, int32_t dv, kda_dtype dtype, int32_t chunk, uint32_t flags,
                            const kda_short_conv *conv_q, const kda_short_conv *conv_k,
                            const kda_short_conv *conv_v, const kda_output_gate *out_gate, void *o,
                            float *S_T, void *workspace, size_t workspace_bytes, kda_stream_t stream);

/*
 * Backward of the prefill (training): the gradients of a loss L with respect
 * to q, k, v, log_alpha, beta and S0, given dL/do and dL/dS_T. The pages
 * mention training but give no backward; the chunked reverse-mode algebra
 * implemented here is stated in csrc/kda_backward.cu. The same inputs and
 * rules as kda_prefill (chunk 64; KDA_FLAG_NO_L2NORM honoured; with
 * KDA_FLAG_SCALAR_GATE, log_alpha and grad_log_alpha are [T][H]: the gradient
 * of the one gate per (token, head) is the sum over the key channels of the
 * broadcast gate's), plus:
 *
 *   dout         [T][H][dv] in the io dtype: dL/do
 *   dS_T         [N][H][dk][dv] fp32: dL/dS_T, or NULL (zero)
 *   grad_q, grad_k        [T][H][dk] fp32 out;  grad_v [T][H][dv] fp32 out
 *   grad_log_alpha        [T][H][dk] fp32 out ([T][H] with KDA_FLAG_SCALAR_GATE);  grad_beta [T][H] fp32 out
 *   grad_S0               [N][H][dk][dv] fp32 out, or NULL (not written)
 *   workspace    kda_backward_workspace_size() bytes, 16-byte aligned: fp32 scratch of
 *                about (11 C dk + 9 C^2 + 3 C dv + 2 dk dv) * 4 bytes (C = 64; 737 KB
 *                at dk = dv = 128) for each of H * (total_tokens / 64 + num_seqs) chunk
 *                slots (at least one per 64-token chunk of every sequence and head;
 *                max_seqlen is not needed), plus about (4 dk + 2) * 4 bytes per (token,
 *                head) and 4 bytes per sequence: 3.0 GB + 0.5 GB for one sequence of 8192
 *                tokens and 32 heads (3.6 GB).
 *
 * fp32 CUDA-core arithmetic (seven launches: the chunk offsets of the
 * sequences, then six; the chunk recurrences split by state column, the
 * value-dimension contractions in shared-memory tiles). It factors
 * e^{G_r - G_i} = e^{G_r} e^{-G_i} inside each chunk:
 * a chunk whose decay range (minus the sum of log_alpha over it) exceeds 60
 * sets device error code 2 (kda_device_error) and its gradients are not valid.
 */
size_t kda_backward_workspace_size(int32_t num_seqs, int64_t total_tokens, int32_t max_seqlen,
                                   int32_t H, int32_t dk, int32_t dv, kda_dtype dtype, int32_t chunk,
                                   uint32_t flags);
kda_status kda_backward(const void *q, const void *k, const void *v, const float *log_alpha,
                        const float *beta, const float *S0, const int32_t *cu_seqlens,
                        int32_t num_seqs, int64_t total_tokens, int32_t max_seqlen, int32_t H,
                        int32_t dk, int32_t dv, kda_dtype dtype, int32_t chunk, uint32_t flags,
                        const void *dout, const float *dS_T, float *grad_q, float *grad_k,
                        float *grad_v, float *grad_log_alpha, float *grad_beta, float *grad_S0, void *workspace,
                        size_t workspace_bytes, kda_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* KDA_H_ */
