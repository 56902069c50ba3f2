/*
 * kda.h -- C ABI of libkda.so: the Kimi Delta Attention (KDA) forward pass on
 * one NVIDIA B200 (sm_100a).
 *
 * What is computed (per sequence n, head h, token t; AliceAI-Foundation KDA
 * write-up, section "二、KDA 线性注意力": the per-token loop, the gate formula,
 * the depthwise causal conv with kernel 4 / padding 3 / no bias + SiLU, and
 * L2-normalised q, k; Ling-3.0-flash-VL config table: kda_safe_gate = true,
 * kda_lower_bound = -5.0):
 *
 *   prologue   x~_t[c] = sum_{j=0..3} conv_w[c][j] * x_{t-3+j}[c]   (x_{<0}: conv history)
 *              x^_t    = SiLU(x~_t)                                   for q, k and v channels
 *              q_t     = q^_t / sqrt(|q^_t|^2 + eps),  k_t likewise   (per head, over d)
 *              g_t[i]  = max(-exp(A_log[h]) * softplus(alpha_t[h][i] + dt_bias[h][i]), lower_bound)
 *              beta_t  = sigmoid(b_t[h])
 *   recurrence S  <- diag(exp(g_t)) S                 S: [d_k, d_v] fp32 state
 *              d_t = beta_t * (v_t - S^T k_t)
 *              S  <- S + k_t d_t^T
 *              o_t = scale * S^T q_t
 *
 * Prefill and decode share the state interface: the final_state a prefill
 * returns seeds kda_decode_step with no recomputation (same write-up, section
 * "五": the prefill/decode kernels share initial_state / final_state), and the
 * conv history is carried as the raw inputs of the last 3 tokens (section "四":
 * kernel - 1 = 3 conv states per channel).
 *
 * Conventions shared by every entry point
 *   - Every pointer is a DEVICE pointer unless stated otherwise; the caller
 *     owns every buffer, including the workspace.  The library allocates no
 *     device memory, creates no streams and is thread-safe across streams;
 *     its only process-wide state is the opt-in benchmark timing of
 *     kda_kernel_timing().
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL = the
 *     legacy default stream).  Return codes report argument checks and launch
 *     errors; device-side conditions are reported by kda_prefill_status().
 *   - Argument errors are detected before any launch: NULL required pointers,
 *     pointers not 16-byte aligned, unsupported shapes.  Nothing is launched
 *     then and the outputs are untouched.
 *   - Layouts are row-major and tokens are packed: dense batches are N
 *     sequences of seq_len tokens back to back (token row = n * seq_len + t);
 *     varlen batches give cu_seqlens [N + 1] (int32, device) with
 *     cu_seqlens[0] = 0 and cu_seqlens[N] = total tokens.
 *   - io dtype (kda_shape.io_dtype): bf16 or fp32 for q, k, v, conv_w, alpha,
 *     b, o and the conv history.  A_log, dt_bias and states are always fp32.
 *   - Channel blocks of the conv: c in [0, H*d) is q, [H*d, 2*H*d) is k,
 *     [2*H*d, 3*H*d) is v; conv_w[blk][c][3] multiplies the current token.
 *
 * Supported shapes: head_dim 64 or 128; num_heads 1..64; any sequence
 * length >= 0.  bf16 with head_dim 128 and lower_bound >= -10 runs the
 * tensor-core chunk path (chunk_prep, with the prologue fused in, then the
 * state pass).  Other combinations (fp32 I/O: the fp32 test mode; head_dim 64)
 * run the prologue kernel and then, for lower_bound >= -10, the same chunkwise
 * algebra on CUDA cores in fp32, or else (or with KDA_FLAG_TOKEN_RECURRENCE) the
 * CUDA-core token loop.  The bound keeps the chunk algebra's split decay factors,
 * which span up to 8 tokens of gate, inside fp32 and bf16 normal range.
 */
#ifndef KDA_H
#define KDA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARGUMENT = 1, /* NULL / misaligned pointer, bad sizes, bad cu_seqlens */
    KDA_ERR_UNSUPPORTED = 2,      /* valid but not implemented (e.g. head_dim 96) */
    KDA_ERR_WORKSPACE = 3,        /* workspace NULL or smaller than *_workspace_size() */
    KDA_ERR_CUDA = 4,             /* a CUDA runtime call or launch failed */
    KDA_ERR_TIMEOUT = 5           /* a bounded device-side wait gave up */
} kda_status;

typedef enum { KDA_BF16 = 0, KDA_FP32 = 1 } kda_dtype;

typedef struct {
    int32_t num_seqs;    /* N: sequences (dense batch size, or number of varlen sequences) */
    int32_t seq_len;     /* dense: tokens per sequence; varlen: total packed tokens */
    int32_t num_heads;   /* H (q, k and v heads alike) */
    int32_t head_dim;    /* d = d_k = d_v: 64 or 128 */
    float lower_bound;   /* safe-gate lower bound on g: -5.0f */
    float l2norm_eps;    /* added to |x|^2 inside the square root: 1e-6f */
    float scale;         /* output scale on S^T q: 1.0f (the pages apply none) */
    int32_t io_dtype;    /* kda_dtype */
    uint32_t flags;      /* KDA_FLAG_* bits; 0 is the configuration the pages run */
} kda_shape;

/* beta = 2 sigmoid(b), in (0, 2), instead of sigmoid(b): the write's transition
 * I - beta k k^T then has eigenvalue 1 - beta in (-1, 1) along k.  The KDA layer's
 * kda_allow_negative_eigenvalues switch (AliceAI-Foundation KDA write-up, section
 * "二": with the switch off, beta is not doubled and stays in (0, 1)). */
#define KDA_FLAG_NEGATIVE_EIGENVALUES 0x1u
/* Where the tensor-core chunk path does not apply (fp32 I/O, head_dim 64), run
 * the recurrence token by token on CUDA cores, the loop exactly as the KDA
 * write-up's section "二" states it, instead of the fp32 chunkwise kernel.  Both
 * compute in fp32; gate bounds below -10 always take the token loop. */
#define KDA_FLAG_TOKEN_RECURRENCE 0x2u
/* For tests of the failure path only; never set it in normal use.  Every
 * bounded device-side wait of the call (the mbarrier waits of chunk
 * preparation, the state pass and the bf16 decode kernels) gives up at its
 * first check.  Each kernel then stops issuing work, waits (with the normal
 * limit) for the copies and tensor-core operations it already started, frees
 * its tensor memory and returns; the call's status word reports
 * KDA_ERR_TIMEOUT and the outputs are unspecified.  The next call without the
 * flag runs normally. */
#define KDA_FLAG_TEST_EXPIRE_WAITS 0x80000000u
#define KDA_FLAGS_KNOWN \
    (KDA_FLAG_NEGATIVE_EIGENVALUES | KDA_FLAG_TOKEN_RECURRENCE | KDA_FLAG_TEST_EXPIRE_WAITS)

/* Bits of the device status word (the first int32 of a prefill workspace, or a
 * decode call's `status`), as kda_device_status() reads them. */
#define KDA_STATUS_BAD_CU_SEQLENS 0x1    /* cu_seqlens malformed (accesses stayed clamped) */
#define KDA_STATUS_TIMEOUT_PREP 0x2      /* a wait of chunk preparation gave up */
#define KDA_STATUS_TIMEOUT_STATE 0x4     /* a wait of the state pass gave up */
#define KDA_STATUS_TIMEOUT_DECODE 0x8    /* a wait of a decode kernel gave up */

/* Bytes of device workspace kda_prefill() needs for this shape (0 on a bad
 * shape).  is_varlen != 0: shape->seq_len is the packed token total (the call
 * will pass cu_seqlens); 0: dense, num_seqs * seq_len tokens. */
size_t kda_prefill_workspace_size(const kda_shape *shape, int is_varlen);

/*
 * kda_prefill -- prologue + recurrence over whole sequences.
 *
 *   q, k, v            [T_total, H*d] io dtype, raw (pre-conv) projections
 *   conv_w             [3, H*d, 4]    io dtype
 *   alpha              [T_total, H, d] io dtype
 *   b                  [T_total, H]   io dtype
 *   A_log              [H]            fp32
 *   dt_bias            [H, d]         fp32
 *   initial_state      [N, H, d, d]   fp32 or NULL (zeros); S[i][j], i = key, j = value
 *   initial_conv_state [N, 3, 3*H*d]  io dtype or NULL (zeros): raw inputs of the
 *                                     3 tokens before each sequence, oldest first
 *   cu_seqlens         [N + 1]        int32 or NULL (dense: N sequences of seq_len)
 *   o                  [T_total, H, d] io dtype, written
 *   final_state        [N, H, d, d]   fp32, written; may equal initial_state
 *   final_conv_state   [N, 3, 3*H*d]  io dtype or NULL; may not overlap the inputs
 *   workspace          >= kda_prefill_workspace_size(shape) bytes, 256-byte aligned
 *
 * A sequence of length 0 copies its initial state (or zeros) to final_state.
 * Bad cu_seqlens (not starting at 0, decreasing, or not ending at T_total)
 * are caught on the device: every access stays clamped in bounds and
 * kda_prefill_status() then returns KDA_ERR_INVALID_ARGUMENT.
 */
kda_status kda_prefill(const kda_shape *shape,
                       const void *q, const void *k, const void *v,
                       const void *conv_w, const void *alpha, const void *b,
                       const float *A_log, const float *dt_bias,
                       const float *initial_state, const void *initial_conv_state,
                       const int32_t *cu_seqlens,
                       void *o, float *final_state, void *final_conv_state,
                       void *workspace, size_t workspace_bytes, void *stream);

/*
 * Output epilogue of the KDA layer, fused into the store of o: the layer's
 * o_norm followed by its sigmoid output gating (AliceAI-Foundation KDA
 * write-up: the layer projects an output_gate, section "二", and ends in o_norm
 * plus sigmoid gating, section "三"; the Ling-3.0-flash-VL weight list names
 * o_norm and g_proj).  Per (token, head), over the head's d value channels:
 *
 *   o[j] <- o[j] / sqrt(mean_j o[j]^2 + eps) * weight[j] * sigmoid(gate[j])
 *
 *   gate    [T_total, H, d] io dtype (prefill) or [N, H, d] (decode): the
 *           output gate before the sigmoid; 16-byte aligned
 *   weight  [d] fp32, shared by the heads; 16-byte aligned
 *   eps     inside the root, added to the mean square (1e-5f); finite, >= 0
 */
typedef struct {
    const void *gate;
    const float *weight;
    float eps;
} kda_output_gate;

/*
 * kda_prefill_gated -- kda_prefill with the output epilogue applied to o
 * (out_gate NULL: exactly kda_prefill).  Same workspace size.
 */
kda_status kda_prefill_gated(const kda_shape *shape,
                             const void *q, const void *k, const void *v,
                             const void *conv_w, const void *alpha, const void *b,
                             const float *A_log, const float *dt_bias,
                             const float *initial_state, const void *initial_conv_state,
                             const int32_t *cu_seqlens, const kda_output_gate *out_gate,
                             void *o, float *final_state, void *final_conv_state,
                             void *workspace, size_t workspace_bytes, void *stream);

/*
 * kda_prefill_ex -- kda_prefill with every optional output, through one
 * argument block (NULL members: not wanted).  kda_prefill and
 * kda_prefill_gated are this call with the extras off.
 *
 *   out_gate           the output epilogue (see kda_output_gate) or NULL
 *   snapshots          [N, snapshot_capacity, H, d, d] fp32 or NULL: state
 *                      snapshots aligned to the sequence start, for prefix
 *                      caching (the "align" state-cache mode and chunked prefill
 *                      the Ling-3.0-flash-VL page runs under vLLM): snapshot j
 *                      of sequence n is the state after its first
 *                      (j + 1) * 64 * snapshot_every tokens, S[i][j] as in
 *                      final_state.  Only whole intervals are written, and at
 *                      most snapshot_capacity per sequence; the rest of the
 *                      buffer is left as it was.
 *   snapshot_every     >= 1: 64-token chunks between snapshots
 *   snapshot_capacity  >= 0: snapshots the buffer holds per sequence
 *   side_stream        a cudaStream_t of the caller's (a high-priority one is
 *                      best) or NULL.  Given one, a dense batch with at least
 *                      256 chunks of 64 tokens per sequence and at most
 *                      (SMs / 2) (sequence, head) pairs runs in time segments:
 *                      chunk preparation of segment s + 1 on `stream` while
 *                      the state pass of segment s runs on `side_stream`,
 *                      ordered by two events the call creates and releases;
 *                      `stream` waits for the last state pass before the call
 *                      returns control of it.  Under stream capture the fork
 *                      and the join are captured with the rest.  NULL: one
 *                      launch of each kernel on `stream` (few long sequences
 *                      then leave most SMs idle during the state pass).
 */
typedef struct {
    const void *q, *k, *v, *conv_w, *alpha, *b;
    const float *A_log, *dt_bias;
    const float *initial_state;
    const void *initial_conv_state;
    const int32_t *cu_seqlens;
    void *o;
    float *final_state;
    void *final_conv_state;
    const kda_output_gate *out_gate;
    float *snapshots;
    int32_t snapshot_every;
    int32_t snapshot_capacity;
    void *side_stream;
} kda_prefill_args;

kda_status kda_prefill_ex(const kda_shape *shape, const kda_prefill_args *args,
                          void *workspace, size_t workspace_bytes, void *stream);

/*
 * kda_prefill_status -- synchronises `stream` and reads the device status word
 * the last kda_prefill() on this workspace left (its first int32): KDA_OK,
 * KDA_ERR_INVALID_ARGUMENT (bad cu_seqlens), KDA_ERR_TIMEOUT (a bounded wait
 * gave up) or KDA_ERR_CUDA.  kda_device_status() is the same call on any
 * status word (a decode call's `status` included).
 */
kda_status kda_prefill_status(const void *workspace, void *stream);
kda_status kda_device_status(const int32_t *word, void *stream);

/*
 * kda_prologue -- the prologue alone (conv4 + SiLU, L2 norm, gate, beta).
 * Same inputs as kda_prefill; outputs
 *   qn, kn, vc        [T_total, H, d] io dtype (L2-normalised q, k; conv'd v)
 *   g                 [T_total, H, d] fp32 (after the lower-bound clamp)
 *   beta              [T_total, H]    fp32
 *   final_conv_state  [N, 3, 3*H*d]   io dtype or NULL, as in kda_prefill
 * Bad cu_seqlens are clamped (no out-of-bounds access) but not reported here.
 * Accuracy: bf16 outputs carry one bf16 rounding (their SiLU takes the hardware tanh
 * approximation, relative error about 2^-11, below it); fp32 outputs and g, beta are
 * within a few fp32 roundings of the exact values.
 */
kda_status kda_prologue(const kda_shape *shape,
                        const void *q, const void *k, const void *v,
                        const void *conv_w, const void *alpha, const void *b,
                        const float *A_log, const float *dt_bias,
                        const void *initial_conv_state, const int32_t *cu_seqlens,
                        void *qn, void *kn, void *vc, float *g, float *beta,
                        void *final_conv_state, void *stream);

/*
 * kda_recurrence -- the recurrence alone, on prepared per-token inputs
 * (what kda_prologue writes):
 *   qn, kn, vc     [T_total, H, d] io dtype
 *   g              [T_total, H, d] fp32, gate values in [lower_bound, 0] (what
 *                  kda_prologue writes; the tensor-core path clamps into that range)
 *   beta           [T_total, H]    fp32
 *   initial_state  [N, H, d, d]    fp32 or NULL (zeros)
 *   cu_seqlens     [N + 1] int32 or NULL (dense)
 *   o              [T_total, H, d] io dtype, written
 *   final_state    [N, H, d, d]    fp32, written; may equal initial_state
 *   workspace      >= kda_recurrence_workspace_size(shape, varlen) bytes,
 *                  256-byte aligned (per-chunk records of the tensor-core path)
 * kda_prologue followed by kda_recurrence computes what kda_prefill computes
 * (kda_prefill fuses the two on the tensor-core path).  kda_prefill_status()
 * reads this workspace's error word the same way; on the tensor-core path it
 * also reports bad cu_seqlens.
 */
size_t kda_recurrence_workspace_size(const kda_shape *shape, int is_varlen);
kda_status kda_recurrence(const kda_shape *shape,
                          const void *qn, const void *kn, const void *vc,
                          const float *g, const float *beta,
                          const float *initial_state, const int32_t *cu_seqlens,
                          void *o, float *final_state,
                          void *workspace, size_t workspace_bytes, void *stream);

/*
 * kda_decode_step -- one new token for each of N sequences, in place.
 *
 *   q, k, v      [N, H*d]       io dtype, raw projections of the new token
 *   alpha        [N, H, d]      io dtype
 *   b            [N, H]         io dtype
 *   conv_w, A_log, dt_bias      as in kda_prefill
 *   state        [N, H, d, d]   fp32, read and overwritten (a prefill's final_state)
 *   conv_state   [N, 3, 3*H*d]  io dtype, read and shifted by one token in place
 *   o            [N, H, d]      io dtype, written
 *
 * shape->seq_len is ignored.  Needs no workspace.
 */
kda_status kda_decode_step(const kda_shape *shape,
                           const void *q, const void *k, const void *v,
                           const void *alpha, const void *b,
                           const void *conv_w, const float *A_log, const float *dt_bias,
                           float *state, void *conv_state, void *o, void *stream);

/*
 * kda_decode_multi -- shape->seq_len (1 to 16) new tokens per sequence in one
 * call, in order, for verifying speculative (MTP) tokens: the KDA layer's
 * model predicts one extra token per step (AliceAI-Foundation KDA write-up,
 * section "六": MTP with num_speculative_tokens 1 generates 2 tokens per forward).
 *
 *   q, k, v      [N, T, H*d]     io dtype, T = shape->seq_len
 *   alpha        [N, T, H, d]    io dtype
 *   b            [N, T, H]       io dtype
 *   out_gate     NULL, or the output epilogue with gate [N, T, H, d]
 *   state        [N, H, d, d]    fp32, in place: the state after all T tokens
 *   conv_state   [N, 3, 3*H*d]   io dtype, shifted by T tokens in place
 *   o            [N, T, H, d]    io dtype
 *   step_states  [N, T, H, d, d] fp32 or NULL: the state after each token, so a
 *                verifier that accepts t tokens resumes from step_states[:, t - 1]
 *                (the conv state it needs is the last 3 raw tokens up to t)
 *
 * T = 1 without step_states is kda_decode_step_gated.  Needs no workspace.
 */
kda_status kda_decode_multi(const kda_shape *shape,
                            const void *q, const void *k, const void *v,
                            const void *alpha, const void *b,
                            const void *conv_w, const float *A_log, const float *dt_bias,
                            const kda_output_gate *out_gate,
                            float *state, void *conv_state, void *o, float *step_states,
                            void *stream);

/*
 * kda_decode_ex -- kda_decode_multi through one argument block, with a device
 * status word.  `status` (device int32, or NULL) is zeroed by the call and
 * gets KDA_STATUS_TIMEOUT_DECODE when a bounded wait of the decode kernel gave
 * up; read it with kda_device_status().  kda_decode_step, kda_decode_step_gated
 * and kda_decode_multi are this call with status NULL.
 */
typedef struct {
    const void *q, *k, *v, *alpha, *b, *conv_w;
    const float *A_log, *dt_bias;
    const kda_output_gate *out_gate;
    float *state;
    void *conv_state;
    void *o;
    float *step_states;
    int32_t *status;
} kda_decode_args;

kda_status kda_decode_ex(const kda_shape *shape, const kda_decode_args *args, void *stream);

/* kda_decode_step with the output epilogue (gate [N, H, d]); out_gate NULL:
 * exactly kda_decode_step. */
kda_status kda_decode_step_gated(const kda_shape *shape,
                                 const void *q, const void *k, const void *v,
                                 const void *alpha, const void *b,
                                 const void *conv_w, const float *A_log, const float *dt_bias,
                                 const kda_output_gate *out_gate,
                                 float *state, void *conv_state, void *o, void *stream);

/*
 * kda_prefill_noalloc -- kda_prefill for callers that cannot allocate device
 * memory.  The pages describe no such variant; it exists for embeddings where
 * cudaMalloc is not allowed or not possible (a caller that owns all device
 * memory and lends the library only its inputs and outputs, code running
 * under an allocator that must not grow, a host callback).
 *
 * Same arguments and results as kda_prefill minus the workspace: what
 * kda_prefill keeps in its workspace (the per-chunk records of the
 * tensor-core path, or the prologue's outputs on the token-kernel path) lives
 * in a library-owned array of KDA_NOALLOC_SCRATCH_BYTES in device memory,
 * which every GPU that loads the library holds until the library is unloaded.
 * The call allocates nothing.
 *
 *   - A shape whose intermediates need more than KDA_NOALLOC_SCRATCH_BYTES
 *     (bf16, d = 128: a 74,752-byte record per 64-token chunk and head, about
 *     1.2 KiB per token per head, e.g. 896 tokens at 32 heads) returns
 *     KDA_ERR_WORKSPACE and launches nothing.
 *   - The first call on each device looks up that device's address of the
 *     array (cudaGetSymbolAddress, with the device current) and keeps it for
 *     the life of the process.  Make that first call before any stream
 *     capture, and do not call this entry point on a device after a
 *     cudaDeviceReset() of it: the kept address would be stale.
 *   - The shape rules are kda_prefill's (the same checks, the same codes).
 *   - All calls share the one array and it keeps the previous call's
 *     contents; calls that overlap on the GPU (other streams, other threads)
 *     race with each other.  Serialise them.
 *   - Device-side conditions (bad cu_seqlens, a bounded wait that gave up)
 *     are not reported by this entry point; use kda_prefill to see them.
 */
#define KDA_NOALLOC_SCRATCH_BYTES (32u << 20)
kda_status kda_prefill_noalloc(const kda_shape *shape,
                               const void *q, const void *k, const void *v,
                               const void *conv_w, const void *alpha, const void *b,
                               const float *A_log, const float *dt_bias,
                               const float *initial_state, const void *initial_conv_state,
                               const int32_t *cu_seqlens,
                               void *o, float *final_state, void *final_conv_state,
                               void *stream);

/*
 * kda_kernel_timing / kda_kernel_times -- per-kernel device time of the
 * tensor-core chunk path, for benchmarks.  The pages describe no such facility.
 *
 * kda_kernel_timing(1) makes every later kda_prefill / kda_prefill_noalloc /
 * kda_recurrence call that takes the chunk path record CUDA events on its
 * stream before chunk_prep, between chunk_prep and the state pass, and after
 * the state pass (up to 4096 calls are kept; later ones are not timed).  In
 * the time-segmented schedule the middle event follows the last segment's
 * chunk_prep, so the two durations are the overlapped part and the tail.
 * kda_kernel_timing(0) stops recording and drops what was kept.
 * kda_kernel_times() waits for the recorded events, writes the mean duration
 * in milliseconds of chunk_prep to *prep_ms and of the state pass to *state_ms
 * over the calls recorded since the last read (both 0 when there were none),
 * returns the number of calls, and forgets them.  Recording is process-wide and
 * not meant for concurrent use from several host threads.  Returns -1 when a
 * CUDA call fails.
 */
int kda_kernel_timing(int enable);
int kda_kernel_times(float *prep_ms, float *state_ms);

/* Static description of a status code (never NULL). */
const char *kda_status_string(kda_status status);

/* Library version as MAJOR * 10000 + MINOR * 100 + PATCH. */
int kda_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H */
