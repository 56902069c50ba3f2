// C ABI of libkda.so (declared in include/kda.h): argument validation,
// workspace layout and kernel dispatch.  Every step of the forward pass runs
// in this library's CUDA kernels; there is no host-side compute path.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>

#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {

kda_status check_shape(const kda_shape *s) {
  if (s == nullptr) return KDA_ERR_INVALID_ARGUMENT;
  if (s->num_seqs < 0 || s->seq_len < 0 || s->num_heads < 1 || s->head_dim < 1)
    return KDA_ERR_INVALID_ARGUMENT;
  if (s->io_dtype != KDA_BF16 && s->io_dtype != KDA_FP32) return KDA_ERR_INVALID_ARGUMENT;
  if (!std::isfinite(s->lower_bound) || !std::isfinite(s->l2norm_eps) || s->l2norm_eps < 0.f ||
      !std::isfinite(s->scale))
    return KDA_ERR_INVALID_ARGUMENT;
  if (s->flags & ~KDA_FLAGS_KNOWN) return KDA_ERR_INVALID_ARGUMENT;
  if (s->head_dim != 64 && s->head_dim != 128) return KDA_ERR_UNSUPPORTED;
  if (s->num_heads > 64) return KDA_ERR_UNSUPPORTED;
  return KDA_OK;
}

}  // namespace kda

namespace {

using namespace kda;

constexpr size_t kAlign = 256;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Total packed tokens: dense N * seq_len, varlen seq_len.
int64_t total_tokens(const kda_shape *s, const int32_t *cu) {
  return cu ? (int64_t)s->seq_len : (int64_t)s->num_seqs * s->seq_len;
}

#define KDA_REQUIRE(p) do { if ((p) == nullptr || !aligned16(p)) return KDA_ERR_INVALID_ARGUMENT; } while (0)
#define KDA_OPTIONAL(p) do { if ((p) != nullptr && !aligned16(p)) return KDA_ERR_INVALID_ARGUMENT; } while (0)

kda_status cuda_status(cudaError_t e) { return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA; }

// The output epilogue's arguments (nullptr: no epilogue).
kda_status check_out_gate(const kda_output_gate *og, int64_t rows) {
  if (og == nullptr) return KDA_OK;
  if (rows > 0 && (og->gate == nullptr || !aligned16(og->gate))) return KDA_ERR_INVALID_ARGUMENT;
  if (og->weight == nullptr || !aligned16(og->weight)) return KDA_ERR_INVALID_ARGUMENT;
  if (!std::isfinite(og->eps) || og->eps < 0.f) return KDA_ERR_INVALID_ARGUMENT;
  return KDA_OK;
}

PrologueArgs make_prologue_args(const kda_shape *s, int64_t T, const void *q, const void *k,
                                const void *v, const void *conv_w, const void *alpha, const void *b,
                                const float *A_log, const float *dt_bias, const void *conv0,
                                const int32_t *cu) {
  PrologueArgs a;
  std::memset(&a, 0, sizeof a);
  a.N = s->num_seqs; a.H = s->num_heads; a.D = s->head_dim; a.seq_len = s->seq_len;
  a.total_tokens = T; a.io_dtype = s->io_dtype; a.cu = cu;
  a.q = q; a.k = k; a.v = v; a.conv_w = conv_w; a.alpha = alpha; a.b = b;
  a.A_log = A_log; a.dt_bias = dt_bias; a.conv0 = conv0;
  a.lower_bound = s->lower_bound; a.eps = s->l2norm_eps;
  a.beta2 = (s->flags & KDA_FLAG_NEGATIVE_EIGENVALUES) != 0;
  return a;
}

RecurrenceArgs make_recurrence_args(const kda_shape *s, int64_t T, const void *qn, const void *kn,
                                    const void *vc, const float *g, const float *beta,
                                    const float *state0, const int32_t *cu, void *o, float *state1) {
  RecurrenceArgs ra;
  std::memset(&ra, 0, sizeof ra);
  ra.N = s->num_seqs; ra.H = s->num_heads; ra.D = s->head_dim;
  ra.seq_len = s->seq_len; ra.total_tokens = T; ra.io_dtype = s->io_dtype;
  ra.cu = cu; ra.qn = qn; ra.kn = kn; ra.vc = vc; ra.g = g; ra.beta = beta;
  ra.state0 = state0; ra.scale = s->scale; ra.o = o; ra.state1 = state1;
  ra.lower_bound = s->lower_bound;
  ra.wait_polls = wait_polls_for(s->flags);
  ra.token_loop = (s->flags & KDA_FLAG_TOKEN_RECURRENCE) != 0;
  return ra;
}

// The status a device status word maps to (bad cu_seqlens before a timeout).
kda_status word_status(int word) {
  if (word == ERR_NONE) return KDA_OK;
  if (word & ERR_BAD_CU_SEQLENS) return KDA_ERR_INVALID_ARGUMENT;
  if (word & (ERR_TIMEOUT_PREP | ERR_TIMEOUT_STATE | ERR_TIMEOUT_DECODE)) return KDA_ERR_TIMEOUT;
  return KDA_ERR_CUDA;
}

}  // namespace

extern "C" {

size_t kda_prefill_workspace_size(const kda_shape *shape, int is_varlen) {
  if (check_shape(shape) != KDA_OK) return 0;
  const int64_t T = is_varlen ? (int64_t)shape->seq_len : (int64_t)shape->num_seqs * shape->seq_len;
  if (check_tokens(T) != KDA_OK) return 0;
  return workspace_layout(shape->num_seqs, shape->num_heads, shape->head_dim, shape->seq_len, T,
                          shape->io_dtype, shape->lower_bound, is_varlen != 0, true).total;
}

size_t kda_recurrence_workspace_size(const kda_shape *shape, int is_varlen) {
  if (check_shape(shape) != KDA_OK) return 0;
  const int64_t T = is_varlen ? (int64_t)shape->seq_len : (int64_t)shape->num_seqs * shape->seq_len;
  if (check_tokens(T) != KDA_OK) return 0;
  return workspace_layout(shape->num_seqs, shape->num_heads, shape->head_dim, shape->seq_len, T,
                          shape->io_dtype, shape->lower_bound, is_varlen != 0, false).total;
}

kda_status kda_prefill(const kda_shape *shape, const void *q, const void *k, const void *v,
                       const void *conv_w, const void *alpha, const void *b, const float *A_log,
                       const float *dt_bias, const float *initial_state,
                       const void *initial_conv_state, const int32_t *cu_seqlens, void *o,
                       float *final_state, void *final_conv_state, void *workspace,
                       size_t workspace_bytes, void *stream_) {
  return kda_prefill_gated(shape, q, k, v, conv_w, alpha, b, A_log, dt_bias, initial_state,
                           initial_conv_state, cu_seqlens, nullptr, o, final_state,
                           final_conv_state, workspace, workspace_bytes, stream_);
}

kda_status kda_prefill_gated(const kda_shape *shape, const void *q, const void *k, const void *v,
                             const void *conv_w, const void *alpha, const void *b,
                             const float *A_log, const float *dt_bias, const float *initial_state,
                             const void *initial_conv_state, const int32_t *cu_seqlens,
                             const kda_output_gate *out_gate, void *o, float *final_state,
                             void *final_conv_state, void *workspace, size_t workspace_bytes,
                             void *stream_) {
  kda_prefill_args a;
  std::memset(&a, 0, sizeof a);
  a.q = q; a.k = k; a.v = v; a.conv_w = conv_w; a.alpha = alpha; a.b = b;
  a.A_log = A_log; a.dt_bias = dt_bias; a.initial_state = initial_state;
  a.initial_conv_state = initial_conv_state; a.cu_seqlens = cu_seqlens;
  a.o = o; a.final_state = final_state; a.final_conv_state = final_conv_state;
  a.out_gate = out_gate;
  a.snapshot_every = 1;
  return kda_prefill_ex(shape, &a, workspace, workspace_bytes, stream_);
}

kda_status kda_prefill_ex(const kda_shape *shape, const kda_prefill_args *args, void *workspace,
                          size_t workspace_bytes, void *stream_) {
  kda_status st = check_shape(shape);
  if (st != KDA_OK) return st;
  if (args == nullptr) return KDA_ERR_INVALID_ARGUMENT;
  if (shape->num_seqs == 0) return KDA_OK;
  const int32_t *cu_seqlens = args->cu_seqlens;
  const int64_t T = total_tokens(shape, cu_seqlens);
  if (check_tokens(T) != KDA_OK) return KDA_ERR_UNSUPPORTED;
  st = check_out_gate(args->out_gate, T);
  if (st != KDA_OK) return st;
  if (T > 0) {
    KDA_REQUIRE(args->q); KDA_REQUIRE(args->k); KDA_REQUIRE(args->v); KDA_REQUIRE(args->alpha);
    KDA_REQUIRE(args->b); KDA_REQUIRE(args->o);
  }
  KDA_REQUIRE(args->conv_w); KDA_REQUIRE(args->A_log); KDA_REQUIRE(args->dt_bias);
  KDA_REQUIRE(args->final_state);
  KDA_OPTIONAL(args->initial_state); KDA_OPTIONAL(args->initial_conv_state);
  KDA_OPTIONAL(args->final_conv_state); KDA_OPTIONAL(args->snapshots);
  if (args->snapshots != nullptr && (args->snapshot_every < 1 || args->snapshot_capacity < 0))
    return KDA_ERR_INVALID_ARGUMENT;
  if (cu_seqlens != nullptr && (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u)) return KDA_ERR_INVALID_ARGUMENT;
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)))
    return KDA_ERR_WORKSPACE;
  const bool varlen = cu_seqlens != nullptr;
  const WsLayout L = workspace_layout(shape->num_seqs, shape->num_heads, shape->head_dim,
                                      shape->seq_len, T, shape->io_dtype, shape->lower_bound,
                                      varlen, true);
  if (workspace_bytes < L.total) return KDA_ERR_WORKSPACE;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  char *ws = static_cast<char *>(workspace);
  int *err = reinterpret_cast<int *>(ws + L.err);

  cudaError_t e = cudaMemsetAsync(err, 0, sizeof(int), stream);
  if (e != cudaSuccess) return KDA_ERR_CUDA;

  PrologueArgs pa = make_prologue_args(shape, T, args->q, args->k, args->v, args->conv_w,
                                       args->alpha, args->b, args->A_log, args->dt_bias,
                                       args->initial_conv_state, cu_seqlens);
  pa.err = err;
  RecurrenceArgs ra = make_recurrence_args(shape, T, nullptr, nullptr, nullptr, nullptr, nullptr,
                                           args->initial_state, cu_seqlens, args->o,
                                           args->final_state);
  ra.err = err;
  if (args->out_gate != nullptr) {
    ra.ogate = args->out_gate->gate; ra.onw = args->out_gate->weight; ra.oeps = args->out_gate->eps;
  }
  if (args->snapshots != nullptr && args->snapshot_capacity > 0) {
    ra.snap = args->snapshots; ra.snap_cap = args->snapshot_capacity;
    ra.snap_every = (int64_t)args->snapshot_every * 64;
  }
  ra.side_stream = static_cast<cudaStream_t>(args->side_stream);
  return cuda_status(run_prefill(pa, ra, args->final_conv_state, varlen, ws, L, stream));
}

kda_status kda_device_status(const int32_t *word_ptr, void *stream_) {
  if (word_ptr == nullptr || (reinterpret_cast<uintptr_t>(word_ptr) & 3u)) return KDA_ERR_INVALID_ARGUMENT;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  if (cudaStreamSynchronize(stream) != cudaSuccess) return KDA_ERR_CUDA;
  int word = 0;
  if (cudaMemcpy(&word, word_ptr, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return KDA_ERR_CUDA;
  return word_status(word);
}

kda_status kda_prefill_status(const void *workspace, void *stream_) {
  return kda_device_status(static_cast<const int32_t *>(workspace), stream_);
}

kda_status kda_prologue(const kda_shape *shape, const void *q, const void *k, const void *v,
                        const void *conv_w, const void *alpha, const void *b, const float *A_log,
                        const float *dt_bias, const void *initial_conv_state,
                        const int32_t *cu_seqlens, void *qn, void *kn, void *vc, float *g,
                        float *beta, void *final_conv_state, void *stream_) {
  kda_status st = check_shape(shape);
  if (st != KDA_OK) return st;
  const int64_t T = total_tokens(shape, cu_seqlens);
  if (check_tokens(T) != KDA_OK) return KDA_ERR_UNSUPPORTED;
  if (shape->num_seqs == 0) return KDA_OK;
  if (T > 0) {
    KDA_REQUIRE(q); KDA_REQUIRE(k); KDA_REQUIRE(v); KDA_REQUIRE(alpha); KDA_REQUIRE(b);
    KDA_REQUIRE(qn); KDA_REQUIRE(kn); KDA_REQUIRE(vc); KDA_REQUIRE(g); KDA_REQUIRE(beta);
  }
  KDA_REQUIRE(conv_w); KDA_REQUIRE(A_log); KDA_REQUIRE(dt_bias);
  KDA_OPTIONAL(initial_conv_state); KDA_OPTIONAL(final_conv_state);
  if (cu_seqlens != nullptr && (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u)) return KDA_ERR_INVALID_ARGUMENT;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  PrologueArgs pa = make_prologue_args(shape, T, q, k, v, conv_w, alpha, b, A_log, dt_bias,
                                       initial_conv_state, cu_seqlens);
  pa.qn = qn; pa.kn = kn; pa.vc = vc; pa.g = g; pa.beta = beta; pa.err = nullptr;
  if (launch_prologue(pa, stream) != cudaSuccess) return KDA_ERR_CUDA;
  if (final_conv_state != nullptr && launch_conv_state_out(pa, final_conv_state, stream) != cudaSuccess)
    return KDA_ERR_CUDA;
  return KDA_OK;
}

kda_status kda_recurrence(const kda_shape *shape, const void *qn, const void *kn, const void *vc,
                          const float *g, const float *beta, const float *initial_state,
                          const int32_t *cu_seqlens, void *o, float *final_state, void *workspace,
                          size_t workspace_bytes, void *stream_) {
  kda_status st = check_shape(shape);
  if (st != KDA_OK) return st;
  if (shape->num_seqs == 0) return KDA_OK;
  const int64_t T = total_tokens(shape, cu_seqlens);
  if (check_tokens(T) != KDA_OK) return KDA_ERR_UNSUPPORTED;
  if (T > 0) {
    KDA_REQUIRE(qn); KDA_REQUIRE(kn); KDA_REQUIRE(vc); KDA_REQUIRE(g); KDA_REQUIRE(beta);
    KDA_REQUIRE(o);
  }
  KDA_REQUIRE(final_state); KDA_OPTIONAL(initial_state);
  if (cu_seqlens != nullptr && (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u)) return KDA_ERR_INVALID_ARGUMENT;
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)))
    return KDA_ERR_WORKSPACE;
  const bool varlen = cu_seqlens != nullptr;
  const WsLayout L = workspace_layout(shape->num_seqs, shape->num_heads, shape->head_dim,
                                      shape->seq_len, T, shape->io_dtype, shape->lower_bound,
                                      varlen, false);
  if (workspace_bytes < L.total) return KDA_ERR_WORKSPACE;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  char *ws = static_cast<char *>(workspace);
  if (cudaMemsetAsync(ws + L.err, 0, sizeof(int), stream) != cudaSuccess) return KDA_ERR_CUDA;
  RecurrenceArgs ra = make_recurrence_args(shape, T, qn, kn, vc, g, beta, initial_state, cu_seqlens,
                                           o, final_state);
  ra.err = reinterpret_cast<int *>(ws + L.err);
  return cuda_status(run_recurrence(ra, varlen, ws, L, stream));
}

kda_status kda_decode_step(const kda_shape *shape, const void *q, const void *k, const void *v,
                           const void *alpha, const void *b, const void *conv_w,
                           const float *A_log, const float *dt_bias, float *state,
                           void *conv_state, void *o, void *stream_) {
  return kda_decode_step_gated(shape, q, k, v, alpha, b, conv_w, A_log, dt_bias, nullptr, state,
                               conv_state, o, stream_);
}

kda_status kda_decode_step_gated(const kda_shape *shape, const void *q, const void *k,
                                 const void *v, const void *alpha, const void *b,
                                 const void *conv_w, const float *A_log, const float *dt_bias,
                                 const kda_output_gate *out_gate, float *state, void *conv_state,
                                 void *o, void *stream_) {
  if (shape == nullptr) return KDA_ERR_INVALID_ARGUMENT;
  kda_shape one = *shape;
  one.seq_len = 1;
  return kda_decode_multi(&one, q, k, v, alpha, b, conv_w, A_log, dt_bias, out_gate, state,
                          conv_state, o, nullptr, stream_);
}

kda_status kda_decode_multi(const kda_shape *shape, const void *q, const void *k, const void *v,
                            const void *alpha, const void *b, const void *conv_w,
                            const float *A_log, const float *dt_bias,
                            const kda_output_gate *out_gate, float *state, void *conv_state,
                            void *o, float *step_states, void *stream_) {
  kda_decode_args a;
  std::memset(&a, 0, sizeof a);
  a.q = q; a.k = k; a.v = v; a.alpha = alpha; a.b = b; a.conv_w = conv_w;
  a.A_log = A_log; a.dt_bias = dt_bias; a.out_gate = out_gate;
  a.state = state; a.conv_state = conv_state; a.o = o; a.step_states = step_states;
  return kda_decode_ex(shape, &a, stream_);
}

kda_status kda_decode_ex(const kda_shape *shape, const kda_decode_args *args, void *stream_) {
  kda_status st = check_shape(shape);
  if (st != KDA_OK) return st;
  if (args == nullptr) return KDA_ERR_INVALID_ARGUMENT;
  if (shape->seq_len < 1 || shape->seq_len > 16) return KDA_ERR_INVALID_ARGUMENT;
  if (args->status != nullptr && (reinterpret_cast<uintptr_t>(args->status) & 3u))
    return KDA_ERR_INVALID_ARGUMENT;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  if (shape->num_seqs == 0)
    return args->status == nullptr ? KDA_OK
                                   : cuda_status(cudaMemsetAsync(args->status, 0, sizeof(int32_t), stream));
  st = check_out_gate(args->out_gate, shape->num_seqs);
  if (st != KDA_OK) return st;
  KDA_REQUIRE(args->q); KDA_REQUIRE(args->k); KDA_REQUIRE(args->v); KDA_REQUIRE(args->alpha);
  KDA_REQUIRE(args->b); KDA_REQUIRE(args->conv_w); KDA_REQUIRE(args->A_log);
  KDA_REQUIRE(args->dt_bias); KDA_REQUIRE(args->state); KDA_REQUIRE(args->conv_state);
  KDA_REQUIRE(args->o); KDA_OPTIONAL(args->step_states);
  DecodeArgs a;
  std::memset(&a, 0, sizeof a);
  a.N = shape->num_seqs; a.H = shape->num_heads; a.D = shape->head_dim; a.io_dtype = shape->io_dtype;
  a.q = args->q; a.k = args->k; a.v = args->v; a.alpha = args->alpha; a.b = args->b;
  a.conv_w = args->conv_w; a.A_log = args->A_log; a.dt_bias = args->dt_bias;
  a.lower_bound = shape->lower_bound; a.eps = shape->l2norm_eps; a.scale = shape->scale;
  a.beta2 = (shape->flags & KDA_FLAG_NEGATIVE_EIGENVALUES) != 0;
  if (args->out_gate != nullptr) {
    a.ogate = args->out_gate->gate; a.onw = args->out_gate->weight; a.oeps = args->out_gate->eps;
  }
  a.ntok = shape->seq_len;
  a.step_states = args->step_states;
  a.state = args->state; a.conv_state = args->conv_state; a.o = args->o;
  a.err = args->status;
  a.wait_polls = wait_polls_for(shape->flags);
  if (a.err != nullptr && cudaMemsetAsync(a.err, 0, sizeof(int32_t), stream) != cudaSuccess)
    return KDA_ERR_CUDA;
  return cuda_status(launch_decode(a, stream));
}

const char *kda_status_string(kda_status status) {
  switch (status) {
    case KDA_OK: return "KDA_OK";
    case KDA_ERR_INVALID_ARGUMENT: return "KDA_ERR_INVALID_ARGUMENT: bad pointer, size or cu_seqlens";
    case KDA_ERR_UNSUPPORTED: return "KDA_ERR_UNSUPPORTED: shape not implemented (head_dim 64/128, heads <= 64)";
    case KDA_ERR_WORKSPACE: return "KDA_ERR_WORKSPACE: workspace missing, misaligned or too small";
    case KDA_ERR_CUDA: return "KDA_ERR_CUDA: a CUDA call or launch failed";
    case KDA_ERR_TIMEOUT: return "KDA_ERR_TIMEOUT: a bounded device wait gave up";
  }
  return "KDA: unknown status";
}

int kda_version(void) { return 100; }

}  // extern "C"
