// kda_prefill_noalloc: the prefill for callers that cannot allocate device
// memory.
//
// kda_prefill asks the caller for a workspace: the prologue's outputs (q, k, v
// after conv / normalisation, the gate and beta) and the error word live
// there between the prologue and recurrence kernels.  Some callers cannot
// provide one: code running where cudaMalloc is forbidden or unavailable
// (inside a host callback, under an allocator that must not grow, or in an
// embedding that owns all device memory and hands out only input/output
// buffers).  This entry point takes its scratch from a fixed-size array in
// device memory that belongs to the library instead.
//
// The array below is reserved on every GPU that loads the library, for as long
// as the library stays loaded.  Host code may not take its address directly:
// on the host the name `g_prefill_scratch` is only a stand-in, so the device
// address is obtained once per device with cudaGetSymbolAddress (while that
// device is current) and then passed to the kernels as a plain pointer.
#include <mutex>

#include "kda_common.cuh"
#include "kda_internal.h"

namespace {

using namespace kda;

static __device__ __align__(256) unsigned char g_prefill_scratch[KDA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mu;
// Looked up once per device and kept for the life of the process; after a
// cudaDeviceReset of a device its entry here would be stale, so the entry point
// must not be used on a device that has been reset.
void *g_scratch_addr[kMaxDevices] = {};

// Device address of this device's copy of the scratch array (set up on first use).
cudaError_t scratch_address(void **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_setup_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_prefill_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

inline bool ok16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" kda_status kda_prefill_noalloc(
    const kda_shape *s, const void *q, const void *k, const void *v, const void *conv_w,
    const void *alpha, const void *b, const float *A_log, const float *dt_bias,
    const float *initial_state, const void *initial_conv_state, const int32_t *cu_seqlens, void *o,
    float *final_state, void *final_conv_state, void *stream_) {
  const kda_status st = check_shape(s);   // the same shape rules as kda_prefill
  if (st != KDA_OK) return st;
  if (s->num_seqs == 0) return KDA_OK;
  const int64_t T = cu_seqlens ? (int64_t)s->seq_len : (int64_t)s->num_seqs * s->seq_len;
  if (check_tokens(T) != KDA_OK) return KDA_ERR_UNSUPPORTED;
  const bool varlen = cu_seqlens != nullptr;
  const WsLayout L = workspace_layout(s->num_seqs, s->num_heads, s->head_dim, s->seq_len, T,
                                      s->io_dtype, s->lower_bound, varlen, true);
  if (L.total > KDA_NOALLOC_SCRATCH_BYTES) return KDA_ERR_WORKSPACE;
  if (T > 0 && (!q || !k || !v || !alpha || !b || !o || !ok16(q) || !ok16(k) || !ok16(v) ||
                !ok16(alpha) || !ok16(b) || !ok16(o)))
    return KDA_ERR_INVALID_ARGUMENT;
  if (!conv_w || !A_log || !dt_bias || !final_state || !ok16(conv_w) || !ok16(A_log) ||
      !ok16(dt_bias) || !ok16(final_state) || !ok16(initial_state) || !ok16(initial_conv_state) ||
      !ok16(final_conv_state))
    return KDA_ERR_INVALID_ARGUMENT;
  if (cu_seqlens != nullptr && (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u))
    return KDA_ERR_INVALID_ARGUMENT;

  void *base = nullptr;
  if (scratch_address(&base) != cudaSuccess) return KDA_ERR_CUDA;
  char *ws = static_cast<char *>(base);
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  // The array keeps the previous call's contents; only the error word must start at zero.
  if (cudaMemsetAsync(ws + L.err, 0, sizeof(int), stream) != cudaSuccess) return KDA_ERR_CUDA;

  PrologueArgs pa{};
  pa.N = s->num_seqs; pa.H = s->num_heads; pa.D = s->head_dim; pa.seq_len = s->seq_len;
  pa.total_tokens = T; pa.io_dtype = s->io_dtype; pa.cu = cu_seqlens;
  pa.q = q; pa.k = k; pa.v = v; pa.conv_w = conv_w; pa.alpha = alpha; pa.b = b;
  pa.A_log = A_log; pa.dt_bias = dt_bias; pa.conv0 = initial_conv_state;
  pa.lower_bound = s->lower_bound; pa.eps = s->l2norm_eps;
  pa.beta2 = (s->flags & KDA_FLAG_NEGATIVE_EIGENVALUES) != 0;
  pa.err = reinterpret_cast<int *>(ws + L.err);

  RecurrenceArgs ra{};
  ra.N = s->num_seqs; ra.H = s->num_heads; ra.D = s->head_dim; ra.seq_len = s->seq_len;
  ra.total_tokens = T; ra.io_dtype = s->io_dtype; ra.cu = cu_seqlens;
  ra.state0 = initial_state; ra.scale = s->scale; ra.o = o; ra.state1 = final_state;
  ra.lower_bound = s->lower_bound; ra.err = pa.err;
  ra.wait_polls = wait_polls_for(s->flags);
  ra.token_loop = (s->flags & KDA_FLAG_TOKEN_RECURRENCE) != 0;
  ra.side_stream = nullptr;   // one launch per kernel: the segmented schedule would create events
  if (run_prefill(pa, ra, final_conv_state, varlen, ws, L, stream) != cudaSuccess) return KDA_ERR_CUDA;
  return KDA_OK;
}
