// Recurrence dispatch: bf16 with head_dim 128 runs the tensor-core chunk path
// (chunk_prep over every (chunk, head), then the sequential state pass); every
// other shape runs the CUDA-core token kernel.
#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {

cudaError_t run_recurrence(const RecurrenceArgs &ra, bool varlen, char *ws, const WsLayout &L,
                           cudaStream_t stream) {
#ifndef KDA_TOKEN_KERNEL_ONLY
  if (L.tc) {
    int32_t *chunk_cu = nullptr;
    if (varlen) {
      chunk_cu = reinterpret_cast<int32_t *>(ws + L.chunk_cu);
      cudaError_t e = launch_chunk_table(ra.cu, ra.N, ra.total_tokens, chunk_cu, stream);
      if (e != cudaSuccess) return e;
    }
    const int64_t slots = max_chunk_slots(ra.N, ra.total_tokens, ra.seq_len, varlen);
    PrepArgs pa{};
    pa.N = ra.N; pa.H = ra.H; pa.seq_len = ra.seq_len; pa.total_tokens = ra.total_tokens;
    pa.cu = ra.cu; pa.chunk_cu = chunk_cu;
    pa.qn = ra.qn; pa.kn = ra.kn; pa.vc = ra.vc; pa.g = ra.g; pa.beta = ra.beta;
    pa.records = ws + L.records; pa.err = ra.err;
    cudaError_t e = launch_chunk_prep(pa, slots, stream);
    if (e != cudaSuccess) return e;
    StateArgs sa{};
    sa.N = ra.N; sa.H = ra.H; sa.seq_len = ra.seq_len; sa.total_tokens = ra.total_tokens;
    sa.cu = ra.cu; sa.chunk_cu = chunk_cu; sa.records = ws + L.records; sa.max_slots = slots;
    sa.state0 = ra.state0; sa.scale = ra.scale; sa.o = ra.o; sa.state1 = ra.state1; sa.err = ra.err;
    return launch_state_pass(sa, stream);
  }
#endif
  return launch_recurrence(ra, stream);
}

}  // namespace kda
