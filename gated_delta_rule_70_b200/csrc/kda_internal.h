// Internal launch interface between the C ABI (kda_api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/kda.h"

namespace kda {

struct PrologueArgs {
  int N, H, D, seq_len;      // seq_len: dense tokens per sequence (unused when cu != nullptr)
  int64_t total_tokens;
  int io_dtype;
  const int32_t *cu;         // [N + 1] or nullptr (dense)
  const void *q, *k, *v;     // [T, H*D] raw
  const void *conv_w;        // [3, H*D, 4]
  const void *alpha;         // [T, H, D]
  const void *b;             // [T, H]
  const float *A_log;        // [H]
  const float *dt_bias;      // [H, D]
  const void *conv0;         // [N, 3, 3*H*D] or nullptr
  float lower_bound, eps;
  int beta2;                 // beta = 2 sigmoid(b) (negative eigenvalues allowed); 0: sigmoid(b)
  void *qn, *kn, *vc;        // [T, H, D] io dtype
  float *g;                  // [T, H, D]
  float *beta;               // [T, H]
  int *err;                  // device error word or nullptr
};

struct RecurrenceArgs {
  int N, H, D, seq_len;
  int64_t total_tokens;
  int io_dtype;
  const int32_t *cu;
  const void *qn, *kn, *vc;  // [T, H, D] io dtype (prologue outputs)
  const float *g;            // [T, H, D]
  const float *beta;         // [T, H]
  const float *state0;       // [N, H, D, D] or nullptr
  float scale;
  float lower_bound;         // gates are taken as clamped into [lower_bound, 0]
  void *o;                   // [T, H, D] io dtype
  float *state1;             // [N, H, D, D]
  int *err;
  // output epilogue: o <- o / sqrt(mean o^2 + oeps) * onw * sigmoid(ogate), or ogate == nullptr
  const void *ogate;         // [T, H, D] io dtype
  const float *onw;          // [D]
  float oeps;
  // state snapshots: snap[(n * snap_cap + j) * H + h] = state after (j + 1) * snap_every
  // tokens of sequence n (snap_every a multiple of 64), j < snap_cap; nullptr: none
  float *snap;
  int64_t snap_every;
  int snap_cap;
  // the caller's side stream for the time-segmented schedule, or nullptr (no segments)
  cudaStream_t side_stream;
  uint32_t wait_polls;       // polls per ordinary bounded wait (kWaitPolls; 0 in the failure test)
  int token_loop;            // off the tensor-core path: the token kernel, not the fp32 chunk kernel
};

struct DecodeArgs {
  int N, H, D;
  int io_dtype;
  const void *q, *k, *v;     // [N, H*D]
  const void *alpha;         // [N, H, D]
  const void *b;             // [N, H]
  const void *conv_w;        // [3, H*D, 4]
  const float *A_log, *dt_bias;
  float lower_bound, eps, scale;
  int beta2;                 // beta = 2 sigmoid(b); 0: sigmoid(b)
  const void *ogate;         // output epilogue [N, ntok, H, D] io dtype, or nullptr
  const float *onw;          // [D]
  float oeps;
  int ntok;                  // tokens per sequence in this call (token inputs [N, ntok, ...]); 0 or 1: one
  float *step_states;        // [N, ntok, H, D, D]: the state after each token, or nullptr
  float *state;              // [N, H, D, D] in place
  void *conv_state;          // [N, 3, 3*H*D] in place
  void *o;                   // [N, H, D]
  int *err;                  // device status word or nullptr
  uint32_t wait_polls;       // polls per ordinary bounded wait
};

// Tensor-core chunk path (bf16, head_dim 128): chunk_prep writes one record
// per (chunk, head); state_pass runs the sequential state chain over them.
// chunk_prep either runs the prologue itself on the raw inputs (fused: the
// prefill entry points) or reads prepared inputs (the recurrence entry point).
struct PrepArgs {
  int N, H, seq_len;
  int64_t total_tokens;
  const int32_t *cu;         // [N + 1] or nullptr (dense)
  const int32_t *chunk_cu;   // [N + 1] chunk prefix (varlen) or nullptr (dense)
  const int4 *slot_info;     // varlen: per chunk slot {sequence, chunk index, first token, tokens}
                             // ({-1, ..} past the last chunk); nullptr (dense)
  float lower_bound, eps;
  int beta2;                 // fused: beta = 2 sigmoid(b); 0: sigmoid(b)
  // fused prologue: raw inputs (q, k, v, alpha read through the tensor maps)
  const void *conv_w;        // [3, H*128, 4] bf16
  const void *b;             // [T, H] bf16
  const float *A_log;        // [H]
  const float *dt_bias;      // [H, 128]
  const void *conv0;         // [N, 3, 3*H*128] bf16 or nullptr
  // prepared inputs
  const void *qn, *kn, *vc;  // [T, H, 128] bf16
  const float *g, *beta;     // [T, H, 128], [T, H]
  void *records;             // [max_slots][H] records of chunkfmt::REC_STRIDE bytes
  int64_t max_slots;         // record slots (set by the launcher)
  int seg_c0, seg_len;       // dense batches: chunks [seg_c0, seg_c0 + seg_len) of every sequence
                             // (seg_len 0: all); varlen batches: unused
  int *err;
  uint32_t wait_polls;       // polls per ordinary bounded wait
  // [T rows][H*128] bf16: q, k, v (67-row boxes: 3 history rows + 64) and alpha (64 rows)
  CUtensorMap map_q, map_k, map_v, map_alpha;
};

struct StateArgs {
  int N, H, seq_len;
  int64_t total_tokens;
  const int32_t *cu, *chunk_cu;
  const int32_t *order;      // varlen: CTA slot -> sequence, longest first; nullptr: identity
  const void *records;
  int64_t max_slots;         // record slots in the workspace (chunks beyond are not read)
  const float *state0;       // [N, H, 128, 128] or nullptr
  int seg_c0, seg_c1;        // chunks [seg_c0, seg_c1) of every sequence (0, INT_MAX: all)
  float scale;
  void *o;                   // [T, H, 128] bf16
  float *state1;
  int *err;
  uint32_t wait_polls;       // polls per ordinary bounded wait
  const float *onw;          // output epilogue weight [128], with map_gate; nullptr: off
  float oeps;
  float *snap;               // state snapshots, as in RecurrenceArgs (every snap_chunks chunks)
  int snap_chunks, snap_cap;
  CUtensorMap map_gate;      // gate [T rows][H*128] bf16, 64-row boxes
};

// Bytes of one chunk record and the number of record slots a shape needs.
constexpr size_t kChunkRecordBytes = 74752;
inline int64_t max_chunk_slots(int N, int64_t total_tokens, int seq_len, bool varlen) {
  return varlen ? (total_tokens + 63) / 64 + N : (int64_t)N * ((seq_len + 63) / 64);
}

// Workspace layout (byte offsets, 256-aligned):
//   error word | qn | kn | vc | g | beta   (prologue outputs; token-kernel prefill only)
//   | chunk table (N+1 int32) | sequence order (N int32, varlen)
//   | slot table (one int4 per chunk slot, varlen) | chunk records   (tensor-core path only)
struct WsLayout {
  size_t err, qn, kn, vc, g, beta, chunk_cu, order, slots, records, total;
  bool tc;   // bf16 with head_dim 128: the tensor-core chunk path
};
// The tensor-core path splits e^{Gamma_t - Gamma_s} around a reference in the middle
// of each sub-block (32 tokens for gate bounds >= -5.02, else 16), so each factor spans
// at most 16 or 8 gates: within 2^{+-116}, inside fp32 / bf16 normal range, for gates
// >= -5.02 or >= -10; shapes with a lower gate bound run the CUDA-core kernels.
constexpr float kTcMinLowerBound = -10.0f;
inline bool use_tensor_core_path(int io_dtype, int D, float lower_bound) {
  return io_dtype == KDA_BF16 && D == 128 && lower_bound >= kTcMinLowerBound;
}
inline WsLayout workspace_layout(int N, int H, int D, int seq_len, int64_t T, int io_dtype,
                                 float lower_bound, bool varlen, bool with_prologue) {
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  const size_t es = io_dtype == KDA_BF16 ? 2 : 4;
  const size_t thd = (size_t)T * H * D;
  WsLayout L{};
  L.tc = use_tensor_core_path(io_dtype, D, lower_bound);
  size_t off = 256;  // error word
  L.err = 0;
  if (with_prologue && !L.tc) {  // the tensor-core path runs the prologue inside chunk_prep
    L.qn = off; off = up(off + thd * es);
    L.kn = off; off = up(off + thd * es);
    L.vc = off; off = up(off + thd * es);
    L.g = off; off = up(off + thd * 4);
    L.beta = off; off = up(off + (size_t)T * H * 4);
  }
  if (L.tc) {
    L.chunk_cu = off; off = up(off + (size_t)(N + 1) * 4);
    if (varlen) {
      L.order = off; off = up(off + (size_t)N * 4);
      L.slots = off; off = up(off + (size_t)max_chunk_slots(N, T, seq_len, varlen) * 16);
    }
    off = (off + 1023) / 1024 * 1024;
    L.records = off;
    off += (size_t)max_chunk_slots(N, T, seq_len, varlen) * H * kChunkRecordBytes;
  }
  L.total = off;
  return L;
}

// Shape checks shared by every entry point: KDA_OK, KDA_ERR_INVALID_ARGUMENT or
// KDA_ERR_UNSUPPORTED.
kda_status check_shape(const kda_shape *s);
// A call's packed token total T: the kernels keep token rows and chunk coordinates in 32 bits.
inline kda_status check_tokens(int64_t T) {
  return T > (int64_t)INT32_MAX - 64 ? KDA_ERR_UNSUPPORTED : KDA_OK;
}
// Polls of one bounded mbarrier wait (each poll is an mbarrier.try_wait, which may
// itself suspend for a while), and the limit every drain of in-flight copies and
// tensor-core work uses after a wait has given up.  A call with
// KDA_FLAG_TEST_EXPIRE_WAITS passes 0 for its ordinary waits, never for a drain.
constexpr uint32_t kWaitPolls = 1u << 22;
inline uint32_t wait_polls_for(uint32_t flags) {
  return (flags & KDA_FLAG_TEST_EXPIRE_WAITS) ? 0u : kWaitPolls;
}

cudaError_t launch_prologue(const PrologueArgs &a, cudaStream_t stream);
// chunk_cu[n] = 64-token chunks before sequence n; also checks cu_seqlens
// (starts at 0, non-decreasing, ends at total) and flags ERR_BAD_CU_SEQLENS in *err.
cudaError_t launch_chunk_table(const int32_t *cu, int N, int64_t total, int32_t *chunk_cu, int *err,
                               cudaStream_t stream);
// order[r] = the sequence with the r-th most 64-token chunks (ties: lower index first), so
// the state pass starts its longest chains first; identity for more than 2048 sequences.
cudaError_t launch_seq_order(const int32_t *cu, int N, int64_t total, int32_t *order, cudaStream_t stream);
// info[s] = {sequence, chunk index, first token, tokens} of chunk slot s < slots, {-1, 0, 0, 0}
// past the last chunk (after launch_chunk_table has written chunk_cu).
cudaError_t launch_slot_table(const int32_t *cu, const int32_t *chunk_cu, int N, int64_t total,
                              int64_t slots, int4 *info, cudaStream_t stream);
// fused: run the prologue on the raw inputs in a.{conv_w, b, A_log, dt_bias, conv0}
// and q, k, v, alpha (tensor maps built here); else read a.{qn, kn, vc, g, beta}.
cudaError_t launch_chunk_prep(PrepArgs a, int64_t max_chunks, bool fused, const void *q,
                              const void *k, const void *v, const void *alpha, cudaStream_t stream);
cudaError_t launch_state_pass(StateArgs a, const void *gate, cudaStream_t stream);
cudaError_t launch_conv_state_out(const PrologueArgs &a, void *out, cudaStream_t stream);
cudaError_t launch_recurrence(const RecurrenceArgs &a, cudaStream_t stream);
// The chunkwise recurrence on CUDA cores in fp32 (prepared inputs, as launch_recurrence).
cudaError_t launch_chunk_simt(const RecurrenceArgs &a, cudaStream_t stream);
// Off the tensor-core path: the fp32 chunk kernel where its split factors fit fp32
// (gate bound >= -10) unless the token loop was asked for, else the token kernel.
inline cudaError_t launch_cuda_core_recurrence(const RecurrenceArgs &a, cudaStream_t stream) {
  return !a.token_loop && a.lower_bound >= kTcMinLowerBound ? launch_chunk_simt(a, stream)
                                                            : launch_recurrence(a, stream);
}
// The recurrence (a4-a8) for RecurrenceArgs `ra` with workspace `ws` laid out by
// workspace_layout(): tensor-core chunk path for bf16 / head_dim 128, else the
// CUDA-core token kernel.
cudaError_t run_recurrence(const RecurrenceArgs &ra, bool varlen, char *ws, const WsLayout &L,
                           cudaStream_t stream);
// The whole prefill (prologue + recurrence + final conv state) for PrologueArgs
// `pa` (inputs, err) and RecurrenceArgs `ra` (state0, scale, o, state1) in a
// workspace laid out by workspace_layout(..., with_prologue = true).
cudaError_t run_prefill(PrologueArgs pa, RecurrenceArgs ra, void *final_conv_state, bool varlen,
                        char *ws, const WsLayout &L, cudaStream_t stream);
cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t stream);

}  // namespace kda
