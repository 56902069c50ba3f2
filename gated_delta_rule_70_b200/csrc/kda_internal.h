// Internal launch interface between the C ABI (kda_api.cu) and the kernels.
#pragma once

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
  void *o;                   // [T, H, D] io dtype
  float *state1;             // [N, H, D, D]
  int *err;
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
  float *state;              // [N, H, D, D] in place
  void *conv_state;          // [N, 3, 3*H*D] in place
  void *o;                   // [N, H, D]
};

cudaError_t launch_prologue(const PrologueArgs &a, cudaStream_t stream);
cudaError_t launch_conv_state_out(const PrologueArgs &a, void *out, cudaStream_t stream);
cudaError_t launch_recurrence(const RecurrenceArgs &a, cudaStream_t stream);
cudaError_t launch_chunk_tc(const RecurrenceArgs &a, cudaStream_t stream);
cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t stream);

}  // namespace kda
