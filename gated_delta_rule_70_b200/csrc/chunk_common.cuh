// Layout helpers shared by the two kernels of the tensor-core chunk path
// (kda_chunk_prep.cu and kda_state_pass.cu).
//
// Shared-memory operand format: token rows of 128 channels, 128-byte swizzle,
// 64-channel atoms (1 KB per 8 rows).  The same bytes are read by an MMA
// descriptor as K-major (K = channels) or MN-major (MN = channels, K = tokens).
//
// The per-chunk record that chunk_prep writes and state_pass reads is stored
// in global memory as the exact byte image state_pass needs in shared memory,
// so a plain bulk copy moves it: no swizzling or tensor map on the way back.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "umma.cuh"

namespace kda {
namespace chunkfmt {

constexpr int CH = 64;    // tokens per chunk
constexpr int DK = 128;   // head dim (d_k = d_v)

// Chunk record (bytes)
constexpr uint32_t REC_WT = 0;        // -W^T: [i = key channel][64 t], MN-major B image, 16 KB
constexpr uint32_t REC_U = 16384;     // U^T: [j = value channel][64 t], K-major A image, 16 KB
constexpr uint32_t REC_AQ = 32768;    // A_qk: [64 t][64 s], K-major image, 8 KB
constexpr uint32_t REC_QT = 40960;    // q e^{Gamma}: token-rows, 16 KB
constexpr uint32_t REC_KH = 57344;    // k e^{Gamma_C - Gamma}: token-rows, 16 KB
constexpr uint32_t REC_EGC = 73728;   // e^{Gamma_C} per key channel: 128 fp32
constexpr uint32_t REC_BYTES = 74240;
constexpr uint32_t REC_STRIDE = 74752;   // 1024-aligned

// Byte offset of (row, channel group cg of 8 channels) in a token-rows operand with `rows` rows.
__device__ __forceinline__ uint32_t tr_off(int rows, int row, int cg) {
  return (uint32_t)((cg >> 3) * rows * 128 + (row >> 3) * 1024 + (row & 7) * 128 +
                    (((cg & 7) ^ (row & 7)) << 4));
}
// Byte offset of (row i, 16-byte chunk c8) in a [rows][64] operand (one atom wide).
__device__ __forceinline__ uint32_t row64_off(int i, int c8) {
  return (uint32_t)((i >> 3) * 1024 + (i & 7) * 128 + ((c8 ^ (i & 7)) << 4));
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&h);
}
__device__ __forceinline__ uint4 pack8(const float (&x)[8]) {
  return make_uint4(pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]), pack_bf16(x[4], x[5]),
                    pack_bf16(x[6], x[7]));
}
__device__ __forceinline__ void unpack8(const uint4 &u, float (&x)[8]) {
  const __nv_bfloat162 *hh = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __bfloat1622float2(hh[i]);
    x[2 * i] = f.x;
    x[2 * i + 1] = f.y;
  }
}

// K-major descriptor over a token-rows operand with `rows` rows, K = 128 channels, k-step s.
__device__ __forceinline__ uint64_t desc_k128(uint32_t base, int rows, int s) {
  return umma::make_desc(base + (uint32_t)((s >> 2) * rows * 128 + (s & 3) * 32), 16, 1024,
                         umma::LAYOUT_SW128);
}
// MN-major descriptor over a 64-token-row operand (MN = 128 channels, K = tokens), k-step s.
__device__ __forceinline__ uint64_t desc_mn_tok(uint32_t base, int s) {
  return umma::make_desc(base + (uint32_t)(s * 2048), 64 * 128, 1024, umma::LAYOUT_SW128);
}
// K-major descriptor over a [rows][64] matrix (one atom wide), k-step s.
__device__ __forceinline__ uint64_t desc_k64(uint32_t base, int s) {
  return umma::make_desc(base + (uint32_t)(s * 32), 16, 1024, umma::LAYOUT_SW128);
}
// MN-major descriptor over [128 K-rows][64] (MN one atom wide), k-step s (16 rows).
__device__ __forceinline__ uint64_t desc_mn_rows(uint32_t base, int s) {
  return umma::make_desc(base + (uint32_t)(s * 2048), 128 * 128, 1024, umma::LAYOUT_SW128);
}

}  // namespace chunkfmt
}  // namespace kda
