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
#include <cuda_fp16.h>
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

// ---- two-lane fp32 arithmetic (sm_100 FFMA2 / FMUL2 / FADD2: each lane rounds
// exactly like the scalar instruction) and bf16 pair conversions
__device__ __forceinline__ float2 f2(float a) { return make_float2(a, a); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
// bf16 pair in one 32-bit word (lower address in the low half) -> (low, high) as fp32
__device__ __forceinline__ float2 bf2_f2(uint32_t u) {
  return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
}
__device__ __forceinline__ uint32_t f2_bf2(float2 v) { return pack_bf16(v.x, v.y); }
__device__ __forceinline__ uint32_t word(const uint4 &u, int i) {
  return i == 0 ? u.x : (i == 1 ? u.y : (i == 2 ? u.z : u.w));
}
__device__ __forceinline__ float2 ex2_2(float2 x) {
  return make_float2(umma::ex2(x.x), umma::ex2(x.y));
}
// SiLU(x) = x sigmoid(x) from h = x/2: with sigmoid(x) = 1/2 + tanh(x/2)/2,
// SiLU(x) = h + h tanh(h), one fma once the tanh is known.  The tanh is taken two
// lanes at a time in half precision on the special-function unit (absolute error
// of the sigmoid about 2^-12, below the bf16 rounding of the result); h itself stays
// fp32, so large |x| (where the half-precision tanh saturates to +-1) still gives
// x or 0.
__device__ __forceinline__ float2 silu2_from_half(float2 h) {
  uint32_t hh, t;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(hh) : "f"(h.y), "f"(h.x));
  asm("tanh.approx.f16x2 %0, %1;" : "=r"(t) : "r"(hh));
  const float2 th = __half22float2(*reinterpret_cast<const __half2 *>(&t));
  return fma2(h, th, h);
}

// sigmoid(x) = 1/2 + tanh(x/2)/2 two lanes at a time, the tanh in half precision
// on the special-function unit (absolute error about 2^-12).
__device__ __forceinline__ float2 sigmoid2(float2 x) {
  const float2 hx = mul2(x, f2(0.5f));
  uint32_t h, t;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(h) : "f"(hx.y), "f"(hx.x));
  asm("tanh.approx.f16x2 %0, %1;" : "=r"(t) : "r"(h));
  const float2 th = __half22float2(*reinterpret_cast<const __half2 *>(&t));
  return fma2(th, f2(0.5f), f2(0.5f));
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
