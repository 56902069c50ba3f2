// Shared device helpers for the KDA kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/kda.h"

namespace kda {

constexpr int KCONV = 4;  // causal conv kernel size; 3 history tokens

// Bits of the device status word (the first int32 of the prefill workspace, or a
// decode call's status word), set with atomicOr.
constexpr int ERR_NONE = 0;
constexpr int ERR_BAD_CU_SEQLENS = KDA_STATUS_BAD_CU_SEQLENS;
constexpr int ERR_TIMEOUT_PREP = KDA_STATUS_TIMEOUT_PREP;
constexpr int ERR_TIMEOUT_STATE = KDA_STATUS_TIMEOUT_STATE;
constexpr int ERR_TIMEOUT_DECODE = KDA_STATUS_TIMEOUT_DECODE;


struct Bf16 {
  using T = __nv_bfloat16;
  static constexpr int kBytes = 2;
};
struct F32 {
  using T = float;
  static constexpr int kBytes = 4;
};

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Load / store 8 consecutive elements (16 B of bf16, 32 B of fp32) as fp32.
__device__ __forceinline__ void load8(const __nv_bfloat16 *p, float (&x)[8]) {
  uint4 u = *reinterpret_cast<const uint4 *>(p);
  const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __bfloat1622float2(h[i]);
    x[2 * i] = f.x;
    x[2 * i + 1] = f.y;
  }
}
__device__ __forceinline__ void load8(const float *p, float (&x)[8]) {
  float4 a = *reinterpret_cast<const float4 *>(p);
  float4 b = *reinterpret_cast<const float4 *>(p + 4);
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
  x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}
// Streaming (read-once) variants: bypass L1 allocation.
__device__ __forceinline__ void load8_stream(const __nv_bfloat16 *p, float (&x)[8]) {
  uint4 u = __ldcs(reinterpret_cast<const uint4 *>(p));
  const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __bfloat1622float2(h[i]);
    x[2 * i] = f.x;
    x[2 * i + 1] = f.y;
  }
}
__device__ __forceinline__ void load8_stream(const float *p, float (&x)[8]) {
  float4 a = __ldcs(reinterpret_cast<const float4 *>(p));
  float4 b = __ldcs(reinterpret_cast<const float4 *>(p + 4));
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
  x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}

__device__ __forceinline__ void store8(__nv_bfloat16 *p, const float (&x)[8]) {
  uint4 u;
  __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
  *reinterpret_cast<uint4 *>(p) = u;
}
__device__ __forceinline__ void store8(float *p, const float (&x)[8]) {
  *reinterpret_cast<float4 *>(p) = make_float4(x[0], x[1], x[2], x[3]);
  *reinterpret_cast<float4 *>(p + 4) = make_float4(x[4], x[5], x[6], x[7]);
}

// Elementwise math on the special-function unit: 2^x and log2(x) by their
// hardware approximations (relative error about 2^-22) and an approximate
// division; every function below is built from its definition on top of them.
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float lg2_approx(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// softplus(x) = log(1 + e^x) in the overflow-free form max(x, 0) + log(1 + e^{-|x|}).
__device__ __forceinline__ float softplus_f(float x) {
  return fmaxf(x, 0.f) + kLn2 * lg2_approx(1.f + ex2_approx(-fabsf(x) * kLog2e));
}
// sigmoid(x) = 1 / (1 + e^{-x}); for x -> -inf the denominator is +inf and the result 0.
__device__ __forceinline__ float sigmoid_f(float x) {
  return __fdividef(1.f, 1.f + ex2_approx(-x * kLog2e));
}
// SiLU(x) = x sigmoid(x)
__device__ __forceinline__ float silu_f(float x) { return __fdividef(x, 1.f + ex2_approx(-x * kLog2e)); }

// Gate: g = max(-exp(A_log) * softplus(alpha + dt_bias), lower_bound); negA = -exp(A_log).
__device__ __forceinline__ float gate_f(float alpha_plus_bias, float negA, float lower_bound) {
  return fmaxf(negA * softplus_f(alpha_plus_bias), lower_bound);
}

// Sequence bounds [start, end) of sequence n, clamped into [0, total] so that a
// malformed cu_seqlens can never produce an out-of-bounds access.
__device__ __forceinline__ void seq_bounds(const int32_t *cu, int n, int seq_len, int64_t total,
                                           int64_t &start, int64_t &end) {
  if (cu == nullptr) {
    start = (int64_t)n * seq_len;
    end = start + seq_len;
  } else {
    int64_t a = cu[n], z = cu[n + 1];
    a = a < 0 ? 0 : (a > total ? total : a);
    z = z < a ? a : (z > total ? total : z);
    start = a;
    end = z;
  }
}

// Sequence index containing packed token row t (binary search over cu_seqlens).
__device__ __forceinline__ int seq_of_token(const int32_t *cu, int N, int seq_len, int64_t t) {
  if (cu == nullptr) return (int)(t / seq_len);
  int lo = 0, hi = N - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if ((int64_t)cu[mid] <= t) lo = mid; else hi = mid - 1;
  }
  return lo;
}

}  // namespace kda
