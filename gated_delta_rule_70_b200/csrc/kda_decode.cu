// KDA decode step: one new token per sequence, fused prologue + in-place state
// update, one CTA per (sequence, head).
//
// The operation is one iteration of the per-token loop of the AliceAI-Foundation
// KDA write-up ("二、KDA 线性注意力"), on the state a prefill left behind (section
// "五": prefill and decode share initial_state / final_state) with the conv
// history advanced by one token (section "四": 3 conv states per channel).
//
// HBM-bound by construction: the CTA issues all loads of its 128x128 fp32 state
// slice (16 x 16-byte loads per thread, fully coalesced rows) before doing the
// token's prologue, so the prologue's latency hides under the state stream;
// each state element is then decayed, reduced, corrected and written back
// exactly once.  o = S'^T q + (q.k) d lets one __syncthreads carry all column
// reductions.
#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {

template <int D>
struct DecSmem {
  float q[D], k[D], eg[D], v[D];
  float red_p[D / 16][D], red_r[D / 16][D], red_qk[D / 16];
  float norm_part[2][D / 32];
  float beta;
};

template <typename T, int D>
__global__ void __launch_bounds__(2 * D, 2)
decode_kernel(DecodeArgs a) {
  constexpr int W = D / 16, CPL = D / 32;
  __shared__ DecSmem<D> sm;
  const int n = blockIdx.x / a.H, h = blockIdx.x % a.H;
  const int w = threadIdx.x / 32, l = threadIdx.x % 32;
  const int H = a.H;
  const int64_t HD = (int64_t)H * D;

  // 1. stream in this (n, h) state slice: rows [16w, 16w+16), columns [CPL*l, CPL*l+CPL)
  float *__restrict__ Sg = a.state + ((int64_t)n * H + h) * D * D;
  float S[16][CPL];
#pragma unroll
  for (int r = 0; r < 16; ++r) {
    const float *src = Sg + (int64_t)(16 * w + r) * D + CPL * l;
    if constexpr (CPL == 4) {
      float4 x = __ldcs(reinterpret_cast<const float4 *>(src));
      S[r][0] = x.x; S[r][1] = x.y; S[r][2] = x.z; S[r][3] = x.w;
    } else {
      float2 x = __ldcs(reinterpret_cast<const float2 *>(src));
      S[r][0] = x.x; S[r][1] = x.y;
    }
  }

  // 2. prologue for this token and head.  Threads [0, D): q and k channel i;
  //    threads [D, 2D): v channel i and the gate of key channel i.
  const T *__restrict__ cw = reinterpret_cast<const T *>(a.conv_w);
  T *__restrict__ cs = reinterpret_cast<T *>(a.conv_state) + (int64_t)n * 3 * 3 * HD;
  const int i = threadIdx.x % D;
  const bool first = threadIdx.x < D;
  auto conv_channel = [&](int blk, const T *x) -> float {
    const int64_t c = (int64_t)blk * HD + h * D + i;
    const float x0 = to_f32(cs[0 * 3 * HD + c]), x1 = to_f32(cs[1 * 3 * HD + c]);
    const float x2 = to_f32(cs[2 * 3 * HD + c]);
    const T xn = x[(int64_t)n * HD + h * D + i];
    float acc = to_f32(cw[c * KCONV + 0]) * x0;
    acc = fmaf(to_f32(cw[c * KCONV + 1]), x1, acc);
    acc = fmaf(to_f32(cw[c * KCONV + 2]), x2, acc);
    acc = fmaf(to_f32(cw[c * KCONV + 3]), to_f32(xn), acc);
    // shift the history in place: this thread is the only reader/writer of channel c
    cs[0 * 3 * HD + c] = cs[1 * 3 * HD + c];
    cs[1 * 3 * HD + c] = cs[2 * 3 * HD + c];
    cs[2 * 3 * HD + c] = xn;
    return silu_f(acc);
  };
  float qv = 0.f, kv = 0.f;
  if (first) {
    qv = conv_channel(0, reinterpret_cast<const T *>(a.q));
    kv = conv_channel(1, reinterpret_cast<const T *>(a.k));
    float sq = qv * qv, sk = kv * kv;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
      sq += __shfl_xor_sync(0xffffffffu, sq, off);
      sk += __shfl_xor_sync(0xffffffffu, sk, off);
    }
    if (l == 0) { sm.norm_part[0][w] = sq; sm.norm_part[1][w] = sk; }
  } else {
    sm.v[i] = conv_channel(2, reinterpret_cast<const T *>(a.v));
    const float al = to_f32(reinterpret_cast<const T *>(a.alpha)[((int64_t)n * H + h) * D + i]);
    const float g = gate_f(al + a.dt_bias[h * D + i], -expf(a.A_log[h]), a.lower_bound);
    sm.eg[i] = expf(g);
    if (i == 0) sm.beta = sigmoid_f(to_f32(reinterpret_cast<const T *>(a.b)[(int64_t)n * H + h]));
  }
  __syncthreads();
  if (first) {
    float sq = 0.f, sk = 0.f;
#pragma unroll
    for (int ww = 0; ww < D / 32; ++ww) { sq += sm.norm_part[0][ww]; sk += sm.norm_part[1][ww]; }
    sm.q[i] = qv * rsqrtf(sq + a.eps);
    sm.k[i] = kv * rsqrtf(sk + a.eps);
  }
  __syncthreads();

  // 3. decay, then the column reductions p = S'^T k and r = S'^T q
  float p[CPL], rr[CPL], qk = 0.f;
#pragma unroll
  for (int c = 0; c < CPL; ++c) { p[c] = 0.f; rr[c] = 0.f; }
#pragma unroll
  for (int r = 0; r < 16; ++r) {
    const int ii = 16 * w + r;
    const float e = sm.eg[ii], kk = sm.k[ii], qq = sm.q[ii];
    qk = fmaf(qq, kk, qk);
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
      S[r][c] *= e;
      p[c] = fmaf(kk, S[r][c], p[c]);
      rr[c] = fmaf(qq, S[r][c], rr[c]);
    }
  }
#pragma unroll
  for (int c = 0; c < CPL; ++c) { sm.red_p[w][CPL * l + c] = p[c]; sm.red_r[w][CPL * l + c] = rr[c]; }
  if (l == 0) sm.red_qk[w] = qk;
  __syncthreads();
  float P[CPL], R[CPL], QK = 0.f;
#pragma unroll
  for (int c = 0; c < CPL; ++c) { P[c] = 0.f; R[c] = 0.f; }
#pragma unroll
  for (int ww = 0; ww < W; ++ww) {
    QK += sm.red_qk[ww];
#pragma unroll
    for (int c = 0; c < CPL; ++c) { P[c] += sm.red_p[ww][CPL * l + c]; R[c] += sm.red_r[ww][CPL * l + c]; }
  }
  const float bt = sm.beta;
  float dl[CPL];
#pragma unroll
  for (int c = 0; c < CPL; ++c) dl[c] = bt * (sm.v[CPL * l + c] - P[c]);
  if (w == 0) {
    T *o = reinterpret_cast<T *>(a.o) + ((int64_t)n * H + h) * D + CPL * l;
#pragma unroll
    for (int c = 0; c < CPL; ++c) o[c] = from_f32<T>(a.scale * fmaf(QK, dl[c], R[c]));
  }

  // 4. write S = S' + k d^T back in place
#pragma unroll
  for (int r = 0; r < 16; ++r) {
    const float kk = sm.k[16 * w + r];
    float *dst = Sg + (int64_t)(16 * w + r) * D + CPL * l;
    if constexpr (CPL == 4) {
      __stcs(reinterpret_cast<float4 *>(dst),
             make_float4(fmaf(kk, dl[0], S[r][0]), fmaf(kk, dl[1], S[r][1]),
                         fmaf(kk, dl[2], S[r][2]), fmaf(kk, dl[3], S[r][3])));
    } else {
      __stcs(reinterpret_cast<float2 *>(dst),
             make_float2(fmaf(kk, dl[0], S[r][0]), fmaf(kk, dl[1], S[r][1])));
    }
  }
}

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t stream) {
  if ((int64_t)a.N * a.H == 0) return cudaSuccess;
  const unsigned grid = (unsigned)(a.N * a.H);
  if (a.io_dtype == KDA_BF16) {
    if (a.D == 128) decode_kernel<__nv_bfloat16, 128><<<grid, 256, 0, stream>>>(a);
    else decode_kernel<__nv_bfloat16, 64><<<grid, 128, 0, stream>>>(a);
  } else {
    if (a.D == 128) decode_kernel<float, 128><<<grid, 256, 0, stream>>>(a);
    else decode_kernel<float, 64><<<grid, 128, 0, stream>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace kda
