// KDA prologue: depthwise causal conv (kernel 4, no bias) + SiLU on q, k, v;
// L2 normalisation of q and k per head; gate g = max(-exp(A_log) *
// softplus(alpha + dt_bias), lower_bound); beta = sigmoid(b).
//
// Source of the operation: AliceAI-Foundation KDA write-up, section
// "二、KDA 线性注意力" (q/k/v_conv1d with kernel 4, padding 3, no bias, SiLU;
// use_qk_l2norm_in_kernel; the gate formula), and the Ling-3.0-flash-VL config
// table (kda_lower_bound = -5.0).
//
// Streaming design: a group of d/8 threads owns one (head, 8-token tile); each
// thread owns 8 consecutive channels and walks the tile's tokens in order,
// keeping the 3-token conv history in registers.  All global traffic is 16-byte
// vector loads/stores; a warp touches 512 contiguous bytes per row (two heads
// of d = 128).  The L2 norm is a shuffle reduction inside the group.  A thread
// works through four phases (q, k, v, then alpha); with bf16 inputs the rows of a
// phase are staged two phases ahead into the thread's own shared-memory slots by
// asynchronous copies, so a thread's loads stay in flight while it computes (the
// registers hold only the phase it works on); a phase's conv weights are requested
// before its rows are waited for.  With bf16 outputs the SiLU takes one special-function
// operation (SiLU(x) = h + h tanh(h), h = x/2): the kernel is close to bound by that unit.
#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {

constexpr int PRO_TPT = 8;       // tokens per thread (one tile)
constexpr int PRO_THREADS = 256;
constexpr int PRO_STAGES = 2;    // phases staged ahead (bf16)
constexpr int PRO_ROWS = PRO_TPT + 3;   // a phase's rows: the 3 history tokens, then the tile
constexpr uint32_t PRO_STAGE_BYTES = PRO_STAGES * PRO_ROWS * PRO_THREADS * 16;   // 88 KB

// 16 bytes global -> shared, asynchronously; src_bytes 0 fills the slot with zeros
// (the source address is then not read, but stays a valid one).
__device__ __forceinline__ void cp_async16(void *dst, const void *src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;"
               :: "r"((uint32_t)__cvta_generic_to_shared(dst)), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N> __device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" :: "n"(N) : "memory");
}

// 8 consecutive elements held undecoded, so a tile's loads can all be issued
// before any arithmetic (one round trip to HBM per tile, not one per token).
template <typename T> struct Raw8;
template <> struct Raw8<__nv_bfloat16> {
  uint4 u;
  __device__ __forceinline__ void load(const __nv_bfloat16 *p) { u = __ldcs(reinterpret_cast<const uint4 *>(p)); }
  __device__ __forceinline__ void zero() { u = make_uint4(0, 0, 0, 0); }
  __device__ __forceinline__ void get(float (&x)[8]) const {
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) { float2 f = __bfloat1622float2(h[i]); x[2 * i] = f.x; x[2 * i + 1] = f.y; }
  }
};
template <> struct Raw8<float> {
  float4 a, b;
  __device__ __forceinline__ void load(const float *p) {
    a = __ldcs(reinterpret_cast<const float4 *>(p));
    b = __ldcs(reinterpret_cast<const float4 *>(p + 4));
  }
  __device__ __forceinline__ void zero() { a = b = make_float4(0.f, 0.f, 0.f, 0.f); }
  __device__ __forceinline__ void get(float (&x)[8]) const {
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  }
};

template <typename T, int D>
__global__ void __launch_bounds__(PRO_THREADS, 2)
prologue_kernel(PrologueArgs a) {
  constexpr int G = D / 8;  // threads per (token, head) row
  const int H = a.H;
  const int64_t HD = (int64_t)H * D;
  const int64_t total = a.total_tokens;
  const int64_t rg = ((int64_t)blockIdx.x * PRO_THREADS + threadIdx.x) / G;
  const int lane_in_group = threadIdx.x % G;
  const int h = (int)(rg % H);
  const int64_t tile = rg / H;
  const int64_t t0 = tile * PRO_TPT;
  if (t0 >= total) return;
  const int64_t t1 = min(t0 + (int64_t)PRO_TPT, total);
  const int c0 = h * D + lane_in_group * 8;  // channel within a q/k/v block
  const T *__restrict__ conv0 = reinterpret_cast<const T *>(a.conv0);

  // Validate cu_seqlens once (block 0, thread 0); bounds are clamped everywhere anyway.
  if (a.cu != nullptr && blockIdx.x == 0 && threadIdx.x == 0 && a.err != nullptr) {
    bool ok = a.cu[0] == 0 && (int64_t)a.cu[a.N] == total;
    for (int n = 0; n < a.N && ok; ++n) ok = a.cu[n + 1] >= a.cu[n];
    if (!ok) atomicOr(a.err, ERR_BAD_CU_SEQLENS);
  }

  const int n0 = seq_of_token(a.cu, a.N, a.seq_len, t0);
  // the G lanes of this row group (all take the same trip counts)
  const unsigned group_mask = (G == 32 ? 0xffffffffu : ((1u << G) - 1u) << ((threadIdx.x % 32) & ~(G - 1)));
  // whole tile inside one sequence: the conv phases take the staged rows; hist_in: its
  // three history tokens belong to the same sequence too (else they come from the conv
  // state or are zeros, loaded as the phase starts)
  bool whole, hist_in;
  {
    int64_t s0, e0;
    seq_bounds(a.cu, n0, a.seq_len, total, s0, e0);
    whole = t0 + PRO_TPT <= e0 && t1 - t0 == PRO_TPT;
    hist_in = t0 - 3 >= s0 && t0 >= 3;
  }

  // bf16: phase p's rows (p = 0, 1, 2: q, k, v at this thread's channels, history tokens
  // t0-3..t0-1 in rows 0-2 and the tile in rows 3..; p = 3: alpha in rows 3..) in slot
  // stage[p % 2][row][thread]; a commit group per phase (empty ones keep the count)
  constexpr bool kStage = sizeof(T) == 2;
  extern __shared__ __align__(16) uint4 pro_stage[];
  auto slot = [&](int p, int r) { return pro_stage + ((p & 1) * PRO_ROWS + r) * PRO_THREADS + threadIdx.x; };
  auto stage_phase = [&](int p) {
    if constexpr (kStage) {
      if (p < 3 && whole) {
        const T *x = reinterpret_cast<const T *>(p == 0 ? a.q : (p == 1 ? a.k : a.v));
        if (hist_in) {
#pragma unroll
          for (int m = 0; m < 3; ++m) cp_async16(slot(p, m), x + (t0 - 3 + m) * HD + c0, 16);
        }
#pragma unroll
        for (int j = 0; j < PRO_TPT; ++j) cp_async16(slot(p, 3 + j), x + (t0 + j) * HD + c0, 16);
      } else if (p == 3) {
        const T *al = reinterpret_cast<const T *>(a.alpha) + h * D + lane_in_group * 8;
#pragma unroll
        for (int j = 0; j < PRO_TPT; ++j)
          cp_async16(slot(p, 3 + j), al + (t0 + j < t1 ? t0 + j : t0) * HD, t0 + j < t1 ? 16u : 0u);
      }
      cp_async_commit();
    }
  };
  stage_phase(0);
  stage_phase(1);
  // b of token t0 + lane (lanes 0..7 of the group; G >= 8), early: each of those lanes
  // writes its token's beta at the end
  const bool has_b = lane_in_group < PRO_TPT && t0 + lane_in_group < t1;
  const float bme = has_b ? to_f32(reinterpret_cast<const T *>(a.b)[(t0 + lane_in_group) * H + h]) : 0.f;

#pragma unroll 1
  for (int blk = 0; blk < 3; ++blk) {
    const T *__restrict__ x = reinterpret_cast<const T *>(blk == 0 ? a.q : (blk == 1 ? a.k : a.v));
    T *__restrict__ y = reinterpret_cast<T *>(blk == 0 ? a.qn : (blk == 1 ? a.kn : a.vc));
    const T *__restrict__ w = reinterpret_cast<const T *>(a.conv_w) + ((int64_t)blk * HD + c0) * KCONV;
    float wr[8][KCONV];  // 8 channels x 4 taps = 32 contiguous elements, 2 channels per load
#pragma unroll
    for (int i = 0; i < 8; i += 2) {   // issued before the wait for the rows: the two latencies overlap
      float t8[8];
      load8(w + i * KCONV, t8);
#pragma unroll
      for (int j = 0; j < KCONV; ++j) { wr[i][j] = t8[j]; wr[i + 1][j] = t8[KCONV + j]; }
    }
    if constexpr (kStage) cp_async_wait<1>();   // phase blk's rows have landed
    // history hist[m][i]: raw input at token (t - 3 + m), m = 0..2
    float hist[3][8];
    int n = n0;
    int64_t s, e;
    seq_bounds(a.cu, n, a.seq_len, total, s, e);
    auto load_history = [&](int64_t t) {
#pragma unroll
      for (int m = 0; m < 3; ++m) {
        const int64_t tm = t - 3 + m;
        const int64_t slot = tm - s + 3;  // history slot; < 0 only for malformed cu_seqlens
        if (tm >= s && tm >= 0) {
          load8(x + tm * HD + c0, hist[m]);
        } else if (conv0 != nullptr && slot >= 0 && slot < 3) {
          load8(conv0 + ((int64_t)n * 3 + slot) * 3 * HD + blk * HD + c0, hist[m]);
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i) hist[m][i] = 0.f;
        }
      }
    };
    bool staged_hist = false;
    if constexpr (kStage) {
      if (whole && hist_in) {
#pragma unroll
        for (int m = 0; m < 3; ++m) {
          Raw8<T> r;
          r.u = *slot(blk, m);
          r.get(hist[m]);
        }
        staged_hist = true;
      }
    }
    if (!staged_hist) load_history(t0);
    // conv + SiLU (+ L2 norm for q, k) of one token whose raw input is xt
    auto emit = [&](int64_t t, const float (&xt)[8]) {
      float yt[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float acc = wr[i][0] * hist[0][i];
        acc = fmaf(wr[i][1], hist[1][i], acc);
        acc = fmaf(wr[i][2], hist[2][i], acc);
        acc = fmaf(wr[i][3], xt[i], acc);
        if constexpr (sizeof(T) == 2) {
          // bf16 outputs: SiLU(x) = h + h tanh(h), h = x/2, with the special-function unit's
          // fp32 tanh (one operation, relative error about 2^-11, under the bf16 rounding
          // that follows); fp32 outputs keep the division form
          const float hx = 0.5f * acc;
          float th;
          asm("tanh.approx.f32 %0, %1;" : "=f"(th) : "f"(hx));
          yt[i] = fmaf(hx, th, hx);
        } else {
          yt[i] = silu_f(acc);
        }
        hist[0][i] = hist[1][i];
        hist[1][i] = hist[2][i];
        hist[2][i] = xt[i];
      }
      if (blk < 2) {
        float ss = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) ss = fmaf(yt[i], yt[i], ss);
#pragma unroll
        for (int off = G / 2; off >= 1; off >>= 1) ss += __shfl_xor_sync(group_mask, ss, off);
        const float r = rsqrtf(ss + a.eps);
#pragma unroll
        for (int i = 0; i < 8; ++i) yt[i] *= r;
      }
      store8(y + (t * H + h) * D + lane_in_group * 8, yt);
    };
    if (whole) {
      // whole tile inside one sequence: every load issued (or staged), then compute
      Raw8<T> raw[PRO_TPT];
#pragma unroll
      for (int j = 0; j < PRO_TPT; ++j) {
        if constexpr (kStage) raw[j].u = *slot(blk, 3 + j);
        else raw[j].load(x + (t0 + j) * HD + c0);
      }
#pragma unroll
      for (int j = 0; j < PRO_TPT; ++j) {
        float xt[8];
        raw[j].get(xt);
        emit(t0 + j, xt);
      }
    } else {
      // tile crosses a sequence boundary or the end: token by token
#pragma unroll 1
      for (int64_t t = t0; t < t1; ++t) {
        if (t >= e) {
          while (n + 1 < a.N && t >= e) { ++n; seq_bounds(a.cu, n, a.seq_len, total, s, e); }
          load_history(t);
        }
        float xt[8];
        load8(x + t * HD + c0, xt);
        emit(t, xt);
      }
    }
    stage_phase(blk + 2);   // into the slots this phase has finished with
  }

  // gate and beta
  const float negA = -expf(a.A_log[h]);
  float bias[8];
  load8(a.dt_bias + h * D + lane_in_group * 8, bias);
  const T *__restrict__ alpha = reinterpret_cast<const T *>(a.alpha);
  Raw8<T> araw[PRO_TPT];
  if constexpr (kStage) cp_async_wait<0>();   // alpha's rows (zeros past the tile)
#pragma unroll
  for (int j = 0; j < PRO_TPT; ++j) {
    if constexpr (kStage) araw[j].u = *slot(3, 3 + j);
    else if (t0 + j < t1) araw[j].load(alpha + ((t0 + j) * H + h) * D + lane_in_group * 8);
    else araw[j].zero();
  }
#pragma unroll
  for (int j = 0; j < PRO_TPT; ++j) {
    const int64_t t = t0 + j;
    if (t >= t1) break;
    float al[8], gt[8];
    araw[j].get(al);
#pragma unroll
    for (int i = 0; i < 8; ++i) gt[i] = gate_f(al[i] + bias[i], negA, a.lower_bound);
    store8(a.g + (t * H + h) * D + lane_in_group * 8, gt);
  }
  if (has_b) a.beta[(t0 + lane_in_group) * H + h] = (a.beta2 ? 2.f : 1.f) * sigmoid_f(bme);
}

// final_conv_state[n][m][c] = raw input of token (end_n - 3 + m), or the
// incoming history / zero when the sequence is shorter than 3 tokens.
template <typename T>
__global__ void conv_state_out_kernel(PrologueArgs a, T *__restrict__ out) {
  const int64_t HD = (int64_t)a.H * a.D;
  const int64_t per_seq = 3 * 3 * HD;
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= per_seq * a.N) return;
  const int n = (int)(idx / per_seq);
  const int m = (int)((idx / (3 * HD)) % 3);
  const int64_t c = idx % (3 * HD);
  int64_t s, e;
  seq_bounds(a.cu, n, a.seq_len, a.total_tokens, s, e);
  const int64_t t = e - 3 + m;
  T val;
  if (t >= s) {
    const int blk = (int)(c / HD);
    const T *x = reinterpret_cast<const T *>(blk == 0 ? a.q : (blk == 1 ? a.k : a.v));
    val = x[t * HD + (c % HD)];
  } else if (a.conv0 != nullptr) {
    val = reinterpret_cast<const T *>(a.conv0)[((int64_t)n * 3 + (t - s + 3)) * 3 * HD + c];
  } else {
    val = from_f32<T>(0.f);
  }
  out[idx] = val;
}

cudaError_t launch_prologue(const PrologueArgs &a, cudaStream_t stream) {
  if (a.total_tokens == 0) return cudaSuccess;
  const int64_t tiles = (a.total_tokens + PRO_TPT - 1) / PRO_TPT;
  const int G = a.D / 8;
  const int64_t threads = tiles * a.H * G;
  const int64_t blocks = (threads + PRO_THREADS - 1) / PRO_THREADS;
  if (a.io_dtype == KDA_BF16) {
    auto kern = a.D == 128 ? prologue_kernel<__nv_bfloat16, 128> : prologue_kernel<__nv_bfloat16, 64>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)PRO_STAGE_BYTES);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)blocks, PRO_THREADS, PRO_STAGE_BYTES, stream>>>(a);
  } else {
    if (a.D == 128) prologue_kernel<float, 128><<<(unsigned)blocks, PRO_THREADS, 0, stream>>>(a);
    else prologue_kernel<float, 64><<<(unsigned)blocks, PRO_THREADS, 0, stream>>>(a);
  }
  return cudaGetLastError();
}

cudaError_t launch_conv_state_out(const PrologueArgs &a, void *out, cudaStream_t stream) {
  const int64_t n = (int64_t)a.N * 9 * a.H * a.D;
  if (n == 0) return cudaSuccess;
  const int threads = 256;
  const unsigned blocks = (unsigned)((n + threads - 1) / threads);
  if (a.io_dtype == KDA_BF16)
    conv_state_out_kernel<__nv_bfloat16><<<blocks, threads, 0, stream>>>(a, (__nv_bfloat16 *)out);
  else
    conv_state_out_kernel<float><<<blocks, threads, 0, stream>>>(a, (float *)out);
  return cudaGetLastError();
}

}  // namespace kda
