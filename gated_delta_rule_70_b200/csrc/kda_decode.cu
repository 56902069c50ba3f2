// KDA decode step: one new token per sequence, fused prologue + in-place state
// update.
//
// The operation is one iteration of the per-token loop of the AliceAI-Foundation
// KDA write-up ("二、KDA 线性注意力"), on the state a prefill left behind (section
// "五": prefill and decode share initial_state / final_state) with the conv
// history advanced by one token (section "四": 3 conv states per channel).
//
// HBM-bound by construction: each state element is read once, decayed, reduced,
// corrected and written back once; o = S'^T q + (q.k) d lets one barrier carry
// all column reductions.  Three kernels:
//   - dec::decode_tma_kernel (bf16, head_dim 128, heads a multiple of 8): one
//     persistent CTA per SM, a producer warp streaming (sequence, head) items
//     through a 3-slot shared-memory ring by bulk copy;
//   - dec::decode_tma_multi_kernel: the same for several tokens per call (or the
//     per-token states), two slots that hold every token's inputs;
//   - decode_kernel (every other shape): one CTA per (sequence, head), which
//     issues all loads of its state slice before the token's prologue so the
//     prologue's latency hides under the state stream.
#include "kda_common.cuh"
#include "kda_internal.h"
#include "umma.cuh"

namespace kda {

template <int D>
struct DecSmem {
  float q[D], k[D], eg[D], v[D];
  float gate[D];   // output gate (epilogue only)
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

  // 2-4, once per token (a.ntok tokens of this sequence, in order; the state stays in
  // registers and the conv history shifts in place between them)
  const T *__restrict__ cw = reinterpret_cast<const T *>(a.conv_w);
  T *__restrict__ cs = reinterpret_cast<T *>(a.conv_state) + (int64_t)n * 3 * 3 * HD;
  const int i = threadIdx.x % D;
  const bool first = threadIdx.x < D;
  const int ntok = a.ntok > 0 ? a.ntok : 1;
#pragma unroll 1
  for (int tt = 0; tt < ntok; ++tt) {
    const int64_t row = (int64_t)n * ntok + tt;   // token row in the [N, ntok, ...] inputs
    // 2. prologue for this token and head.  Threads [0, D): q and k channel i;
    //    threads [D, 2D): v channel i and the gate of key channel i.
    auto conv_channel = [&](int blk, const T *x) -> float {
      const int64_t c = (int64_t)blk * HD + h * D + i;
      const float x0 = to_f32(cs[0 * 3 * HD + c]), x1 = to_f32(cs[1 * 3 * HD + c]);
      const float x2 = to_f32(cs[2 * 3 * HD + c]);
      const T xn = x[row * HD + h * D + i];
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
      const float al = to_f32(reinterpret_cast<const T *>(a.alpha)[(row * H + h) * D + i]);
      const float g = gate_f(al + a.dt_bias[h * D + i], -expf(a.A_log[h]), a.lower_bound);
      sm.eg[i] = expf(g);
      if (i == 0) sm.beta = (a.beta2 ? 2.f : 1.f) * sigmoid_f(to_f32(reinterpret_cast<const T *>(a.b)[row * H + h]));
      if (a.ogate) sm.gate[i] = to_f32(reinterpret_cast<const T *>(a.ogate)[(row * H + h) * D + i]);
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
      T *o = reinterpret_cast<T *>(a.o) + (row * H + h) * D + CPL * l;
      float ov[CPL];
#pragma unroll
      for (int c = 0; c < CPL; ++c) ov[c] = a.scale * fmaf(QK, dl[c], R[c]);
      if (a.ogate) {   // output epilogue: o_norm over the row, then the sigmoid gate
        float ss = 0.f;
#pragma unroll
        for (int c = 0; c < CPL; ++c) ss = fmaf(ov[c], ov[c], ss);
#pragma unroll
        for (int sh = 16; sh >= 1; sh >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, sh);
        const float rn = rsqrtf(ss * (1.f / D) + a.oeps);
#pragma unroll
        for (int c = 0; c < CPL; ++c) ov[c] = ov[c] * rn * a.onw[CPL * l + c] * sigmoid_f(sm.gate[CPL * l + c]);
      }
#pragma unroll
      for (int c = 0; c < CPL; ++c) o[c] = from_f32<T>(ov[c]);
    }

    // 4. S = S' + k d^T (in registers); the state after this token when asked for
#pragma unroll
    for (int r = 0; r < 16; ++r) {
      const float kk = sm.k[16 * w + r];
#pragma unroll
      for (int c = 0; c < CPL; ++c) S[r][c] = fmaf(kk, dl[c], S[r][c]);
    }
    if (a.step_states != nullptr) {
      float *dst = a.step_states + (row * H + h) * D * D;
#pragma unroll
      for (int r = 0; r < 16; ++r)
#pragma unroll
        for (int c = 0; c < CPL; ++c) __stcs(dst + (int64_t)(16 * w + r) * D + CPL * l + c, S[r][c]);
    }
    __syncthreads();   // every read of this token's shared values is done
  }

  // 5. write the state back in place
#pragma unroll
  for (int r = 0; r < 16; ++r) {
    float *dst = Sg + (int64_t)(16 * w + r) * D + CPL * l;
    if constexpr (CPL == 4) {
      __stcs(reinterpret_cast<float4 *>(dst), make_float4(S[r][0], S[r][1], S[r][2], S[r][3]));
    } else {
      __stcs(reinterpret_cast<float2 *>(dst), make_float2(S[r][0], S[r][1]));
    }
  }
}

cudaError_t launch_decode_simt(const DecodeArgs &a, cudaStream_t stream);

// ---------------------------------------------------------------------------
// bf16, head_dim 128, H % 8 == 0: persistent and pipelined.  One CTA per SM walks
// the (sequence, head) items.  A producer warp brings each item's 64 KB state and
// its token's inputs (q, k, v, the 3-token conv history, alpha, the sequence's
// row of b, the head's conv weights and dt_bias) by bulk copy two items ahead
// into a 3-slot ring, and sends the updated state back by an asynchronous bulk
// store; eight compute warps run the prologue and the state update in shared
// memory.  Under a saturated HBM the bulk-copy issue itself stalls for about as
// long as an item's arithmetic, so it lives in its own warp.
namespace dec {

constexpr int NC = 256;                             // compute threads (warps 0-7)
constexpr int NT = NC + 32;                         // + the producer warp (warp 8)
constexpr int D = 128;
constexpr uint32_t S_STATE = 0;                     // fp32 [128][128]
constexpr uint32_t S_QKV = 65536;                   // bf16 q, k, v of the token: 3 x 256 B
constexpr uint32_t S_HIST = S_QKV + 768;            // bf16 conv history [slot m][tensor]: 9 x 256 B
constexpr uint32_t S_ALPHA = S_HIST + 2304;         // bf16 [128]
constexpr uint32_t S_W = S_ALPHA + 256;             // bf16 conv weights [tensor][128][4]: 3 x 1 KB
constexpr uint32_t S_DTB = S_W + 3072;              // fp32 dt_bias [128]
constexpr uint32_t S_B = S_DTB + 512;               // bf16 b of the token's sequence row [H <= 64]
constexpr uint32_t S_GATE = S_B + 128;              // bf16 output gate [128] (epilogue only)
constexpr uint32_t SLOT = S_GATE + 256;             // 72,832 B per item
constexpr int NSLOT = 3;
constexpr uint32_t OFF_SCR = NSLOT * SLOT;
template <int NS>
struct ScratchT {
  float q[D], k[D], eg[D], v[D];
  float red_p[NC / 32][D], red_r[NC / 32][D], red_qk[NC / 32];
  float norm_part[2][4];
  float alog[64];
  float onw[D];     // output epilogue weight
  float beta;
  int fail;
  int req[NS];      // requests issued per slot (for the error path)
  uint64_t full[NS], empty[NS];
};
using Scratch = ScratchT<NSLOT>;
constexpr uint32_t SMEM_BYTES = OFF_SCR + sizeof(Scratch);
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
static_assert(SLOT % 16 == 0 && S_QKV % 16 == 0 && S_HIST % 16 == 0 && S_W % 16 == 0 && S_DTB % 16 == 0 &&
              S_B % 16 == 0 && S_GATE % 16 == 0, "bulk copy alignment");
constexpr uint32_t BAR_COMPUTE = 1;                 // named barrier of the compute warps

__global__ void __launch_bounds__(NT, 1) decode_tma_kernel(DecodeArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  Scratch &sc = *reinterpret_cast<Scratch *>(smem + OFF_SCR);
  const int tid = threadIdx.x, w = tid >> 5, l = tid & 31;
  const int H = a.H;
  const int64_t HD = (int64_t)H * D;
  const int items = a.N * H;
  const int G = gridDim.x;
  const __nv_bfloat16 *cw = reinterpret_cast<const __nv_bfloat16 *>(a.conv_w);
  __nv_bfloat16 *cs = reinterpret_cast<__nv_bfloat16 *>(a.conv_state);

  if (tid == 0) {
    for (int i = 0; i < NSLOT; ++i) {
      umma::mbar_init(&sc.full[i], 1);
      umma::mbar_init(&sc.empty[i], NC);
      sc.req[i] = 0;
    }
    umma::mbar_fence_init();
    sc.fail = 0;
  }
  // A_log of every head, once: a plain load inside the loop would queue behind
  // the bulk traffic for about one item's time
  if (tid < H) sc.alog[tid] = a.A_log[tid];
  const bool gated = a.ogate != nullptr;
  if (gated && tid < D) sc.onw[tid] = a.onw[tid];
  __syncthreads();

  if (w == NC / 32) {
    // ---------------- producer warp
    // everything item `it` reads, into ring slot `slot` (lanes 0-18: one copy each)
    auto request = [&](int it, int slot) {
      const int n = it / H, h = it % H;
      uint8_t *base = smem + slot * SLOT;
      uint64_t *bar = &sc.full[slot];
      if (l == 0) {
        umma::mbar_arrive_expect_tx(bar, S_B + 2 * H + (gated ? 2 * D : 0));
        ++sc.req[slot];
      }
      __syncwarp();
      if (l == 0) {
        umma::bulk_g2s(base + S_STATE, a.state + (int64_t)it * D * D, D * D * 4, bar);
      } else if (l < 4) {
        const void *tok = l == 1 ? a.q : (l == 2 ? a.k : a.v);
        umma::bulk_g2s(base + S_QKV + (l - 1) * 256,
                       reinterpret_cast<const __nv_bfloat16 *>(tok) + (int64_t)n * HD + h * D, 256, bar);
      } else if (l < 13) {
        const int m = (l - 4) / 3, blk = (l - 4) % 3;
        umma::bulk_g2s(base + S_HIST + (m * 3 + blk) * 256,
                       cs + ((int64_t)n * 3 + m) * 3 * HD + blk * HD + h * D, 256, bar);
      } else if (l == 13) {
        umma::bulk_g2s(base + S_ALPHA, reinterpret_cast<const __nv_bfloat16 *>(a.alpha) + (int64_t)it * D, 256, bar);
      } else if (l < 17) {
        const int blk = l - 14;
        umma::bulk_g2s(base + S_W + blk * 1024, cw + ((int64_t)blk * HD + h * D) * KCONV, 1024, bar);
      } else if (l == 17) {
        umma::bulk_g2s(base + S_DTB, a.dt_bias + h * D, 512, bar);
      } else if (l == 18) {   // the row of b for sequence n (2H bytes, 16-byte aligned for H % 8 == 0)
        umma::bulk_g2s(base + S_B, reinterpret_cast<const __nv_bfloat16 *>(a.b) + (int64_t)n * H, 2 * H, bar);
      } else if (l == 19 && gated) {
        umma::bulk_g2s(base + S_GATE, reinterpret_cast<const __nv_bfloat16 *>(a.ogate) + (int64_t)it * D,
                       2 * D, bar);
      }
      __syncwarp();
    };
    int it = blockIdx.x;
    if (it < items) request(it, 0);
    if (it + G < items) request(it + G, 1);
#pragma unroll 1
    for (int j = 0; it < items; ++j, it += G) {
      const int slot = j % NSLOT;
      // item j's state is final in its slot: store it
      int ok = l == 0 ? (int)umma::mbar_wait_bounded(&sc.empty[slot], (j / NSLOT) & 1, a.wait_polls) : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) { sc.fail = 1; break; }
      if (l == 0) {
        umma::bulk_s2g(a.state + (int64_t)it * D * D, smem + slot * SLOT + S_STATE, D * D * 4);
        umma::bulk_commit();
      }
      // two items ahead, into the slot item j-1 used: only its store (not item j's)
      // must have finished reading shared memory
      if (it + 2 * G < items) {
        if (l == 0) umma::bulk_wait_read<1>();
        __syncwarp();
        request(it + 2 * G, (j + 2) % NSLOT);
      }
      if (*(volatile int *)&sc.fail) break;
    }
    // the stores read shared memory until they finish: wait before the CTA can leave
    if (l == 0) umma::bulk_wait<0>();
    if (*(volatile int *)&sc.fail) {
      // copies requested into a slot may still be landing: wait (bounded) for each slot's last
      if (l < NSLOT && sc.req[l] > 0) (void)umma::mbar_wait_bounded(&sc.full[l], (sc.req[l] - 1) & 1, kWaitPolls);
    }
  } else {
    // ---------------- compute warps
    const bool first = tid < D;
    const int i = tid % D;   // q/k channel (first half) or v / gate channel (second half)
#pragma unroll 1
    for (int k = 0, it = blockIdx.x; it < items; ++k, it += G) {
      const int slot = k % NSLOT;
      const int n = it / H, h = it % H;
      uint8_t *base = smem + slot * SLOT;
      float *S_s = reinterpret_cast<float *>(base + S_STATE);
      // all compute threads agree to go on: the slot has landed and nobody failed.
      // The barrier also closes every read of the previous item's scratch values.
      const bool landed = umma::mbar_wait_bounded(&sc.full[slot], (k / NSLOT) & 1, a.wait_polls);
      if (!umma::named_sync_and(BAR_COMPUTE, NC, landed && !*(volatile int *)&sc.fail)) {
        if (tid == 0) sc.fail = 1;
        break;
      }

      // 1. prologue of this token: conv4 + SiLU per channel; the history shifts by one
      const __nv_bfloat16 *qkv = reinterpret_cast<const __nv_bfloat16 *>(base + S_QKV);
      const __nv_bfloat16 *hist = reinterpret_cast<const __nv_bfloat16 *>(base + S_HIST);
      const __nv_bfloat16 *wts = reinterpret_cast<const __nv_bfloat16 *>(base + S_W);
      auto conv_channel = [&](int blk) -> float {
        const __nv_bfloat16 *wc = wts + (blk * D + i) * KCONV;
        const __nv_bfloat16 h0 = hist[(0 * 3 + blk) * D + i], h1 = hist[(1 * 3 + blk) * D + i];
        const __nv_bfloat16 h2 = hist[(2 * 3 + blk) * D + i], xn = qkv[blk * D + i];
        float acc = __bfloat162float(wc[0]) * __bfloat162float(h0);
        acc = fmaf(__bfloat162float(wc[1]), __bfloat162float(h1), acc);
        acc = fmaf(__bfloat162float(wc[2]), __bfloat162float(h2), acc);
        acc = fmaf(__bfloat162float(wc[3]), __bfloat162float(xn), acc);
        __nv_bfloat16 *c = cs + (int64_t)n * 3 * 3 * HD + blk * HD + h * D + i;   // slot m at + m * 3 * HD
        c[0] = h1;
        c[3 * HD] = h2;
        c[6 * HD] = xn;
        return silu_f(acc);
      };
      float qv = 0.f, kv = 0.f;
      if (first) {
        qv = conv_channel(0);
        kv = conv_channel(1);
        float sq = qv * qv, sk = kv * kv;
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) {
          sq += __shfl_xor_sync(0xffffffffu, sq, off);
          sk += __shfl_xor_sync(0xffffffffu, sk, off);
        }
        if (l == 0) { sc.norm_part[0][w] = sq; sc.norm_part[1][w] = sk; }
      } else {
        sc.v[i] = conv_channel(2);
        const float al = __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(base + S_ALPHA)[i]);
        const float g = gate_f(al + reinterpret_cast<const float *>(base + S_DTB)[i], -expf(sc.alog[h]),
                               a.lower_bound);
        sc.eg[i] = expf(g);
        if (i == 0)
          sc.beta = (a.beta2 ? 2.f : 1.f) *
                    sigmoid_f(__bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(base + S_B)[h]));
      }
      umma::named_sync(BAR_COMPUTE, NC);
      if (first) {
        const float sq = sc.norm_part[0][0] + sc.norm_part[0][1] + sc.norm_part[0][2] + sc.norm_part[0][3];
        const float sk = sc.norm_part[1][0] + sc.norm_part[1][1] + sc.norm_part[1][2] + sc.norm_part[1][3];
        sc.q[i] = qv * rsqrtf(sq + a.eps);
        sc.k[i] = kv * rsqrtf(sk + a.eps);
      }
      umma::named_sync(BAR_COMPUTE, NC);

      // 2. decay, then the column reductions p = S'^T k and r = S'^T q
      //    (warp w: rows 16w..16w+15; lane l: columns 4l..4l+3)
      float S[16][4];
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        const float4 x = *reinterpret_cast<const float4 *>(S_s + (16 * w + r) * D + 4 * l);
        S[r][0] = x.x; S[r][1] = x.y; S[r][2] = x.z; S[r][3] = x.w;
      }
      float p[4] = {0.f, 0.f, 0.f, 0.f}, rr[4] = {0.f, 0.f, 0.f, 0.f}, qk = 0.f;
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        const int ii = 16 * w + r;
        const float e = sc.eg[ii], kk = sc.k[ii], qq = sc.q[ii];
        qk = fmaf(qq, kk, qk);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          S[r][c] *= e;
          p[c] = fmaf(kk, S[r][c], p[c]);
          rr[c] = fmaf(qq, S[r][c], rr[c]);
        }
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) { sc.red_p[w][4 * l + c] = p[c]; sc.red_r[w][4 * l + c] = rr[c]; }
      if (l == 0) sc.red_qk[w] = qk;
      umma::named_sync(BAR_COMPUTE, NC);
      float P[4] = {0.f, 0.f, 0.f, 0.f}, R[4] = {0.f, 0.f, 0.f, 0.f}, QK = 0.f;
#pragma unroll
      for (int ww = 0; ww < NC / 32; ++ww) {
        QK += sc.red_qk[ww];
#pragma unroll
        for (int c = 0; c < 4; ++c) { P[c] += sc.red_p[ww][4 * l + c]; R[c] += sc.red_r[ww][4 * l + c]; }
      }
      const float bt = sc.beta;
      float dl[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) dl[c] = bt * (sc.v[4 * l + c] - P[c]);
      if (w == 0) {
        __nv_bfloat16 *o = reinterpret_cast<__nv_bfloat16 *>(a.o) + (int64_t)it * D + 4 * l;
        float ov[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) ov[c] = a.scale * fmaf(QK, dl[c], R[c]);
        if (gated) {   // output epilogue: o_norm over the row, then the sigmoid gate
          float ss = 0.f;
#pragma unroll
          for (int c = 0; c < 4; ++c) ss = fmaf(ov[c], ov[c], ss);
#pragma unroll
          for (int sh = 16; sh >= 1; sh >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, sh);
          const float rn = rsqrtf(ss * (1.f / D) + a.oeps);
          const __nv_bfloat16 *gr = reinterpret_cast<const __nv_bfloat16 *>(base + S_GATE) + 4 * l;
#pragma unroll
          for (int c = 0; c < 4; ++c)
            ov[c] = ov[c] * rn * sc.onw[4 * l + c] * sigmoid_f(__bfloat162float(gr[c]));
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) o[c] = __float2bfloat16_rn(ov[c]);
      }
      // 3. S = S' + k d^T, back into the slot; the producer stores it
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        const float kk = sc.k[16 * w + r];
        *reinterpret_cast<float4 *>(S_s + (16 * w + r) * D + 4 * l) =
            make_float4(fmaf(kk, dl[0], S[r][0]), fmaf(kk, dl[1], S[r][1]), fmaf(kk, dl[2], S[r][2]),
                        fmaf(kk, dl[3], S[r][3]));
      }
      umma::fence_proxy_async_smem();
      umma::mbar_arrive(&sc.empty[slot]);
    }
  }
  __syncthreads();
  if (tid == 0 && *(volatile int *)&sc.fail && a.err) atomicOr(a.err, ERR_TIMEOUT_DECODE);
}

// ---------------------------------------------------------------------------
// Multi-token variant (2 to MT_MAX tokens per sequence in one call, optionally the
// state after each token): the same producer / compute split, with two ring slots
// that hold the state and every token's inputs.  The conv history and the call's
// tokens sit in one raw-row array per tensor (rows 0-2 the history, row 3 + t token
// t), so token t's conv reads rows t .. t+3 and the new history is rows T .. T+2.
// The state stays in registers across the tokens; the per-token states leave from
// registers as 16-byte row stores.
constexpr int MT_MAX = 16;
constexpr uint32_t M_STATE = 0;                            // fp32 [128][128]
constexpr uint32_t M_RAWT = (3 + MT_MAX) * 256;            // bf16 raw rows of one tensor: [3 + MT_MAX][128]
constexpr uint32_t M_RAW = 65536;                          // [tensor][row][128]
constexpr uint32_t M_ALPHA = M_RAW + 3 * M_RAWT;           // bf16 [MT_MAX][128]
constexpr uint32_t M_W = M_ALPHA + MT_MAX * 256;           // bf16 conv weights [tensor][128][4]
constexpr uint32_t M_DTB = M_W + 3072;                     // fp32 dt_bias [128]
constexpr uint32_t M_B = M_DTB + 512;                      // bf16 b of the sequence's rows [MT_MAX][H <= 64]
constexpr uint32_t M_GATE = M_B + MT_MAX * 128;            // bf16 output gate [MT_MAX][128]
constexpr uint32_t M_SLOT = M_GATE + MT_MAX * 256;         // 93,952 B per item
constexpr int M_NSLOT = 2;
constexpr uint32_t M_OFF_SCR = M_NSLOT * M_SLOT;
using MScratch = ScratchT<M_NSLOT>;
constexpr uint32_t M_SMEM_BYTES = M_OFF_SCR + sizeof(MScratch);
static_assert(M_SMEM_BYTES <= 232448, "shared memory budget");
static_assert(M_SLOT % 16 == 0 && M_RAW % 16 == 0 && M_RAWT % 16 == 0 && M_ALPHA % 16 == 0 && M_W % 16 == 0 &&
              M_DTB % 16 == 0 && M_B % 16 == 0 && M_GATE % 16 == 0 && M_OFF_SCR % 16 == 0, "bulk copy alignment");

__global__ void __launch_bounds__(NT, 1) decode_tma_multi_kernel(DecodeArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  MScratch &sc = *reinterpret_cast<MScratch *>(smem + M_OFF_SCR);
  const int tid = threadIdx.x, w = tid >> 5, l = tid & 31;
  const int H = a.H, T = a.ntok;
  const int64_t HD = (int64_t)H * D;
  const int items = a.N * H;
  const int G = gridDim.x;
  const __nv_bfloat16 *cw = reinterpret_cast<const __nv_bfloat16 *>(a.conv_w);
  __nv_bfloat16 *cs = reinterpret_cast<__nv_bfloat16 *>(a.conv_state);

  if (tid == 0) {
    for (int i = 0; i < M_NSLOT; ++i) {
      umma::mbar_init(&sc.full[i], 1);
      umma::mbar_init(&sc.empty[i], NC);
      sc.req[i] = 0;
    }
    umma::mbar_fence_init();
    sc.fail = 0;
  }
  if (tid < H) sc.alog[tid] = a.A_log[tid];
  const bool gated = a.ogate != nullptr;
  if (gated && tid < D) sc.onw[tid] = a.onw[tid];
  __syncthreads();

  if (w == NC / 32) {
    // ---------------- producer warp: everything item `it` reads, into ring slot `slot`
    const int ncopy = 1 + 9 + 3 * T + T + 3 + 1 + 1 + (gated ? T : 0);
    const uint32_t bytes = D * D * 4 + 9 * 256 + 4 * T * 256 + 3072 + 512 + 2 * T * H + (gated ? T * 256 : 0);
    auto request = [&](int it, int slot) {
      const int n = it / H, h = it % H;
      uint8_t *base = smem + slot * M_SLOT;
      uint64_t *bar = &sc.full[slot];
      if (l == 0) {
        umma::mbar_arrive_expect_tx(bar, bytes);
        ++sc.req[slot];
      }
      __syncwarp();
      for (int c = l; c < ncopy; c += 32) {
        int k = c;
        if (k == 0) {
          umma::bulk_g2s(base + M_STATE, a.state + (int64_t)it * D * D, D * D * 4, bar);
        } else if ((k -= 1) < 9) {   // conv history: slot m of tensor blk into raw row m
          const int m = k / 3, blk = k % 3;
          umma::bulk_g2s(base + M_RAW + blk * M_RAWT + m * 256, cs + ((int64_t)n * 3 + m) * 3 * HD + blk * HD + h * D,
                         256, bar);
        } else if ((k -= 9) < 3 * T) {   // token t of tensor blk into raw row 3 + t
          const int blk = k / T, t = k % T;
          const void *tok = blk == 0 ? a.q : (blk == 1 ? a.k : a.v);
          umma::bulk_g2s(base + M_RAW + blk * M_RAWT + (3 + t) * 256,
                         reinterpret_cast<const __nv_bfloat16 *>(tok) + ((int64_t)n * T + t) * HD + h * D, 256, bar);
        } else if ((k -= 3 * T) < T) {
          umma::bulk_g2s(base + M_ALPHA + k * 256,
                         reinterpret_cast<const __nv_bfloat16 *>(a.alpha) + (((int64_t)n * T + k) * H + h) * D, 256, bar);
        } else if ((k -= T) < 3) {
          umma::bulk_g2s(base + M_W + k * 1024, cw + ((int64_t)k * HD + h * D) * KCONV, 1024, bar);
        } else if ((k -= 3) == 0) {
          umma::bulk_g2s(base + M_DTB, a.dt_bias + h * D, 512, bar);
        } else if (k == 1) {   // the T rows of b of sequence n (16-byte aligned for H % 8 == 0)
          umma::bulk_g2s(base + M_B, reinterpret_cast<const __nv_bfloat16 *>(a.b) + (int64_t)n * T * H, 2 * T * H, bar);
        } else {
          const int t = k - 2;
          umma::bulk_g2s(base + M_GATE + t * 256,
                         reinterpret_cast<const __nv_bfloat16 *>(a.ogate) + (((int64_t)n * T + t) * H + h) * D, 256, bar);
        }
      }
      __syncwarp();
    };
    int it = blockIdx.x;
    if (it < items) request(it, 0);
    if (it + G < items) request(it + G, 1);
#pragma unroll 1
    for (int j = 0; it < items; ++j, it += G) {
      const int slot = j & 1;
      // item j's final state is in its slot: store it
      int ok = l == 0 ? (int)umma::mbar_wait_bounded(&sc.empty[slot], (j >> 1) & 1, a.wait_polls) : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) { sc.fail = 1; break; }
      if (l == 0) {
        umma::bulk_s2g(a.state + (int64_t)it * D * D, smem + slot * M_SLOT + M_STATE, D * D * 4);
        if (a.step_states != nullptr) {   // the state after the last token is the final state
          const int n = it / H, h = it % H;
          umma::bulk_s2g(a.step_states + (((int64_t)n * T + T - 1) * H + h) * D * D,
                         smem + slot * M_SLOT + M_STATE, D * D * 4);
        }
        umma::bulk_commit();
      }
      // two items ahead, into this same slot once the store has read it
      if (it + 2 * G < items) {
        if (l == 0) umma::bulk_wait_read<0>();
        __syncwarp();
        request(it + 2 * G, slot);
      }
      if (*(volatile int *)&sc.fail) break;
    }
    if (l == 0) umma::bulk_wait<0>();
    if (*(volatile int *)&sc.fail) {
      if (l < M_NSLOT && sc.req[l] > 0) (void)umma::mbar_wait_bounded(&sc.full[l], (sc.req[l] - 1) & 1, kWaitPolls);
    }
  } else {
    // ---------------- compute warps
    const bool first = tid < D;
    const int i = tid % D;   // q/k channel (first half) or v / gate channel (second half)
#pragma unroll 1
    for (int kk = 0, it = blockIdx.x; it < items; ++kk, it += G) {
      const int slot = kk & 1;
      const int n = it / H, h = it % H;
      uint8_t *base = smem + slot * M_SLOT;
      float *S_s = reinterpret_cast<float *>(base + M_STATE);
      const bool landed = umma::mbar_wait_bounded(&sc.full[slot], (kk >> 1) & 1, a.wait_polls);
      if (!umma::named_sync_and(BAR_COMPUTE, NC, landed && !*(volatile int *)&sc.fail)) {
        if (tid == 0) sc.fail = 1;
        break;
      }
      // the state, rows 16w..16w+15, columns 4l..4l+3, into registers for all T tokens
      float S[16][4];
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        const float4 x = *reinterpret_cast<const float4 *>(S_s + (16 * w + r) * D + 4 * l);
        S[r][0] = x.x; S[r][1] = x.y; S[r][2] = x.z; S[r][3] = x.w;
      }
      const __nv_bfloat16 *raw = reinterpret_cast<const __nv_bfloat16 *>(base + M_RAW);
      const __nv_bfloat16 *wts = reinterpret_cast<const __nv_bfloat16 *>(base + M_W);
#pragma unroll 1
      for (int t = 0; t < T; ++t) {
        const int64_t row = (int64_t)n * T + t;   // token row in the [N, T, ...] inputs
        // 1. prologue of token t: conv4 + SiLU over raw rows t .. t+3 of the channel
        auto conv_channel = [&](int blk) -> float {
          const __nv_bfloat16 *wc = wts + (blk * D + i) * KCONV;
          const __nv_bfloat16 *x = raw + (blk * (3 + MT_MAX) + t) * D + i;
          float acc = __bfloat162float(wc[0]) * __bfloat162float(x[0]);
          acc = fmaf(__bfloat162float(wc[1]), __bfloat162float(x[D]), acc);
          acc = fmaf(__bfloat162float(wc[2]), __bfloat162float(x[2 * D]), acc);
          acc = fmaf(__bfloat162float(wc[3]), __bfloat162float(x[3 * D]), acc);
          return silu_f(acc);
        };
        float qv = 0.f, kv = 0.f;
        if (first) {
          qv = conv_channel(0);
          kv = conv_channel(1);
          float sq = qv * qv, sk = kv * kv;
#pragma unroll
          for (int off = 16; off >= 1; off >>= 1) {
            sq += __shfl_xor_sync(0xffffffffu, sq, off);
            sk += __shfl_xor_sync(0xffffffffu, sk, off);
          }
          if (l == 0) { sc.norm_part[0][w] = sq; sc.norm_part[1][w] = sk; }
        } else {
          sc.v[i] = conv_channel(2);
          const float al = __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(base + M_ALPHA)[t * D + i]);
          const float g = gate_f(al + reinterpret_cast<const float *>(base + M_DTB)[i], -expf(sc.alog[h]),
                                 a.lower_bound);
          sc.eg[i] = expf(g);
          if (i == 0)
            sc.beta = (a.beta2 ? 2.f : 1.f) *
                      sigmoid_f(__bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(base + M_B)[t * H + h]));
        }
        umma::named_sync(BAR_COMPUTE, NC);
        if (first) {
          const float sq = sc.norm_part[0][0] + sc.norm_part[0][1] + sc.norm_part[0][2] + sc.norm_part[0][3];
          const float sk = sc.norm_part[1][0] + sc.norm_part[1][1] + sc.norm_part[1][2] + sc.norm_part[1][3];
          sc.q[i] = qv * rsqrtf(sq + a.eps);
          sc.k[i] = kv * rsqrtf(sk + a.eps);
        }
        umma::named_sync(BAR_COMPUTE, NC);

        // 2. decay, then the column reductions p = S'^T k and r = S'^T q
        float p[4] = {0.f, 0.f, 0.f, 0.f}, rr[4] = {0.f, 0.f, 0.f, 0.f}, qk = 0.f;
#pragma unroll
        for (int r = 0; r < 16; ++r) {
          const int ii = 16 * w + r;
          const float e = sc.eg[ii], k_ = sc.k[ii], q_ = sc.q[ii];
          qk = fmaf(q_, k_, qk);
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            S[r][c] *= e;
            p[c] = fmaf(k_, S[r][c], p[c]);
            rr[c] = fmaf(q_, S[r][c], rr[c]);
          }
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) { sc.red_p[w][4 * l + c] = p[c]; sc.red_r[w][4 * l + c] = rr[c]; }
        if (l == 0) sc.red_qk[w] = qk;
        umma::named_sync(BAR_COMPUTE, NC);
        float P[4] = {0.f, 0.f, 0.f, 0.f}, R[4] = {0.f, 0.f, 0.f, 0.f}, QK = 0.f;
#pragma unroll
        for (int ww = 0; ww < NC / 32; ++ww) {
          QK += sc.red_qk[ww];
#pragma unroll
          for (int c = 0; c < 4; ++c) { P[c] += sc.red_p[ww][4 * l + c]; R[c] += sc.red_r[ww][4 * l + c]; }
        }
        const float bt = sc.beta;
        float dl[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) dl[c] = bt * (sc.v[4 * l + c] - P[c]);
        if (w == 0) {
          __nv_bfloat16 *o = reinterpret_cast<__nv_bfloat16 *>(a.o) + (row * H + h) * D + 4 * l;
          float ov[4];
#pragma unroll
          for (int c = 0; c < 4; ++c) ov[c] = a.scale * fmaf(QK, dl[c], R[c]);
          if (gated) {   // output epilogue: o_norm over the row, then the sigmoid gate
            float ss = 0.f;
#pragma unroll
            for (int c = 0; c < 4; ++c) ss = fmaf(ov[c], ov[c], ss);
#pragma unroll
            for (int sh = 16; sh >= 1; sh >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, sh);
            const float rn = rsqrtf(ss * (1.f / D) + a.oeps);
            const __nv_bfloat16 *gr = reinterpret_cast<const __nv_bfloat16 *>(base + M_GATE) + t * D + 4 * l;
#pragma unroll
            for (int c = 0; c < 4; ++c)
              ov[c] = ov[c] * rn * sc.onw[4 * l + c] * sigmoid_f(__bfloat162float(gr[c]));
          }
#pragma unroll
          for (int c = 0; c < 4; ++c) o[c] = __float2bfloat16_rn(ov[c]);
        }
        // 3. S = S' + k d^T in registers; the state after this token when asked for
#pragma unroll
        for (int r = 0; r < 16; ++r) {
          const float k_ = sc.k[16 * w + r];
#pragma unroll
          for (int c = 0; c < 4; ++c) S[r][c] = fmaf(k_, dl[c], S[r][c]);
        }
        if (a.step_states != nullptr && t + 1 < T) {   // (the last one leaves with the slot)
          float *dst = a.step_states + (row * H + h) * D * D;
#pragma unroll
          for (int r = 0; r < 16; ++r)
            __stcs(reinterpret_cast<float4 *>(dst + (int64_t)(16 * w + r) * D + 4 * l),
                   make_float4(S[r][0], S[r][1], S[r][2], S[r][3]));
        }
        umma::named_sync(BAR_COMPUTE, NC);   // every read of this token's shared values is done
      }
      // 4. the conv history after the call: raw rows T .. T+2 (channel i of q, k / of v)
#pragma unroll
      for (int bb = 0; bb < 2; ++bb) {
        const int blk = first ? bb : 2;
        if (bb == 1 && !first) break;
#pragma unroll
        for (int m = 0; m < 3; ++m)
          cs[((int64_t)n * 3 + m) * 3 * HD + blk * HD + h * D + i] = raw[(blk * (3 + MT_MAX) + T + m) * D + i];
      }
      // 5. the final state back into the slot; the producer stores it
#pragma unroll
      for (int r = 0; r < 16; ++r)
        *reinterpret_cast<float4 *>(S_s + (16 * w + r) * D + 4 * l) = make_float4(S[r][0], S[r][1], S[r][2], S[r][3]);
      umma::fence_proxy_async_smem();
      umma::mbar_arrive(&sc.empty[slot]);
    }
  }
  __syncthreads();
  if (tid == 0 && *(volatile int *)&sc.fail && a.err) atomicOr(a.err, ERR_TIMEOUT_DECODE);
}

}  // namespace dec

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t stream) {
  if ((int64_t)a.N * a.H == 0) return cudaSuccess;
  if (a.io_dtype == KDA_BF16 && a.D == 128 && a.H % 8 == 0 && a.ntok <= 1 && a.step_states == nullptr) {
    cudaError_t e = cudaFuncSetAttribute(dec::decode_tma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)dec::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    const int items = a.N * a.H;
    dec::decode_tma_kernel<<<items < sms ? items : sms, dec::NT, dec::SMEM_BYTES, stream>>>(a);
    return cudaGetLastError();
  }
  if (a.io_dtype == KDA_BF16 && a.D == 128 && a.H % 8 == 0 && a.H <= 64 && a.ntok >= 1 &&
      a.ntok <= dec::MT_MAX) {   // several tokens, or the per-token states
    cudaError_t e = cudaFuncSetAttribute(dec::decode_tma_multi_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dec::M_SMEM_BYTES);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    const int items = a.N * a.H;
    dec::decode_tma_multi_kernel<<<items < sms ? items : sms, dec::NT, dec::M_SMEM_BYTES, stream>>>(a);
    return cudaGetLastError();
  }
  return launch_decode_simt(a, stream);
}

cudaError_t launch_decode_simt(const DecodeArgs &a, cudaStream_t stream) {
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
