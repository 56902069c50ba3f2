// KDA token recurrence on CUDA cores (fp32 arithmetic), one CTA per
// (sequence, head).  Used for the fp32 I/O test mode and head_dim 64, where
// the tensor-core chunk kernel (bf16 operands) does not apply.
//
// Per token, in the order of the AliceAI-Foundation KDA write-up's per-token
// loop ("二、KDA 线性注意力"): S <- diag(e^g) S; p = S^T k; d = beta (v - p);
// S <- S + k d^T; o = S^T q.  Using o = S'^T q + (q.k) d (S' the decayed
// state) every thread reads its slice of S once per token and all column
// reductions share one __syncthreads.
//
// Thread layout (D = 128: 8 warps): warp w owns key rows [16w, 16w + 16),
// lane l owns value columns [CPL*l, CPL*l + CPL) with CPL = D/32; the state
// slice lives in registers for the whole sequence.
//
// Optional output epilogue (the layer's o_norm and sigmoid output gate, same
// write-up sections "二" and "三"): warp 0 holds a token's whole o row, so
// o <- o / sqrt(mean o^2 + eps) * w * sigmoid(gate) takes one warp reduction;
// the gate rows are staged with the token tile.
#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {

constexpr int REC_TT = 32;  // tokens staged in shared memory per tile

template <int D>
struct RecSmem {
  float k[REC_TT][D], q[REC_TT][D], eg[REC_TT][D], v[REC_TT][D];
  float beta[REC_TT];
  float red_p[2][D / 16][D], red_r[2][D / 16][D], red_qk[2][D / 16];
  float gate[REC_TT][D];     // output gate of the tile (epilogue only)
};

template <typename T, int D>
__global__ void __launch_bounds__(2 * D)
recurrence_kernel(RecurrenceArgs a) {
  constexpr int W = D / 16, CPL = D / 32, NT = 2 * D;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  RecSmem<D> &sm = *reinterpret_cast<RecSmem<D> *>(smem_raw);
  const int n = blockIdx.x / a.H, h = blockIdx.x % a.H;
  const int w = threadIdx.x / 32, l = threadIdx.x % 32;
  const int H = a.H;
  int64_t s0, s1;
  seq_bounds(a.cu, n, a.seq_len, a.total_tokens, s0, s1);

  float S[16][CPL];
  const int64_t sbase = ((int64_t)n * H + h) * D * D;
#pragma unroll
  for (int r = 0; r < 16; ++r) {
    const int i = 16 * w + r;
#pragma unroll
    for (int c = 0; c < CPL; ++c)
      S[r][c] = a.state0 ? a.state0[sbase + (int64_t)i * D + CPL * l + c] : 0.f;
  }

  const T *__restrict__ qn = reinterpret_cast<const T *>(a.qn);
  const T *__restrict__ kn = reinterpret_cast<const T *>(a.kn);
  const T *__restrict__ vc = reinterpret_cast<const T *>(a.vc);
  T *__restrict__ o = reinterpret_cast<T *>(a.o);
  const T *__restrict__ og = reinterpret_cast<const T *>(a.ogate);
  float onw[CPL];   // epilogue weight of this lane's channels
#pragma unroll
  for (int c = 0; c < CPL; ++c) onw[c] = og ? a.onw[CPL * l + c] : 0.f;
  int buf = 0;

  for (int64_t tile0 = s0; tile0 < s1; tile0 += REC_TT) {
    const int nt = (int)min((int64_t)REC_TT, s1 - tile0);
    __syncthreads();  // previous tile fully consumed
    for (int idx = threadIdx.x; idx < nt * D; idx += NT) {
      const int tt = idx / D, i = idx % D;
      const int64_t off = ((tile0 + tt) * H + h) * D + i;
      sm.k[tt][i] = to_f32(kn[off]);
      sm.q[tt][i] = to_f32(qn[off]);
      sm.v[tt][i] = to_f32(vc[off]);
      sm.eg[tt][i] = expf(a.g[off]);
      if (og) sm.gate[tt][i] = to_f32(og[off]);
    }
    for (int tt = threadIdx.x; tt < nt; tt += NT) sm.beta[tt] = a.beta[(tile0 + tt) * H + h];
    __syncthreads();

    for (int tt = 0; tt < nt; ++tt) {
      float p[CPL], rr[CPL], qk = 0.f;
#pragma unroll
      for (int c = 0; c < CPL; ++c) { p[c] = 0.f; rr[c] = 0.f; }
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        const int i = 16 * w + r;
        const float e = sm.eg[tt][i], kk = sm.k[tt][i], qq = sm.q[tt][i];
        qk = fmaf(qq, kk, qk);
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
          S[r][c] *= e;
          p[c] = fmaf(kk, S[r][c], p[c]);
          rr[c] = fmaf(qq, S[r][c], rr[c]);
        }
      }
#pragma unroll
      for (int c = 0; c < CPL; ++c) {
        sm.red_p[buf][w][CPL * l + c] = p[c];
        sm.red_r[buf][w][CPL * l + c] = rr[c];
      }
      if (l == 0) sm.red_qk[buf][w] = qk;
      __syncthreads();
      float P[CPL], R[CPL], QK = 0.f;
#pragma unroll
      for (int c = 0; c < CPL; ++c) { P[c] = 0.f; R[c] = 0.f; }
#pragma unroll
      for (int ww = 0; ww < W; ++ww) {
        QK += sm.red_qk[buf][ww];
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
          P[c] += sm.red_p[buf][ww][CPL * l + c];
          R[c] += sm.red_r[buf][ww][CPL * l + c];
        }
      }
      const float bt = sm.beta[tt];
      float dl[CPL];
#pragma unroll
      for (int c = 0; c < CPL; ++c) dl[c] = bt * (sm.v[tt][CPL * l + c] - P[c]);
      if (w == 0) {
        const int64_t off = ((tile0 + tt) * H + h) * D + CPL * l;
        float ov[CPL];
#pragma unroll
        for (int c = 0; c < CPL; ++c) ov[c] = a.scale * fmaf(QK, dl[c], R[c]);
        if (og) {   // o_norm over the row (RMS with the weight), then the sigmoid gate
          float ss = 0.f;
#pragma unroll
          for (int c = 0; c < CPL; ++c) ss = fmaf(ov[c], ov[c], ss);
#pragma unroll
          for (int sh = 16; sh >= 1; sh >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, sh);
          const float rn = rsqrtf(ss * (1.f / D) + a.oeps);
#pragma unroll
          for (int c = 0; c < CPL; ++c) ov[c] = ov[c] * rn * onw[c] * sigmoid_f(sm.gate[tt][CPL * l + c]);
        }
#pragma unroll
        for (int c = 0; c < CPL; ++c) o[off + c] = from_f32<T>(ov[c]);
      }
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        const float kk = sm.k[tt][16 * w + r];
#pragma unroll
        for (int c = 0; c < CPL; ++c) S[r][c] = fmaf(kk, dl[c], S[r][c]);
      }
      if (a.snap != nullptr) {   // state snapshot after every snap_every tokens of the sequence
        const int64_t done = tile0 + tt + 1 - s0;
        if (done % a.snap_every == 0 && done / a.snap_every <= a.snap_cap) {
          float *dst = a.snap + (((int64_t)n * a.snap_cap + done / a.snap_every - 1) * H + h) * D * D;
#pragma unroll
          for (int r = 0; r < 16; ++r)
#pragma unroll
            for (int c = 0; c < CPL; ++c) __stcs(dst + (int64_t)(16 * w + r) * D + CPL * l + c, S[r][c]);
        }
      }
      buf ^= 1;
    }
  }

#pragma unroll
  for (int r = 0; r < 16; ++r) {
    const int i = 16 * w + r;
#pragma unroll
    for (int c = 0; c < CPL; ++c) a.state1[sbase + (int64_t)i * D + CPL * l + c] = S[r][c];
  }
}

template <typename T, int D>
static cudaError_t launch_rec_t(const RecurrenceArgs &a, cudaStream_t stream) {
  const size_t smem = sizeof(RecSmem<D>);
  cudaError_t e = cudaFuncSetAttribute(recurrence_kernel<T, D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  recurrence_kernel<T, D><<<a.N * a.H, 2 * D, smem, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_recurrence(const RecurrenceArgs &a, cudaStream_t stream) {
  if ((int64_t)a.N * a.H == 0) return cudaSuccess;
  if (a.io_dtype == KDA_BF16)
    return a.D == 128 ? launch_rec_t<__nv_bfloat16, 128>(a, stream)
                      : launch_rec_t<__nv_bfloat16, 64>(a, stream);
  return a.D == 128 ? launch_rec_t<float, 128>(a, stream) : launch_rec_t<float, 64>(a, stream);
}

}  // namespace kda
