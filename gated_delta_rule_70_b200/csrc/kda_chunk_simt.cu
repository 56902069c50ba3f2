// KDA chunkwise recurrence on CUDA cores in fp32: the fp32 test mode.
//
// The per-token loop of the AliceAI-Foundation KDA write-up ("二、KDA 线性注意力":
// S <- diag(e^g) S; d = beta (v - S^T k); S <- S + k d^T; o = S^T q) evaluated one
// 64-token chunk at a time in the same re-associated form the tensor-core path
// (kda_chunk_prep.cu + kda_state_pass.cu) uses, but with every operand and product
// in fp32 and accurate expf.  It runs the chunk algebra on the GPU to the fp32
// tolerance, so the factorisation itself is checked there and not only in bf16.
// With Gamma the in-chunk cumulative gate (per key channel):
//   A_kk[t,s] = beta_t sum_c k_tc k_sc e^{Gamma_tc - Gamma_sc}   (s < t)
//   A_qk[t,s] = sum_c q_tc k_sc e^{Gamma_tc - Gamma_sc}          (s <= t)
//   (I + A_kk) [W | U] = diag(beta) [k e^{Gamma} | v]          (forward substitution)
//   D = U - W S,  O = (q e^{Gamma}) S + A_qk D,  S' = diag(e^{Gamma_C}) S + (k e^{Gamma_C - Gamma})^T D
// The pairwise factor e^{Gamma_t - Gamma_s} is split as in the tensor-core path:
// 16-token sub-blocks, reference m_I = Gamma after the block's 8th token,
// L = x e^{Gamma - m_I}, R = k e^{m_I - Gamma}, and e^{m_I - m_J} <= 1 between blocks,
// so no factor leaves e^{+-8 |g|max} (fp32 range for gate bounds >= -10).
//
// One CTA of 256 threads per (sequence, head), chunks in order; the d_k x d_v state
// stays in shared memory for the whole sequence.  This is a test mode: it favours
// the plainest loops over speed.
#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {
namespace csimt {

constexpr int C = 64;       // tokens per chunk
constexpr int NB = 4;       // 16-token sub-blocks per chunk
constexpr int NT = 256;

// Shared-memory floats of the kernel for head dim D.
template <int D> constexpr int smem_floats() {
  return D * D           // S [d_k][d_v]
         + 4 * C * D     // Lq, Lk, Rk, V tiles [C][D]
         + C * C         // A: A_qk on and below the diagonal, beta A_kk transposed above it
         + 20 * D        // m_I, Gamma_C, e^{m_I - m_J} (6 pairs), e^{m_I}, e^{Gamma_C - m_I}, e^{Gamma_C}
         + C;            // beta
}

// The index of block pair (I, J), I > J, in the e^{m_I - m_J} table.
__device__ __forceinline__ int pair_index(int I, int J) { return I * (I - 1) / 2 + J; }

template <typename T, int D>
__global__ void __launch_bounds__(NT) chunk_simt_kernel(const RecurrenceArgs a) {
  extern __shared__ __align__(16) float sm[];
  float *S = sm;                 // [D][D]
  float *Lq = S + D * D;         // q -> q e^{Gamma - m_I} -> q e^{Gamma}; then O
  float *Lk = Lq + C * D;        // k -> k e^{Gamma - m_I} -> k e^{Gamma} -> W
  float *Rk = Lk + C * D;        // g -> Gamma -> k e^{m_I - Gamma} -> k e^{Gamma_C - Gamma}
  float *Vt = Rk + C * D;        // v -> U -> D
  float *A = Vt + C * D;         // [C][C]
  float *cm = A + C * C;         // [NB][D] references m_I
  float *cgc = cm + NB * D;      // [D] Gamma_C
  float *eij = cgc + D;          // [6][D] e^{m_I - m_J}
  float *eM = eij + 6 * D;       // [NB][D] e^{m_I}
  float *eCM = eM + NB * D;      // [NB][D] e^{Gamma_C - m_I}
  float *eGC = eCM + NB * D;     // [D] e^{Gamma_C}
  float *bet = eGC + D;          // [C]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = a.H;
  const int n = blockIdx.x / H, h = blockIdx.x % H;
  int64_t s0, s1;
  seq_bounds(a.cu, n, a.seq_len, a.total_tokens, s0, s1);
  const int64_t sg = ((int64_t)n * H + h) * D * D;
  for (int idx = tid; idx < D * D; idx += NT) S[idx] = a.state0 ? a.state0[sg + idx] : 0.f;

  const T *__restrict__ qn = reinterpret_cast<const T *>(a.qn);
  const T *__restrict__ kn = reinterpret_cast<const T *>(a.kn);
  const T *__restrict__ vc = reinterpret_cast<const T *>(a.vc);
  const T *__restrict__ og = reinterpret_cast<const T *>(a.ogate);
  T *__restrict__ o = reinterpret_cast<T *>(a.o);

  const int nchunks = (int)((s1 - s0 + C - 1) / C);
  for (int ci = 0; ci < nchunks; ++ci) {
    const int64_t c0 = s0 + (int64_t)ci * C;
    const int nt = (int)min((int64_t)C, s1 - c0);
    __syncthreads();   // the previous chunk's tiles have been read

    // 1. the chunk's inputs (rows past the sequence: zeros, so they change nothing)
    for (int idx = tid; idx < C * D; idx += NT) {
      const int t = idx / D, i = idx % D;
      float q = 0.f, k = 0.f, v = 0.f, g = 0.f;
      if (t < nt) {
        const int64_t off = ((c0 + t) * H + h) * D + i;
        q = to_f32(qn[off]);
        k = to_f32(kn[off]);
        v = to_f32(vc[off]);
        g = fminf(fmaxf(a.g[off], a.lower_bound), 0.f);
      }
      Lq[idx] = q; Lk[idx] = k; Rk[idx] = g; Vt[idx] = v;
    }
    if (tid < C) bet[tid] = tid < nt ? a.beta[(c0 + tid) * H + h] : 0.f;
    __syncthreads();

    // 2. Gamma (in place of g), the block references and the per-channel constants
    if (tid < D) {
      const int c = tid;
      float acc = 0.f;
      for (int t = 0; t < C; ++t) {
        acc += Rk[t * D + c];
        Rk[t * D + c] = acc;
        if ((t & 15) == 7) cm[(t >> 4) * D + c] = acc;
      }
      cgc[c] = acc;
      eGC[c] = expf(acc);
      for (int I = 0; I < NB; ++I) {
        const float m = cm[I * D + c];
        eM[I * D + c] = expf(m);
        eCM[I * D + c] = expf(acc - m);
        for (int J = 0; J < I; ++J) eij[pair_index(I, J) * D + c] = expf(m - cm[J * D + c]);
      }
    }
    __syncthreads();

    // 3. the split factors
    for (int idx = tid; idx < C * D; idx += NT) {
      const int t = idx / D, c = idx % D;
      const float m = cm[(t >> 4) * D + c], G = Rk[idx];
      const float k = Lk[idx];
      const float e1 = expf(G - m);
      Lq[idx] *= e1;
      Lk[idx] = k * e1;
      Rk[idx] = k * expf(m - G);
    }
    __syncthreads();

    // 4. A_qk (s <= t) at A[t][s]; beta_t A_kk[t][s] (s < t) at A[s][t]
    for (int idx = tid; idx < C * C; idx += NT) {
      const int t = idx / C, s = idx % C;
      if (s > t) continue;
      const int I = t >> 4, J = s >> 4;
      const float *lq = Lq + t * D, *lk = Lk + t * D, *rk = Rk + s * D;
      float aq = 0.f, ak = 0.f;
      if (I == J) {
        for (int c = 0; c < D; ++c) {
          aq = fmaf(lq[c], rk[c], aq);
          ak = fmaf(lk[c], rk[c], ak);
        }
      } else {
        const float *e = eij + pair_index(I, J) * D;
        for (int c = 0; c < D; ++c) {
          const float r = e[c] * rk[c];
          aq = fmaf(lq[c], r, aq);
          ak = fmaf(lk[c], r, ak);
        }
      }
      A[t * C + s] = aq;
      if (s < t) A[s * C + t] = bet[t] * ak;
    }
    __syncthreads();

    // 5. [W | U] by forward substitution: X[t] = beta_t rhs[t] - sum_{s<t} beta_t A_kk[t][s] X[s],
    //    rhs = [k e^{Gamma} | v]; each thread owns one right-hand-side column, in place
    for (int col = tid; col < 2 * D; col += NT) {
      float *X = col < D ? Lk + col : Vt + (col - D);
      for (int t = 0; t < C; ++t) {
        float r = X[t * D];
        if (col < D) r *= eM[(t >> 4) * D + col];   // k e^{Gamma} = (k e^{Gamma - m_I}) e^{m_I}
        float acc = bet[t] * r;
        for (int s = 0; s < t; ++s) acc = fmaf(-A[s * C + t], X[s * D], acc);
        X[t * D] = acc;
      }
    }
    // q e^{Gamma} and k e^{Gamma_C - Gamma} from the split factors
    for (int idx = tid; idx < C * D; idx += NT) {
      const int t = idx / D, c = idx % D, I = t >> 4;
      Lq[idx] *= eM[I * D + c];
      Rk[idx] *= eCM[I * D + c];
    }
    __syncthreads();

    // 6. D = U - W S (in place of U)
    for (int idx = tid; idx < C * D; idx += NT) {
      const int t = idx / D, j = idx % D;
      const float *w = Lk + t * D;
      float acc = Vt[idx];
      for (int i = 0; i < D; ++i) acc = fmaf(-w[i], S[i * D + j], acc);
      Vt[idx] = acc;
    }
    __syncthreads();

    // 7. O = (q e^{Gamma}) S + A_qk D, scaled (in place of W, which is no longer needed)
    for (int idx = tid; idx < C * D; idx += NT) {
      const int t = idx / D, j = idx % D;
      const float *qt = Lq + t * D;
      float acc = 0.f;
      for (int i = 0; i < D; ++i) acc = fmaf(qt[i], S[i * D + j], acc);
      for (int s = 0; s <= t; ++s) acc = fmaf(A[t * C + s], Vt[s * D + j], acc);
      Lk[idx] = a.scale * acc;
    }
    __syncthreads();

    // 8. S <- diag(e^{Gamma_C}) S + (k e^{Gamma_C - Gamma})^T D, and o (with the epilogue)
    for (int idx = tid; idx < D * D; idx += NT) {
      const int i = idx / D, j = idx % D;
      float acc = eGC[i] * S[idx];
      for (int t = 0; t < C; ++t) acc = fmaf(Rk[t * D + i], Vt[t * D + j], acc);
      S[idx] = acc;
    }
    for (int t = warp; t < nt; t += NT / 32) {   // a warp per token row
      const float *orow = Lk + t * D;
      const int64_t off = ((c0 + t) * H + h) * D;
      float rn = 1.f;
      if (og) {   // o_norm over the row (RMS with the weight), then the sigmoid gate
        float ss = 0.f;
        for (int j = lane; j < D; j += 32) ss = fmaf(orow[j], orow[j], ss);
        for (int sh = 16; sh >= 1; sh >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, sh);
        rn = rsqrtf(ss * (1.f / D) + a.oeps);
      }
      for (int j = lane; j < D; j += 32) {
        float ov = orow[j];
        if (og) ov = ov * rn * a.onw[j] * sigmoid_f(to_f32(og[off + j]));
        o[off + j] = from_f32<T>(ov);
      }
    }
    __syncthreads();

    // 9. a state snapshot after every snap_every tokens of the sequence (whole chunks only)
    if (a.snap != nullptr && nt == C) {
      const int64_t done = (int64_t)(ci + 1) * C;
      if (done % a.snap_every == 0 && done / a.snap_every <= a.snap_cap) {
        float *dst = a.snap + (((int64_t)n * a.snap_cap + done / a.snap_every - 1) * H + h) * D * D;
        for (int idx = tid; idx < D * D; idx += NT) __stcs(dst + idx, S[idx]);
      }
    }
  }
  __syncthreads();
  for (int idx = tid; idx < D * D; idx += NT) a.state1[sg + idx] = S[idx];
}

template <typename T, int D>
cudaError_t launch_t(const RecurrenceArgs &a, cudaStream_t stream) {
  const size_t smem = (size_t)smem_floats<D>() * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(chunk_simt_kernel<T, D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  chunk_simt_kernel<T, D><<<a.N * a.H, NT, smem, stream>>>(a);
  return cudaGetLastError();
}

static_assert(smem_floats<128>() * 4 <= 232448, "shared memory budget");

}  // namespace csimt

cudaError_t launch_chunk_simt(const RecurrenceArgs &a, cudaStream_t stream) {
  if ((int64_t)a.N * a.H == 0) return cudaSuccess;
  if (a.io_dtype == KDA_BF16)
    return a.D == 128 ? csimt::launch_t<__nv_bfloat16, 128>(a, stream)
                      : csimt::launch_t<__nv_bfloat16, 64>(a, stream);
  return a.D == 128 ? csimt::launch_t<float, 128>(a, stream) : csimt::launch_t<float, 64>(a, stream);
}

}  // namespace kda
