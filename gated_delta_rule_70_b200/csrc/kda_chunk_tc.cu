// KDA chunkwise prefill on the 5th-generation tensor cores (tcgen05 + TMEM),
// bf16 operands with fp32 accumulation, head_dim 128, one CTA per
// (sequence, head), 64-token chunks.
//
// The recurrence of the AliceAI-Foundation KDA write-up ("二、KDA 线性注意力":
// S <- diag(e^g) S; d = beta (v - S^T k); S <- S + k d^T; o = S^T q) is
// evaluated per chunk in the WY / UT form.  With Gamma_t the in-chunk
// cumulative gate (per key channel),
//   A_kk[t,s] = sum_c k_tc k_sc e^{Gamma_tc - Gamma_sc}   (s < t)
//   A_qk[t,s] = sum_c q_tc k_sc e^{Gamma_tc - Gamma_sc}   (s <= t)
//   T  = (I + diag(beta) A_kk)^{-1},   T_b = T diag(beta)
//   W  = T_b (k e^{Gamma}),   U = T_b v
//   D  = U - W S            (the chunk's delta rows)
//   O  = (q e^{Gamma}) S + A_qk D
//   S' = diag(e^{Gamma_C}) S + (k e^{Gamma_C - Gamma})^T D
// which is the token loop re-associated (no approximation).
//
// Numerics: Gamma reaches 64 * (-5) = -320 inside a chunk, so e^{-Gamma}
// overflows fp32.  The pairwise factor e^{Gamma_t - Gamma_s} is therefore only
// ever split around a reference point close to both tokens: 16-token sub-blocks
// I with r_I = Gamma at the end of block I-1.  Diagonal blocks use
// (q|k)_t e^{Gamma_t - r_I} against k_s e^{r_I - Gamma_s} (factors within
// e^{+-80}); a row in block I against earlier blocks uses the reference r_I on
// both sides (both factors <= 1).  The operands e^{Gamma}, e^{Gamma_C - Gamma}
// are <= 1.
//
// Everything with a 128-wide dimension sits on the MMA's M = 128 axis: the
// state is kept transposed, S^T [d_v lanes x d_k columns] fp32 in TMEM, with a
// bf16 copy in TMEM as the A operand of S^T W^T and S^T Q~^T; D^T lives in
// TMEM the same way.  Shared-memory operands all use one format: token rows
// of 128 channels, 128-byte swizzle, 64-channel atoms; a descriptor reads it
// as K-major (K = channels) or MN-major (MN = channels, K = tokens).
#include "kda_common.cuh"
#include "kda_internal.h"
#include "umma.cuh"

namespace kda {
namespace chunk {

constexpr int CH = 64;        // tokens per chunk
constexpr int DK = 128;       // head dim (d_k = d_v)
constexpr int SB = 16;        // sub-block for the decay references
constexpr int NT = 256;       // threads per CTA
constexpr int TSS = 68;       // fp32 row stride of the solve scratch

// Shared-memory byte offsets (base aligned to 1024).
constexpr uint32_t OFF_L = 0;                       // [q rows 0..63 | k rows 64..127] x 128 ch: 32 KB
constexpr uint32_t OFF_R = OFF_L + 32768;           // R_all: 160 rows x 128 ch: 40 KB
constexpr uint32_t OFF_KT = OFF_R + 40960;          // k e^{Gamma}: 16 KB
constexpr uint32_t OFF_QT = OFF_KT + 16384;         // q e^{Gamma}: 16 KB
constexpr uint32_t OFF_KH = OFF_QT + 16384;         // k e^{Gamma_C - Gamma}: 16 KB
constexpr uint32_t OFF_V = OFF_KH + 16384;          // v: 16 KB
constexpr uint32_t OFF_TB = OFF_V + 16384;          // T_b [t][s] bf16: 8 KB
constexpr uint32_t OFF_AQ = OFF_TB + 8192;          // A_qk [t][s] bf16: 8 KB
constexpr uint32_t OFF_WT = OFF_AQ + 8192;          // -W^T [i][t] bf16 (MN-major B): 16 KB
constexpr uint32_t OFF_SB = OFF_WT + 16384;         // diag(beta) A_kk fp32 [64][TSS]
constexpr uint32_t OFF_ST = OFF_SB + 64 * TSS * 4;  // T fp32 [64][TSS]
constexpr uint32_t OFF_MISC = OFF_ST + 64 * TSS * 4;
// misc: beta[64], egC[128] (e^{Gamma_C}), wtot[8][128] (per-warp gate sums)
constexpr uint32_t OFF_BETA = OFF_MISC;
constexpr uint32_t OFF_EGC = OFF_BETA + 256;
constexpr uint32_t OFF_WTOT = OFF_EGC + 512;
constexpr uint32_t OFF_BAR = OFF_WTOT + 4096;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 64;
constexpr uint32_t SMEM_ALLOC = SMEM_BYTES + 1024;   // slack for the 1024-byte alignment

// R_all rows: [0,64) diagonal-reference rows, then R_1 (16 rows), R_2 (32), R_3 (48).
__host__ __device__ constexpr int r_row0(int I) { return I == 1 ? 64 : (I == 2 ? 80 : 112); }

// TMEM columns (512 allocated)
constexpr uint32_t TM_S32 = 0;     // S^T fp32, 128 cols
constexpr uint32_t TM_S16 = 128;   // S^T bf16 A operand, 64 cols
constexpr uint32_t TM_P = 192;     // intra products, 160 cols (later O^T, 64 cols)
constexpr uint32_t TM_O = 192;
constexpr uint32_t TM_W = 352;     // W^T fp32, 64 cols
constexpr uint32_t TM_D = 416;     // D^T fp32 (starts as U^T), 64 cols
constexpr uint32_t TM_D16 = 480;   // D^T bf16 A operand, 32 cols

constexpr uint32_t WAIT_POLLS = 1u << 24;   // bounded mbarrier waits

// Byte offset of (row, channel group cg of 8) in a token-rows SW128 operand with
// `rows` rows: atom = cg / 8 (64 channels), 16-byte chunk = cg % 8 swizzled by row % 8.
__device__ __forceinline__ uint32_t tr_off(int rows, int row, int cg) {
  return (uint32_t)((cg >> 3) * rows * 128 + (row >> 3) * 1024 + (row & 7) * 128 +
                    (((cg & 7) ^ (row & 7)) << 4));
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&h);
}
__device__ __forceinline__ uint4 pack8(const float (&x)[8]) {
  return make_uint4(pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]), pack_bf16(x[4], x[5]),
                    pack_bf16(x[6], x[7]));
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
// K-major descriptor over a [64 rows][64] matrix (one atom wide), k-step s.
__device__ __forceinline__ uint64_t desc_k64(uint32_t base, int s) {
  return umma::make_desc(base + (uint32_t)(s * 32), 16, 1024, umma::LAYOUT_SW128);
}
// MN-major descriptor over W^T stored [i rows][64 t] (MN = t, one atom), k-step s (16 channels).
__device__ __forceinline__ uint64_t desc_mn_wt(uint32_t base, int s) {
  return umma::make_desc(base + (uint32_t)(s * 2048), 128 * 128, 1024, umma::LAYOUT_SW128);
}

struct Ctx {
  uint8_t *smem;
  uint32_t sbase;     // shared address of smem
  uint32_t tmem;      // TMEM base address
  uint64_t *bar;      // MMA completion barrier
  uint32_t phase;
  bool ok;
  int *err;
};

// All threads: wait for the MMA barrier's next phase (bounded).  The outcome is
// voted block-wide so every thread takes the same path afterwards.
__device__ __forceinline__ void wait_mma(Ctx &c) {
  bool mine = c.ok && umma::mbar_wait_bounded(c.bar, c.phase, WAIT_POLLS);
  const bool all = __syncthreads_and(mine) != 0;
  if (c.ok && !all && threadIdx.x == 0 && c.err) atomicExch(c.err, ERR_TIMEOUT);
  c.ok = all;
  c.phase ^= 1u;
  umma::fence_after_sync();
}

// Threads: make generic smem writes and tcgen05.st visible, then rendezvous.
__device__ __forceinline__ void publish() {
  umma::fence_proxy_async_smem();
  umma::fence_before_sync();
  __syncthreads();
  umma::fence_after_sync();
}

template <int NCOLS>
__device__ __forceinline__ void tmem_row_load(uint32_t taddr, float (&x)[NCOLS]) {
  static_assert(NCOLS % 16 == 0, "");
#pragma unroll
  for (int c = 0; c < NCOLS; c += 16) {
    uint32_t r[16];
    umma::tmem_ld16(taddr + c, r);
    umma::tmem_wait_ld();
#pragma unroll
    for (int j = 0; j < 16; ++j) x[c + j] = __uint_as_float(r[j]);
  }
}

__global__ void __launch_bounds__(NT, 1) chunk_kernel(RecurrenceArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n = blockIdx.x / a.H, h = blockIdx.x % a.H;
  const int H = a.H;
  int64_t s0, s1;
  seq_bounds(a.cu, n, a.seq_len, a.total_tokens, s0, s1);
  const int64_t L = s1 - s0;

  float *beta_s = reinterpret_cast<float *>(smem + OFF_BETA);
  float *egc = reinterpret_cast<float *>(smem + OFF_EGC);
  float *wtot = reinterpret_cast<float *>(smem + OFF_WTOT);
  float *sBm = reinterpret_cast<float *>(smem + OFF_SB);
  float *sTm = reinterpret_cast<float *>(smem + OFF_ST);
  uint64_t *bar = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + OFF_BAR + 16);

  Ctx cx;
  cx.smem = smem;
  cx.sbase = umma::smem_u32(smem);
  cx.bar = bar;
  cx.phase = 0;
  cx.ok = true;
  cx.err = a.err;

  if (warp == 0) {
    umma::tmem_alloc(tmem_slot, 512);
    umma::tmem_relinquish();
  }
  if (tid == 0) {
    umma::mbar_init(bar, 1);
    umma::mbar_fence_init();
  }
  umma::fence_before_sync();
  __syncthreads();
  umma::fence_after_sync();
  cx.tmem = *tmem_slot;

  const __nv_bfloat16 *__restrict__ qn = reinterpret_cast<const __nv_bfloat16 *>(a.qn);
  const __nv_bfloat16 *__restrict__ kn = reinterpret_cast<const __nv_bfloat16 *>(a.kn);
  const __nv_bfloat16 *__restrict__ vc = reinterpret_cast<const __nv_bfloat16 *>(a.vc);
  __nv_bfloat16 *__restrict__ o = reinterpret_cast<__nv_bfloat16 *>(a.o);
  const int64_t sbase_g = ((int64_t)n * H + h) * DK * DK;

  // Epilogue role: warps 0..3 own TMEM lanes 32w..32w+31 (row j of S^T, D^T, O^T).
  const bool epi = warp < 4;
  const int jrow = warp * 32 + lane;                     // valid when epi
  const uint32_t lane_base = (uint32_t)(warp & 3) * 32u << 16;

  // ---- initial state: S^T[j][i] = S0[i][j] into TMEM (fp32 and bf16 copies)
  if (epi) {
#pragma unroll 1
    for (int c = 0; c < DK; c += 16) {
      uint32_t r[16];
#pragma unroll
      for (int jj = 0; jj < 16; ++jj) {
        float x = a.state0 ? a.state0[sbase_g + (int64_t)(c + jj) * DK + jrow] : 0.f;
        r[jj] = __float_as_uint(x);
      }
      umma::tmem_st16(cx.tmem + lane_base + TM_S32 + c, r);
    }
#pragma unroll 1
    for (int c = 0; c < DK; c += 32) {   // bf16 copy: 32 channels -> 16 columns
      uint32_t r[16];
#pragma unroll
      for (int jj = 0; jj < 16; ++jj) {
        float x0 = a.state0 ? a.state0[sbase_g + (int64_t)(c + 2 * jj) * DK + jrow] : 0.f;
        float x1 = a.state0 ? a.state0[sbase_g + (int64_t)(c + 2 * jj + 1) * DK + jrow] : 0.f;
        r[jj] = pack_bf16(x0, x1);
      }
      umma::tmem_st16(cx.tmem + lane_base + TM_S16 + c / 2, r);
    }
    umma::tmem_wait_st();
  }
  publish();

  // Elementwise role mapping: 16 channel groups x 16 token groups of 4 tokens.
  const int cg = tid & 15, tg = tid >> 4;
  const int blkI = tg >> 2;                               // sub-block of this thread's tokens

  const int nchunks = (int)((L + CH - 1) / CH);
#pragma unroll 1
  for (int ch = 0; ch < nchunks && cx.ok; ++ch) {
    const int64_t c0 = s0 + (int64_t)ch * CH;
    // ------------------------------------------------ E: load, cumulative gate, operands
    float qv[4][8], kv[4][8], gv[4][8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int t = tg * 4 + j;
      const bool valid = c0 + t < s1;
      const int64_t off = ((c0 + t) * H + h) * DK + cg * 8;
      float vv[8];
      if (valid) {
        load8(qn + off, qv[j]);
        load8(kn + off, kv[j]);
        load8(vc + off, vv);
        load8(a.g + off, gv[j]);
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) { qv[j][i] = 0.f; kv[j][i] = 0.f; vv[i] = 0.f; gv[j][i] = 0.f; }
      }
      *reinterpret_cast<uint4 *>(smem + OFF_V + tr_off(64, t, cg)) = pack8(vv);
      if (cg == 0) beta_s[t] = valid ? a.beta[(c0 + t) * H + h] : 0.f;
    }
    // local inclusive cumsum over this thread's 4 tokens
#pragma unroll
    for (int j = 1; j < 4; ++j)
#pragma unroll
      for (int i = 0; i < 8; ++i) gv[j][i] += gv[j - 1][i];
    // the upper half-warp (token group 2w+1) adds the lower half's total
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float lo = __shfl_up_sync(0xffffffffu, gv[3][i], 16);
      if (lane >= 16) {
#pragma unroll
        for (int j = 0; j < 4; ++j) gv[j][i] += lo;
      }
    }
    if (lane >= 16) {
#pragma unroll
      for (int i = 0; i < 8; ++i) wtot[warp * 128 + cg * 8 + i] = gv[3][i];
    }
    __syncthreads();
    // prefix over earlier warps; references r_I = Gamma at the end of block I-1
    float pre[8], rI[8], rI1[8], gC[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) { pre[i] = 0.f; rI[i] = 0.f; rI1[i] = 0.f; gC[i] = 0.f; }
    float rAll[5][8];  // r_0 .. r_4 (r_4 = Gamma_C)
#pragma unroll
    for (int i = 0; i < 8; ++i) rAll[0][i] = 0.f;
#pragma unroll
    for (int w2 = 0; w2 < 8; ++w2) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float x = wtot[w2 * 128 + cg * 8 + i];
        if (w2 < warp) pre[i] += x;
        gC[i] += x;
        if (w2 % 2 == 1) rAll[(w2 + 1) / 2][i] = gC[i];
      }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      rI[i] = rAll[blkI][i];
      rI1[i] = rAll[blkI + 1][i];
#pragma unroll
      for (int j = 0; j < 4; ++j) gv[j][i] += pre[i];
    }
    if (tid < 16) {
#pragma unroll
      for (int i = 0; i < 8; ++i) egc[tid * 8 + i] = expf(gC[i]);
    }
    // per-thread constants
    float eR[8], bdI[8], cx2[4][8];  // e^{r_I}, e^{r_{I+1} - r_I}, e^{r_{I'} - r_{I+1}} (I' = I+1..4)
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      eR[i] = expf(rI[i]);
      bdI[i] = expf(rI1[i] - rI[i]);
#pragma unroll
      for (int ip = 0; ip < 4; ++ip)
        cx2[ip][i] = (ip + 1 > blkI) ? expf(rAll[ip + 1][i] - rI1[i]) : 0.f;
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int t = tg * 4 + j;
      float Lq[8], Lk[8], Rd[8], Qt[8], Kt[8], Kh[8], u[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float e1 = expf(gv[j][i] - rI[i]);       // <= 1
        const float rd = expf(rI[i] - gv[j][i]);       // >= 1, <= e^80
        Lq[i] = qv[j][i] * e1;
        Lk[i] = kv[j][i] * e1;
        Rd[i] = kv[j][i] * rd;
        Qt[i] = Lq[i] * eR[i];
        Kt[i] = Lk[i] * eR[i];
        u[i] = rd * bdI[i];                            // e^{r_{I+1} - Gamma_t} in [e^-80, 1]
        Kh[i] = kv[j][i] * u[i] * cx2[3][i];           // e^{Gamma_C - Gamma_t}
      }
      *reinterpret_cast<uint4 *>(smem + OFF_L + tr_off(128, t, cg)) = pack8(Lq);
      *reinterpret_cast<uint4 *>(smem + OFF_L + tr_off(128, 64 + t, cg)) = pack8(Lk);
      *reinterpret_cast<uint4 *>(smem + OFF_R + tr_off(160, t, cg)) = pack8(Rd);
      *reinterpret_cast<uint4 *>(smem + OFF_QT + tr_off(64, t, cg)) = pack8(Qt);
      *reinterpret_cast<uint4 *>(smem + OFF_KT + tr_off(64, t, cg)) = pack8(Kt);
      *reinterpret_cast<uint4 *>(smem + OFF_KH + tr_off(64, t, cg)) = pack8(Kh);
      // rows of R_{I'} for every later block I' (reference r_{I'})
#pragma unroll
      for (int ip = 1; ip < 4; ++ip) {
        if (ip > blkI) {
          float Rx[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) Rx[i] = kv[j][i] * u[i] * cx2[ip - 1][i];
          *reinterpret_cast<uint4 *>(smem + OFF_R + tr_off(160, r_row0(ip) + t, cg)) = pack8(Rx);
        }
      }
    }
    publish();

    // ------------------------------------------------ MMA 1: [Lq; Lk] x R_all^T -> P
    if (tid == 0) {
      const uint32_t idesc = umma::make_idesc_bf16(128, 160, 0, 0);
#pragma unroll 1
      for (int s = 0; s < DK / 16; ++s)
        umma::mma_ss(cx.tmem + TM_P, desc_k128(cx.sbase + OFF_L, 128, s),
                     desc_k128(cx.sbase + OFF_R, 160, s), idesc, s > 0);
      umma::mma_commit(bar);
    }
    wait_mma(cx);

    // ------------------------------------------------ E-1: assemble A_qk (bf16) and diag(beta) A_kk
    if (epi) {
      const int t = jrow & 63;
      const bool is_q = jrow < 64;
      const int I = t >> 4;
      float rowv[64];
#pragma unroll
      for (int s = 0; s < 64; ++s) rowv[s] = 0.f;
      // P columns in 16-wide chunks: 0..3 diagonal-reference blocks, 4 = R_1, 5..6 = R_2,
      // 7..9 = R_3.  Every lane loads every chunk (tcgen05.ld is warp-uniform) and keeps
      // the ones its sub-block I uses.
#pragma unroll
      for (int cc = 0; cc < 10; ++cc) {
        uint32_t r[16];
        umma::tmem_ld16(cx.tmem + lane_base + TM_P + cc * 16, r);
        umma::tmem_wait_ld();
        const int want = cc < 4 ? cc : (cc == 4 ? 1 : (cc < 7 ? 2 : 3));
        const int sblk = cc < 4 ? cc : (cc == 4 ? 0 : (cc < 7 ? cc - 5 : cc - 7));
        if (I == want) {
#pragma unroll
          for (int e = 0; e < 16; ++e) rowv[sblk * 16 + e] = __uint_as_float(r[e]);
        }
      }
      const float bt = is_q ? 1.f : beta_s[t];
#pragma unroll
      for (int s = 0; s < 64; ++s) {
        const bool keep = is_q ? (s <= t) : (s < t);
        rowv[s] = keep ? rowv[s] * bt : 0.f;
      }
      if (is_q) {
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) {
          float x8[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) x8[i] = rowv[c8 * 8 + i];
          *reinterpret_cast<uint4 *>(smem + OFF_AQ + tr_off(64, t, c8)) = pack8(x8);
        }
      } else {
#pragma unroll
        for (int s = 0; s < 64; ++s) sBm[t * TSS + s] = rowv[s];
      }
    }
    umma::tmem_wait_ld();
    publish();

    // ------------------------------------------------ E-2: T = (I + B)^{-1}, T_b = T diag(beta)
    if (tid < 64) {  // diagonal 16x16 blocks: thread = (block, column)
      const int I = tid >> 4, c = tid & 15, o16 = I * 16;
      float x[16];
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        float acc = (r == c) ? 1.f : 0.f;
        if (r > c) {
#pragma unroll
          for (int m = 0; m < 16; ++m)
            if (m >= c && m < r) acc -= sBm[(o16 + r) * TSS + o16 + m] * x[m];
        }
        x[r] = acc;
      }
#pragma unroll
      for (int r = 0; r < 16; ++r) sTm[(o16 + r) * TSS + o16 + c] = x[r];
    }
    __syncthreads();
#pragma unroll 1
    for (int d = 1; d < 4; ++d) {
      // X_IJ = sum_{K=J}^{I-1} B_IK T_KJ, kept in the unused upper block (J, I) of sBm
      for (int e = tid; e < (4 - d) * 256; e += NT) {
        const int J = e >> 8, I = J + d, r = (e >> 4) & 15, c = e & 15;
        float acc = 0.f;
        for (int K = J; K < I; ++K)
#pragma unroll
          for (int m = 0; m < 16; ++m)
            acc += sBm[(I * 16 + r) * TSS + K * 16 + m] * sTm[(K * 16 + m) * TSS + J * 16 + c];
        sBm[(J * 16 + r) * TSS + I * 16 + c] = acc;
      }
      __syncthreads();
      for (int e = tid; e < (4 - d) * 256; e += NT) {
        const int J = e >> 8, I = J + d, r = (e >> 4) & 15, c = e & 15;
        float acc = 0.f;
#pragma unroll
        for (int m = 0; m < 16; ++m)
          if (m <= r) acc -= sTm[(I * 16 + r) * TSS + I * 16 + m] * sBm[(J * 16 + m) * TSS + I * 16 + c];
        sTm[(I * 16 + r) * TSS + J * 16 + c] = acc;
      }
      __syncthreads();
    }
    for (int e = tid; e < 64 * 8; e += NT) {  // T_b rows as bf16, K-major [t][s]
      const int t = e >> 3, c8 = e & 7;
      float x8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int s = c8 * 8 + i;
        x8[i] = s <= t ? sTm[t * TSS + s] * beta_s[s] : 0.f;
      }
      *reinterpret_cast<uint4 *>(smem + OFF_TB + tr_off(64, t, c8)) = pack8(x8);
    }
    publish();

    // ------------------------------------------------ MMA 2: W^T = Kt^T T_b^T, U^T = V^T T_b^T
    if (tid == 0) {
      const uint32_t idesc = umma::make_idesc_bf16(128, 64, 1, 0);
#pragma unroll 1
      for (int s = 0; s < CH / 16; ++s) {
        umma::mma_ss(cx.tmem + TM_W, desc_mn_tok(cx.sbase + OFF_KT, s),
                     desc_k64(cx.sbase + OFF_TB, s), idesc, s > 0);
        umma::mma_ss(cx.tmem + TM_D, desc_mn_tok(cx.sbase + OFF_V, s),
                     desc_k64(cx.sbase + OFF_TB, s), idesc, s > 0);
      }
      umma::mma_commit(bar);
    }
    wait_mma(cx);

    // ------------------------------------------------ E-3: -W^T to smem (MN-major B, rows = channel)
    if (epi) {
      float w[64];
      tmem_row_load<64>(cx.tmem + lane_base + TM_W, w);
      const int i = jrow;  // lane = key channel
#pragma unroll
      for (int c8 = 0; c8 < 8; ++c8) {
        float x8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) x8[e] = -w[c8 * 8 + e];
        *reinterpret_cast<uint4 *>(smem + OFF_WT + (uint32_t)((i >> 3) * 1024 + (i & 7) * 128 +
                                                             ((c8 ^ (i & 7)) << 4))) = pack8(x8);
      }
    }
    umma::tmem_wait_ld();
    publish();

    // ------------------------------------------------ MMA 3: D^T += S^T (-W^T); O^T = S^T Qt^T
    if (tid == 0) {
      const uint32_t id_d = umma::make_idesc_bf16(128, 64, 0, 1);
      const uint32_t id_o = umma::make_idesc_bf16(128, 64, 0, 0);
#pragma unroll 1
      for (int s = 0; s < DK / 16; ++s) {
        const uint32_t a_t = cx.tmem + TM_S16 + (uint32_t)(s * 8);
        umma::mma_ts(cx.tmem + TM_D, a_t, desc_mn_wt(cx.sbase + OFF_WT, s), id_d, 1);
        umma::mma_ts(cx.tmem + TM_O, a_t, desc_k128(cx.sbase + OFF_QT, 64, s), id_o, s > 0);
      }
      umma::mma_commit(bar);
    }
    wait_mma(cx);

    // ------------------------------------------------ E-4: D^T -> bf16 A operand; decay S^T
    if (epi) {
      float dl[64];
      tmem_row_load<64>(cx.tmem + lane_base + TM_D, dl);
#pragma unroll
      for (int c = 0; c < 32; c += 16) {
        uint32_t r[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) r[e] = pack_bf16(dl[2 * (c + e)], dl[2 * (c + e) + 1]);
        umma::tmem_st16(cx.tmem + lane_base + TM_D16 + c, r);
      }
#pragma unroll 1
      for (int c = 0; c < DK; c += 16) {
        uint32_t r[16];
        umma::tmem_ld16(cx.tmem + lane_base + TM_S32 + c, r);
        umma::tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * egc[c + e]);
        umma::tmem_st16(cx.tmem + lane_base + TM_S32 + c, r);
      }
      umma::tmem_wait_st();
    }
    publish();

    // ------------------------------------------------ MMA 4: O^T += D^T A_qk^T; S^T += D^T Kh
    if (tid == 0) {
      const uint32_t id_o = umma::make_idesc_bf16(128, 64, 0, 0);
      const uint32_t id_s = umma::make_idesc_bf16(128, 128, 0, 1);
#pragma unroll 1
      for (int s = 0; s < CH / 16; ++s) {
        const uint32_t a_t = cx.tmem + TM_D16 + (uint32_t)(s * 8);
        umma::mma_ts(cx.tmem + TM_O, a_t, desc_k64(cx.sbase + OFF_AQ, s), id_o, 1);
        umma::mma_ts(cx.tmem + TM_S32, a_t, desc_mn_tok(cx.sbase + OFF_KH, s), id_s, 1);
      }
      umma::mma_commit(bar);
    }
    wait_mma(cx);

    // ------------------------------------------------ E-5: store O; refresh the bf16 state copy
    if (epi) {
      const int j = jrow;
#pragma unroll 1
      for (int c = 0; c < CH; c += 16) {
        uint32_t r[16];
        umma::tmem_ld16(cx.tmem + lane_base + TM_O + c, r);
        umma::tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int t = c + e;
          if (c0 + t < s1)
            o[((c0 + t) * H + h) * DK + j] = __float2bfloat16_rn(a.scale * __uint_as_float(r[e]));
        }
      }
#pragma unroll 1
      for (int c = 0; c < DK; c += 32) {
        uint32_t r0[16], r1[16], p[16];
        umma::tmem_ld16(cx.tmem + lane_base + TM_S32 + c, r0);
        umma::tmem_ld16(cx.tmem + lane_base + TM_S32 + c + 16, r1);
        umma::tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          p[e] = pack_bf16(__uint_as_float(r0[2 * e]), __uint_as_float(r0[2 * e + 1]));
          p[8 + e] = pack_bf16(__uint_as_float(r1[2 * e]), __uint_as_float(r1[2 * e + 1]));
        }
        umma::tmem_st16(cx.tmem + lane_base + TM_S16 + c / 2, p);
      }
      umma::tmem_wait_st();
    }
    publish();
  }

  // ---- final state: S[i][j] = S^T[j][i]
  if (epi) {
#pragma unroll 1
    for (int c = 0; c < DK; c += 16) {
      uint32_t r[16];
      umma::tmem_ld16(cx.tmem + lane_base + TM_S32 + c, r);
      umma::tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 16; ++e) a.state1[sbase_g + (int64_t)(c + e) * DK + jrow] = __uint_as_float(r[e]);
    }
  }
  umma::fence_before_sync();
  __syncthreads();
  if (warp == 0) umma::tmem_dealloc(cx.tmem, 512);
}

}  // namespace chunk

cudaError_t launch_chunk_tc(const RecurrenceArgs &a, cudaStream_t stream) {
  if ((int64_t)a.N * a.H == 0) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(chunk::chunk_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)chunk::SMEM_ALLOC);
  if (e != cudaSuccess) return e;
  chunk::chunk_kernel<<<a.N * a.H, chunk::NT, chunk::SMEM_ALLOC, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace kda
