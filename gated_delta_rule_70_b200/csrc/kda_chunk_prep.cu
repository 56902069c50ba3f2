// KDA chunk preparation: everything in a 64-token chunk that does not depend
// on the recurrent state, for every (chunk, head).
//
// The recurrence of the AliceAI-Foundation KDA write-up ("二、KDA 线性注意力":
// S <- diag(e^g) S; d = beta (v - S^T k); S <- S + k d^T; o = S^T q) is
// evaluated per chunk in the WY / UT form.  With Gamma_t the in-chunk
// cumulative gate (per key channel),
//   A_kk[t,s] = sum_c k_tc k_sc e^{Gamma_tc - Gamma_sc}   (s < t)
//   A_qk[t,s] = sum_c q_tc k_sc e^{Gamma_tc - Gamma_sc}   (s <= t)
//   T  = (I + diag(beta) A_kk)^{-1},   T_b = T diag(beta)
//   W  = T_b (k e^{Gamma}),   U = T_b v
// and the state pass (kda_state_pass.cu) then needs only
//   D  = U - W S,   O = (q e^{Gamma}) S + A_qk D,   S' = diag(e^{Gamma_C}) S + (k e^{Gamma_C - Gamma})^T D.
// This kernel writes -W^T, U^T, A_qk, q e^{Gamma}, k e^{Gamma_C - Gamma} and
// e^{Gamma_C} of each (chunk, head) as one record, already in the
// shared-memory image the state pass copies in.
//
// Numerics: Gamma reaches 64 * (-5) = -320 inside a chunk, so e^{-Gamma}
// overflows fp32.  The pairwise factor e^{Gamma_t - Gamma_s} is only ever split
// around a reference close to both tokens: 16-token sub-blocks I with r_I =
// Gamma at the end of block I-1.  Diagonal blocks use (q|k)_t e^{Gamma_t - r_I}
// against k_s e^{r_I - Gamma_s} (factors within e^{+-80}); a row in block I
// against earlier blocks uses r_I on both sides (factors <= 1).  Exponentials
// run on the special-function unit in base 2; every other decay factor is a
// product of terms ordered so that no intermediate overflows.
//
// Structure: one CTA of 8 warps per (chunk, head), two CTAs per SM so that one
// item's memory and tensor-core waits overlap the other's arithmetic.
// Tensor-core work (tcgen05, fp32 accumulation in TMEM):
//   [Lq; Lk] x R_all^T (M=128, N=160, K=128) -> A_qk and A_kk blocks
//   W^T = K~^T T_b^T and U^T = V^T T_b^T      (M=128, N=64, K=64)
// The 64x64 unit-lower-triangular solve runs in shared memory (16x16 blocks).
#include <algorithm>

#include "chunk_common.cuh"
#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {
namespace prep {

using namespace chunkfmt;

constexpr int NT = 256;
constexpr int TSS = 68;      // fp32 row stride of the solve scratch
constexpr float LOG2E = 1.4426950408889634f;

// Shared memory (byte offsets from a 1024-aligned base); two CTAs fit on one SM.
constexpr uint32_t OFF_L = 0;                 // [q rows 0..63 | k rows 64..127] x 128 ch: 32 KB
constexpr uint32_t OFF_R = 32768;             // R_all: 160 rows x 128 ch: 40 KB
constexpr uint32_t OFF_SB = 0;                // diag(beta) A_kk fp32 [64][TSS] (after the intra MMA)
constexpr uint32_t OFF_ST = 64 * TSS * 4;     // T fp32 [64][TSS]
constexpr uint32_t OFF_TB = 35840;            // T_b [t][s] bf16, 8 KB
constexpr uint32_t OFF_KT = 73728;            // k e^{Gamma}: 16 KB
constexpr uint32_t OFF_V = 90112;             // v: 16 KB
constexpr uint32_t OFF_BETA = 106496;         // beta[64]
constexpr uint32_t OFF_WTOT = OFF_BETA + 256; // per-warp gate sums [8][128], then their prefixes
constexpr uint32_t OFF_RB = OFF_WTOT + 4096;  // Gamma at the end of blocks 0..3 [4][128]
constexpr uint32_t OFF_BAR = OFF_RB + 2048;   // mbarrier + TMEM address
constexpr uint32_t SMEM_BYTES = OFF_BAR + 64;
constexpr uint32_t SMEM_ALLOC = SMEM_BYTES + 1024;
static_assert(OFF_ST + 64 * TSS * 4 <= OFF_TB && OFF_TB + 8192 <= OFF_KT, "solve scratch overlaps");
static_assert(OFF_TB % 1024 == 0 && OFF_KT % 1024 == 0 && OFF_V % 1024 == 0, "SW128 alignment");
static_assert(2 * SMEM_ALLOC <= 231424, "two CTAs per SM");

// R_all rows: [0,64) diagonal-reference rows, then R_1 (16 rows), R_2 (32), R_3 (48).
__host__ __device__ constexpr int r_row0(int I) { return I == 1 ? 64 : (I == 2 ? 80 : 112); }

// TMEM columns (256 allocated): intra products; after they are read, W^T and U^T
constexpr uint32_t TM_P = 0;
constexpr uint32_t TM_W = 0;
constexpr uint32_t TM_U = 64;

constexpr uint32_t WAIT_POLLS = 1u << 22;

__device__ __forceinline__ bool wait_vote(uint64_t *bar, uint32_t parity, bool ok) {
  const bool mine = ok && umma::mbar_wait_bounded(bar, parity, WAIT_POLLS);
  const bool all = __syncthreads_and(mine) != 0;
  umma::fence_after_sync();
  return all;
}

__global__ void __launch_bounds__(NT, 2) chunk_prep_kernel(const __grid_constant__ PrepArgs a) {
  const int H = a.H;
  const int h = blockIdx.x % H;
  const int64_t gchunk = blockIdx.x / H;
  // locate (sequence, chunk): dense batches by division, varlen by the chunk table
  int n;
  int64_t cidx;
  if (a.chunk_cu == nullptr) {
    const int64_t per = (a.seq_len + CH - 1) / CH;
    if (per == 0 || gchunk >= per * a.N) return;
    n = (int)(gchunk / per);
    cidx = gchunk % per;
  } else {
    if (gchunk >= a.chunk_cu[a.N] || gchunk >= a.max_slots) return;
    int lo = 0, hi = a.N - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if ((int64_t)a.chunk_cu[mid] <= gchunk) lo = mid; else hi = mid - 1;
    }
    n = lo;
    cidx = gchunk - a.chunk_cu[n];
  }
  int64_t s0, s1;
  seq_bounds(a.cu, n, a.seq_len, a.total_tokens, s0, s1);
  const int64_t c0 = s0 + cidx * CH;
  if (c0 >= s1) return;   // only for malformed cu_seqlens / chunk tables

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  uint8_t *rec = reinterpret_cast<uint8_t *>(a.records) + (gchunk * H + h) * (int64_t)REC_STRIDE;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int cg = tid & 15, tg = tid >> 4, blkI = warp >> 1;   // tokens 4tg..4tg+3; block warp/2
  float *beta_s = reinterpret_cast<float *>(smem + OFF_BETA);
  float *wtot = reinterpret_cast<float *>(smem + OFF_WTOT);
  float *rbs = reinterpret_cast<float *>(smem + OFF_RB);
  float *sBm = reinterpret_cast<float *>(smem + OFF_SB);
  float *sTm = reinterpret_cast<float *>(smem + OFF_ST);
  uint64_t *bar = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + OFF_BAR + 8);
  const uint32_t sbase = umma::smem_u32(smem);
  const uint32_t lane_base = (uint32_t)(warp & 3) * 32u << 16;
  const __nv_bfloat16 *__restrict__ qn = reinterpret_cast<const __nv_bfloat16 *>(a.qn);
  const __nv_bfloat16 *__restrict__ kn = reinterpret_cast<const __nv_bfloat16 *>(a.kn);
  const __nv_bfloat16 *__restrict__ vc = reinterpret_cast<const __nv_bfloat16 *>(a.vc);

  // ---------------------------------------------------------------- loads (all issued first)
  uint4 qr[4], kr[4], vr[4];
  float g2[4][8];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int t = tg * 4 + j;
    const int64_t off = ((c0 + t) * H + h) * DK + cg * 8;
    if (c0 + t < s1) {
      qr[j] = __ldcs(reinterpret_cast<const uint4 *>(qn + off));
      kr[j] = __ldcs(reinterpret_cast<const uint4 *>(kn + off));
      vr[j] = __ldcs(reinterpret_cast<const uint4 *>(vc + off));
      const float4 ga = __ldcs(reinterpret_cast<const float4 *>(a.g + off));
      const float4 gb = __ldcs(reinterpret_cast<const float4 *>(a.g + off + 4));
      g2[j][0] = ga.x; g2[j][1] = ga.y; g2[j][2] = ga.z; g2[j][3] = ga.w;
      g2[j][4] = gb.x; g2[j][5] = gb.y; g2[j][6] = gb.z; g2[j][7] = gb.w;
    } else {
      qr[j] = kr[j] = vr[j] = make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int i = 0; i < 8; ++i) g2[j][i] = 0.f;
    }
  }
  float btj = 0.f;
  if (tid < 64 && c0 + tid < s1) btj = __ldcs(a.beta + (c0 + tid) * H + h);

  if (warp == 0) {
    umma::tmem_alloc(tmem_slot, 256);
    umma::tmem_relinquish();
  }
  if (tid == 32) {
    umma::mbar_init(bar, 1);
    umma::mbar_fence_init();
  }

  // ---------------------------------------------------------------- cumulative gate (base 2)
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    g2[0][i] *= LOG2E;
#pragma unroll
    for (int j = 1; j < 4; ++j) g2[j][i] = fmaf(g2[j][i], LOG2E, g2[j - 1][i]);
    const float lo = __shfl_up_sync(0xffffffffu, g2[3][i], 16);
    if (lane >= 16) {
#pragma unroll
      for (int j = 0; j < 4; ++j) g2[j][i] += lo;
    }
  }
  if (lane >= 16) {
    *reinterpret_cast<float4 *>(wtot + warp * 128 + cg * 8) = make_float4(g2[3][0], g2[3][1], g2[3][2], g2[3][3]);
    *reinterpret_cast<float4 *>(wtot + warp * 128 + cg * 8 + 4) = make_float4(g2[3][4], g2[3][5], g2[3][6], g2[3][7]);
  }
#pragma unroll
  for (int j = 0; j < 4; ++j)
    *reinterpret_cast<uint4 *>(smem + OFF_V + tr_off(64, tg * 4 + j, cg)) = vr[j];
  if (tid < 64) beta_s[tid] = btj;
  umma::fence_before_sync();
  __syncthreads();
  umma::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  // per channel: exclusive prefix of the warp sums (in place) and Gamma at block ends
  if (tid < 128) {
    float acc = 0.f;
#pragma unroll
    for (int w2 = 0; w2 < 8; ++w2) {
      const float x = wtot[w2 * 128 + tid];
      wtot[w2 * 128 + tid] = acc;
      acc += x;
      if (w2 & 1) rbs[(w2 >> 1) * 128 + tid] = acc;
    }
    reinterpret_cast<float *>(rec + REC_EGC)[tid] = umma::ex2(acc);   // e^{Gamma_C}
  }
  __syncthreads();

  // ---------------------------------------------------------------- operands
  {
    float rI[8], rI1[8], rC[8];
    {
      const float4 p0 = *reinterpret_cast<const float4 *>(wtot + warp * 128 + cg * 8);
      const float4 p1 = *reinterpret_cast<const float4 *>(wtot + warp * 128 + cg * 8 + 4);
      const float pre[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
      for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int i = 0; i < 8; ++i) g2[j][i] += pre[i];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        rI[i] = blkI == 0 ? 0.f : rbs[(blkI - 1) * 128 + cg * 8 + i];
        rI1[i] = rbs[blkI * 128 + cg * 8 + i];
        rC[i] = rbs[3 * 128 + cg * 8 + i];
      }
    }
    float eR[8], cK[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      eR[i] = umma::ex2(rI[i]);            // e^{r_I}
      cK[i] = umma::ex2(rC[i] - rI1[i]);   // e^{Gamma_C - r_{I+1}}
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int t = tg * 4 + j;
      float q[8], k[8], Lq[8], Lk[8], Rd[8], Qt[8], Kt[8], Kh[8], u[8];
      unpack8(qr[j], q);
      unpack8(kr[j], k);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float e1 = umma::ex2(g2[j][i] - rI[i]);    // <= 1
        const float rd = umma::ex2(rI[i] - g2[j][i]);    // in [1, 2^116)
        u[i] = umma::ex2(rI1[i] - g2[j][i]);             // e^{r_{I+1} - Gamma_t} in (0, 1]
        Lq[i] = q[i] * e1;
        Lk[i] = k[i] * e1;
        Rd[i] = k[i] * rd;
        Qt[i] = Lq[i] * eR[i];
        Kt[i] = Lk[i] * eR[i];
        Kh[i] = k[i] * u[i] * cK[i];                      // e^{Gamma_C - Gamma_t}
      }
      *reinterpret_cast<uint4 *>(smem + OFF_L + tr_off(128, t, cg)) = pack8(Lq);
      *reinterpret_cast<uint4 *>(smem + OFF_L + tr_off(128, 64 + t, cg)) = pack8(Lk);
      *reinterpret_cast<uint4 *>(smem + OFF_R + tr_off(160, t, cg)) = pack8(Rd);
      *reinterpret_cast<uint4 *>(smem + OFF_KT + tr_off(64, t, cg)) = pack8(Kt);
      *reinterpret_cast<uint4 *>(rec + REC_QT + tr_off(64, t, cg)) = pack8(Qt);
      *reinterpret_cast<uint4 *>(rec + REC_KH + tr_off(64, t, cg)) = pack8(Kh);
#pragma unroll
      for (int ip = 1; ip < 4; ++ip) {   // rows of R_ip (reference r_ip) for later blocks
        if (ip > blkI) {
          float Rx[8];
#pragma unroll
          for (int i = 0; i < 8; ++i)
            Rx[i] = k[i] * umma::ex2(rbs[(ip - 1) * 128 + cg * 8 + i] - g2[j][i]);   // e^{r_ip - Gamma_t} <= 1
          *reinterpret_cast<uint4 *>(smem + OFF_R + tr_off(160, r_row0(ip) + t, cg)) = pack8(Rx);
        }
      }
    }
  }
  umma::fence_proxy_async_smem();
  __syncthreads();

  // ---------------------------------------------------------------- intra MMA
  bool ok = true;
  uint32_t phase = 0;
  if (tid == 0) {
    umma::fence_after_sync();
    const uint32_t idesc = umma::make_idesc_bf16(128, 160, 0, 0);
#pragma unroll
    for (int s = 0; s < DK / 16; ++s)
      umma::mma_ss(tmem + TM_P, desc_k128(sbase + OFF_L, 128, s), desc_k128(sbase + OFF_R, 160, s),
                   idesc, s > 0);
    umma::mma_commit(bar);
  }
  ok = wait_vote(bar, phase, ok);
  phase ^= 1u;

  // ---------------------------------------------------------------- A_qk (bf16) and diag(beta) A_kk
  if (ok && warp < 4) {
    const int r = warp * 32 + lane;
    const int t = r & 63;
    const bool is_q = r < 64;
    const int I = t >> 4;
    float rowv[64];
#pragma unroll
    for (int s = 0; s < 64; ++s) rowv[s] = 0.f;
    // P columns in 16-wide groups: 0..3 diagonal blocks, 4 = R_1, 5..6 = R_2, 7..9 = R_3.
    // tcgen05.ld is warp-uniform: every lane loads every group and keeps its own.
#pragma unroll
    for (int c32 = 0; c32 < 5; ++c32) {
      uint32_t rr[32];
      umma::tmem_ld32(tmem + lane_base + TM_P + c32 * 32, rr);
      umma::tmem_wait_ld();
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int cc = c32 * 2 + half;
        const int want = cc < 4 ? cc : (cc == 4 ? 1 : (cc < 7 ? 2 : 3));
        const int sblk = cc < 4 ? cc : (cc == 4 ? 0 : (cc < 7 ? cc - 5 : cc - 7));
        if (I == want) {
#pragma unroll
          for (int e = 0; e < 16; ++e) rowv[sblk * 16 + e] = __uint_as_float(rr[half * 16 + e]);
        }
      }
    }
    if (is_q) {
#pragma unroll
      for (int c8 = 0; c8 < 8; ++c8) {
        float x8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) x8[i] = (c8 * 8 + i <= t) ? rowv[c8 * 8 + i] : 0.f;
        *reinterpret_cast<uint4 *>(rec + REC_AQ + tr_off(64, t, c8)) = pack8(x8);
      }
    } else {
      const float bt = beta_s[t];
#pragma unroll
      for (int s4 = 0; s4 < 16; ++s4) {
        float4 v;
        v.x = (4 * s4 + 0 < t) ? rowv[4 * s4 + 0] * bt : 0.f;
        v.y = (4 * s4 + 1 < t) ? rowv[4 * s4 + 1] * bt : 0.f;
        v.z = (4 * s4 + 2 < t) ? rowv[4 * s4 + 2] * bt : 0.f;
        v.w = (4 * s4 + 3 < t) ? rowv[4 * s4 + 3] * bt : 0.f;
        *reinterpret_cast<float4 *>(sBm + t * TSS + 4 * s4) = v;
      }
    }
  }
  umma::fence_before_sync();
  __syncthreads();

  // ---------------------------------------------------------------- T = (I + B)^{-1}
  if (warp < 4) {  // diagonal 16x16 blocks: warp = block, lane = column (lanes 16..31 mirror)
    const int o16 = warp * 16, cidx2 = lane & 15;
    float x[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) {
      float acc = 0.f;
#pragma unroll
      for (int m = 0; m < r; ++m) acc = fmaf(sBm[(o16 + r) * TSS + o16 + m], x[m], acc);
      x[r] = r < cidx2 ? 0.f : (r == cidx2 ? 1.f : -acc);
    }
    if (lane < 16) {
#pragma unroll
      for (int r = 0; r < 16; ++r) sTm[(o16 + r) * TSS + o16 + cidx2] = x[r];
    }
  }
  __syncthreads();
  // Off-diagonal blocks by distance d = I - J: X_IJ = sum_K B_IK T_KJ (kept in the unused
  // upper block (J, I)), then T_IJ = -T_II X_IJ.  B rows are read as float4.
#pragma unroll
  for (int d = 1; d < 4; ++d) {
    for (int e = tid; e < (4 - d) * 256; e += NT) {
      const int J = e >> 8, I = J + d, r = (e >> 4) & 15, cc = e & 15;
      float acc = 0.f;
#pragma unroll
      for (int kb = 0; kb < d; ++kb) {
        const int K = J + kb;
        const float4 *brow = reinterpret_cast<const float4 *>(sBm + (I * 16 + r) * TSS + K * 16);
#pragma unroll
        for (int m4 = 0; m4 < 4; ++m4) {
          const float4 bv = brow[m4];
          acc = fmaf(bv.x, sTm[(K * 16 + 4 * m4 + 0) * TSS + J * 16 + cc], acc);
          acc = fmaf(bv.y, sTm[(K * 16 + 4 * m4 + 1) * TSS + J * 16 + cc], acc);
          acc = fmaf(bv.z, sTm[(K * 16 + 4 * m4 + 2) * TSS + J * 16 + cc], acc);
          acc = fmaf(bv.w, sTm[(K * 16 + 4 * m4 + 3) * TSS + J * 16 + cc], acc);
        }
      }
      sBm[(J * 16 + r) * TSS + I * 16 + cc] = acc;
    }
    __syncthreads();
    for (int e = tid; e < (4 - d) * 256; e += NT) {
      const int J = e >> 8, I = J + d, r = (e >> 4) & 15, cc = e & 15;
      const float4 *trow = reinterpret_cast<const float4 *>(sTm + (I * 16 + r) * TSS + I * 16);
      float acc = 0.f;
#pragma unroll
      for (int m4 = 0; m4 < 4; ++m4) {
        const float4 tv = trow[m4];   // row r of T_II (entries right of the diagonal masked)
        const int m = 4 * m4;
        acc = fmaf(m + 0 <= r ? tv.x : 0.f, sBm[(J * 16 + m + 0) * TSS + I * 16 + cc], acc);
        acc = fmaf(m + 1 <= r ? tv.y : 0.f, sBm[(J * 16 + m + 1) * TSS + I * 16 + cc], acc);
        acc = fmaf(m + 2 <= r ? tv.z : 0.f, sBm[(J * 16 + m + 2) * TSS + I * 16 + cc], acc);
        acc = fmaf(m + 3 <= r ? tv.w : 0.f, sBm[(J * 16 + m + 3) * TSS + I * 16 + cc], acc);
      }
      sTm[(I * 16 + r) * TSS + J * 16 + cc] = -acc;
    }
    __syncthreads();
  }
#pragma unroll
  for (int it = 0; it < 2; ++it) {  // T_b rows as bf16, K-major [t][s]
    const int e = tid + it * NT;
    const int t = e >> 3, c8 = e & 7;
    float x8[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int s = c8 * 8 + i;
      x8[i] = s <= t ? sTm[t * TSS + s] * beta_s[s] : 0.f;
    }
    *reinterpret_cast<uint4 *>(smem + OFF_TB + tr_off(64, t, c8)) = pack8(x8);
  }
  umma::fence_proxy_async_smem();
  umma::fence_before_sync();
  __syncthreads();

  // ---------------------------------------------------------------- W^T, U^T (P has been read)
  if (tid == 0) {
    umma::fence_after_sync();
    const uint32_t idesc = umma::make_idesc_bf16(128, 64, 1, 0);
#pragma unroll
    for (int s = 0; s < CH / 16; ++s) {
      umma::mma_ss(tmem + TM_W, desc_mn_tok(sbase + OFF_KT, s), desc_k64(sbase + OFF_TB, s), idesc, s > 0);
      umma::mma_ss(tmem + TM_U, desc_mn_tok(sbase + OFF_V, s), desc_k64(sbase + OFF_TB, s), idesc, s > 0);
    }
    umma::mma_commit(bar);
  }
  ok = wait_vote(bar, phase, ok);

  // ---------------------------------------------------------------- -W^T (warps 0-3), U^T (4-7) rows
  if (ok) {
    const int i = (warp & 3) * 32 + lane;   // TMEM lane: key channel (W^T) / value channel (U^T)
    const bool isW = warp < 4;
    const float sign = isW ? -1.f : 1.f;
    uint8_t *dst = rec + (isW ? REC_WT : REC_U);
#pragma unroll
    for (int c32 = 0; c32 < 2; ++c32) {
      uint32_t rr[32];
      umma::tmem_ld32(tmem + lane_base + (isW ? TM_W : TM_U) + c32 * 32, rr);
      umma::tmem_wait_ld();
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        float x8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) x8[e] = sign * __uint_as_float(rr[q4 * 8 + e]);
        *reinterpret_cast<uint4 *>(dst + row64_off(i, c32 * 4 + q4)) = pack8(x8);
      }
    }
  }
  if (!ok && tid == 0 && a.err) atomicExch(a.err, ERR_TIMEOUT);
  umma::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    umma::fence_after_sync();
    umma::tmem_dealloc(tmem, 256);
  }
}

// chunk_cu[n] = number of 64-token chunks in sequences 0..n-1 (one thread; N is small).
__global__ void chunk_table_kernel(const int32_t *cu, int N, int64_t total, int32_t *chunk_cu) {
  if (blockIdx.x != 0 || threadIdx.x != 0) return;
  int32_t acc = 0;
  for (int n = 0; n < N; ++n) {
    int64_t s, e;
    seq_bounds(cu, n, 0, total, s, e);
    chunk_cu[n] = acc;
    acc += (int32_t)((e - s + CH - 1) / CH);
  }
  chunk_cu[N] = acc;
}

}  // namespace prep

static_assert(kChunkRecordBytes == chunkfmt::REC_STRIDE, "record size");

cudaError_t launch_chunk_table(const int32_t *cu, int N, int64_t total, int32_t *chunk_cu,
                               cudaStream_t stream) {
  prep::chunk_table_kernel<<<1, 32, 0, stream>>>(cu, N, total, chunk_cu);
  return cudaGetLastError();
}

cudaError_t launch_chunk_prep(PrepArgs a, int64_t max_chunks, cudaStream_t stream) {
  if (max_chunks == 0 || a.H == 0) return cudaSuccess;
  a.max_slots = max_chunks;
  cudaError_t e = cudaFuncSetAttribute(prep::chunk_prep_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)prep::SMEM_ALLOC);
  if (e != cudaSuccess) return e;
  prep::chunk_prep_kernel<<<(unsigned)(max_chunks * a.H), prep::NT, prep::SMEM_ALLOC, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace kda
