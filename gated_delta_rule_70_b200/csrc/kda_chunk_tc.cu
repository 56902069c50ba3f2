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
// overflows fp32.  The pairwise factor e^{Gamma_t - Gamma_s} is only ever split
// around a reference point close to both tokens: 16-token sub-blocks I with
// r_I = Gamma at the end of block I-1.  Diagonal blocks use (q|k)_t
// e^{Gamma_t - r_I} against k_s e^{r_I - Gamma_s} (factors within e^{+-80}); a
// row in block I against earlier blocks uses r_I on both sides (factors <= 1).
// Exponentials run on the special-function unit in base 2 (gates are scaled by
// log2 e once); every other decay factor is a product of per-block constants
// ordered so that no intermediate leaves the fp32 range.
//
// Layout: the 128-wide dimension always sits on the MMA's M = 128 axis.  The
// state is kept transposed, S^T [d_v lanes x d_k columns] fp32 in TMEM, with a
// bf16 copy in TMEM as the A operand of S^T W^T and S^T Q~^T; D^T lives in TMEM
// the same way.  Shared-memory operands share one format: token rows of 128
// channels, 128-byte swizzle, 64-channel atoms, read by a descriptor as K-major
// (K = channels) or MN-major (MN = channels, K = tokens).
//
// Pipeline (warp specialization, 384 threads):
//   stage A, warps 0-7: loads, cumulative gate, operands; intra MMA; A_qk and
//     diag(beta) A_kk; the 64x64 unit-lower-triangular solve; W^T, U^T MMAs
//     -- everything that does not depend on the state, one chunk ahead;
//   stage B, warps 8-11: D^T = U^T - S^T W^T, O^T, the state update and the
//     output store -- the sequential chain through S.
// Stage A hands chunk c to stage B through mbarriers; the operands stage B
// reads (Q~, K^, A_qk, e^{Gamma_C}) are double-buffered by chunk parity, and the
// L / R operand region is reused for the solve once the intra MMA has read it.
#include "kda_common.cuh"
#include "kda_internal.h"
#include "umma.cuh"

namespace kda {
namespace chunk {

constexpr int CH = 64;       // tokens per chunk
constexpr int DK = 128;      // head dim (d_k = d_v)
constexpr int NT = 384;      // threads per CTA
constexpr int NTA = 256;     // stage A threads (warps 0-7)
constexpr int NTB = 128;     // stage B threads (warps 8-11)
constexpr int TSS = 68;      // fp32 row stride of the solve scratch
constexpr float LOG2E = 1.4426950408889634f;

// Shared memory (byte offsets from a 1024-aligned base)
constexpr uint32_t OFF_L = 0;                 // [q rows 0..63 | k rows 64..127] x 128 ch: 32 KB
constexpr uint32_t OFF_R = 32768;             // R_all: 160 rows x 128 ch: 40 KB
constexpr uint32_t OFF_SB = 0;                // diag(beta) A_kk fp32 [64][TSS] (after the intra MMA)
constexpr uint32_t OFF_ST = 64 * TSS * 4;     // T fp32 [64][TSS]
constexpr uint32_t OFF_TB = 35840;            // T_b [t][s] bf16, 8 KB
constexpr uint32_t OFF_KT = 73728;            // k e^{Gamma}: 16 KB
constexpr uint32_t OFF_V = 90112;             // v: 16 KB
constexpr uint32_t OFF_QT = 106496;           // q e^{Gamma}: 2 x 16 KB (chunk parity)
constexpr uint32_t OFF_KH = 139264;           // k e^{Gamma_C - Gamma}: 2 x 16 KB
constexpr uint32_t OFF_AQ = 172032;           // A_qk [t][s] bf16: 2 x 8 KB
constexpr uint32_t OFF_WT = 188416;           // -W^T [i][t] bf16 (MN-major B): 16 KB
constexpr uint32_t OFF_BETA = 204800;         // beta[64]
constexpr uint32_t OFF_EGC = OFF_BETA + 256;  // e^{Gamma_C}: 2 x 128
constexpr uint32_t OFF_WTOT = OFF_EGC + 1024; // per-warp gate sums [8][128]
constexpr uint32_t OFF_BAR = OFF_WTOT + 4096; // mbarriers + TMEM address
constexpr uint32_t SMEM_BYTES = OFF_BAR + 128;
constexpr uint32_t SMEM_ALLOC = SMEM_BYTES + 1024;
static_assert(OFF_ST + 64 * TSS * 4 <= OFF_TB && OFF_TB + 8192 <= OFF_KT, "solve scratch overlaps");
static_assert(OFF_TB % 1024 == 0 && OFF_KT % 1024 == 0 && OFF_WT % 1024 == 0, "SW128 alignment");
static_assert(SMEM_ALLOC <= 232448, "shared memory budget");

// R_all rows: [0,64) diagonal-reference rows, then R_1 (16 rows), R_2 (32), R_3 (48).
__host__ __device__ constexpr int r_row0(int I) { return I == 1 ? 64 : (I == 2 ? 80 : 112); }

// TMEM columns (512 allocated)
constexpr uint32_t TM_S32 = 0;     // S^T fp32, 128 cols
constexpr uint32_t TM_S16 = 128;   // S^T bf16 A operand, 64 cols
constexpr uint32_t TM_D = 192;     // U^T, then D^T (fp32), 64 cols
constexpr uint32_t TM_D16 = 256;   // D^T bf16 A operand, 32 cols
constexpr uint32_t TM_O = 288;     // O^T fp32, 64 cols
constexpr uint32_t TM_P = 352;     // intra products, 160 cols; later W^T (first 64)
constexpr uint32_t TM_W = 352;

constexpr uint32_t WAIT_POLLS = 1u << 22;   // bounded mbarrier waits

enum Bar { B_MMA_A = 0, B_MMA_B, B_FULL0, B_FULL1, B_EMPTY0, B_EMPTY1, B_DFREE, B_COUNT };

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
__device__ __forceinline__ void unpack8(const uint4 &u, float (&x)[8]) {
  const __nv_bfloat162 *hh = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __bfloat1622float2(hh[i]);
    x[2 * i] = f.x;
    x[2 * i + 1] = f.y;
  }
}

__device__ __forceinline__ uint64_t desc_k128(uint32_t base, int rows, int s) {
  return umma::make_desc(base + (uint32_t)((s >> 2) * rows * 128 + (s & 3) * 32), 16, 1024,
                         umma::LAYOUT_SW128);
}
__device__ __forceinline__ uint64_t desc_mn_tok(uint32_t base, int s) {
  return umma::make_desc(base + (uint32_t)(s * 2048), 64 * 128, 1024, umma::LAYOUT_SW128);
}
__device__ __forceinline__ uint64_t desc_k64(uint32_t base, int s) {
  return umma::make_desc(base + (uint32_t)(s * 32), 16, 1024, umma::LAYOUT_SW128);
}
__device__ __forceinline__ uint64_t desc_mn_wt(uint32_t base, int s) {
  return umma::make_desc(base + (uint32_t)(s * 2048), 128 * 128, 1024, umma::LAYOUT_SW128);
}

struct Shared {
  uint8_t *smem;
  uint32_t sbase, tmem;
  uint64_t *bar;
  int *err;
};

// Bounded wait, then a warp-group vote so every thread of the group agrees.
__device__ __forceinline__ bool wait_vote(uint64_t *bar, uint32_t parity, bool ok, uint32_t bar_id,
                                          uint32_t nthreads) {
  const bool mine = ok && umma::mbar_wait_bounded(bar, parity, WAIT_POLLS);
  const bool all = umma::named_sync_and(bar_id, nthreads, mine);
  umma::fence_after_sync();
  return all;
}

// --------------------------------------------------------------------- stage A helpers

// Operand rows for this thread's 4 tokens; sub-block I known at compile time.
// g2[j][i]: cumulative gate in base 2 at token j (chunk-relative), channel i;
// rb[m][i]: its value at the end of block m-1 (rb[0] = 0, rb[4] = Gamma_C).
template <int I>
__device__ __forceinline__ void emit_operands(uint8_t *smem, int b, int tg, int cg,
                                              const uint4 (&qr)[4], const uint4 (&kr)[4],
                                              const float (&g2)[4][8], const float (&rb)[5][8]) {
  float eR[8], bd[8], cl[4 - I][8];  // cl[m]: 2^{rb[I+1+m] - rb[I+1]}
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    eR[i] = umma::ex2(rb[I][i]);
    bd[i] = umma::ex2(rb[I + 1][i] - rb[I][i]);
#pragma unroll
    for (int m = 0; m < 4 - I; ++m) cl[m][i] = umma::ex2(rb[I + 1 + m][i] - rb[I + 1][i]);
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int t = tg * 4 + j;
    float q[8], k[8], Lq[8], Lk[8], Rd[8], Qt[8], Kt[8], Kh[8], u[8];
    unpack8(qr[j], q);
    unpack8(kr[j], k);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float e1 = umma::ex2(g2[j][i] - rb[I][i]);   // <= 1
      const float rd = umma::ex2(rb[I][i] - g2[j][i]);   // in [1, 2^116)
      Lq[i] = q[i] * e1;
      Lk[i] = k[i] * e1;
      Rd[i] = k[i] * rd;
      Qt[i] = Lq[i] * eR[i];
      Kt[i] = Lk[i] * eR[i];
      u[i] = rd * bd[i];                                  // e^{r_{I+1} - Gamma_t} in (0, 1]
      Kh[i] = k[i] * u[i] * cl[3 - I][i];                 // e^{Gamma_C - Gamma_t}
    }
    *reinterpret_cast<uint4 *>(smem + OFF_L + tr_off(128, t, cg)) = pack8(Lq);
    *reinterpret_cast<uint4 *>(smem + OFF_L + tr_off(128, 64 + t, cg)) = pack8(Lk);
    *reinterpret_cast<uint4 *>(smem + OFF_R + tr_off(160, t, cg)) = pack8(Rd);
    *reinterpret_cast<uint4 *>(smem + OFF_QT + b * 16384 + tr_off(64, t, cg)) = pack8(Qt);
    *reinterpret_cast<uint4 *>(smem + OFF_KT + tr_off(64, t, cg)) = pack8(Kt);
    *reinterpret_cast<uint4 *>(smem + OFF_KH + b * 16384 + tr_off(64, t, cg)) = pack8(Kh);
#pragma unroll
    for (int ip = I + 1; ip < 4; ++ip) {   // rows of R_ip (reference r_ip) for later blocks
      float Rx[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) Rx[i] = k[i] * u[i] * cl[ip - I - 1][i];
      *reinterpret_cast<uint4 *>(smem + OFF_R + tr_off(160, r_row0(ip) + t, cg)) = pack8(Rx);
    }
  }
}

__device__ void stage_a(const RecurrenceArgs &a, const Shared &sh, int h, int64_t s0, int64_t s1,
                        int nchunks) {
  uint8_t *smem = sh.smem;
  uint64_t *bar = sh.bar;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int cg = tid & 15, tg = tid >> 4, blkI = warp >> 1;
  const int H = a.H;
  float *beta_s = reinterpret_cast<float *>(smem + OFF_BETA);
  float *wtot = reinterpret_cast<float *>(smem + OFF_WTOT);
  float *sBm = reinterpret_cast<float *>(smem + OFF_SB);
  float *sTm = reinterpret_cast<float *>(smem + OFF_ST);
  const uint32_t lane_base = (uint32_t)(warp & 3) * 32u << 16;
  const __nv_bfloat16 *__restrict__ qn = reinterpret_cast<const __nv_bfloat16 *>(a.qn);
  const __nv_bfloat16 *__restrict__ kn = reinterpret_cast<const __nv_bfloat16 *>(a.kn);
  const __nv_bfloat16 *__restrict__ vc = reinterpret_cast<const __nv_bfloat16 *>(a.vc);
  uint32_t ph_mma = 0;
  bool ok = true;

  auto prefetch_chunk = [&](int c) {  // one bulk L2 prefetch per (token row, tensor)
    const int t = tid & 63, which = tid >> 6;
    const int64_t row = s0 + (int64_t)c * CH + t;
    if (row < s1) {
      const int64_t off = (row * H + h) * DK;
      if (which == 0) umma::prefetch_l2(qn + off, 256);
      else if (which == 1) umma::prefetch_l2(kn + off, 256);
      else if (which == 2) umma::prefetch_l2(vc + off, 256);
      else umma::prefetch_l2(a.g + off, 512);
    }
  };
  prefetch_chunk(0);

#pragma unroll 1
  for (int c = 0; c < nchunks; ++c) {
    const int b = c & 1;
    const int64_t c0 = s0 + (int64_t)c * CH;
    // ---------------------------------------------------------------- loads (all issued first)
    uint4 qr[4], kr[4], vr[4];
    float g2[4][8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int t = tg * 4 + j;
      const int64_t off = ((c0 + t) * H + h) * DK + cg * 8;
      if (c0 + t < s1) {
        qr[j] = __ldg(reinterpret_cast<const uint4 *>(qn + off));
        kr[j] = __ldg(reinterpret_cast<const uint4 *>(kn + off));
        vr[j] = __ldg(reinterpret_cast<const uint4 *>(vc + off));
        const float4 ga = __ldg(reinterpret_cast<const float4 *>(a.g + off));
        const float4 gb = __ldg(reinterpret_cast<const float4 *>(a.g + off + 4));
        g2[j][0] = ga.x; g2[j][1] = ga.y; g2[j][2] = ga.z; g2[j][3] = ga.w;
        g2[j][4] = gb.x; g2[j][5] = gb.y; g2[j][6] = gb.z; g2[j][7] = gb.w;
      } else {
        qr[j] = kr[j] = vr[j] = make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int i = 0; i < 8; ++i) g2[j][i] = 0.f;
      }
    }
    float btj[4] = {0.f, 0.f, 0.f, 0.f};
    if (cg == 0) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int64_t row = c0 + tg * 4 + j;
        if (row < s1) btj[j] = __ldg(a.beta + row * H + h);
      }
    }
    if (c + 1 < nchunks) prefetch_chunk(c + 1);
    // buffers of parity b are free once stage B has finished chunk c-2
    if (c >= 2) {
      ok = wait_vote(&bar[B_EMPTY0 + b], ((c - 2) >> 1) & 1, ok, 1, NTA);
      if (!ok) break;
    }
    // ---------------------------------------------------------------- cumulative gate (base 2)
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int i = 0; i < 8; ++i) g2[j][i] *= LOG2E;
#pragma unroll
    for (int j = 1; j < 4; ++j)
#pragma unroll
      for (int i = 0; i < 8; ++i) g2[j][i] += g2[j - 1][i];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float lo = __shfl_up_sync(0xffffffffu, g2[3][i], 16);
      if (lane >= 16) {
#pragma unroll
        for (int j = 0; j < 4; ++j) g2[j][i] += lo;
      }
    }
    if (lane >= 16) {
      *reinterpret_cast<float4 *>(wtot + warp * 128 + cg * 8) =
          make_float4(g2[3][0], g2[3][1], g2[3][2], g2[3][3]);
      *reinterpret_cast<float4 *>(wtot + warp * 128 + cg * 8 + 4) =
          make_float4(g2[3][4], g2[3][5], g2[3][6], g2[3][7]);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j)
      *reinterpret_cast<uint4 *>(smem + OFF_V + tr_off(64, tg * 4 + j, cg)) = vr[j];
    if (cg == 0) {
#pragma unroll
      for (int j = 0; j < 4; ++j) beta_s[tg * 4 + j] = btj[j];
    }
    umma::named_sync(1, NTA);
    // prefix over earlier warps; rb[m] = Gamma at the end of block m-1
    float rb[5][8], pre[8];
    {
      float acc[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) { acc[i] = 0.f; rb[0][i] = 0.f; pre[i] = 0.f; }
#pragma unroll
      for (int w2 = 0; w2 < 8; ++w2) {
        const float4 x0 = *reinterpret_cast<const float4 *>(wtot + w2 * 128 + cg * 8);
        const float4 x1 = *reinterpret_cast<const float4 *>(wtot + w2 * 128 + cg * 8 + 4);
        const float x[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (w2 == warp) pre[i] = acc[i];
          acc[i] += x[i];
          if (w2 & 1) rb[(w2 + 1) >> 1][i] = acc[i];
        }
      }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int i = 0; i < 8; ++i) g2[j][i] += pre[i];
    if (tid < 16) {
      float *egc = reinterpret_cast<float *>(smem + OFF_EGC) + b * 128;
      *reinterpret_cast<float4 *>(egc + tid * 8) =
          make_float4(umma::ex2(rb[4][0]), umma::ex2(rb[4][1]), umma::ex2(rb[4][2]), umma::ex2(rb[4][3]));
      *reinterpret_cast<float4 *>(egc + tid * 8 + 4) =
          make_float4(umma::ex2(rb[4][4]), umma::ex2(rb[4][5]), umma::ex2(rb[4][6]), umma::ex2(rb[4][7]));
    }
    switch (blkI) {  // warp-uniform
      case 0: emit_operands<0>(smem, b, tg, cg, qr, kr, g2, rb); break;
      case 1: emit_operands<1>(smem, b, tg, cg, qr, kr, g2, rb); break;
      case 2: emit_operands<2>(smem, b, tg, cg, qr, kr, g2, rb); break;
      default: emit_operands<3>(smem, b, tg, cg, qr, kr, g2, rb); break;
    }
    umma::fence_proxy_async_smem();
    umma::named_sync(1, NTA);

    // ---------------------------------------------------------------- intra MMA
    if (tid == 0) {
      umma::fence_after_sync();
      const uint32_t idesc = umma::make_idesc_bf16(128, 160, 0, 0);
#pragma unroll
      for (int s = 0; s < DK / 16; ++s)
        umma::mma_ss(sh.tmem + TM_P, desc_k128(sh.sbase + OFF_L, 128, s),
                     desc_k128(sh.sbase + OFF_R, 160, s), idesc, s > 0);
      umma::mma_commit(&bar[B_MMA_A]);
    }
    ok = wait_vote(&bar[B_MMA_A], ph_mma, ok, 1, NTA);
    ph_mma ^= 1u;
    if (!ok) break;

    // ---------------------------------------------------------------- A_qk (bf16) and diag(beta) A_kk
    if (warp < 4) {
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
        umma::tmem_ld32(sh.tmem + lane_base + TM_P + c32 * 32, rr);
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
        uint8_t *aq = smem + OFF_AQ + b * 8192;
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) {
          float x8[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) x8[i] = (c8 * 8 + i <= t) ? rowv[c8 * 8 + i] : 0.f;
          *reinterpret_cast<uint4 *>(aq + tr_off(64, t, c8)) = pack8(x8);
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
    umma::named_sync(1, NTA);

    // ---------------------------------------------------------------- T = (I + B)^{-1}
    if (warp < 4) {  // diagonal 16x16 blocks: warp = block, lane = column (lanes 16..31 mirror)
      const int o16 = warp * 16, cidx = lane & 15;
      float x[16];
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        float acc = 0.f;
#pragma unroll
        for (int m = 0; m < r; ++m) acc = fmaf(sBm[(o16 + r) * TSS + o16 + m], x[m], acc);
        // column cidx of the inverse: 0 above the diagonal, 1 on it, forward substitution below
        x[r] = r < cidx ? 0.f : (r == cidx ? 1.f : -acc);
      }
      if (lane < 16) {
#pragma unroll
        for (int r = 0; r < 16; ++r) sTm[(o16 + r) * TSS + o16 + cidx] = x[r];
      }
    }
    umma::named_sync(1, NTA);
#pragma unroll 1
    for (int d = 1; d < 4; ++d) {
      // X_IJ = sum_{K=J}^{I-1} B_IK T_KJ, kept in the unused upper block (J, I) of sBm
      for (int e = tid; e < (4 - d) * 256; e += NTA) {
        const int J = e >> 8, I = J + d, r = (e >> 4) & 15, cc = e & 15;
        float acc = 0.f;
        for (int K = J; K < I; ++K) {
#pragma unroll
          for (int m = 0; m < 16; ++m)
            acc = fmaf(sBm[(I * 16 + r) * TSS + K * 16 + m], sTm[(K * 16 + m) * TSS + J * 16 + cc], acc);
        }
        sBm[(J * 16 + r) * TSS + I * 16 + cc] = acc;
      }
      umma::named_sync(1, NTA);
      // T_IJ = -T_II X_IJ
      for (int e = tid; e < (4 - d) * 256; e += NTA) {
        const int J = e >> 8, I = J + d, r = (e >> 4) & 15, cc = e & 15;
        float acc = 0.f;
#pragma unroll
        for (int m = 0; m < 16; ++m) {
          const float tv = m <= r ? sTm[(I * 16 + r) * TSS + I * 16 + m] : 0.f;
          acc = fmaf(tv, sBm[(J * 16 + m) * TSS + I * 16 + cc], acc);
        }
        sTm[(I * 16 + r) * TSS + J * 16 + cc] = -acc;
      }
      umma::named_sync(1, NTA);
    }
    for (int e = tid; e < 64 * 8; e += NTA) {  // T_b rows as bf16, K-major [t][s]
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
    umma::named_sync(1, NTA);

    // ---------------------------------------------------------------- W^T, U^T
    // U^T goes to the D region: stage B must be done with chunk c-1's D^T (and W^T).
    if (c >= 1) {
      ok = wait_vote(&bar[B_DFREE], (c - 1) & 1, ok, 1, NTA);
      if (!ok) break;
    }
    if (tid == 0) {
      const uint32_t idesc = umma::make_idesc_bf16(128, 64, 1, 0);
#pragma unroll
      for (int s = 0; s < CH / 16; ++s) {
        umma::mma_ss(sh.tmem + TM_W, desc_mn_tok(sh.sbase + OFF_KT, s),
                     desc_k64(sh.sbase + OFF_TB, s), idesc, s > 0);
        umma::mma_ss(sh.tmem + TM_D, desc_mn_tok(sh.sbase + OFF_V, s),
                     desc_k64(sh.sbase + OFF_TB, s), idesc, s > 0);
      }
      umma::mma_commit(&bar[B_MMA_A]);
    }
    ok = wait_vote(&bar[B_MMA_A], ph_mma, ok, 1, NTA);
    ph_mma ^= 1u;
    if (!ok) break;

    // ---------------------------------------------------------------- -W^T to smem (rows = channel)
    if (warp < 4) {
      const int i = warp * 32 + lane;
#pragma unroll
      for (int c32 = 0; c32 < 2; ++c32) {
        uint32_t rr[32];
        umma::tmem_ld32(sh.tmem + lane_base + TM_W + c32 * 32, rr);
        umma::tmem_wait_ld();
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const int c8 = c32 * 4 + q4;
          float x8[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) x8[e] = -__uint_as_float(rr[q4 * 8 + e]);
          *reinterpret_cast<uint4 *>(smem + OFF_WT + (uint32_t)((i >> 3) * 1024 + (i & 7) * 128 +
                                                               ((c8 ^ (i & 7)) << 4))) = pack8(x8);
        }
      }
    }
    umma::fence_proxy_async_smem();
    umma::fence_before_sync();
    umma::named_sync(1, NTA);
    if (tid == 0) umma::mbar_arrive(&bar[B_FULL0 + b]);
  }
  if (!ok && tid == 0 && sh.err) atomicExch(sh.err, ERR_TIMEOUT);
}

// --------------------------------------------------------------------- stage B

__device__ void stage_b(const RecurrenceArgs &a, const Shared &sh, int n, int h, int64_t s0,
                        int64_t s1, int nchunks) {
  uint8_t *smem = sh.smem;
  uint64_t *bar = sh.bar;
  const int tb = threadIdx.x - NTA;          // 0..127
  const int wb = tb >> 5;
  const int j = tb;                          // TMEM lane: value channel of S^T, D^T, O^T
  const uint32_t lane_base = (uint32_t)wb * 32u << 16;
  const int H = a.H;
  const int64_t sg = ((int64_t)n * H + h) * DK * DK;
  __nv_bfloat16 *__restrict__ o = reinterpret_cast<__nv_bfloat16 *>(a.o);
  uint32_t ph_mma = 0;
  bool ok = true;

  // initial state: S^T[j][i] = S0[i][j] (fp32 and bf16 copies)
#pragma unroll 1
  for (int c = 0; c < DK; c += 32) {
    uint32_t r[32], p[16];
#pragma unroll
    for (int e = 0; e < 32; ++e)
      r[e] = __float_as_uint(a.state0 ? a.state0[sg + (int64_t)(c + e) * DK + j] : 0.f);
#pragma unroll
    for (int e = 0; e < 16; ++e) p[e] = pack_bf16(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1]));
    umma::tmem_st32(sh.tmem + lane_base + TM_S32 + c, r);
    umma::tmem_st16(sh.tmem + lane_base + TM_S16 + c / 2, p);
  }
  umma::tmem_wait_st();
  umma::fence_before_sync();
  umma::named_sync(2, NTB);

#pragma unroll 1
  for (int c = 0; c < nchunks; ++c) {
    const int b = c & 1;
    const int64_t c0 = s0 + (int64_t)c * CH;
    ok = wait_vote(&bar[B_FULL0 + b], (c >> 1) & 1, ok, 2, NTB);
    if (!ok) break;
    // D^T += S^T (-W^T), committed alone (the next step needs only D^T); then O^T = S^T Q~^T
    if (tb == 0) {
      const uint32_t id_d = umma::make_idesc_bf16(128, 64, 0, 1);
      const uint32_t id_o = umma::make_idesc_bf16(128, 64, 0, 0);
#pragma unroll
      for (int s = 0; s < DK / 16; ++s)
        umma::mma_ts(sh.tmem + TM_D, sh.tmem + TM_S16 + (uint32_t)(s * 8),
                     desc_mn_wt(sh.sbase + OFF_WT, s), id_d, 1);
      umma::mma_commit(&bar[B_MMA_B]);
#pragma unroll
      for (int s = 0; s < DK / 16; ++s)
        umma::mma_ts(sh.tmem + TM_O, sh.tmem + TM_S16 + (uint32_t)(s * 8),
                     desc_k128(sh.sbase + OFF_QT + b * 16384, 64, s), id_o, s > 0);
    }
    ok = wait_vote(&bar[B_MMA_B], ph_mma, ok, 2, NTB);
    ph_mma ^= 1u;
    if (!ok) break;
    // D^T -> bf16 A operand; decay S^T columns by e^{Gamma_C}
    {
      uint32_t r0[32], r1[32], p[32];
      umma::tmem_ld32(sh.tmem + lane_base + TM_D, r0);
      umma::tmem_ld32(sh.tmem + lane_base + TM_D + 32, r1);
      umma::tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        p[e] = pack_bf16(__uint_as_float(r0[2 * e]), __uint_as_float(r0[2 * e + 1]));
        p[16 + e] = pack_bf16(__uint_as_float(r1[2 * e]), __uint_as_float(r1[2 * e + 1]));
      }
      umma::tmem_st32(sh.tmem + lane_base + TM_D16, p);
      const float *egc = reinterpret_cast<const float *>(smem + OFF_EGC) + b * 128;
#pragma unroll 1
      for (int cc = 0; cc < DK; cc += 32) {
        uint32_t s[32];
        umma::tmem_ld32(sh.tmem + lane_base + TM_S32 + cc, s);
        umma::tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) s[e] = __float_as_uint(__uint_as_float(s[e]) * egc[cc + e]);
        umma::tmem_st32(sh.tmem + lane_base + TM_S32 + cc, s);
      }
      umma::tmem_wait_st();
    }
    umma::fence_before_sync();
    umma::named_sync(2, NTB);
    if (tb == 0) {
      umma::mbar_arrive(&bar[B_DFREE]);      // D region and W^T are free for chunk c+1
      umma::fence_after_sync();
      // S^T += D^T K^ (the chain) first, then O^T += D^T A_qk^T
      const uint32_t id_o = umma::make_idesc_bf16(128, 64, 0, 0);
      const uint32_t id_s = umma::make_idesc_bf16(128, 128, 0, 1);
#pragma unroll
      for (int s = 0; s < CH / 16; ++s)
        umma::mma_ts(sh.tmem + TM_S32, sh.tmem + TM_D16 + (uint32_t)(s * 8),
                     desc_mn_tok(sh.sbase + OFF_KH + b * 16384, s), id_s, 1);
#pragma unroll
      for (int s = 0; s < CH / 16; ++s)
        umma::mma_ts(sh.tmem + TM_O, sh.tmem + TM_D16 + (uint32_t)(s * 8),
                     desc_k64(sh.sbase + OFF_AQ + b * 8192, s), id_o, 1);
      umma::mma_commit(&bar[B_MMA_B]);
    }
    ok = wait_vote(&bar[B_MMA_B], ph_mma, ok, 2, NTB);
    ph_mma ^= 1u;
    if (!ok) break;
    if (tb == 0) umma::mbar_arrive(&bar[B_EMPTY0 + b]);  // chunk c's parity-b buffers are free
    // refresh the bf16 state copy (next chunk's A operand), then store O
    {
#pragma unroll 1
      for (int cc = 0; cc < DK; cc += 32) {
        uint32_t s[32], p[16];
        umma::tmem_ld32(sh.tmem + lane_base + TM_S32 + cc, s);
        umma::tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) p[e] = pack_bf16(__uint_as_float(s[2 * e]), __uint_as_float(s[2 * e + 1]));
        umma::tmem_st16(sh.tmem + lane_base + TM_S16 + cc / 2, p);
      }
      uint32_t r0[32], r1[32];
      umma::tmem_ld32(sh.tmem + lane_base + TM_O, r0);
      umma::tmem_ld32(sh.tmem + lane_base + TM_O + 32, r1);
      umma::tmem_wait_ld();
      umma::tmem_wait_st();
      const int nvalid = (int)min((int64_t)CH, s1 - c0);
      __nv_bfloat16 *orow = o + (c0 * H + h) * DK + j;
#pragma unroll
      for (int t = 0; t < 32; ++t)
        if (t < nvalid) orow[(int64_t)t * H * DK] = __float2bfloat16_rn(a.scale * __uint_as_float(r0[t]));
#pragma unroll
      for (int t = 0; t < 32; ++t)
        if (t + 32 < nvalid)
          orow[(int64_t)(t + 32) * H * DK] = __float2bfloat16_rn(a.scale * __uint_as_float(r1[t]));
    }
    umma::fence_before_sync();
    umma::named_sync(2, NTB);
  }
  // final state: S[i][j] = S^T[j][i]
  if (ok) {
#pragma unroll 1
    for (int cc = 0; cc < DK; cc += 32) {
      uint32_t s[32];
      umma::tmem_ld32(sh.tmem + lane_base + TM_S32 + cc, s);
      umma::tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 32; ++e) a.state1[sg + (int64_t)(cc + e) * DK + j] = __uint_as_float(s[e]);
    }
  }
  if (!ok && tb == 0 && sh.err) atomicExch(sh.err, ERR_TIMEOUT);
}

__global__ void __launch_bounds__(NT, 1) chunk_kernel(RecurrenceArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5;
  const int n = blockIdx.x / a.H, h = blockIdx.x % a.H;
  int64_t s0, s1;
  seq_bounds(a.cu, n, a.seq_len, a.total_tokens, s0, s1);
  const int nchunks = (int)((s1 - s0 + CH - 1) / CH);

  uint64_t *bar = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + OFF_BAR + 8 * B_COUNT);
  if (warp == 0) {
    umma::tmem_alloc(tmem_slot, 512);
    umma::tmem_relinquish();
  }
  if (tid == 32) {
    for (int i = 0; i < B_COUNT; ++i) umma::mbar_init(&bar[i], 1);
    umma::mbar_fence_init();
  }
  umma::fence_before_sync();
  __syncthreads();
  umma::fence_after_sync();

  Shared sh;
  sh.smem = smem;
  sh.sbase = umma::smem_u32(smem);
  sh.tmem = *tmem_slot;
  sh.bar = bar;
  sh.err = a.err;

  if (tid < NTA) stage_a(a, sh, h, s0, s1, nchunks);
  else stage_b(a, sh, n, h, s0, s1, nchunks);

  umma::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    umma::fence_after_sync();
    umma::tmem_dealloc(sh.tmem, 512);
  }
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
