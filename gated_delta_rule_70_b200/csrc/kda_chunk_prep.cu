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
// shared-memory image the state pass copies in.  A_qk and -W^T | U^T are built in
// that image in free shared memory and leave by one bulk store each; the two token-row
// parts are stored directly (whole 256-byte rows per half-warp).
//
// Prologue (fused variant, the prefill entry points): the chunk's raw q, k, v
// (with the 3 tokens before it for the causal conv) and alpha arrive by TMA;
// conv4 + SiLU, the L2 norm of q and k, the gate and beta are computed here,
// so those intermediates never travel through device memory.  The other
// variant reads them prepared (the recurrence entry point).  Elementwise work
// runs two fp32 lanes per instruction; the SiLU's sigmoid is 1/2 + tanh(x/2)/2
// with the tanh on the special-function unit: fp32 for v, half precision for q and
// k, two lanes at a time (absolute error about 2^-12 either way, under the bf16
// rounding of q, k, v); the gate and every decay factor stay in fp32.
//
// Numerics: Gamma reaches 64 * (-5) = -320 inside a chunk, so e^{-Gamma}
// overflows fp32.  The pairwise factor e^{Gamma_t - Gamma_s} is only ever split
// around a reference close to both tokens: the sub-block I of a token (16 or 32
// tokens, kSub) has the reference m_I = Gamma after its (kSub/2)-th token.  A
// token's L-side factor e^{Gamma_t - m_I} and R-side factor e^{m_I - Gamma_t} then
// stay within e^{+-(kSub/2) |g|max}: with 16-token blocks 2^{+-116} at a gate bound of
// -10, with 32-token blocks 2^{+-116} at -5.02, so neither overflows nor drops to a
// subnormal the exponential would flush.  The host takes 32-token blocks whenever
// the bound allows it (the pages' -5 does).  A row in block I against an earlier
// block J uses k_s e^{m_J - Gamma_s} times e^{m_I - m_J} <= 1.  Per element only two
// exponentials are taken, e^{Gamma_t - m_I} and e^{m_I - Gamma_t}; every other
// factor is one of them times a per-channel constant of the chunk, all in base 2 on
// the special-function unit.
//
// Structure: one CTA of 8 warps per (chunk, head), two CTAs per SM so that one
// item's memory and tensor-core waits overlap the other's arithmetic.
// Tensor-core work (tcgen05, fp32 accumulation in TMEM):
//   [Lq; Lk] x R_all^T (M=128, N=160 or 96, K=128) -> A_qk and A_kk blocks
//   W^T = K~^T T_b^T and U^T = V^T T_b^T      (M=128, N=64, K=64)
// The 64x64 unit-lower-triangular solve runs in shared memory: 16x16 diagonal
// blocks by forward substitution, then the off-diagonal blocks as products of
// 16x16 blocks on the warp-level tensor-core path (mma.sync, tf32 operands,
// fp32 accumulation): first the blocks next to the diagonal, then the lower-left
// 32x32 half from the two 32x32 diagonal halves.
#include <algorithm>

#include "chunk_common.cuh"
#include "kda_common.cuh"
#include "kda_internal.h"
#include "tma_host.h"

namespace kda {
namespace prep {

using namespace chunkfmt;

constexpr int NT = 256;
constexpr int TSS = 68;      // fp32 row stride of diag(beta) A_kk (ldmatrix rows in distinct banks)
constexpr int TST = 72;      // fp32 row stride of T (a B fragment's rows c, c+4 and columns g: distinct banks)
constexpr int TSX = 40;      // fp32 row stride of the 32 x 32 intermediate of the solve (likewise)
constexpr float LOG2E = 1.4426950408889634f;

// Shared memory (byte offsets from a 1024-aligned base); two CTAs fit on one SM.
// Prologue staging (fused variant), read before the operands are written:
constexpr int RAW_ROWS = CH + 3;              // tokens c0-3 .. c0+63
constexpr uint32_t RAW_ROW = DK * 2;          // 256 B per token row
constexpr uint32_t OFF_RAWQ = 0;
constexpr uint32_t OFF_RAWK = 17408;
constexpr uint32_t OFF_RAWV = 34816;
constexpr uint32_t OFF_RAWA = 52224;          // alpha: 64 rows
// Intra-chunk MMA operands:
constexpr uint32_t OFF_L = 0;                 // [q rows 0..63 | k rows 64..127] x 128 ch: 32 KB
constexpr uint32_t OFF_R = 32768;             // R_all: up to 160 rows x 128 ch: 40 KB
// Once the intra-chunk MMA has completed:
constexpr uint32_t OFF_SB = 0;                // diag(beta) A_kk fp32 [64][TSS]
constexpr uint32_t OFF_ST = 64 * TSS * 4;     // T fp32 [64][TST]
constexpr uint32_t OFF_TB = 35840;            // T_b [t][s] bf16, 8 KB (before it: the solve's X [32][TSX])
// Record parts staged in their record image, then sent by one bulk store each
// (a lane per 128-byte row would scatter 16-byte pieces over 32 rows per store):
constexpr uint32_t OFF_AQS = 45056;           // A_qk, 8 KB (after the intra MMA, beside the solve)
constexpr uint32_t OFF_WUS = 0;               // -W^T | U^T, 32 KB (after the W/U MMA)
constexpr uint32_t OFF_KT = 73728;            // k e^{Gamma}: 16 KB
constexpr uint32_t OFF_V = 90112;             // v: 16 KB (written as soon as v is known)
// The conv weights as the prologue uses them: fp32 tap pairs (w_t of channels 2p and 2p+1),
// [tensor][pair p][taps 0-1 | taps 2-3][channel group cg][16 B], 2 KB per tensor.  They land
// as bf16 [tensor][channel][4 taps] (read as they are, a thread's 16-byte reads fell 8-way on
// the same banks and each pair took a dozen unpacking instructions); in the k e^{Gamma}
// area, which the operands fill only later.
constexpr uint32_t OFF_WRL = OFF_KT;
// Per-channel constants of the chunk (after the prologue, which stages the conv
// weights and dt_bias of the head in the same bytes):
constexpr uint32_t OFF_C = 106496;
constexpr uint32_t OFF_WCONV = OFF_C;         // [3][128 channels][4 taps] bf16, 1 KB per tensor
constexpr uint32_t OFF_DTB = OFF_C + 3 * 1024;   // [128] fp32
constexpr uint32_t C_M = OFF_C;               // m_0..m_3 (block references), Gamma_C  [5][128]
constexpr uint32_t OFF_WTOT = OFF_C + 4096;   // per-warp gate sums [8][128], then their prefixes
constexpr uint32_t OFF_BETA = OFF_C + 8192;   // beta[64]
constexpr uint32_t OFF_BAR = OFF_BETA + 256;  // MMA barrier, TMA barrier, TMEM address, OFF_PEND
constexpr uint32_t OFF_PEND = OFF_BAR + 20;   // the phase a failed wait left outstanding
constexpr uint32_t SMEM_BYTES = OFF_BAR + 64;
constexpr uint32_t TMA_BYTES = 3 * RAW_ROWS * RAW_ROW + CH * RAW_ROW + 3 * 1024 + 512;
static_assert(OFF_RAWK >= RAW_ROWS * RAW_ROW && OFF_RAWV >= OFF_RAWK + RAW_ROWS * RAW_ROW &&
              OFF_RAWA >= OFF_RAWV + RAW_ROWS * RAW_ROW && OFF_RAWA + CH * RAW_ROW <= OFF_KT,
              "prologue staging overlaps");
static_assert(OFF_ST + 64 * TST * 4 <= OFF_TB && OFF_TB + 8192 <= OFF_KT && OFF_V + 16384 <= OFF_C &&
                  32 * TSX * 4 <= 8192 && OFF_ST % 16 == 0,
              "solve scratch overlaps");
static_assert(OFF_TB % 1024 == 0 && OFF_KT % 1024 == 0 && OFF_V % 1024 == 0 && OFF_R % 1024 == 0,
              "SW128 alignment");
static_assert(OFF_WRL + 3 * 2048 <= OFF_V, "re-laid conv weights");
static_assert(OFF_TB + 8192 <= OFF_AQS && OFF_AQS + 8192 <= OFF_KT && OFF_WUS + 32768 <= OFF_TB &&
              REC_U == REC_WT + 16384 && REC_WT == 0, "record staging");
static_assert(OFF_DTB + 512 <= OFF_WTOT && C_M + 2560 <= OFF_WTOT, "constant area");
static_assert(OFF_DTB % 16 == 0 && OFF_WCONV % 16 == 0, "bulk copy alignment");

// A per-channel vector of 128 floats is stored as two halves: channels 8c..8c+3
// of every channel group c, then channels 8c+4..8c+7, so that the 8-channel
// group of a thread is two 16-byte reads that fall in distinct banks.
__device__ __forceinline__ int cpos(int ch) { return ((ch & 7) >> 2) * 64 + (ch >> 3) * 4 + (ch & 3); }
static_assert(2 * (SMEM_BYTES + 1024) <= 233472, "two CTAs per SM");

// R_all rows: [0,64) diagonal-block rows (every token against its own block's
// reference), then R_I for each later block I: the tokens of the blocks before I
// against block I's reference.  16-token blocks: R_1 (16 rows), R_2 (32), R_3 (48),
// 160 rows in all; 32-token blocks: R_1 (32 rows), 96 rows in all.
template <int kSub> __host__ __device__ constexpr int r_rows() { return kSub == 32 ? 96 : 160; }
template <int kSub> __host__ __device__ constexpr int r_row0(int I) {
  return kSub == 32 ? 64 : (I == 1 ? 64 : (I == 2 ? 80 : 112));
}

// TMEM columns (256 allocated): intra products; after they are read, W^T and U^T
constexpr uint32_t TM_P = 0;
constexpr uint32_t TM_W = 0;
constexpr uint32_t TM_U = 64;

// Bounded waits.  Each CTA has at most one asynchronous phase outstanding at a time
// (the input copies, then each MMA commit, every one waited before the next is
// issued).  When a wait gives up, the CTA issues nothing more, records that phase in
// shared memory (barrier offset and parity) and, before it frees its tensor memory and
// leaves, waits for it once more with the full limit, so no copy or MMA of this CTA can
// still be writing when it is gone.
// Only thread 0 issues MMAs and bulk stores and drains, and it wrote the record
// itself; the other threads read it only after a later block barrier.
__device__ __forceinline__ bool failed(const uint8_t *smem) {
  return *reinterpret_cast<const volatile uint32_t *>(smem + OFF_PEND) != 0;
}
// CTA-wide: every thread waits (`polls` polls) and they vote; no wait once failed.
// Returns whether this and every earlier wait succeeded.
__device__ __forceinline__ bool vote(uint8_t *smem, uint32_t bar_off, uint32_t parity, uint32_t polls) {
  const bool before = !failed(smem);
  const bool mine = before && umma::mbar_wait_bounded(reinterpret_cast<uint64_t *>(smem + bar_off), parity, polls);
  const bool all = __syncthreads_and(mine) != 0;
  umma::fence_after_sync();
  if (before && !all && threadIdx.x == 0)
    *reinterpret_cast<volatile uint32_t *>(smem + OFF_PEND) = bar_off | parity;   // bar_off > 0
  return all;
}
// After a failure, thread 0 waits out the outstanding phase with the full limit.
__device__ __forceinline__ void drain(uint8_t *smem) {
  const uint32_t p = *reinterpret_cast<const volatile uint32_t *>(smem + OFF_PEND);
  if (p != 0) (void)umma::mbar_wait_bounded(reinterpret_cast<uint64_t *>(smem + (p & ~7u)), p & 1u, kWaitPolls);
}

// 16 x 8 x 16 tiles of the solve on the warp-level tensor-core path (tf32 operands, fp32
// accumulation), over row-major fp32 matrices in shared memory.
// d += A[ra..ra+16)[ca..ca+16) * B[rb..rb+16)[cb..cb+8)   (A at shared address abase, row stride lda)
__device__ __forceinline__ void tile_mma(float (&d)[4], uint32_t abase, int lda, int ra, int ca,
                                         const float *bm, int ldb, int rb, int cb, int lane) {
  const int mi = lane >> 3, g = lane >> 2, c = lane & 3;
#pragma unroll
  for (int kk = 0; kk < 2; ++kk) {
    uint32_t a[4];
    umma::ldsm_x4(abase + (uint32_t)(((ra + (lane & 7) + (mi & 1) * 8) * lda + ca + 8 * kk + (mi >> 1) * 4) * 4), a);
    const uint32_t b0 = __float_as_uint(bm[(rb + 8 * kk + c) * ldb + cb + g]);
    const uint32_t b1 = __float_as_uint(bm[(rb + 8 * kk + c + 4) * ldb + cb + g]);
    umma::mma_tf32(d, a, b0, b1);
  }
}
// m[r0..r0+16)[c0..c0+8) = sgn * d
__device__ __forceinline__ void tile_store(float *m, int ld, int r0, int c0, int lane, const float (&d)[4], float sgn) {
  const int g = lane >> 2, c = lane & 3;
  *reinterpret_cast<float2 *>(m + (r0 + g) * ld + c0 + 2 * c) = make_float2(sgn * d[0], sgn * d[1]);
  *reinterpret_cast<float2 *>(m + (r0 + g + 8) * ld + c0 + 2 * c) = make_float2(sgn * d[2], sgn * d[3]);
}

// The (sequence, chunk) of chunk slot `gchunk`: dense batches by a 32-bit division,
// varlen by one load from the slot table (every CTA pays for this before its first copy).
// False for slots past the last chunk.
__device__ __forceinline__ bool locate(const PrepArgs &a, int64_t gchunk, int &n, int64_t &c0, int &nt,
                                       int64_t &cidx) {
  if (a.slot_info != nullptr) {
    if (gchunk >= a.max_slots) return false;
    const int4 si = a.slot_info[gchunk];
    if (si.x < 0) return false;
    n = si.x;
    cidx = si.y;
    c0 = si.z;
    nt = si.w;
    return true;
  }
  const uint32_t per = ((uint32_t)a.seq_len + CH - 1) / CH;
  if (per == 0 || gchunk >= (int64_t)per * a.N) return false;
  const uint32_t g32 = (uint32_t)gchunk, n32 = g32 / per;   // gchunk < the grid < 2^31
  n = (int)n32;
  cidx = g32 - n32 * per;
  int64_t s0, s1;
  seq_bounds(a.cu, n, a.seq_len, a.total_tokens, s0, s1);
  c0 = s0 + cidx * CH;
  if (c0 >= s1) return false;   // only for malformed cu_seqlens / chunk tables
  nt = (int)(s1 - c0 < CH ? s1 - c0 : CH);   // valid tokens in this chunk
  return true;
}

template <bool kFused, int kSub>
__global__ void __launch_bounds__(NT, 2) chunk_prep_kernel(const __grid_constant__ PrepArgs a) {
  static_assert(kSub == 16 || kSub == 32, "sub-block length");
  constexpr int NB = CH / kSub;            // sub-blocks per chunk
  constexpr int RR = r_rows<kSub>();       // rows of R_all
  const int H = a.H;
  const uint32_t gq = blockIdx.x / (uint32_t)H;
  const int h = (int)(blockIdx.x - gq * (uint32_t)H);
  int64_t gchunk = gq;
  if (a.chunk_cu == nullptr && a.seg_len > 0) {   // a time segment of a dense batch
    const uint32_t per = ((uint32_t)a.seq_len + CH - 1) / CH;
    const uint32_t sq = gq / (uint32_t)a.seg_len;
    const uint32_t cidx = (uint32_t)a.seg_c0 + (gq - sq * (uint32_t)a.seg_len);
    if (cidx >= per) return;
    gchunk = (int64_t)sq * per + cidx;
  }
  int n, nt;
  int64_t c0, cidx;
  if (!locate(a, gchunk, n, c0, nt, cidx)) return;

  extern __shared__ __align__(1024) uint8_t smem[];
  if (umma::smem_u32(smem) & 1023u) {   // the swizzled operands need a 1024-byte aligned base
    if (threadIdx.x == 0 && a.err) atomicOr(a.err, ERR_TIMEOUT_PREP);
    return;
  }
  uint8_t *rec = reinterpret_cast<uint8_t *>(a.records) + (gchunk * H + h) * (int64_t)REC_STRIDE;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int cg = tid & 15, tg = tid >> 4;   // tokens 4tg..4tg+3 (warp w: tokens 8w..8w+7)
  const int blkI = warp / (kSub / 8);        // their sub-block
  float *beta_s = reinterpret_cast<float *>(smem + OFF_BETA);
  float *wtot = reinterpret_cast<float *>(smem + OFF_WTOT);
  float *sBm = reinterpret_cast<float *>(smem + OFF_SB);
  float *sTm = reinterpret_cast<float *>(smem + OFF_ST);
  uint64_t *bar_mma = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
  uint64_t *bar_tma = bar_mma + 1;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + OFF_BAR + 16);
  const uint32_t sbase = umma::smem_u32(smem);
  const uint32_t lane_base = (uint32_t)(warp & 3) * 32u << 16;

  if (warp == 1) {
    // barriers, then at once the chunk's input copies: their latency overlaps the
    // TMEM allocation and the first block barrier
    if (lane == 0) {
      umma::mbar_init(bar_mma, 1);
      umma::mbar_init(bar_tma, 1);
      umma::mbar_fence_init();
      *reinterpret_cast<uint32_t *>(smem + OFF_PEND) = 0u;
    }
    __syncwarp();
    if constexpr (kFused) {
      if (lane == 0) {
        umma::mbar_arrive_expect_tx(bar_tma, TMA_BYTES);
        const int x = h * DK;
        umma::tma_load_2d(smem + OFF_RAWQ, &a.map_q, x, (int)c0 - 3, bar_tma);
        umma::tma_load_2d(smem + OFF_RAWK, &a.map_k, x, (int)c0 - 3, bar_tma);
        umma::tma_load_2d(smem + OFF_RAWV, &a.map_v, x, (int)c0 - 3, bar_tma);
        umma::tma_load_2d(smem + OFF_RAWA, &a.map_alpha, x, (int)c0, bar_tma);
      }
      __syncwarp();
      // one copy per tensor: under load every copy instruction costs about as much
      // to issue as a few KB of data, so the weights come as 3 x 1 KB
      if (lane < 3) {   // conv weights of tensor `lane`
        const __nv_bfloat16 *cw = reinterpret_cast<const __nv_bfloat16 *>(a.conv_w);
        umma::bulk_g2s(smem + OFF_WCONV + lane * 1024, cw + ((int64_t)lane * H + h) * DK * KCONV, 1024, bar_tma);
      } else if (lane == 3) {
        umma::bulk_g2s(smem + OFF_DTB, a.dt_bias + h * DK, 512, bar_tma);
      }
    }
  }
  if (warp == 0) {
    umma::tmem_alloc(tmem_slot, 256);
    umma::tmem_relinquish();
  }
  umma::fence_before_sync();
  __syncthreads();
  umma::fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  // ---------------------------------------------------------------- inputs
  uint4 qb[4], kb[4];          // bf16 q, k (normalised) of this thread's 4 tokens x 8 channels
  float2 g2[4][4];             // gate in base 2, [token][channel pair]
  float btj = 0.f;             // beta of token tid (tid < 64)
  if constexpr (kFused) {
    const float negA = -expf(a.A_log[h]);
    const float lb2 = a.lower_bound * LOG2E;
    if (tid < 64 && tid < nt)
      btj = (a.beta2 ? 2.f : 1.f) *
            sigmoid_f(__bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(a.b)[(c0 + tid) * H + h]));
    // causal-conv history of a sequence's first chunk: the caller's conv state or zeros
    const bool hist = cidx == 0 && tg == 0;
    uint4 hraw[3][3];
    if (hist) {
      const __nv_bfloat16 *c0p = reinterpret_cast<const __nv_bfloat16 *>(a.conv0);
#pragma unroll
      for (int blk = 0; blk < 3; ++blk)
#pragma unroll
        for (int m = 0; m < 3; ++m)
          hraw[blk][m] = c0p != nullptr
                             ? *reinterpret_cast<const uint4 *>(
                                   c0p + (((int64_t)n * 3 + m) * 3 + blk) * H * DK + h * DK + cg * 8)
                             : make_uint4(0, 0, 0, 0);
    }
    (void)vote(smem, OFF_BAR + 8, 0, a.wait_polls);   // bar_tma
    if (tid < 192) {   // conv weights / 2 into fp32 tap pairs (one channel pair each): the
                       // conv then yields x/2, the argument SiLU's tanh form starts from
      const int blk = tid >> 6, cgw = (tid >> 2) & 15, pw = tid & 3;
      const uint4 wq = *reinterpret_cast<const uint4 *>(smem + OFF_WCONV + blk * 1024 + cgw * 64 + pw * 16);
      const float2 wa = mul2(bf2_f2(wq.x), f2(0.5f)), wb = mul2(bf2_f2(wq.y), f2(0.5f));
      const float2 wc = mul2(bf2_f2(wq.z), f2(0.5f)), wd = mul2(bf2_f2(wq.w), f2(0.5f));
      uint8_t *dw = smem + OFF_WRL + blk * 2048 + pw * 512 + cgw * 16;
      *reinterpret_cast<float4 *>(dw) = make_float4(wa.x, wc.x, wa.y, wc.y);         // taps 0, 1
      *reinterpret_cast<float4 *>(dw + 256) = make_float4(wb.x, wd.x, wb.y, wd.y);   // taps 2, 3
    }
    if (hist) {
#pragma unroll
      for (int blk = 0; blk < 3; ++blk)
#pragma unroll
        for (int m = 0; m < 3; ++m)   // only this thread reads these 16 bytes
          *reinterpret_cast<uint4 *>(smem + (blk == 0 ? OFF_RAWQ : blk == 1 ? OFF_RAWK : OFF_RAWV) +
                                     m * RAW_ROW + cg * 16) = hraw[blk][m];
    }
    __syncthreads();   // the re-laid conv weights
    // conv4 + SiLU (+ L2 norm over the head's 128 channels for q and k), two
    // channels at a time; v first, it goes straight into its operand tile
#pragma unroll
    for (int bi = 0; bi < 3; ++bi) {
      const int blk = bi == 0 ? 2 : bi - 1;
      const uint8_t *raw = smem + (blk == 0 ? OFF_RAWQ : blk == 1 ? OFF_RAWK : OFF_RAWV) + cg * 16;
      uint4 xr[7];   // input rows 4tg .. 4tg+6 (tokens 4tg-3 .. 4tg+3), 8 channels each
#pragma unroll
      for (int r = 0; r < 7; ++r) xr[r] = *reinterpret_cast<const uint4 *>(raw + (4 * tg + r) * RAW_ROW);
      float2 y[4][4];
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        // tap t of channels 2p and 2p+1 as one fp32 pair w_t
        const float4 wl = *reinterpret_cast<const float4 *>(smem + OFF_WRL + blk * 2048 + p * 512 + cg * 16);
        const float4 wh = *reinterpret_cast<const float4 *>(smem + OFF_WRL + blk * 2048 + p * 512 + 256 + cg * 16);
        const float2 w0 = make_float2(wl.x, wl.y), w1 = make_float2(wl.z, wl.w);
        const float2 w2 = make_float2(wh.x, wh.y), w3 = make_float2(wh.z, wh.w);
        float2 x[7];
#pragma unroll
        for (int r = 0; r < 7; ++r) x[r] = bf2_f2(word(xr[r], p));
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float2 acc = mul2(w0, x[j]);   // x/2, exactly (the weights are halved)
          acc = fma2(w1, x[j + 1], acc);
          acc = fma2(w2, x[j + 2], acc);
          acc = fma2(w3, x[j + 3], acc);
          if (blk == 2) {   // v: the fp32 tanh, one special-function operation per lane
            float t0, t1;
            asm("tanh.approx.f32 %0, %1;" : "=f"(t0) : "f"(acc.x));
            asm("tanh.approx.f32 %0, %1;" : "=f"(t1) : "f"(acc.y));
            y[j][p] = fma2(acc, make_float2(t0, t1), acc);
          } else {
            y[j][p] = silu2_from_half(acc);
          }
        }
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (blk < 2) {
          float2 ss = mul2(y[j][0], y[j][0]);
#pragma unroll
          for (int p = 1; p < 4; ++p) ss = fma2(y[j][p], y[j][p], ss);
          float s1 = ss.x + ss.y;
#pragma unroll
          for (int off = 8; off >= 1; off >>= 1) s1 += __shfl_xor_sync(0xffffffffu, s1, off);
          const float2 rn = f2(rsqrtf(s1 + a.eps));
#pragma unroll
          for (int p = 0; p < 4; ++p) y[j][p] = mul2(y[j][p], rn);
        }
        const uint4 packed = make_uint4(f2_bf2(y[j][0]), f2_bf2(y[j][1]), f2_bf2(y[j][2]), f2_bf2(y[j][3]));
        if (blk == 0) qb[j] = packed;
        else if (blk == 1) kb[j] = packed;
        else *reinterpret_cast<uint4 *>(smem + OFF_V + tr_off(64, tg * 4 + j, cg)) = packed;
      }
    }
    // gate g = max(-exp(A_log) softplus(alpha + dt_bias), lower_bound), kept in base 2:
    // g log2(e) = -exp(A_log) log2(1 + 2^{x log2 e}).  Where the exponential overflows the
    // gate is -inf before the clamp, which then gives the lower bound, as it should.
    float2 bias[4];
    {
      const float4 b0 = *reinterpret_cast<const float4 *>(smem + OFF_DTB + cg * 32);
      const float4 b1 = *reinterpret_cast<const float4 *>(smem + OFF_DTB + cg * 32 + 16);
      bias[0] = make_float2(b0.x, b0.y); bias[1] = make_float2(b0.z, b0.w);
      bias[2] = make_float2(b1.x, b1.y); bias[3] = make_float2(b1.z, b1.w);
#pragma unroll
      for (int p = 0; p < 4; ++p) bias[p] = mul2(bias[p], f2(LOG2E));   // (alpha + dt_bias) log2 e by one fma
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint4 ar = *reinterpret_cast<const uint4 *>(smem + OFF_RAWA + (4 * tg + j) * RAW_ROW + cg * 16);
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        const float2 l = add2(ex2_2(fma2(bf2_f2(word(ar, p)), f2(LOG2E), bias[p])), f2(1.f));
        const float2 g = mul2(make_float2(lg2_approx(l.x), lg2_approx(l.y)), f2(negA));
        g2[j][p] = make_float2(fmaxf(g.x, lb2), fmaxf(g.y, lb2));
      }
    }
    if (nt < CH) {   // a sequence's last chunk: tokens past its end take no part (q, k, v, gate 0)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (4 * tg + j >= nt) {
          qb[j] = kb[j] = make_uint4(0u, 0u, 0u, 0u);
          *reinterpret_cast<uint4 *>(smem + OFF_V + tr_off(64, tg * 4 + j, cg)) = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
          for (int p = 0; p < 4; ++p) g2[j][p] = f2(0.f);
        }
      }
    }
  } else {
    const __nv_bfloat16 *__restrict__ qn = reinterpret_cast<const __nv_bfloat16 *>(a.qn);
    const __nv_bfloat16 *__restrict__ kn = reinterpret_cast<const __nv_bfloat16 *>(a.kn);
    const __nv_bfloat16 *__restrict__ vc = reinterpret_cast<const __nv_bfloat16 *>(a.vc);
    uint4 vr[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int t = tg * 4 + j;
      const int64_t off = ((c0 + t) * H + h) * DK + cg * 8;
      if (t < nt) {
        qb[j] = __ldcs(reinterpret_cast<const uint4 *>(qn + off));
        kb[j] = __ldcs(reinterpret_cast<const uint4 *>(kn + off));
        vr[j] = __ldcs(reinterpret_cast<const uint4 *>(vc + off));
        const float4 ga = __ldcs(reinterpret_cast<const float4 *>(a.g + off));
        const float4 gb = __ldcs(reinterpret_cast<const float4 *>(a.g + off + 4));
        const float gg[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
#pragma unroll
        for (int p = 0; p < 4; ++p)
          g2[j][p] = make_float2(fminf(fmaxf(gg[2 * p], a.lower_bound), 0.f) * LOG2E,
                                 fminf(fmaxf(gg[2 * p + 1], a.lower_bound), 0.f) * LOG2E);
      } else {
        qb[j] = kb[j] = vr[j] = make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int p = 0; p < 4; ++p) g2[j][p] = f2(0.f);
      }
    }
    if (tid < 64 && tid < nt) btj = __ldcs(a.beta + (c0 + tid) * H + h);
#pragma unroll
    for (int j = 0; j < 4; ++j)   // v is the U operand as it is: straight into its tile
      *reinterpret_cast<uint4 *>(smem + OFF_V + tr_off(64, tg * 4 + j, cg)) = vr[j];
  }

  // ---------------------------------------------------------------- cumulative gate
#pragma unroll
  for (int p = 0; p < 4; ++p) {
#pragma unroll
    for (int j = 1; j < 4; ++j) g2[j][p] = add2(g2[j][p], g2[j - 1][p]);
    const float2 lo = make_float2(__shfl_up_sync(0xffffffffu, g2[3][p].x, 16),
                                  __shfl_up_sync(0xffffffffu, g2[3][p].y, 16));
    if (lane >= 16) {
#pragma unroll
      for (int j = 0; j < 4; ++j) g2[j][p] = add2(g2[j][p], lo);
    }
  }
  if (lane >= 16) {
    *reinterpret_cast<float4 *>(wtot + warp * 128 + cg * 4) = make_float4(g2[3][0].x, g2[3][0].y, g2[3][1].x, g2[3][1].y);
    *reinterpret_cast<float4 *>(wtot + warp * 128 + 64 + cg * 4) = make_float4(g2[3][2].x, g2[3][2].y, g2[3][3].x, g2[3][3].y);
  }
  if (tid < 64) beta_s[tid] = btj;
  __syncthreads();   // also: every read of the prologue staging is done
  // per channel: exclusive prefix of the warp sums (in place), the block references
  // m_I (Gamma after token kSub I + kSub/2 - 1, the end of warp (kSub/8) I + kSub/16 - 1)
  // and Gamma_C
  if (tid < 128) {
    const int pc = cpos(tid);   // this thread's channel, in the split-half layout
    float acc = 0.f, m[NB];
#pragma unroll
    for (int w2 = 0; w2 < 8; ++w2) {
      const float x = wtot[w2 * 128 + pc];
      wtot[w2 * 128 + pc] = acc;
      acc += x;
      if (w2 % (kSub / 8) == kSub / 16 - 1) m[w2 / (kSub / 8)] = acc;
    }
    float *cf = reinterpret_cast<float *>(smem);
#pragma unroll
    for (int I = 0; I < NB; ++I) cf[C_M / 4 + I * 128 + pc] = m[I];
    cf[C_M / 4 + 4 * 128 + pc] = acc;
    reinterpret_cast<float *>(rec + REC_EGC)[tid] = umma::ex2(acc);   // e^{Gamma_C}
  }
  __syncthreads();

  // ---------------------------------------------------------------- operands
  const uint32_t coff = (uint32_t)cg * 16;
  auto lds_pairs = [&](uint32_t off, float2 (&x)[4]) {   // this thread's 8 channels of a split-half vector
    const float4 u = *reinterpret_cast<const float4 *>(smem + off + coff);
    const float4 w = *reinterpret_cast<const float4 *>(smem + off + 256 + coff);
    x[0] = make_float2(u.x, u.y); x[1] = make_float2(u.z, u.w);
    x[2] = make_float2(w.x, w.y); x[3] = make_float2(w.z, w.w);
  };
  {
    float2 pre[4];
    lds_pairs(OFF_WTOT + warp * 512, pre);
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int p = 0; p < 4; ++p) g2[j][p] = add2(g2[j][p], pre[p]);   // Gamma_t (base 2)
  }
  {  // L side: Lq = q e^{Gamma - m_I}, Lk likewise; q e^{Gamma}, k e^{Gamma}
    float2 nm[4], eM[4];
    lds_pairs(C_M + blkI * 512, nm);
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      eM[p] = ex2_2(nm[p]);
      nm[p] = mul2(nm[p], f2(-1.f));
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int t = tg * 4 + j;
      uint32_t Lq[4], Lk[4], Qt[4], Kt[4];
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        const float2 e1 = ex2_2(add2(g2[j][p], nm[p]));   // within 2^{+-8|g|max}
        const float2 lq = mul2(bf2_f2(word(qb[j], p)), e1);
        const float2 lk = mul2(bf2_f2(word(kb[j], p)), e1);
        Lq[p] = f2_bf2(lq);
        Lk[p] = f2_bf2(lk);
        Qt[p] = f2_bf2(mul2(lq, eM[p]));
        Kt[p] = f2_bf2(mul2(lk, eM[p]));
      }
      *reinterpret_cast<uint4 *>(smem + OFF_L + tr_off(128, t, cg)) = make_uint4(Lq[0], Lq[1], Lq[2], Lq[3]);
      *reinterpret_cast<uint4 *>(smem + OFF_L + tr_off(128, 64 + t, cg)) = make_uint4(Lk[0], Lk[1], Lk[2], Lk[3]);
      *reinterpret_cast<uint4 *>(smem + OFF_KT + tr_off(64, t, cg)) = make_uint4(Kt[0], Kt[1], Kt[2], Kt[3]);
      *reinterpret_cast<uint4 *>(rec + REC_QT + tr_off(64, t, cg)) = make_uint4(Qt[0], Qt[1], Qt[2], Qt[3]);
    }
  }
  {  // R side: kd = k e^{m_I - Gamma} (the diagonal-block row); R rows of the later
     // blocks I' = kd e^{m_I' - m_I}; k e^{Gamma_C - Gamma} = kd e^{Gamma_C - m_I}
    float2 m[4], cK[4], c1[4], c2[4], c3[4];
    lds_pairs(C_M + blkI * 512, m);
    {
      float2 gc[4];
      lds_pairs(C_M + 4 * 512, gc);
#pragma unroll
      for (int p = 0; p < 4; ++p) cK[p] = ex2_2(add2(gc[p], mul2(m[p], f2(-1.f))));   // <= 1
    }
    auto later = [&](int I2, float2 (&c)[4]) {   // 2^{m_I2 - m_I} <= 1 (32-token blocks: its root)
      float2 mi[4];
      lds_pairs(C_M + I2 * 512, mi);
#pragma unroll
      for (int p = 0; p < 4; ++p)
        c[p] = ex2_2(mul2(add2(mi[p], mul2(m[p], f2(-1.f))), f2(kSub == 32 ? 0.5f : 1.f)));
    };
    // The row against the next block's reference is kd 2^{m_{I+1} - m_I}.  With 16-token
    // blocks the constant spans 16 gates; with 32-token blocks it would span 32 (2^-231 at
    // a bound of -5, flushed to zero) while kd and the L factor reach 2^+-115, so there the
    // constant is c = 2^{(m_1 - m_0) / 2}, 16 gates, applied twice: kd c c flushes to zero
    // only where the true product is below 2^-18 of q.k.
    if (blkI < NB - 1) later(blkI + 1, c1);
    if constexpr (NB > 2) {
      if (blkI < NB - 2) later(blkI + 2, c2);
      if (blkI < NB - 3) later(blkI + 3, c3);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int t = tg * 4 + j;
      uint32_t Rd[4], Kh[4], K1[4], K2[4], K3[4];
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        const float2 kd = mul2(bf2_f2(word(kb[j], p)),
                               ex2_2(fma2(g2[j][p], f2(-1.f), m[p])));   // within 2^{+-8|g|max}
        Rd[p] = f2_bf2(kd);
        Kh[p] = f2_bf2(mul2(kd, cK[p]));
        if constexpr (kSub == 32)
          K1[p] = blkI < NB - 1 ? f2_bf2(mul2(mul2(kd, c1[p]), c1[p])) : 0u;
        else
          K1[p] = blkI < NB - 1 ? f2_bf2(mul2(kd, c1[p])) : 0u;
        if constexpr (NB > 2) {
          K2[p] = blkI < NB - 2 ? f2_bf2(mul2(kd, c2[p])) : 0u;
          K3[p] = blkI < NB - 3 ? f2_bf2(mul2(kd, c3[p])) : 0u;
        }
      }
      *reinterpret_cast<uint4 *>(smem + OFF_R + tr_off(RR, t, cg)) = make_uint4(Rd[0], Rd[1], Rd[2], Rd[3]);
      *reinterpret_cast<uint4 *>(rec + REC_KH + tr_off(64, t, cg)) = make_uint4(Kh[0], Kh[1], Kh[2], Kh[3]);
      if (blkI < NB - 1)
        *reinterpret_cast<uint4 *>(smem + OFF_R + tr_off(RR, r_row0<kSub>(blkI + 1) + t, cg)) =
            make_uint4(K1[0], K1[1], K1[2], K1[3]);
      if constexpr (NB > 2) {
        if (blkI < NB - 2)
          *reinterpret_cast<uint4 *>(smem + OFF_R + tr_off(RR, r_row0<kSub>(blkI + 2) + t, cg)) =
              make_uint4(K2[0], K2[1], K2[2], K2[3]);
        if (blkI < NB - 3)
          *reinterpret_cast<uint4 *>(smem + OFF_R + tr_off(RR, r_row0<kSub>(3) + t, cg)) =
              make_uint4(K3[0], K3[1], K3[2], K3[3]);
      }
    }
  }
  umma::fence_proxy_async_smem();
  __syncthreads();

  // ---------------------------------------------------------------- intra MMA
  uint32_t phase = 0;
  if (tid == 0 && !failed(smem)) {
    umma::fence_after_sync();
    const uint32_t idesc = umma::make_idesc_bf16(128, RR, 0, 0);
#pragma unroll
    for (int s = 0; s < DK / 16; ++s)
      umma::mma_ss(tmem + TM_P, desc_k128(sbase + OFF_L, 128, s), desc_k128(sbase + OFF_R, RR, s),
                   idesc, s > 0);
    umma::mma_commit(bar_mma);
  }
  bool ok = vote(smem, OFF_BAR, phase, a.wait_polls);   // bar_mma
  phase ^= 1u;

  // ---------------------------------------------------------------- A_qk (bf16) and diag(beta) A_kk
  // Warp w reads TMEM lanes 32(w&3)..: q rows (w&3 = 0, 1) or k rows (2, 3) of
  // tokens 32p..32p+31, p = w & 1.  Warps 0-3 take column groups 0-1 (s = 0..31),
  // warps 4-7 (the same lane quadrants) groups 2-3.  A column group of row t comes
  // from the diagonal product (t's own block, masked) or from R_I (an earlier block).
  // 32-token blocks: a warp's lanes are exactly one block.  16-token blocks: lane half
  // hh gives the block I = 2p + hh; tcgen05.ld is warp-uniform, so both halves load
  // both candidates and keep their own.  Blocks of diag(beta) A_kk right of the
  // diagonal are never read, so only A_qk gets explicit zeros.
  if (ok) {
    const int p = warp & 1, hh = lane >> 4;
    const int t = 32 * p + lane;
    const bool is_q = (warp & 3) < 2;
    const bool upper = warp >= 4;
    const float bt = is_q ? 1.f : beta_s[t];
    const uint32_t tb = tmem + lane_base + TM_P;
    auto emit = [&](int gi, const uint32_t (&v)[16], bool zero, bool diag) {
      if (is_q) {   // A_qk row t, s <= t, bf16 into the record
        uint32_t w8[8];
#pragma unroll
        for (int e2 = 0; e2 < 8; ++e2) {
          const int s = 16 * gi + 2 * e2;
          const bool k0 = !zero && (!diag || s <= t), k1 = !zero && (!diag || s + 1 <= t);
          w8[e2] = pack_bf16(k0 ? __uint_as_float(v[2 * e2]) : 0.f, k1 ? __uint_as_float(v[2 * e2 + 1]) : 0.f);
        }
        *reinterpret_cast<uint4 *>(smem + OFF_AQS + tr_off(64, t, 2 * gi)) = make_uint4(w8[0], w8[1], w8[2], w8[3]);
        *reinterpret_cast<uint4 *>(smem + OFF_AQS + tr_off(64, t, 2 * gi + 1)) = make_uint4(w8[4], w8[5], w8[6], w8[7]);
      } else {      // beta_t A_kk row t, s < t, fp32 into the solve scratch
        float4 *dst = reinterpret_cast<float4 *>(sBm + t * TSS + 16 * gi);
#pragma unroll
        for (int e4 = 0; e4 < 4; ++e4) {
          const int s = 16 * gi + 4 * e4;
          const float2 lo = mul2(make_float2(__uint_as_float(v[4 * e4]), __uint_as_float(v[4 * e4 + 1])), f2(bt));
          const float2 hi = mul2(make_float2(__uint_as_float(v[4 * e4 + 2]), __uint_as_float(v[4 * e4 + 3])), f2(bt));
          const bool k0 = !zero && (!diag || s < t), k1 = !zero && (!diag || s + 1 < t);
          const bool k2 = !zero && (!diag || s + 2 < t), k3 = !zero && (!diag || s + 3 < t);
          dst[e4] = make_float4(k0 ? lo.x : 0.f, k1 ? lo.y : 0.f, k2 ? hi.x : 0.f, k3 ? hi.y : 0.f);
        }
      }
    };
    uint32_t va[16], vb2[16], v[16];
    if constexpr (kSub == 32) {
      (void)vb2; (void)v; (void)hh;
      uint32_t vc[16];
      if (p == 0) {
        if (!upper) {          // block 0, groups 0-1: the diagonal product, columns 0..31
          umma::tmem_ld16(tb + 0, va);
          umma::tmem_ld16(tb + 16, vc);
          umma::tmem_wait_ld();
          emit(0, va, false, true);
          emit(1, vc, false, true);
        } else if (is_q) {     // block 0 against block 1: zero
#pragma unroll
          for (int e = 0; e < 16; ++e) va[e] = 0u;
          emit(2, va, true, false);
          emit(3, va, true, false);
        }
      } else if (!upper) {     // block 1 against block 0: R_1, columns 64..95
        umma::tmem_ld16(tb + 64, va);
        umma::tmem_ld16(tb + 80, vc);
        umma::tmem_wait_ld();
        emit(0, va, false, false);
        emit(1, vc, false, false);
      } else {                 // block 1, groups 2-3: the diagonal product, columns 32..63
        umma::tmem_ld16(tb + 32, va);
        umma::tmem_ld16(tb + 48, vc);
        umma::tmem_wait_ld();
        emit(2, va, false, true);
        emit(3, vc, false, true);
      }
    } else if (p == 0) {
      if (!upper) {
        // gi 0: lo = diagonal (col 0), hi = R_1 (col 64); gi 1: hi = diagonal (col 16)
        uint32_t vc[16];
        umma::tmem_ld16(tb + 0, va);
        umma::tmem_ld16(tb + 64, vb2);
        umma::tmem_ld16(tb + 16, vc);
        umma::tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) v[e] = hh ? vb2[e] : va[e];
        emit(0, v, false, hh == 0);
        emit(1, vc, hh == 0, true);
      } else if (is_q) {   // groups 2-3 of blocks 0-1: zero
#pragma unroll
        for (int e = 0; e < 16; ++e) va[e] = 0u;
        emit(2, va, true, false);
        emit(3, va, true, false);
      }
    } else if (!upper) {
      // gi 0: lo = R_2 (col 80), hi = R_3 (col 112); gi 1: 96 / 128
      uint32_t vc[16], vd[16];
      umma::tmem_ld16(tb + 80, va);
      umma::tmem_ld16(tb + 112, vb2);
      umma::tmem_ld16(tb + 96, vc);
      umma::tmem_ld16(tb + 128, vd);
      umma::tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 16; ++e) v[e] = hh ? vb2[e] : va[e];
      emit(0, v, false, false);
#pragma unroll
      for (int e = 0; e < 16; ++e) v[e] = hh ? vd[e] : vc[e];
      emit(1, v, false, false);
    } else {
      // gi 2: lo = diagonal (col 32), hi = R_3 (col 144); gi 3: hi = diagonal (col 48)
      uint32_t vc[16];
      umma::tmem_ld16(tb + 32, va);
      umma::tmem_ld16(tb + 144, vb2);
      umma::tmem_ld16(tb + 48, vc);
      umma::tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 16; ++e) v[e] = hh ? vb2[e] : va[e];
      emit(2, v, false, hh == 0);
      emit(3, vc, hh == 0, true);
    }
  }
  umma::fence_proxy_async_smem();   // A_qk staged: visible to the bulk store
  umma::fence_before_sync();
  __syncthreads();
  if (tid == 0 && !failed(smem)) {
    umma::bulk_s2g(rec + REC_AQ, smem + OFF_AQS, 8192);
    umma::bulk_commit();
  }

  // ---------------------------------------------------------------- T = (I + B)^{-1}
  // The 16 x 16 diagonal blocks D_I by forward substitution; then products of 16 x 16 blocks,
  // each warp a 16 x 8 tile (columns 8 nh .. 8 nh + 7 of a block) on the warp-level tensor-core
  // path:  T_10 = -D_1 (B_10 D_0),  T_32 = -D_3 (B_32 D_2);  then the lower-left 32 x 32 half
  //   X = B_[10] T_[00]:  X_a0 = B_a0 D_0 + B_a1 T_10,  X_a1 = B_a1 D_1   (a = 2, 3)
  //   T_[10] = -T_[11] X:  T_2b = -D_2 X_2b,  T_3b = -(T_32 X_2b + D_3 X_3b).
  if (warp < 4) {  // diagonal blocks: warp = block, lane = column (lanes 16..31 mirror)
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
      for (int r = 0; r < 16; ++r) sTm[(o16 + r) * TST + o16 + cidx2] = x[r];
    }
  }
  __syncthreads();
  {
    const uint32_t aB = sbase + OFF_SB, aT = sbase + OFF_ST;
    float *sX = reinterpret_cast<float *>(smem + OFF_TB);
    const int nh = warp & 1;
    float xa[4] = {0.f, 0.f, 0.f, 0.f}, xb[4] = {0.f, 0.f, 0.f, 0.f};
    const int ia = 16 * (2 + ((warp - 4) >> 1));   // warps 4-7: row block a of X
    if (warp < 4) {   // T_10 (warps 0, 1) and T_32 (warps 2, 3)
      const int i = 16 * ((warp >> 1) * 2 + 1), j = i - 16;
      tile_mma(xa, aB, TSS, i, j, sTm, TST, j, j + 8 * nh, lane);    // B_ij D_j, parked where T_ij goes
      tile_store(sTm, TST, i, j + 8 * nh, lane, xa, 1.f);
      __syncwarp();
      tile_mma(xb, aT, TST, i, i, sTm, TST, i, j + 8 * nh, lane);    // D_i (B_ij D_j)
      __syncwarp();
      tile_store(sTm, TST, i, j + 8 * nh, lane, xb, -1.f);
    } else {          // B_a0 D_0 and X_a1 = B_a1 D_1 (need no T_10)
      tile_mma(xa, aB, TSS, ia, 0, sTm, TST, 0, 8 * nh, lane);
      tile_mma(xb, aB, TSS, ia, 16, sTm, TST, 16, 16 + 8 * nh, lane);
    }
    __syncthreads();
    if (warp >= 4) {  // X_a0 = B_a0 D_0 + B_a1 T_10
      tile_mma(xa, aB, TSS, ia, 16, sTm, TST, 16, 8 * nh, lane);
      tile_store(sX, TSX, ia - 32, 8 * nh, lane, xa, 1.f);
      tile_store(sX, TSX, ia - 32, 16 + 8 * nh, lane, xb, 1.f);
    }
    __syncthreads();
    {                 // T_ab, a = 2 + warp / 4, b = (warp / 2) % 2
      const int a = 2 + (warp >> 2), b = (warp >> 1) & 1;
      float y[4] = {0.f, 0.f, 0.f, 0.f};
      tile_mma(y, aT, TST, 16 * a, 32, sX, TSX, 0, 16 * b + 8 * nh, lane);       // T_a2 X_2b
      if (a == 3) tile_mma(y, aT, TST, 48, 48, sX, TSX, 16, 16 * b + 8 * nh, lane);   // D_3 X_3b
      tile_store(sTm, TST, 16 * a, 16 * b + 8 * nh, lane, y, -1.f);
    }
  }
  __syncthreads();
#pragma unroll
  for (int it = 0; it < 2; ++it) {  // T_b rows as bf16, K-major [t][s]
    const int e = tid + it * NT;
    const int t = e >> 3, c8 = e & 7;
    const float4 t0 = *reinterpret_cast<const float4 *>(sTm + t * TST + c8 * 8);
    const float4 t1 = *reinterpret_cast<const float4 *>(sTm + t * TST + c8 * 8 + 4);
    const float4 b0 = *reinterpret_cast<const float4 *>(beta_s + c8 * 8);
    const float4 b1 = *reinterpret_cast<const float4 *>(beta_s + c8 * 8 + 4);
    const float2 p0 = mul2(make_float2(t0.x, t0.y), make_float2(b0.x, b0.y));
    const float2 p1 = mul2(make_float2(t0.z, t0.w), make_float2(b0.z, b0.w));
    const float2 p2 = mul2(make_float2(t1.x, t1.y), make_float2(b1.x, b1.y));
    const float2 p3 = mul2(make_float2(t1.z, t1.w), make_float2(b1.z, b1.w));
    const float x8[8] = {p0.x, p0.y, p1.x, p1.y, p2.x, p2.y, p3.x, p3.y};
    uint32_t w4[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int s0 = c8 * 8 + 2 * i;
      w4[i] = pack_bf16(s0 <= t ? x8[2 * i] : 0.f, s0 + 1 <= t ? x8[2 * i + 1] : 0.f);
    }
    *reinterpret_cast<uint4 *>(smem + OFF_TB + tr_off(64, t, c8)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
  }
  umma::fence_proxy_async_smem();
  umma::fence_before_sync();
  __syncthreads();

  // ---------------------------------------------------------------- W^T, U^T (P has been read)
  if (tid == 0 && !failed(smem)) {
    umma::fence_after_sync();
    const uint32_t idesc_w = umma::make_idesc_bf16(128, 64, 1, 0, 1);   // -W^T: A negated
    const uint32_t idesc_u = umma::make_idesc_bf16(128, 64, 1, 0);
#pragma unroll
    for (int s = 0; s < CH / 16; ++s) {
      umma::mma_ss(tmem + TM_W, desc_mn_tok(sbase + OFF_KT, s), desc_k64(sbase + OFF_TB, s), idesc_w, s > 0);
      umma::mma_ss(tmem + TM_U, desc_mn_tok(sbase + OFF_V, s), desc_k64(sbase + OFF_TB, s), idesc_u, s > 0);
    }
    umma::mma_commit(bar_mma);
  }
  ok = vote(smem, OFF_BAR, phase, a.wait_polls);   // bar_mma

  // ---------------------------------------------------------------- -W^T (warps 0-3), U^T (4-7) rows
  if (ok) {
    const int i = (warp & 3) * 32 + lane;   // TMEM lane: key channel (W^T) / value channel (U^T)
    const bool isW = warp < 4;
    uint8_t *dst = smem + OFF_WUS + (isW ? REC_WT : REC_U);
    uint32_t rr[2][32];   // both column halves in flight before one wait
    umma::tmem_ld32(tmem + lane_base + (isW ? TM_W : TM_U), rr[0]);
    umma::tmem_ld32(tmem + lane_base + (isW ? TM_W : TM_U) + 32, rr[1]);
    umma::tmem_wait_ld();
#pragma unroll
    for (int c32 = 0; c32 < 2; ++c32) {
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        uint32_t w4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
          w4[e] = pack_bf16(__uint_as_float(rr[c32][q4 * 8 + 2 * e]), __uint_as_float(rr[c32][q4 * 8 + 2 * e + 1]));
        *reinterpret_cast<uint4 *>(dst + row64_off(i, c32 * 4 + q4)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
      }
    }
  }
  umma::fence_proxy_async_smem();   // -W^T | U^T staged: visible to the bulk store
  umma::fence_before_sync();
  __syncthreads();
  if (tid == 0) {
    if (!failed(smem)) {
      umma::bulk_s2g(rec + REC_WT, smem + OFF_WUS, 32768);
      umma::bulk_commit();
    } else {
      drain(smem);
      if (a.err) atomicOr(a.err, ERR_TIMEOUT_PREP);
    }
    umma::bulk_wait_read<0>();   // shared memory must stay until every store has read it
  }
  if (warp == 0) {
    umma::fence_after_sync();
    umma::tmem_dealloc(tmem, 256);
  }
}

// chunk_cu[n] = number of 64-token chunks before sequence n (varlen batches);
// also checks cu_seqlens: starts at 0, never decreases, ends at the token total.
__global__ void chunk_table_kernel(const int32_t *cu, int N, int64_t total, int32_t *chunk_cu, int *err) {
  if (blockIdx.x != 0 || threadIdx.x != 0) return;
  bool good = cu[0] == 0 && (int64_t)cu[N] == total;
  int32_t acc = 0;
  for (int n = 0; n < N; ++n) {
    good = good && cu[n + 1] >= cu[n];
    int64_t s, e;
    seq_bounds(cu, n, 0, total, s, e);
    chunk_cu[n] = acc;
    acc += (int32_t)((e - s + CH - 1) / CH);
  }
  chunk_cu[N] = acc;
  if (!good && err != nullptr) atomicOr(err, ERR_BAD_CU_SEQLENS);
}

// Per chunk slot of a varlen batch: its sequence, chunk index, first token and token count,
// so that a chunk_prep CTA needs one load, not a binary search over chunk_cu.
__global__ void slot_table_kernel(const int32_t *cu, const int32_t *chunk_cu, int N, int64_t total,
                                  int64_t slots, int4 *info) {
  const int64_t nchunks = chunk_cu[N];
  for (int64_t s = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; s < slots;
       s += (int64_t)gridDim.x * blockDim.x) {
    int4 r = make_int4(-1, 0, 0, 0);
    if (s < nchunks) {
      int lo = 0, hi = N - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if ((int64_t)chunk_cu[mid] <= s) lo = mid; else hi = mid - 1;
      }
      int64_t s0, s1;
      seq_bounds(cu, lo, 0, total, s0, s1);
      const int64_t cidx = s - chunk_cu[lo], c0 = s0 + cidx * CH;
      if (c0 < s1) r = make_int4(lo, (int)cidx, (int)c0, (int)(s1 - c0 < CH ? s1 - c0 : CH));
    }
    info[s] = r;
  }
}

// order[r] = the sequence with the r-th most chunks (ties: lower index first); one CTA:
// the chunk counts go to shared memory, then each thread ranks its sequences against all.
constexpr int kOrderMaxSeqs = 2048;
__global__ void __launch_bounds__(1024) seq_order_kernel(const int32_t *cu, int N, int64_t total,
                                                         int32_t *order) {
  __shared__ int32_t nch[kOrderMaxSeqs];
  if (N > kOrderMaxSeqs) {   // many short sequences: the tail matters little, keep the order
    for (int n = threadIdx.x; n < N; n += blockDim.x) order[n] = n;
    return;
  }
  for (int n = threadIdx.x; n < N; n += blockDim.x) {
    int64_t s, e;
    seq_bounds(cu, n, 0, total, s, e);
    nch[n] = (int32_t)((e - s + CH - 1) / CH);
  }
  __syncthreads();
  for (int n = threadIdx.x; n < N; n += blockDim.x) {
    const int32_t c = nch[n];
    int rank = 0;
    for (int m = 0; m < N; ++m) rank += (nch[m] > c) | (nch[m] == c && m < n);
    order[rank] = n;
  }
}

}  // namespace prep

static_assert(kChunkRecordBytes == chunkfmt::REC_STRIDE, "record size");

cudaError_t launch_seq_order(const int32_t *cu, int N, int64_t total, int32_t *order, cudaStream_t stream) {
  if (N <= 0) return cudaSuccess;
  prep::seq_order_kernel<<<1, 1024, 0, stream>>>(cu, N, total, order);
  return cudaGetLastError();
}

cudaError_t launch_slot_table(const int32_t *cu, const int32_t *chunk_cu, int N, int64_t total,
                              int64_t slots, int4 *info, cudaStream_t stream) {
  if (slots <= 0) return cudaSuccess;
  const int64_t blocks = (slots + 255) / 256;
  prep::slot_table_kernel<<<(unsigned)(blocks < 1024 ? blocks : 1024), 256, 0, stream>>>(cu, chunk_cu, N, total,
                                                                                       slots, info);
  return cudaGetLastError();
}

cudaError_t launch_chunk_table(const int32_t *cu, int N, int64_t total, int32_t *chunk_cu, int *err,
                               cudaStream_t stream) {
  prep::chunk_table_kernel<<<1, 32, 0, stream>>>(cu, N, total, chunk_cu, err);
  return cudaGetLastError();
}

namespace {
template <bool kFused, int kSub>
cudaError_t launch_prep_sub(const PrepArgs &a, int64_t max_chunks, cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(prep::chunk_prep_kernel<kFused, kSub>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)prep::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  prep::chunk_prep_kernel<kFused, kSub><<<(unsigned)(max_chunks * a.H), prep::NT, prep::SMEM_BYTES, stream>>>(a);
  return cudaGetLastError();
}
// 32-token sub-blocks split each decay factor over at most 16 gates: within 2^{+-116}
// (the margin the 16-token blocks keep at a bound of -10) while |lower_bound| <= 5.02.
constexpr float kSub32MinLowerBound = -5.02f;
template <bool kFused>
cudaError_t launch_prep_variant(const PrepArgs &a, int64_t max_chunks, cudaStream_t stream) {
  return a.lower_bound >= kSub32MinLowerBound ? launch_prep_sub<kFused, 32>(a, max_chunks, stream)
                                              : launch_prep_sub<kFused, 16>(a, max_chunks, stream);
}
}  // namespace

cudaError_t launch_chunk_prep(PrepArgs a, int64_t max_chunks, bool fused, const void *q,
                              const void *k, const void *v, const void *alpha, cudaStream_t stream) {
  if (max_chunks == 0 || a.H == 0 || a.total_tokens == 0) return cudaSuccess;
  a.max_slots = max_chunks;
  if (a.chunk_cu == nullptr && a.seg_len > 0) max_chunks = (int64_t)a.N * a.seg_len;   // grid of a segment
  if (!fused) return launch_prep_variant<false>(a, max_chunks, stream);
  const uint64_t rows = (uint64_t)a.total_tokens, cols = (uint64_t)a.H * chunkfmt::DK;
  const CUtensorMapDataType bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if (!encode_rows(&a.map_q, q, bf, 2, rows, cols, cols, prep::RAW_ROWS, chunkfmt::DK) ||
      !encode_rows(&a.map_k, k, bf, 2, rows, cols, cols, prep::RAW_ROWS, chunkfmt::DK) ||
      !encode_rows(&a.map_v, v, bf, 2, rows, cols, cols, prep::RAW_ROWS, chunkfmt::DK) ||
      !encode_rows(&a.map_alpha, alpha, bf, 2, rows, cols, cols, chunkfmt::CH, chunkfmt::DK))
    return cudaErrorInvalidValue;
  return launch_prep_variant<true>(a, max_chunks, stream);
}

}  // namespace kda
