// KDA state pass: the sequential part of the chunkwise recurrence, one CTA per
// (sequence, head), on tcgen05 tensor cores with the fp32 state resident in
// TMEM.
//
// Per 64-token chunk, with the record chunk_prep wrote (-W^T, U^T, A_qk,
// q e^{Gamma}, k e^{Gamma_C - Gamma}, e^{Gamma_C}):
//   D^T = U^T - S^T W^T
//   O^T = S^T (q e^{Gamma})^T + D^T A_qk^T
//   S^T <- S^T diag(e^{Gamma_C}) + D^T (k e^{Gamma_C - Gamma})
// i.e. the per-token loop of the AliceAI-Foundation KDA write-up ("二、KDA
// 线性注意力": decay, predict, correct, write, read) re-associated per chunk.
//
// The state is kept transposed: S^T [d_v lanes x d_k columns] fp32 in TMEM
// (M = 128 on the value channel), with a bf16 copy in TMEM as the A operand.
// Records arrive by one contiguous bulk copy each (they are stored as their
// shared-memory image), double-buffered: the copy of chunk c+2 starts as soon
// as chunk c's MMAs have read its buffer.
//
// Only D stands between one chunk's state and the next, so the chain per chunk
// is: the S^T W^T MMA -> D + U to bf16 -> the state-update MMA -> the state's
// bf16 copy.  The pass that makes that copy also applies the next chunk's decay
// to the fp32 state (the next record is normally resident by then), and O is
// double-buffered in TMEM so that chunk c-1's output leaves while chunk c's
// MMAs run: transposed through shared memory into 16-byte row stores.
#include "chunk_common.cuh"
#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {
namespace spass {

using namespace chunkfmt;

constexpr int NT = 128;
constexpr uint32_t OFF_REC0 = 0;
constexpr uint32_t OFF_REC1 = REC_STRIDE;
constexpr uint32_t OFF_OST = 2 * REC_STRIDE;   // o of one chunk, bf16 [64 t][128 j]: 16 KB
constexpr uint32_t OFF_BAR = OFF_OST + CH * DK * 2;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 64;
constexpr uint32_t SMEM_ALLOC = SMEM_BYTES + 1024;
static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
static_assert(REC_STRIDE % 1024 == 0, "SW128 alignment");

// TMEM columns (512 allocated)
constexpr uint32_t TM_S32 = 0;     // S^T fp32, 128 cols
constexpr uint32_t TM_S16 = 128;   // S^T bf16 A operand, 64 cols
constexpr uint32_t TM_D = 192;     // D^T fp32, 64 cols; its bf16 copy (32 cols) is packed in place
constexpr uint32_t TM_O = 256;     // O^T fp32, 2 x 64 cols (chunk parity)

constexpr uint32_t WAIT_POLLS = 1u << 22;
enum { B_FULL0 = 0, B_FULL1, B_D, B_S, B_COUNT };

__device__ __forceinline__ bool wait_vote(uint64_t *bar, uint32_t parity, bool ok) {
  const bool mine = ok && umma::mbar_wait_bounded(bar, parity, WAIT_POLLS);
  const bool all = __syncthreads_and(mine) != 0;
  umma::fence_after_sync();
  return all;
}

__global__ void __launch_bounds__(NT, 1) state_pass_kernel(StateArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5;
  const int H = a.H;
  const int n = blockIdx.x / H, h = blockIdx.x % H;
  int64_t s0, s1;
  seq_bounds(a.cu, n, a.seq_len, a.total_tokens, s0, s1);
  int nchunks = (int)((s1 - s0 + CH - 1) / CH);
  int64_t chunk0 = a.chunk_cu ? (int64_t)a.chunk_cu[n] : (int64_t)n * ((a.seq_len + CH - 1) / CH);
  // only malformed cu_seqlens (overlapping clamped sequences) can exceed the record slots
  if (chunk0 < 0 || chunk0 > a.max_slots) chunk0 = a.max_slots;
  if (chunk0 + nchunks > a.max_slots) nchunks = (int)(a.max_slots - chunk0);
  const uint8_t *recs = reinterpret_cast<const uint8_t *>(a.records);
  auto rec_ptr = [&](int c) { return recs + ((chunk0 + c) * H + h) * (int64_t)REC_STRIDE; };

  uint64_t *bar = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + OFF_BAR + 8 * B_COUNT);
  const uint32_t sbase = umma::smem_u32(smem);
  const int j = tid;                                  // TMEM lane = value channel
  const uint32_t lane_base = (uint32_t)warp * 32u << 16;
  const int64_t sg = ((int64_t)n * H + h) * DK * DK;
  __nv_bfloat16 *__restrict__ o = reinterpret_cast<__nv_bfloat16 *>(a.o);

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
  const uint32_t tmem = *tmem_slot;

  // first two records in flight
  if (tid == 0) {
    for (int c = 0; c < 2 && c < nchunks; ++c) {
      umma::mbar_arrive_expect_tx(&bar[B_FULL0 + c], REC_BYTES);
      umma::bulk_g2s(smem + (c ? OFF_REC1 : OFF_REC0), rec_ptr(c), REC_BYTES, &bar[B_FULL0 + c]);
    }
  }
  // initial state: S^T[j][i] = S0[i][j] (fp32 and bf16 copies)
#pragma unroll 1
  for (int c = 0; c < DK; c += 32) {
    uint32_t r[32], p[16];
#pragma unroll
    for (int e = 0; e < 32; ++e)
      r[e] = __float_as_uint(a.state0 ? a.state0[sg + (int64_t)(c + e) * DK + j] : 0.f);
#pragma unroll
    for (int e = 0; e < 16; ++e) p[e] = pack_bf16(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1]));
    umma::tmem_st32(tmem + lane_base + TM_S32 + c, r);
    umma::tmem_st16(tmem + lane_base + TM_S16 + c / 2, p);
  }
  umma::tmem_wait_st();
  umma::fence_before_sync();
  __syncthreads();

  // o of chunk cc (its O^T in TMEM columns ocol): lane j holds column j of the
  // chunk's 64 rows; a shared-memory transpose turns them into 16-byte row stores
  __nv_bfloat16 *ost = reinterpret_cast<__nv_bfloat16 *>(smem + OFF_OST);
  auto emit_o = [&](int cc, uint32_t ocol) {
    uint32_t r[2][32];
    umma::tmem_ld32(tmem + lane_base + ocol, r[0]);
    umma::tmem_ld32(tmem + lane_base + ocol + 32, r[1]);
    umma::tmem_wait_ld();
#pragma unroll
    for (int t = 0; t < CH; ++t) ost[t * DK + j] = __float2bfloat16_rn(a.scale * __uint_as_float(r[t >> 5][t & 31]));
    __syncthreads();
    const int64_t c0 = s0 + (int64_t)cc * CH;
    const int nvalid = (int)min((int64_t)CH, s1 - c0);
#pragma unroll
    for (int k = 0; k < CH * DK / 8 / NT; ++k) {
      const int q = tid + k * NT, t = q >> 4, c16 = q & 15;
      if (t < nvalid)
        *reinterpret_cast<uint4 *>(o + ((c0 + t) * H + h) * DK + c16 * 8) =
            *reinterpret_cast<const uint4 *>(ost + t * DK + c16 * 8);
    }
    __syncthreads();
  };
  // S^T columns *= e^{Gamma_C} of the record at rb; with bf16: also refresh the bf16 copy first
  auto state_pass_over = [&](uint32_t rb, bool decay, bool bf16) {
    const float4 *egc = reinterpret_cast<const float4 *>(smem + rb + REC_EGC);
#pragma unroll
    for (int cc = 0; cc < DK; cc += 64) {
      uint32_t x[2][32];
      umma::tmem_ld32(tmem + lane_base + TM_S32 + cc, x[0]);
      umma::tmem_ld32(tmem + lane_base + TM_S32 + cc + 32, x[1]);
      umma::tmem_wait_ld();
      if (bf16) {
        uint32_t p[32];
#pragma unroll
        for (int e = 0; e < 32; ++e)
          p[e] = pack_bf16(__uint_as_float(x[e >> 4][(e & 15) * 2]), __uint_as_float(x[e >> 4][(e & 15) * 2 + 1]));
        umma::tmem_st32(tmem + lane_base + TM_S16 + cc / 2, p);
      }
      if (decay) {
#pragma unroll
        for (int e4 = 0; e4 < 16; ++e4) {
          const float4 g = egc[cc / 4 + e4];
          uint32_t *y = &x[e4 >> 3][(e4 & 7) * 4];
          const float2 lo = mul2(make_float2(__uint_as_float(y[0]), __uint_as_float(y[1])), make_float2(g.x, g.y));
          const float2 hi = mul2(make_float2(__uint_as_float(y[2]), __uint_as_float(y[3])), make_float2(g.z, g.w));
          y[0] = __float_as_uint(lo.x); y[1] = __float_as_uint(lo.y);
          y[2] = __float_as_uint(hi.x); y[3] = __float_as_uint(hi.y);
        }
        umma::tmem_st32(tmem + lane_base + TM_S32 + cc, x[0]);
        umma::tmem_st32(tmem + lane_base + TM_S32 + cc + 32, x[1]);
      }
    }
    umma::tmem_wait_st();
  };

  bool ok = true;
#pragma unroll 1
  for (int c = 0; c < nchunks; ++c) {
    const int b = c & 1;
    const uint32_t rb = b ? OFF_REC1 : OFF_REC0;
    const uint32_t ocol = TM_O + (uint32_t)b * 64;
    ok = wait_vote(&bar[B_FULL0 + b], (c >> 1) & 1, ok);
    if (!ok) break;
    if (c == 0) {   // the first chunk's decay (later ones ride on the previous chunk's last pass)
      state_pass_over(rb, true, false);
      umma::fence_before_sync();
      __syncthreads();
      umma::fence_after_sync();
    }
    // D^T = S^T (-W^T) (committed alone: the chain needs only D^T); O^T = S^T Q~^T
    if (tid == 0) {
      const uint32_t id_d = umma::make_idesc_bf16(128, 64, 0, 1);
      const uint32_t id_o = umma::make_idesc_bf16(128, 64, 0, 0);
#pragma unroll
      for (int s = 0; s < DK / 16; ++s)
        umma::mma_ts(tmem + TM_D, tmem + TM_S16 + (uint32_t)(s * 8), desc_mn_rows(sbase + rb + REC_WT, s),
                     id_d, s > 0);
      umma::mma_commit(&bar[B_D]);
#pragma unroll
      for (int s = 0; s < DK / 16; ++s)
        umma::mma_ts(tmem + ocol, tmem + TM_S16 + (uint32_t)(s * 8), desc_k128(sbase + rb + REC_QT, 64, s),
                     id_o, s > 0);
    }
    // while those run: the previous chunk's o
    if (c > 0) emit_o(c - 1, TM_O + (uint32_t)(b ^ 1) * 64);
    ok = wait_vote(&bar[B_D], c & 1, ok);
    if (!ok) break;
    // D^T + U^T -> bf16 A operand, packed over the first 32 columns of D
    {
      uint32_t r[2][32], p[32];
      umma::tmem_ld32(tmem + lane_base + TM_D, r[0]);
      umma::tmem_ld32(tmem + lane_base + TM_D + 32, r[1]);
      umma::tmem_wait_ld();
      const uint8_t *urow = smem + rb + REC_U;
#pragma unroll
      for (int c8 = 0; c8 < 8; ++c8) {
        const uint4 u = *reinterpret_cast<const uint4 *>(urow + row64_off(j, c8));   // tokens 8c8 .. 8c8+7
        const uint32_t *x = &r[c8 >> 2][(c8 & 3) * 8];
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const float2 d = add2(make_float2(__uint_as_float(x[2 * w]), __uint_as_float(x[2 * w + 1])),
                                bf2_f2(word(u, w)));
          p[4 * c8 + w] = f2_bf2(d);
        }
      }
      umma::tmem_st32(tmem + lane_base + TM_D, p);
      umma::tmem_wait_st();
    }
    umma::fence_before_sync();
    __syncthreads();
    if (tid == 0) {
      umma::fence_after_sync();
      // S^T += D^T K^ first (the chain), then O^T += D^T A_qk^T
      const uint32_t id_s = umma::make_idesc_bf16(128, 128, 0, 1);
      const uint32_t id_o = umma::make_idesc_bf16(128, 64, 0, 0);
#pragma unroll
      for (int s = 0; s < CH / 16; ++s)
        umma::mma_ts(tmem + TM_S32, tmem + TM_D + (uint32_t)(s * 8), desc_mn_tok(sbase + rb + REC_KH, s),
                     id_s, 1);
#pragma unroll
      for (int s = 0; s < CH / 16; ++s)
        umma::mma_ts(tmem + ocol, tmem + TM_D + (uint32_t)(s * 8), desc_k64(sbase + rb + REC_AQ, s), id_o, 1);
      umma::mma_commit(&bar[B_S]);
    }
    ok = wait_vote(&bar[B_S], c & 1, ok);
    if (!ok) break;
    // this buffer has been read: start the copy of chunk c+2 into it
    if (tid == 0 && c + 2 < nchunks) {
      umma::mbar_arrive_expect_tx(&bar[B_FULL0 + b], REC_BYTES);
      umma::bulk_g2s(smem + rb, rec_ptr(c + 2), REC_BYTES, &bar[B_FULL0 + b]);
    }
    // the next chunk's A operand (bf16 copy of the state) and its decay, in one pass
    if (c + 1 < nchunks) {
      ok = wait_vote(&bar[B_FULL0 + (b ^ 1)], ((c + 1) >> 1) & 1, ok);
      if (!ok) break;
      state_pass_over(b ? OFF_REC0 : OFF_REC1, true, true);
    }
    umma::fence_before_sync();
    __syncthreads();
  }
  if (ok) {
    if (nchunks > 0) emit_o(nchunks - 1, TM_O + (uint32_t)((nchunks - 1) & 1) * 64);
    // final state: S[i][j] = S^T[j][i]
#pragma unroll 1
    for (int cc = 0; cc < DK; cc += 32) {
      uint32_t s[32];
      umma::tmem_ld32(tmem + lane_base + TM_S32 + cc, s);
      umma::tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 32; ++e) a.state1[sg + (int64_t)(cc + e) * DK + j] = __uint_as_float(s[e]);
    }
  } else {
    // a copy may still be in flight into this CTA's shared memory: wait (bounded) for it
    for (int c = 0; c < 2; ++c) (void)umma::mbar_wait_bounded(&bar[B_FULL0 + c], 0, WAIT_POLLS);
    if (tid == 0 && a.err) atomicExch(a.err, ERR_TIMEOUT);
  }
  umma::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    umma::fence_after_sync();
    umma::tmem_dealloc(tmem, 512);
  }
}

}  // namespace spass

cudaError_t launch_state_pass(const StateArgs &a, cudaStream_t stream) {
  if ((int64_t)a.N * a.H == 0) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(spass::state_pass_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)spass::SMEM_ALLOC);
  if (e != cudaSuccess) return e;
  spass::state_pass_kernel<<<a.N * a.H, spass::NT, spass::SMEM_ALLOC, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace kda
