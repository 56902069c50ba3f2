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
// shared-memory image), double-buffered.
//
// Only D stands between one chunk's state and the next, so the chain per chunk
// is: the S^T W^T MMA -> D + U to bf16 -> the state-update MMA -> the state's
// bf16 copy; the output MMAs fill the tensor pipe while the chain's epilogue
// steps run.  Warp-specialised roles:
//   warps 0-7   the chain: two warpgroups over the same TMEM lanes (warp w reads
//               lane quadrant w % 4), each taking half of the columns of every
//               step (D to bf16; the state's bf16 copy and its decay);
//   warps 8-11  the output: each chunk's O^T leaves TMEM, transposed through
//               shared memory into 16-byte row stores, off the chain;
//   warp 12     MMA issue; warp 13 record copies; warp 14 output-gate copies;
//   warp 15     waits on the mbarriers the D MMA also depends on (the chunk's record
//               has landed, its O^T buffer is free), so the MMA-issuing thread
//               waits on none (a thread that issues tcgen05 MMAs sees even a
//               completed mbarrier phase several hundred cycles late).
// The chain hands its bf16 copies to the MMA warp at named barriers ("the bf16
// state copy is ready", with warp 15; "D in bf16 is ready"), a few tens of cycles
// each.  The other hand-offs are mbarriers: the MMA commits, "chunk c's MMAs are
// done" (its record buffer is free; its O^T can leave) and "O^T of chunk c has
// left" (its TMEM buffer is free).  O^T has four TMEM buffers (chunk index mod 4).
//
// Optional output epilogue (the layer's o_norm and sigmoid output gate, same
// write-up sections "二" and "三"): o <- o / sqrt(mean o^2 + eps) * w * sigmoid(gate)
// per (token, head).  Warp 14 streams the chunk's gate tile by TMA into one of two
// slots; the transpose then stages o in fp32 so that the norm sees it unrounded.
#include "chunk_common.cuh"
#include "kda_common.cuh"
#include "kda_internal.h"
#include "tma_host.h"
#include "umma.cuh"

namespace kda {
namespace spass {

using namespace chunkfmt;

constexpr int NCH = 256;         // chain threads (warps 0-7)
constexpr int NO = 128;          // output threads (warps 8-11)
constexpr int W_MMA = 12, W_REC = 13, W_GATE = 14, W_WAIT = 15;
constexpr int NT = 512;
constexpr uint32_t BAR_OUT = 1;   // named barrier of the output warps
constexpr uint32_t BAR_GO_D = 2;  // chain + waiter -> MMA warp: chunk c's D / O MMAs may go
constexpr uint32_t BAR_GO_S = 3;  // chain -> MMA warp: chunk c's state / O MMAs may go
// Every thread of the chain, the waiter and the MMA warp meets at BAR_GO_D once per chunk,
// and the chain and the MMA warp at BAR_GO_S, whatever happens (no role leaves its loop
// early), so no role can run a barrier generation ahead of another.
constexpr uint32_t N_GO_D = NCH + 64;
constexpr uint32_t N_GO_S = NCH + 32;
constexpr uint32_t OFF_REC0 = 0;
constexpr uint32_t OFF_REC1 = REC_STRIDE;
constexpr uint32_t OFF_OST = 2 * REC_STRIDE;   // o of one chunk, [64 t][128 j]: bf16, or fp32 when gated
constexpr uint32_t OFF_GATE = OFF_OST + CH * DK * 4;   // output gate tiles, 2 x bf16 [64 t][128 j]
constexpr uint32_t GATE_BYTES = CH * DK * 2;
constexpr uint32_t OFF_BAR = OFF_GATE + 2 * GATE_BYTES;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 256;
constexpr uint32_t SMEM_ALLOC = SMEM_BYTES + 1024;
static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
static_assert(REC_STRIDE % 1024 == 0, "SW128 alignment");

// TMEM columns (512 allocated).  The bf16 state copy and D are read only by MMAs
// that precede, in the tensor pipe's order, the next write of them: one buffer each.
constexpr uint32_t TM_S32 = 0;     // S^T fp32, 128 cols
constexpr uint32_t TM_S16 = 128;   // S^T bf16 A operand, 64 cols
constexpr uint32_t TM_D = 192;     // D^T fp32, 64 cols; its bf16 copy is packed in place:
                                   // tokens 0-31 into cols 0-15, tokens 32-63 into cols 32-47
constexpr uint32_t TM_O = 256;     // O^T fp32, 4 x 64 cols (chunk index mod 4)
constexpr int NOBUF = 4;
__device__ __forceinline__ uint32_t o_cols(int c) { return TM_O + (uint32_t)(c & (NOBUF - 1)) * 64; }
// bf16 D^T columns of MMA k-step s (tokens 16s .. 16s+15), packed where each warpgroup read them
__device__ __forceinline__ uint32_t d16_col(int s) { return TM_D + (uint32_t)(32 * (s >> 1) + 8 * (s & 1)); }

// B_OC / B_OE: one per O^T buffer (commit of chunk c's MMAs / its O^T has left TMEM)
enum { B_FULL0 = 0, B_FULL1, B_D, B_S, B_REL0, B_REL1, B_OC0, B_OC1, B_OC2, B_OC3,
       B_OE0, B_OE1, B_OE2, B_OE3, B_G0, B_G1, B_GE0, B_GE1, B_COUNT };
constexpr uint32_t BAR_AREA = 256;
static_assert(8 * B_COUNT + 16 <= BAR_AREA, "barrier area");

__global__ void __launch_bounds__(NT, 1) state_pass_kernel(const __grid_constant__ StateArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = a.H;
  const int n = a.order != nullptr ? a.order[blockIdx.x / H] : (int)(blockIdx.x / H);
  const int h = blockIdx.x % H;
  int64_t s0, s1;
  seq_bounds(a.cu, n, a.seq_len, a.total_tokens, s0, s1);
  // this launch's chunks [k0, k1) of the sequence (a time segment, or all of it)
  const int nall = (int)((s1 - s0 + CH - 1) / CH);
  const int k0 = min(a.seg_c0, nall), k1 = min(a.seg_c1, nall);
  int nchunks = k1 - k0;
  const int64_t t0 = s0 + (int64_t)k0 * CH;   // first token of chunk 0 of this launch
  int64_t chunk0 = (a.chunk_cu ? (int64_t)a.chunk_cu[n] : (int64_t)n * ((a.seq_len + CH - 1) / CH)) + k0;
  // only malformed cu_seqlens (overlapping clamped sequences) can exceed the record slots
  if (chunk0 < 0 || chunk0 > a.max_slots) chunk0 = a.max_slots;
  if (chunk0 + nchunks > a.max_slots) nchunks = (int)(a.max_slots - chunk0);
  const uint8_t *recs = reinterpret_cast<const uint8_t *>(a.records);
  auto rec_ptr = [&](int c) { return recs + ((chunk0 + c) * H + h) * (int64_t)REC_STRIDE; };
  auto rec_off = [](int c) { return (c & 1) ? OFF_REC1 : OFF_REC0; };

  uint64_t *bar = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + OFF_BAR + 8 * B_COUNT);
  int *fail = reinterpret_cast<int *>(smem + OFF_BAR + 8 * B_COUNT + 8);
  const uint32_t sbase = umma::smem_u32(smem);

  if (warp == 0) {
    umma::tmem_alloc(tmem_slot, 512);
    umma::tmem_relinquish();
  }
  if (tid == 32) {
    for (int i = 0; i < B_COUNT; ++i)
      umma::mbar_init(&bar[i], ((i >= B_OE0 && i <= B_OE3) || i == B_GE0 || i == B_GE1) ? NO / 32 : 1);
    umma::mbar_fence_init();
    *fail = 0;
  }
  umma::fence_before_sync();
  __syncthreads();
  umma::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const bool gated = a.onw != nullptr;

  // Bounded wait; once any wait anywhere has given up (the shared fail flag), later
  // waits return at once, so every role runs out its loop without stalling and every
  // thread of a role keeps the same control flow (addresses never depend on data).
  auto wait_one = [&](uint64_t *bb, uint32_t parity) {
    if (*(volatile int *)fail == 0 && !umma::mbar_wait_bounded(bb, parity, a.wait_polls))
      *(volatile int *)fail = 1;
    umma::fence_after_sync();
  };

  // The issuing warps run their loops with all 32 lanes (only lane 0 issues): a wait
  // made by one lane while the rest of its warp sits at the block barrier at the end
  // costs several hundred cycles even on a completed barrier.  wait_warp makes the
  // outcome warp-uniform.
  auto wait_warp = [&](uint64_t *bb, uint32_t parity) -> bool {
    bool ok = *(volatile int *)fail == 0 && umma::mbar_wait_bounded(bb, parity, a.wait_polls);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok && lane == 0) *(volatile int *)fail = 1;
    umma::fence_after_sync();
    return ok;
  };

  if (warp >= W_MMA) {
    if (warp == W_GATE && gated) {
      // ---------------------------------------------------------- output-gate copies
      // chunk c's 64 gate rows into slot c % 2 once chunk c-2's o has left it
      int issued = 0;
      for (int c = 0; c < nchunks; ++c) {
        if (c >= 2 && !wait_warp(&bar[B_GE0 + (c & 1)], ((c >> 1) - 1) & 1)) break;
        if (lane == 0) {
          umma::mbar_arrive_expect_tx(&bar[B_G0 + (c & 1)], GATE_BYTES);
          umma::tma_load_2d(smem + OFF_GATE + (c & 1) * GATE_BYTES, &a.map_gate, h * DK,
                            (int)(t0 + (int64_t)c * CH), &bar[B_G0 + (c & 1)]);
        }
        __syncwarp();
        issued = c + 1;
      }
      // copies still in flight into this CTA's shared memory: wait (bounded) for them
      for (int k = issued - 2 < 0 ? 0 : issued - 2; k < issued; ++k)
        (void)umma::mbar_wait_bounded(&bar[B_G0 + (k & 1)], (k >> 1) & 1, kWaitPolls);
    } else if (warp == W_REC) {
      // ---------------------------------------------------------- record copies
      // chunk c+2 goes into chunk c's buffer once every MMA of chunk c is done (the
      // chain reads U and e^{Gamma_C} from it before the hand-offs those MMAs need)
      int c = 0;
      for (; c < 2 && c < nchunks; ++c) {
        if (lane == 0) {
          umma::mbar_arrive_expect_tx(&bar[B_FULL0 + c], REC_BYTES);
          umma::bulk_g2s(smem + rec_off(c), rec_ptr(c), REC_BYTES, &bar[B_FULL0 + c]);
        }
      }
      __syncwarp();
      int issued = c;
      for (c = 0; c + 2 < nchunks; ++c) {
        if (!wait_warp(&bar[B_REL0 + (c & 1)], (c >> 1) & 1)) break;
        if (lane == 0) {
          umma::mbar_arrive_expect_tx(&bar[B_FULL0 + (c & 1)], REC_BYTES);
          umma::bulk_g2s(smem + rec_off(c), rec_ptr(c + 2), REC_BYTES, &bar[B_FULL0 + (c & 1)]);
        }
        __syncwarp();
        issued = c + 3;
      }
      for (int k = issued - 2 < 0 ? 0 : issued - 2; k < issued; ++k)
        (void)umma::mbar_wait_bounded(&bar[B_FULL0 + (k & 1)], (k >> 1) & 1, kWaitPolls);
    } else if (warp == W_WAIT) {
      // ---------------------------------------------------------- waits for the MMA issue
      // This warp meets the chain and the MMA warp at BAR_GO_D once per chunk, every chunk,
      // whatever happens (after a failed wait the mbarrier waits return at once and the MMA
      // warp issues nothing), so no role can be left waiting at it.
      // Chunk c+1's record and O^T buffer (normally long ready) are waited for while chunk
      // c's state MMA and bf16 state copy run: even a completed wait costs a few hundred
      // cycles, and only the bf16 state copy should stand before the D MMA.
      auto pre = [&](int cc) {
        (void)(wait_warp(&bar[B_FULL0 + (cc & 1)], (cc >> 1) & 1) &&
               (cc < NOBUF || wait_warp(&bar[B_OE0 + (cc & (NOBUF - 1))], ((cc / NOBUF) - 1) & 1)));
      };
      if (nchunks > 0) pre(0);
      for (int c = 0; c < nchunks; ++c) {
        umma::named_sync(BAR_GO_D, N_GO_D);   // with the chain's bf16 state copy of chunk c
        if (c + 1 < nchunks) pre(c + 1);
      }
    } else if (warp == W_MMA) {
      // ---------------------------------------------------------- MMA issue
      const uint32_t id_d = umma::make_idesc_bf16(128, 64, 0, 1);
      const uint32_t id_o = umma::make_idesc_bf16(128, 64, 0, 0);
      const uint32_t id_s = umma::make_idesc_bf16(128, 128, 0, 1);
      uint64_t *last = nullptr;   // the barrier of the last commit and the phase it completes
      uint32_t last_parity = 0;
      // released by the chain and the waiter warp (the same named-barrier steps for every
      // chunk); after a failed wait anywhere nothing more is issued (warp-uniform)
      auto go = [&](uint32_t id, uint32_t count) -> bool {
        umma::named_sync(id, count);
        umma::fence_after_sync();
        return !__any_sync(0xffffffffu, *(volatile int *)fail != 0);
      };
      bool issuing = true;
      for (int c = 0; c < nchunks; ++c) {
        const int b = c & 1;
        const uint32_t rb = sbase + rec_off(c);
        const int ob = c & (NOBUF - 1);
        const uint32_t ocol = tmem + o_cols(c);
        issuing = go(BAR_GO_D, N_GO_D) && issuing;
        if (issuing && lane == 0) {
          // D^T = S^T (-W^T) (the chain: committed alone), then O^T = S^T Q~^T
#pragma unroll
          for (int s = 0; s < DK / 16; ++s)
            umma::mma_ts(tmem + TM_D, tmem + TM_S16 + (uint32_t)(s * 8), desc_mn_rows(rb + REC_WT, s), id_d, s > 0);
          umma::mma_commit(&bar[B_D]);
#pragma unroll
          for (int s = 0; s < DK / 16; ++s)
            umma::mma_ts(ocol, tmem + TM_S16 + (uint32_t)(s * 8), desc_k128(rb + REC_QT, 64, s), id_o, s > 0);
        }
        __syncwarp();
        if (issuing) {
          last = &bar[B_D];
          last_parity = c & 1;
        }
        issuing = go(BAR_GO_S, N_GO_S) && issuing;
        if (issuing && lane == 0) {
          // S^T += D^T K^ (the chain), then O^T += D^T A_qk^T
#pragma unroll
          for (int s = 0; s < CH / 16; ++s)
            umma::mma_ts(tmem + TM_S32, tmem + d16_col(s), desc_mn_tok(rb + REC_KH, s), id_s, 1);
          umma::mma_commit(&bar[B_S]);
#pragma unroll
          for (int s = 0; s < CH / 16; ++s)
            umma::mma_ts(ocol, tmem + d16_col(s), desc_k64(rb + REC_AQ, s), id_o, 1);
          umma::mma_commit(&bar[B_REL0 + b]);
          umma::mma_commit(&bar[B_OC0 + ob]);
        }
        __syncwarp();
        if (issuing) {
          last = &bar[B_OC0 + ob];
          last_parity = (c / NOBUF) & 1;
        }
      }
      // nothing of this CTA's may still run on the tensor cores when TMEM is freed
      if (last != nullptr) (void)umma::mbar_wait_bounded(last, last_parity, kWaitPolls);
    }
  } else if (warp >= NCH / 32) {
    // ------------------------------------------------------------ output (warps 8-11)
    const int ot = tid - NCH;                           // 0..127
    const int j = (warp & 3) * 32 + lane;               // TMEM lane = value channel
    const uint32_t lane_base = (uint32_t)(warp & 3) * 32u << 16;
    __nv_bfloat16 *__restrict__ o = reinterpret_cast<__nv_bfloat16 *>(a.o);
    __nv_bfloat16 *ost = reinterpret_cast<__nv_bfloat16 *>(smem + OFF_OST);
    float *ost32 = reinterpret_cast<float *>(smem + OFF_OST);
    float2 onw[4];   // epilogue weight of this thread's 8 channels (c16 = ot & 15 in every row pass)
    if (gated) {
      const float4 w0 = *reinterpret_cast<const float4 *>(a.onw + (ot & 15) * 8);
      const float4 w1 = *reinterpret_cast<const float4 *>(a.onw + (ot & 15) * 8 + 4);
      onw[0] = make_float2(w0.x, w0.y); onw[1] = make_float2(w0.z, w0.w);
      onw[2] = make_float2(w1.x, w1.y); onw[3] = make_float2(w1.z, w1.w);
    } else {
      onw[0] = onw[1] = onw[2] = onw[3] = f2(0.f);
    }
#pragma unroll 1
    for (int c = 0; c < nchunks; ++c) {
      const int ob = c & (NOBUF - 1);
      wait_one(&bar[B_OC0 + ob], (c / NOBUF) & 1);
      uint32_t r[2][32];
      umma::tmem_ld32(tmem + lane_base + o_cols(c), r[0]);
      umma::tmem_ld32(tmem + lane_base + o_cols(c) + 32, r[1]);
      umma::tmem_wait_ld();
      // O^T of chunk c is in registers: its TMEM buffer is free for chunk c+4
      umma::fence_before_sync();
      __syncwarp();
      if (lane == 0) umma::mbar_arrive(&bar[B_OE0 + ob]);
      const int64_t c0 = t0 + (int64_t)c * CH;
      const int nvalid = (int)min((int64_t)CH, s1 - c0);
      if (!gated) {
#pragma unroll
        for (int t = 0; t < CH; ++t)
          ost[t * DK + j] = __float2bfloat16_rn(a.scale * __uint_as_float(r[t >> 5][t & 31]));
        umma::named_sync(BAR_OUT, NO);
#pragma unroll
        for (int k = 0; k < CH * DK / 8 / NO; ++k) {
          const int q = ot + k * NO, t = q >> 4, c16 = q & 15;
          if (t < nvalid)
            *reinterpret_cast<uint4 *>(o + ((c0 + t) * H + h) * DK + c16 * 8) =
                *reinterpret_cast<const uint4 *>(ost + t * DK + c16 * 8);
        }
        umma::named_sync(BAR_OUT, NO);
      } else {
        // o in fp32 through shared memory; a token's 128 channels then sit in 16
        // consecutive lanes (8 each): the mean square by a 16-lane butterfly
#pragma unroll
        for (int t = 0; t < CH; ++t) ost32[t * DK + j] = a.scale * __uint_as_float(r[t >> 5][t & 31]);
        wait_one(&bar[B_G0 + (c & 1)], (c >> 1) & 1);
        umma::named_sync(BAR_OUT, NO);
        const uint8_t *gt = smem + OFF_GATE + (c & 1) * GATE_BYTES;
#pragma unroll 2
        for (int k = 0; k < CH * DK / 8 / NO; ++k) {
          const int q = ot + k * NO, t = q >> 4, c16 = q & 15;
          const float4 x0 = *reinterpret_cast<const float4 *>(ost32 + t * DK + c16 * 8);
          const float4 x1 = *reinterpret_cast<const float4 *>(ost32 + t * DK + c16 * 8 + 4);
          const uint4 graw = *reinterpret_cast<const uint4 *>(gt + t * (DK * 2) + c16 * 16);
          float2 x[4] = {make_float2(x0.x, x0.y), make_float2(x0.z, x0.w), make_float2(x1.x, x1.y),
                         make_float2(x1.z, x1.w)};
          float2 ss = mul2(x[0], x[0]);
#pragma unroll
          for (int e = 1; e < 4; ++e) ss = fma2(x[e], x[e], ss);
          float s2 = ss.x + ss.y;
#pragma unroll
          for (int off = 8; off >= 1; off >>= 1) s2 += __shfl_xor_sync(0xffffffffu, s2, off);
          const float rn = rsqrtf(s2 * (1.f / DK) + a.oeps);
          uint32_t w4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 sg = sigmoid2(bf2_f2(word(graw, e)));
            w4[e] = f2_bf2(mul2(mul2(x[e], f2(rn)), mul2(onw[e], sg)));
          }
          if (t < nvalid)
            *reinterpret_cast<uint4 *>(o + ((c0 + t) * H + h) * DK + c16 * 8) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
        umma::named_sync(BAR_OUT, NO);
        if (lane == 0) umma::mbar_arrive(&bar[B_GE0 + (c & 1)]);   // gate slot c % 2 is free again
      }
    }
  } else {
    // ------------------------------------------------------------ chain (warps 0-7)
    // Warp w reads TMEM lane quadrant w % 4; warpgroup hf = w / 4 takes tokens
    // 32hf .. 32hf+31 of D and key channels 64hf .. 64hf+63 of the state.
    const int hf = warp >> 2;
    const int j = (warp & 3) * 32 + lane;               // TMEM lane = value channel
    const uint32_t lane_base = (uint32_t)(warp & 3) * 32u << 16;
    const int64_t sg = ((int64_t)n * H + h) * DK * DK;
    // the snapshot slot that takes the state after chunk cc of this launch (a whole chunk), or nullptr
    auto snap_after = [&](int cl) -> float * {
      const int cc = cl + k0;   // chunk index within the sequence
      if (a.snap == nullptr || a.snap_chunks < 1 || (cc + 1) % a.snap_chunks != 0) return nullptr;
      const int js = (cc + 1) / a.snap_chunks - 1;
      if (js >= a.snap_cap) return nullptr;
      return a.snap + (((int64_t)n * a.snap_cap + js) * H + h) * DK * DK;
    };
    // this warp's TMEM stores are done: meet the MMA warp at named barrier `id` (the
    // canonical hand-off of tcgen05 stores to a tcgen05.mma issued by another thread)
    auto handoff_go = [&](uint32_t id, uint32_t count) {
      umma::tmem_wait_st();
      umma::fence_before_sync();
      umma::named_sync(id, count);
    };
    // This warpgroup's 64 S^T columns (key channels 64hf ..) *= e^{Gamma_C} of the record at rb;
    // with s16: also write their bf16 copy first; with snap: store the state as it stands
    // (before that decay) there, S[i][j] row-major
    const uint32_t scol = TM_S32 + 64 * hf;
    auto state_pass_over = [&](uint32_t rb, bool s16, float *snap) {
      const float4 *egc = reinterpret_cast<const float4 *>(smem + rb + REC_EGC) + 16 * hf;
      uint32_t x[2][32];
#pragma unroll
      for (int q = 0; q < 2; ++q) umma::tmem_ld32(tmem + lane_base + scol + q * 32, x[q]);
      umma::tmem_wait_ld();
      if (s16) {
        uint32_t p[32];
#pragma unroll
        for (int e = 0; e < 32; ++e)
          p[e] = pack_bf16(__uint_as_float(x[e >> 4][(e & 15) * 2]), __uint_as_float(x[e >> 4][(e & 15) * 2 + 1]));
        umma::tmem_st32(tmem + lane_base + TM_S16 + 32 * hf, p);
        handoff_go(BAR_GO_D, N_GO_D);   // the next D / O MMAs need only this copy
      }
      if (snap != nullptr) {   // lane j holds column j of S: each row store is 128 contiguous floats
#pragma unroll
        for (int i = 0; i < 64; ++i)
          __stcs(snap + (int64_t)(64 * hf + i) * DK + j, __uint_as_float(x[i >> 5][i & 31]));
      }
#pragma unroll
      for (int e4 = 0; e4 < 16; ++e4) {
        const float4 g = egc[e4];
        uint32_t *y = &x[e4 >> 3][(e4 & 7) * 4];
        const float2 lo = mul2(make_float2(__uint_as_float(y[0]), __uint_as_float(y[1])), make_float2(g.x, g.y));
        const float2 hi = mul2(make_float2(__uint_as_float(y[2]), __uint_as_float(y[3])), make_float2(g.z, g.w));
        y[0] = __float_as_uint(lo.x); y[1] = __float_as_uint(lo.y);
        y[2] = __float_as_uint(hi.x); y[3] = __float_as_uint(hi.y);
      }
#pragma unroll
      for (int q = 0; q < 2; ++q) umma::tmem_st32(tmem + lane_base + scol + q * 32, x[q]);
    };

    // initial state: S^T[j][i] = S0[i][j] (fp32, and the bf16 copy), key channels 64hf ..
#pragma unroll 1
    for (int c = 64 * hf; c < 64 * hf + 64; c += 32) {
      uint32_t r[32], p[16];
#pragma unroll
      for (int e = 0; e < 32; ++e)
        r[e] = __float_as_uint(a.state0 ? a.state0[sg + (int64_t)(c + e) * DK + j] : 0.f);
#pragma unroll
      for (int e = 0; e < 16; ++e) p[e] = pack_bf16(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1]));
      umma::tmem_st32(tmem + lane_base + TM_S32 + c, r);
      umma::tmem_st16(tmem + lane_base + TM_S16 + c / 2, p);
    }
    if (nchunks > 0) {   // chunk 0's decay
      wait_one(&bar[B_FULL0], 0);
      umma::tmem_wait_st();
      state_pass_over(OFF_REC0, false, nullptr);
    }
    if (nchunks > 0) handoff_go(BAR_GO_D, N_GO_D);
#pragma unroll 1
    for (int c = 0; c < nchunks; ++c) {
      const uint32_t rb = rec_off(c);
      // (complete already, as the D MMA needed it: makes U visible here; waited before B_D
      // because even a complete barrier's wait costs a few hundred cycles)
      wait_one(&bar[B_FULL0 + (c & 1)], (c >> 1) & 1);
      wait_one(&bar[B_D], c & 1);
      // D^T + U^T -> bf16 A operand: this warpgroup's tokens 32hf .. 32hf+31, packed over
      // the first 16 of the 32 columns it read
      {
        uint32_t r[32], p[16];
        umma::tmem_ld32(tmem + lane_base + TM_D + 32 * hf, r);
        uint4 u[4];
        const uint8_t *urow = smem + rb + REC_U;
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8) u[c8] = *reinterpret_cast<const uint4 *>(urow + row64_off(j, 4 * hf + c8));
        umma::tmem_wait_ld();
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8) {   // tokens 32hf + 8c8 .. +7
          const uint32_t *x = &r[c8 * 8];
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            const float2 d = add2(make_float2(__uint_as_float(x[2 * w]), __uint_as_float(x[2 * w + 1])),
                                  bf2_f2(word(u[c8], w)));
            p[4 * c8 + w] = f2_bf2(d);
          }
        }
        umma::tmem_st16(tmem + lane_base + TM_D + 32 * hf, p);
      }
      handoff_go(BAR_GO_S, N_GO_S);
      if (c + 1 < nchunks) wait_one(&bar[B_FULL0 + ((c + 1) & 1)], ((c + 1) >> 1) & 1);   // its e^{Gamma_C}
      wait_one(&bar[B_S], c & 1);
      // the next chunk's bf16 state copy (handed off first), then its decay
      if (c + 1 < nchunks) state_pass_over(rec_off(c + 1), true, snap_after(c));
    }
    if (*(volatile int *)fail == 0) {
      // final state: S[i][j] = S^T[j][i] (and the last snapshot when this launch ends on one)
      umma::tmem_wait_st();
      // (a segment that ends inside the sequence ends on a whole chunk)
      float *last = nchunks > 0 && (k1 < nall ||
                                    (s1 - s0) % ((int64_t)CH * (a.snap_chunks > 0 ? a.snap_chunks : 1)) == 0)
                        ? snap_after(nchunks - 1) : nullptr;
#pragma unroll 1
      for (int cc = 64 * hf; cc < 64 * hf + 64; cc += 32) {
        uint32_t x[32];
        umma::tmem_ld32(tmem + lane_base + TM_S32 + cc, x);
        umma::tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          a.state1[sg + (int64_t)(cc + e) * DK + j] = __uint_as_float(x[e]);
          if (last != nullptr) last[(int64_t)(cc + e) * DK + j] = __uint_as_float(x[e]);
        }
      }
    }
  }
  umma::fence_before_sync();
  __syncthreads();
  if (tid == 0 && *(volatile int *)fail != 0 && a.err) atomicOr(a.err, ERR_TIMEOUT_STATE);
  if (warp == 0) {
    umma::fence_after_sync();
    umma::tmem_dealloc(tmem, 512);
  }
}

}  // namespace spass

cudaError_t launch_state_pass(StateArgs a, const void *gate, cudaStream_t stream) {
  if ((int64_t)a.N * a.H == 0) return cudaSuccess;
  if (a.onw != nullptr) {   // output epilogue: the gate [T rows][H * 128] in 64-row tiles
    if (gate == nullptr || a.total_tokens == 0) {
      a.onw = nullptr;
    } else {
      const uint64_t rows = (uint64_t)a.total_tokens, cols = (uint64_t)a.H * chunkfmt::DK;
      if (!encode_rows(&a.map_gate, gate, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, rows, cols, cols,
                       chunkfmt::CH, chunkfmt::DK))
        return cudaErrorInvalidValue;
    }
  }
  cudaError_t e = cudaFuncSetAttribute(spass::state_pass_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)spass::SMEM_ALLOC);
  if (e != cudaSuccess) return e;
  spass::state_pass_kernel<<<a.N * a.H, spass::NT, spass::SMEM_ALLOC, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace kda
