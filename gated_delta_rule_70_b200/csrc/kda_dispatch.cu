// Dispatch of the recurrence and of the whole prefill.
//
// bf16 with head_dim 128 (and a gate bound the chunk factorisation can hold)
// runs the tensor-core chunk path: chunk_prep over every (chunk, head), then
// the sequential state pass.  For a prefill chunk_prep also runs the prologue
// on the raw inputs, so conv'd / normalised q, k, v and the gates never travel
// through device memory.  Every other shape runs the prologue kernel and the
// CUDA-core token kernel.
#include <climits>
#include <mutex>
#include <vector>

#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {

namespace {

// Optional per-kernel timing of the chunk path (kda_kernel_timing / kda_kernel_times).
struct KernelClock {
  std::mutex mu;
  bool on = false;
  std::vector<cudaEvent_t> ev;   // 3 per recorded call
};
KernelClock g_clock;
constexpr size_t kMaxTimedCalls = 4096;

void drop_events_locked() {
  for (cudaEvent_t e : g_clock.ev) cudaEventDestroy(e);
  g_clock.ev.clear();
}

// Records one event on `stream` when timing is on and this call is being timed.
void clock_mark(bool timed, cudaStream_t stream) {
  if (!timed) return;
  cudaEvent_t e;
  if (cudaEventCreate(&e) != cudaSuccess) return;
  cudaEventRecord(e, stream);
  std::lock_guard<std::mutex> lock(g_clock.mu);
  g_clock.ev.push_back(e);
}

bool clock_begin() {
  std::lock_guard<std::mutex> lock(g_clock.mu);
  return g_clock.on && g_clock.ev.size() / 3 < kMaxTimedCalls;
}

// Time segments: when a dense batch has few (sequence, head) chains, the state pass
// occupies few SMs for a long time while the rest idle.  Given a side stream by the
// caller, the chunks are then split into segments of kSegChunks: chunk_prep of segment
// s+1 runs on the caller's stream while the state pass of segment s runs on the side
// stream (the state passes carry the state from one segment to the next through
// final_state).  Only stream order and two events, created and released by the call,
// connect the two: no kernel waits on another.  (Measured on the 1 x 262144 x 32
// prefill: segments of 32, 64, 128, 256 and 512 chunks gave 12.3, 10.9, 10.1, 10.2 and
// 10.6 ms.)
constexpr int kSegChunks = 128;

// The call's two events (prep of a segment done; the last state pass done).
struct SegEvents {
  cudaEvent_t prep = nullptr, pass = nullptr;
  cudaError_t create() {
    cudaError_t e = cudaEventCreateWithFlags(&prep, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&pass, cudaEventDisableTiming);
    return e;
  }
  // (an event may be destroyed while work that records or waits on it is pending)
  ~SegEvents() {
    if (prep) cudaEventDestroy(prep);
    if (pass) cudaEventDestroy(pass);
  }
};

cudaError_t run_chunk_path(PrepArgs pa, const RecurrenceArgs &ra, bool varlen, bool fused,
                           const PrologueArgs *raw, char *ws, const WsLayout &L,
                           cudaStream_t stream) {
  int32_t *chunk_cu = nullptr, *order = nullptr;
  int4 *slot_info = nullptr;
  const int64_t slots = max_chunk_slots(ra.N, ra.total_tokens, ra.seq_len, varlen);
  if (varlen) {
    chunk_cu = reinterpret_cast<int32_t *>(ws + L.chunk_cu);
    order = reinterpret_cast<int32_t *>(ws + L.order);
    slot_info = reinterpret_cast<int4 *>(ws + L.slots);
    cudaError_t e = launch_chunk_table(ra.cu, ra.N, ra.total_tokens, chunk_cu, ra.err, stream);
    if (e == cudaSuccess) e = launch_slot_table(ra.cu, chunk_cu, ra.N, ra.total_tokens, slots, slot_info, stream);
    if (e == cudaSuccess) e = launch_seq_order(ra.cu, ra.N, ra.total_tokens, order, stream);
    if (e != cudaSuccess) return e;
  }
  pa.N = ra.N; pa.H = ra.H; pa.seq_len = ra.seq_len; pa.total_tokens = ra.total_tokens;
  pa.cu = ra.cu; pa.chunk_cu = chunk_cu; pa.slot_info = slot_info;
  pa.records = ws + L.records; pa.err = ra.err; pa.wait_polls = ra.wait_polls;
  StateArgs sa{};
  sa.N = ra.N; sa.H = ra.H; sa.seq_len = ra.seq_len; sa.total_tokens = ra.total_tokens;
  sa.cu = ra.cu; sa.chunk_cu = chunk_cu; sa.order = order; sa.records = ws + L.records; sa.max_slots = slots;
  sa.state0 = ra.state0; sa.scale = ra.scale; sa.o = ra.o; sa.state1 = ra.state1; sa.err = ra.err;
  sa.wait_polls = ra.wait_polls;
  sa.seg_c0 = 0; sa.seg_c1 = INT_MAX;
  if (ra.ogate != nullptr) { sa.onw = ra.onw; sa.oeps = ra.oeps; }
  if (ra.snap != nullptr) { sa.snap = ra.snap; sa.snap_chunks = (int)(ra.snap_every / 64); sa.snap_cap = ra.snap_cap; }
  const void *rq = raw ? raw->q : nullptr, *rk = raw ? raw->k : nullptr;
  const void *rv = raw ? raw->v : nullptr, *ralpha = raw ? raw->alpha : nullptr;

  const int64_t per = varlen ? 0 : (ra.seq_len + 63) / 64;
  cudaStream_t side = ra.side_stream;
  SegEvents ev;
  bool segmented = !varlen && per >= 2 * kSegChunks && ra.state1 != nullptr && side != nullptr;
  if (segmented) {
    int dev = 0, sms = 0;
    cudaError_t e0 = cudaGetDevice(&dev);
    if (e0 == cudaSuccess) e0 = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e0 != cudaSuccess) return e0;
    segmented = 2 * (int64_t)ra.N * ra.H <= sms;
    if (segmented && (e0 = ev.create()) != cudaSuccess) return e0;
  }

  const bool timed = clock_begin();
  clock_mark(timed, stream);
  cudaError_t e = cudaSuccess;
  if (!segmented) {
    e = launch_chunk_prep(pa, slots, fused, rq, rk, rv, ralpha, stream);
    clock_mark(timed, stream);
    if (e == cudaSuccess) e = launch_state_pass(sa, ra.ogate, stream);
    else clock_mark(timed, stream);   // keep the events in triples
    clock_mark(timed, stream);
    return e;
  }
  // segment s: chunk_prep on `stream`, then (after it, on the side stream) the state pass,
  // which starts from the state the previous segment's pass left in final_state
  const int nseg = (int)((per + kSegChunks - 1) / kSegChunks);
  for (int sg = 0; sg < nseg && e == cudaSuccess; ++sg) {
    pa.seg_c0 = sg * kSegChunks;
    pa.seg_len = kSegChunks;
    e = launch_chunk_prep(pa, slots, fused, rq, rk, rv, ralpha, stream);
    if (e == cudaSuccess) e = cudaEventRecord(ev.prep, stream);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(side, ev.prep, 0);
    if (e == cudaSuccess) {
      StateArgs ss = sa;
      ss.seg_c0 = sg * kSegChunks;
      ss.seg_c1 = sg + 1 == nseg ? INT_MAX : (sg + 1) * kSegChunks;
      if (sg > 0) ss.state0 = ra.state1;
      e = launch_state_pass(ss, ra.ogate, side);
    }
  }
  clock_mark(timed, stream);
  // the caller's stream continues only after the last state pass (also on an error, so
  // that nothing of this call is left running unordered)
  cudaError_t e2 = cudaEventRecord(ev.pass, side);
  if (e2 == cudaSuccess) e2 = cudaStreamWaitEvent(stream, ev.pass, 0);
  clock_mark(timed, stream);
  return e != cudaSuccess ? e : e2;
}

}  // namespace

cudaError_t run_recurrence(const RecurrenceArgs &ra, bool varlen, char *ws, const WsLayout &L,
                           cudaStream_t stream) {
#ifndef KDA_TOKEN_KERNEL_ONLY
  if (L.tc) {
    PrepArgs pa{};
    pa.qn = ra.qn; pa.kn = ra.kn; pa.vc = ra.vc; pa.g = ra.g; pa.beta = ra.beta;
    pa.lower_bound = ra.lower_bound;
    return run_chunk_path(pa, ra, varlen, false, nullptr, ws, L, stream);
  }
#endif
  return launch_cuda_core_recurrence(ra, stream);
}

cudaError_t run_prefill(PrologueArgs pa, RecurrenceArgs ra, void *final_conv_state, bool varlen,
                        char *ws, const WsLayout &L, cudaStream_t stream) {
  cudaError_t e = cudaSuccess;
#ifndef KDA_TOKEN_KERNEL_ONLY
  if (L.tc) {
    PrepArgs p{};
    p.lower_bound = pa.lower_bound; p.eps = pa.eps; p.beta2 = pa.beta2;
    p.conv_w = pa.conv_w; p.b = pa.b; p.A_log = pa.A_log; p.dt_bias = pa.dt_bias; p.conv0 = pa.conv0;
    e = run_chunk_path(p, ra, varlen, true, &pa, ws, L, stream);
  } else
#endif
  {
    pa.qn = ws + L.qn; pa.kn = ws + L.kn; pa.vc = ws + L.vc;
    pa.g = reinterpret_cast<float *>(ws + L.g);
    pa.beta = reinterpret_cast<float *>(ws + L.beta);
    if ((e = launch_prologue(pa, stream)) != cudaSuccess) return e;
    ra.qn = pa.qn; ra.kn = pa.kn; ra.vc = pa.vc; ra.g = pa.g; ra.beta = pa.beta;
    e = launch_cuda_core_recurrence(ra, stream);
  }
  if (e != cudaSuccess) return e;
  if (final_conv_state != nullptr) e = launch_conv_state_out(pa, final_conv_state, stream);
  return e;
}

}  // namespace kda

extern "C" int kda_kernel_timing(int enable) {
  std::lock_guard<std::mutex> lock(kda::g_clock.mu);
  kda::g_clock.on = enable != 0;
  if (!kda::g_clock.on) kda::drop_events_locked();
  return 0;
}

extern "C" int kda_kernel_times(float *prep_ms, float *state_ms) {
  std::lock_guard<std::mutex> lock(kda::g_clock.mu);
  const size_t calls = kda::g_clock.ev.size() / 3;
  double a = 0.0, b = 0.0;
  bool ok = true;
  for (size_t c = 0; c < calls && ok; ++c) {
    cudaEvent_t *e = &kda::g_clock.ev[3 * c];
    float x = 0.f, y = 0.f;
    ok = cudaEventSynchronize(e[2]) == cudaSuccess && cudaEventElapsedTime(&x, e[0], e[1]) == cudaSuccess &&
         cudaEventElapsedTime(&y, e[1], e[2]) == cudaSuccess;
    a += x;
    b += y;
  }
  kda::drop_events_locked();
  if (prep_ms) *prep_ms = calls && ok ? (float)(a / calls) : 0.f;
  if (state_ms) *state_ms = calls && ok ? (float)(b / calls) : 0.f;
  return ok ? (int)calls : -1;
}
