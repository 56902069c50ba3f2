#!/usr/bin/env python
"""KDA forward benchmark on B200: prefill tokens/s (+ % of bf16 tensor peak) and
decode-step state GB/s (+ % of HBM), one JSON line on stdout.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Workloads (seeded, synthetic; see gated_delta_rule_70_b200/workloads.py):
  prefill  B=4, T=8192, H=32, d=128, bf16 I/O, fp32 state   (the step that `value` times)
  decode   256 sequences x 32 heads, d=128, state from a T=1024 prefill, 64 steps

A "step" is one kda_prefill call over the whole batch (chunk_prep with the
fused prologue, the state pass, the final conv-state copy), issued through the
C ABI with every input already resident in HBM.  The inputs (1.3 GB) are
larger than L2, so no flush is needed between steps.  Per-kernel durations come
from CUDA events the library records on the launching stream between its
kernels (kda_kernel_timing) inside the timed region.  `e2e` repeats the step through the same
C ABI with host (pinned) inputs: H2D copies, the prefill and the D2H read of
o and the final state are all inside its timed region, pipelined over three
streams with two device buffer sets (one step's H2D overlaps the previous
step's prefill and D2H).

Multi-GPU (torchrun, one process per GPU): the (sequence, head) units are
independent, so every rank runs its own batch with no data-path collective
(weak scaling); time is the max over ranks.

--impl reference times the fp64 CPU oracle (the CPU baseline) on a bounded
sample of the same workload on this host's cores; rank 0 only.
"""

from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

# DRAM bytes (read + write) of one chunk_prep launch on 4x8192x32: an ncu capture of the
# 1x8192x32 launch scaled by the chunk-heads (x4); None while the kernel has changed since
# the capture.
CHUNK_PREP_TRAFFIC_BYTES = 4 * (269.281536e6 + 254.379008e6)

HBM_FALLBACK_GBS = 6650.0
BF16_FALLBACK_TFLOPS = 1590.0
C = 64  # chunk length used for the algorithmic flop count


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": HBM_FALLBACK_GBS, "bf16_tflops": BF16_FALLBACK_TFLOPS,
            "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def prefill_flops_per_token_head(d: int, c: int = C) -> float:
    """Algorithmic flops of the chunked form per (token, head): C(3dk + 2dv) + 6 dk dv + C^2/3."""
    return c * (3 * d + 2 * d) + 6 * d * d + c * c / 3.0


def prefill_algorithmic_bytes(tokens: int, seqs: int, H: int, d: int, esz: int = 2) -> int:
    """The fused minimum a prefill must move: q, k, v and alpha in (4 H d), b in (H), o out
    (H d), all in the io dtype (41,024 B per token at H = 32, d = 128 bf16), plus the fp32
    initial and final states (2 N H d^2 x 4 B)."""
    return tokens * (4 * H * d * esz + H * esz + H * d * esz) + 2 * seqs * H * d * d * 4


def prologue_bytes_per_token_head(d: int, esz: int = 2) -> int:
    """The standalone prologue: q, k, v, alpha (4 d) and b in; q, k, v out (3 d) in the io
    dtype, g (d) and beta out in fp32: 2,310 B at d = 128 bf16."""
    return 4 * d * esz + esz + 3 * d * esz + 4 * d + 4


# ---------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for nm, val in zip(names, f[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": float(np.median(sm)) if sm else None,
                "sm_max_mhz": float(max(smax)) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- our arm

def run_ours(args, rank, world, local_rank):
    import torch
    from gated_delta_rule_70_b200 import build as kbuild
    from gated_delta_rule_70_b200 import kda
    from gated_delta_rule_70_b200 import workloads as W

    if rank == 0:
        kbuild.build_library()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    peaks = measured_peaks()

    if args.only == "decode":   # profiling run: the decode kernels on a random state
        sd, dec_ms, dec_gated_ms, dec_mtp_ms = decode_figures(dev, torch.cuda.current_stream(dev),
                                                              seeded=False)
        return {"metric": "decode only (profiling run)", "ms_per_step": float(np.median(dec_ms)),
                "output_gate_ms_per_step": dec_gated_ms,
                "two_tokens_with_step_states_ms_per_call": dec_mtp_ms} if rank == 0 else None

    s = W.spec("prefill_4x8k")
    if args.batch != 4:   # profiling runs: the same distributions on fewer sequences
        s = W.Spec("prefill_%dx8k" % args.batch, "bf16", [8192] * args.batch, H=32, d=128, seed=1,
                   s0_std=0.02)
    inp = W.make_inputs(s)
    N, H, d = s.num_seqs, s.H, s.d
    T_total = s.total_tokens
    up = lambda a: W.to_device(a, dev)
    q, k, v = up(inp["q"]), up(inp["k"]), up(inp["v"])
    conv_w, alpha, b = up(inp["conv_w"]), up(inp["alpha"]), up(inp["b"])
    A_log, dt_bias, S0 = up(inp["A_log"]), up(inp["dt_bias"]), up(inp["S0"])
    bf = torch.bfloat16
    fc = torch.empty((N, 3, 3 * H * d), dtype=bf, device=dev)
    o = torch.empty((T_total, H, d), dtype=bf, device=dev)
    fs = torch.empty((N, H, d, d), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    ws = torch.empty(kda.prefill_workspace_size(kda.make_shape(N, s.seq_lens[0], H, d, bf), False),
                     dtype=torch.uint8, device=dev)

    if args.only == "prologue":   # profiling run: the standalone prologue alone
        pro_ms = time_prologue(q, k, v, conv_w, alpha, b, A_log, dt_bias, N, stream, args.warmup,
                               args.steps)
        gbs = prologue_bytes_per_token_head(d) * T_total * H / (pro_ms * 1e-3) / 1e9
        return {"metric": "prologue only (profiling run)", "ms": pro_ms, "GB_s": gbs,
                "frac_of_measured_hbm": gbs / peaks["hbm_gbs"]} if rank == 0 else None

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        kda.prefill(q, k, v, conv_w, alpha, b, A_log, dt_bias, initial_state=S0, num_seqs=N,
                    out=o, final_state=fs, final_conv_state=fc, workspace=ws, check=False)
        if ev is not None:
            ev[1].record(stream)

    launches_per_step = 3  # chunk_prep (with the prologue), state_pass, final conv-state copy

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)

    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.3)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    kda.kernel_timing(True)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    elapsed_ms = t_start.elapsed_time(t_end)
    call_ms = float(np.mean([e[0].elapsed_time(e[1]) for e in evs]))
    timed_calls, prep_ms, state_ms = kda.kernel_times()
    kda.kernel_timing(False)

    # ---- the standalone prologue (conv4 + SiLU, L2 norm, gate, beta) on the same inputs
    pro_ms = time_prologue(q, k, v, conv_w, alpha, b, A_log, dt_bias, N, stream, args.warmup,
                           args.steps)
    pro_bytes = prologue_bytes_per_token_head(d) * T_total * H

    if args.only == "prefill":
        clock_info = clocks.stop()
        line = {"metric": "prefill only (profiling run)", "ms_per_step": elapsed_ms / args.steps,
                "kernels_ms": {"prefill_call": call_ms, "chunk_prep": prep_ms, "state_pass": state_ms},
                "clocks": clock_info}
        return line if rank == 0 else None

    # ---- decode workload (state from a T=1024 prefill), timed per step
    sd, dec_ms, dec_gated_ms, dec_mtp_ms = decode_figures(dev, stream)
    clock_info = clocks.stop()

    # ---- the other prefill workloads (reported beside the headline, not in `value`)
    extra = {}
    if not args.no_extra:
        for wname in ("long_256k", "varlen_32"):
            extra[wname] = time_prefill_workload(W.spec(wname), dev, stream, args.warmup,
                                                 max(3, min(args.steps, 5)), peaks)
        if args.batch == 4:   # the headline prefill with the output epilogue fused in
            extra["prefill_4x8k_output_gate"] = time_prefill_workload(
                W.spec("prefill_4x8k"), dev, stream, args.warmup, max(3, min(args.steps, 10)), peaks,
                gated=True)

    # ---- e2e through the C ABI with host buffers.  Pipelined over three streams with two
    # device buffer sets: step i+1's H2D (its own stream) overlaps step i's prefill (the
    # caller's stream) and step i's D2H (a third stream); PCIe carries both directions at
    # once.  Every step copies its inputs in and its o and final state out; the timed
    # region runs from the first H2D to the last D2H.
    pin = lambda t: t.detach().cpu().pin_memory()
    hq, hk, hv, ha, hb, hS0 = pin(q), pin(k), pin(v), pin(alpha), pin(b), pin(S0)
    ho = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    hs = torch.empty(fs.shape, dtype=fs.dtype).pin_memory()
    e2e_steps = 0 if args.no_e2e else max(1, min(args.steps, 10))
    slots = [(q, k, v, alpha, b, S0, o, fs)]
    if e2e_steps:
        slots.append(tuple(torch.empty_like(t) for t in slots[0]))
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()
    in_ready, done, out_free = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    used = [False, False]

    def e2e_step(i):
        sl = i % 2
        dq, dk, dv, da, db, dS0, do, dfs = slots[sl]
        with torch.cuda.stream(s_in):
            if used[sl]:
                s_in.wait_event(done[sl])        # step i-2's prefill has read this slot
            for dst, src in ((dq, hq), (dk, hk), (dv, hv), (da, ha), (db, hb), (dS0, hS0)):
                dst.copy_(src, non_blocking=True)
            in_ready[sl].record(s_in)
        stream.wait_event(in_ready[sl])
        if used[sl]:
            stream.wait_event(out_free[sl])      # step i-2's outputs have left this slot
        kda.prefill(dq, dk, dv, conv_w, da, db, A_log, dt_bias, initial_state=dS0, num_seqs=N,
                    out=do, final_state=dfs, workspace=ws, want_conv_state=False, check=False)
        done[sl].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(done[sl])
            ho.copy_(do, non_blocking=True)
            hs.copy_(dfs, non_blocking=True)
            out_free[sl].record(s_out)
        used[sl] = True

    for i in range(2 if e2e_steps else 0):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    s_in.wait_event(e0)
    s_out.wait_event(e0)
    for i in range(e2e_steps):
        e2e_step(i)
    stream.wait_stream(s_in)
    stream.wait_stream(s_out)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1) / e2e_steps if e2e_steps else float("nan")
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, ha, hb, hS0))
    d2h = ho.numel() * ho.element_size() + hs.numel() * hs.element_size()

    # ---- max over ranks
    from gated_delta_rule_70_b200 import dist as kdist
    elapsed_ms, e2e_ms = kdist.max_over_ranks([elapsed_ms, 0.0 if args.no_e2e else e2e_ms], device=dev)
    if not kdist.report_rank(rank):
        return None

    ms_per_step = elapsed_ms / args.steps
    tokens = T_total * world
    value = kdist.whole_job_rate(T_total, world, ms_per_step)
    flops = prefill_flops_per_token_head(d) * T_total * H
    tc_tflops = flops / (ms_per_step * 1e-3) / 1e12
    # Algorithmic bytes of the step (the fused minimum: inputs once, o and the states once),
    # credited to the dominant kernel's time and to the whole step.  Beside them, each
    # kernel's own bytes: chunk_prep reads the raw q, k, v, alpha and b and writes one
    # 74,240-byte record per (chunk, head); the state pass reads the records and the initial
    # state and writes o and the final state.  The records' round trip is traffic the
    # two-kernel split adds, not algorithmic work.
    esz = 2
    alg_bytes = prefill_algorithmic_bytes(T_total, N, H, d, esz)
    chunks = N * ((s.seq_lens[0] + 63) // 64)
    rec_written = 74240
    prep_bytes = T_total * H * (4 * d * esz + esz) + chunks * H * rec_written
    state_bytes = chunks * H * rec_written + T_total * H * d * esz + 2 * N * H * d * d * 4
    dominant = ("chunk_prep", prep_ms, prep_bytes) if prep_ms >= state_ms else \
        ("state_pass", state_ms, state_bytes)
    dom_gbs = alg_bytes / (dominant[1] * 1e-3) / 1e9 if dominant[1] > 0 else 0.0
    dom_own_gbs = dominant[2] / (dominant[1] * 1e-3) / 1e9 if dominant[1] > 0 else 0.0
    step_gbs = alg_bytes / (ms_per_step * 1e-3) / 1e9
    dec_step_ms = float(np.median(dec_ms))
    dec_bytes = decode_bytes(sd.num_seqs, sd.H, sd.d)
    dec_gbs = dec_bytes / (dec_step_ms * 1e-3) / 1e9
    # two tokens per call with the state after each kept: one state read, two states written
    # (the per-token ones; the last is also the in-place state), the second token's inputs
    mtp_bytes = decode_bytes(sd.num_seqs, sd.H, sd.d) + 2 * sd.num_seqs * sd.H * sd.d * sd.d * 4 + \
        2 * sd.num_seqs * sd.H * sd.d * 2 * 5
    line = {
        "metric": "KDA prefill tokens/s and % bf16 TC peak; decode state GB/s vs HBM peak",
        "value": value,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": "prefill B=%d T=8192 H=32 d=128 bf16 I/O fp32 state (S0~N(0,0.02))" % args.batch,
                   "global_batch": args.batch * world, "seq_len": 8192, "heads": H, "head_dim": d,
                   "parallelism": "dp%d (independent sequences per rank)" % world,
                   "l2": "inputs 1.3 GB > 126 MB L2, no flush"},
        "tc": {"algorithmic_tflops": tc_tflops, "flop_per_token_head": prefill_flops_per_token_head(d),
               "frac_of_measured_bf16": tc_tflops / peaks["bf16_tflops"],
               "frac_of_2250_datasheet": tc_tflops / 2250.0},
        "kernels_ms": {"prefill_call": call_ms, "chunk_prep": prep_ms, "state_pass": state_ms,
                       "timed_calls": timed_calls},
        "roofline": {"kernel": dominant[0], "bound": "hbm", "achieved": dom_gbs,
                     "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": dom_gbs / peaks["hbm_gbs"],
                     "traffic": (CHUNK_PREP_TRAFFIC_BYTES * args.batch / 4
                                 if dominant[0] == "chunk_prep" and CHUNK_PREP_TRAFFIC_BYTES else None),
                     "algorithmic_bytes": alg_bytes,
                     "algorithmic_bytes_rule": "41,024 B per token (q, k, v, alpha, b in; o out; "
                                               "bf16) + 2 N H d^2 x 4 B of fp32 state",
                     "kernel_ms": dominant[1],
                     "step": {"ms": ms_per_step, "achieved": step_gbs,
                              "frac": step_gbs / peaks["hbm_gbs"]},
                     "kernel_bytes": dominant[2], "kernel_bytes_gbs": dom_own_gbs,
                     "kernel_bytes_frac": dom_own_gbs / peaks["hbm_gbs"],
                     "record_round_trip_bytes": 2 * chunks * H * rec_written,
                     "peak_source": peaks["source"] + " (burst copy)"},
        "prologue": {"kernel": "prologue_kernel (kda_prologue, standalone)", "ms": pro_ms,
                     "algorithmic_bytes": pro_bytes,
                     "bytes_rule": "2,310 B per token-head (q, k, v, alpha, b in; q, k, v, g, "
                                   "beta out)",
                     "GB_s": pro_bytes / (pro_ms * 1e-3) / 1e9,
                     "frac_of_measured_hbm": pro_bytes / (pro_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                     "frac_of_8000_datasheet": pro_bytes / (pro_ms * 1e-3) / 1e9 / 8000.0},
        "decode": {"workload": "256 seqs x 32 heads, d=128, fp32 state, 64 steps",
                   "ms_per_step": dec_step_ms, "algorithmic_bytes": dec_bytes, "GB_s": dec_gbs,
                   "frac_of_measured_hbm": dec_gbs / peaks["hbm_gbs"],
                   "frac_of_8000_datasheet": dec_gbs / 8000.0,
                   "tokens_per_s": sd.num_seqs / (dec_step_ms * 1e-3),
                   "output_gate_ms_per_step": dec_gated_ms,
                   "two_tokens_with_step_states_ms_per_call": dec_mtp_ms,
                   "two_tokens_GB_s": mtp_bytes / (dec_mtp_ms * 1e-3) / 1e9,
                   "two_tokens_frac_of_measured_hbm": mtp_bytes / (dec_mtp_ms * 1e-3) / 1e9 /
                   peaks["hbm_gbs"],
                   "gpu_launches": 64 + 64 + 32,   # one per decode call, in its own timed regions
                   "two_tokens_algorithmic_bytes": mtp_bytes},
        "e2e": None if args.no_e2e else {
            "value": tokens / (e2e_ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "steps": e2e_steps,
            "schedule": "pipelined: H2D, prefill and D2H on three streams, two device buffer sets"},
        "other_workloads": extra,
        "gpu_launches": launches_per_step * args.steps,   # the timed prefill steps
        "clocks": clock_info,
        "peaks": peaks,
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(seconds=args.cpu_seconds)
    return line


def time_prologue(q, k, v, conv_w, alpha, b, A_log, dt_bias, N, stream, warmup, steps):
    """Mean ms of one kda_prologue call over the batch (outputs preallocated), CUDA events on
    the launching stream."""
    import torch
    from gated_delta_rule_70_b200 import kda
    T, H, d = alpha.shape
    dev = q.device
    out = tuple(torch.empty((T, H, d), dtype=q.dtype, device=dev) for _ in range(3)) + \
        (torch.empty((T, H, d), dtype=torch.float32, device=dev),
         torch.empty((T, H), dtype=torch.float32, device=dev), None)

    def one():
        kda.prologue(q, k, v, conv_w, alpha, b, A_log, dt_bias, num_seqs=N, out=out)

    for _ in range(warmup):
        one()
    e = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    e[0].record(stream)
    for _ in range(steps):
        one()
    e[1].record(stream)
    torch.cuda.synchronize(dev)
    return e[0].elapsed_time(e[1]) / steps


def decode_figures(dev, stream, seeded=True):
    """Decode timings on the 256 x 32 workload: 64 single-token steps (median per step), the
    same steps with the output epilogue, and 32 two-token calls with per-token states.
    seeded: the state comes from the workload's T=1024 prefill (else a random one, for
    profiling runs that must hold little device memory)."""
    import torch
    from gated_delta_rule_70_b200 import kda
    from gated_delta_rule_70_b200 import workloads as W
    bf = torch.bfloat16
    sd = W.spec("decode_256")
    dup = lambda a: W.to_device(a, dev)
    if seeded:   # the workload's own state: a T=1024 prefill of every sequence
        dinp = W.make_inputs(sd)
        d_o, d_state, d_conv = kda.prefill(dup(dinp["q"]), dup(dinp["k"]), dup(dinp["v"]),
                                           dup(dinp["conv_w"]), dup(dinp["alpha"]),
                                           dup(dinp["b"]), dup(dinp["A_log"]),
                                           dup(dinp["dt_bias"]), num_seqs=sd.num_seqs)
        del dinp, d_o
        torch.cuda.empty_cache()
    else:        # profiling runs: an N(0, 0.02) state and conv history of the same shapes
        rng = np.random.default_rng(0)
        d_state = dup(0.02 * rng.standard_normal((sd.num_seqs, sd.H, sd.d, sd.d), dtype=np.float32))
        d_conv = dup(W.bf16_bits(rng.standard_normal((sd.num_seqs, 3, 3 * sd.H * sd.d),
                                                     dtype=np.float32)))
    dsteps = [W.make_decode_step(sd, i) for i in range(64)]
    dsteps = [{kk: dup(vv) for kk, vv in x.items()} for x in dsteps]
    d_cw, d_A, d_dt = dup(W.make_params(sd)["conv_w"]), dup(W.make_params(sd)["A_log"]), \
        dup(W.make_params(sd)["dt_bias"])
    d_out = torch.empty((sd.num_seqs, sd.H, sd.d), dtype=bf, device=dev)

    def dstep(x):
        kda.decode_step(x["q"], x["k"], x["v"], x["alpha"], x["b"], d_cw, d_A, d_dt, d_state,
                        d_conv, out=d_out)

    for i in range(3):
        dstep(dsteps[i])
    torch.cuda.synchronize(dev)
    de = [torch.cuda.Event(enable_timing=True) for _ in range(65)]
    for i in range(64):
        de[i].record(stream)
        dstep(dsteps[i])
    de[64].record(stream)
    torch.cuda.synchronize(dev)
    dec_ms = [de[i].elapsed_time(de[i + 1]) for i in range(64)]
    # the same steps with the output epilogue fused in
    dG = W.make_output_gate(sd, sd.num_seqs)
    d_gate, d_w = dup(dG["gate"]), dup(dG["o_norm_weight"])

    def dstep_gated(x):
        kda.decode_step(x["q"], x["k"], x["v"], x["alpha"], x["b"], d_cw, d_A, d_dt, d_state,
                        d_conv, out_gate=d_gate, o_norm_weight=d_w, out=d_out)

    for i in range(3):
        dstep_gated(dsteps[i])
    de[0].record(stream)
    for i in range(64):
        dstep_gated(dsteps[i])
    de[1].record(stream)
    torch.cuda.synchronize(dev)
    dec_gated_ms = de[0].elapsed_time(de[1]) / 64
    # two tokens per sequence per call (a speculative token verified), with the state after
    # each token kept: 32 calls over the same 64 tokens
    mtp_x = [{kk: torch.stack([dsteps[2 * c][kk], dsteps[2 * c + 1][kk]], dim=1).contiguous()
              for kk in dsteps[0]} for c in range(32)]
    mtp_states = torch.empty((sd.num_seqs, 2, sd.H, sd.d, sd.d), dtype=torch.float32, device=dev)
    mtp_out = torch.empty((sd.num_seqs, 2, sd.H, sd.d), dtype=bf, device=dev)

    def dstep_mtp(x):
        kda.decode_multi(x["q"], x["k"], x["v"], x["alpha"], x["b"], d_cw, d_A, d_dt, d_state,
                         d_conv, step_states=mtp_states, out=mtp_out)

    for c in range(3):
        dstep_mtp(mtp_x[c])
    de[0].record(stream)
    for c in range(32):
        dstep_mtp(mtp_x[c])
    de[1].record(stream)
    torch.cuda.synchronize(dev)
    dec_mtp_ms = de[0].elapsed_time(de[1]) / 32
    del mtp_x, mtp_states
    return sd, dec_ms, dec_gated_ms, dec_mtp_ms

def time_prefill_workload(s, dev, stream, warmup, steps, peaks, gated=False):
    """One kda_prefill over a whole workload (inputs resident in HBM), timed with CUDA
    events on the launching stream; chunk_prep / state-pass split from the library's
    kernel timing.  gated: with the output epilogue (o_norm and sigmoid output gate)."""
    import torch
    from gated_delta_rule_70_b200 import kda
    from gated_delta_rule_70_b200 import workloads as W

    params = {k: W.to_device(v, dev) for k, v in W.make_params(s).items()}
    T = s.total_tokens
    H, d = s.H, s.d
    bf = torch.bfloat16
    q, k, v = (torch.empty((T, H * d), dtype=bf, device=dev) for _ in range(3))
    alpha = torch.empty((T, H, d), dtype=bf, device=dev)
    b = torch.empty((T, H), dtype=bf, device=dev)
    blk = 65536
    for t0 in range(0, T, blk):   # host generation in slices, uploaded as they come
        t1 = min(T, t0 + blk)
        tok = W.make_tokens(s, t0, t1)
        for name, dst in (("q", q), ("k", k), ("v", v), ("alpha", alpha), ("b", b)):
            dst[t0:t1].copy_(W.to_device(tok[name], dev))
        del tok
    S0 = W.make_initial_state(s)
    S0 = W.to_device(S0, dev) if S0 is not None else None
    cu = W.to_device(s.cu_seqlens, dev) if s.varlen else None
    N = s.num_seqs
    o = torch.empty((T, H, d), dtype=bf, device=dev)
    fs = torch.empty((N, H, d, d), dtype=torch.float32, device=dev)
    fc = torch.empty((N, 3, 3 * H * d), dtype=bf, device=dev)
    seq_len = T if s.varlen else s.seq_lens[0]
    ws = torch.empty(kda.prefill_workspace_size(kda.make_shape(N, seq_len, H, d, bf), s.varlen),
                     dtype=torch.uint8, device=dev)
    gate = wgt = None
    if gated:
        G = W.make_output_gate(s, T)
        gate, wgt = W.to_device(G["gate"], dev), W.to_device(G["o_norm_weight"], dev)
        del G

    def step():
        kda.prefill(q, k, v, params["conv_w"], alpha, b, params["A_log"], params["dt_bias"],
                    initial_state=S0, cu_seqlens=cu, num_seqs=N, out=o, final_state=fs,
                    final_conv_state=fc, workspace=ws, out_gate=gate, o_norm_weight=wgt,
                    check=False)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize(dev)
    kda.kernel_timing(True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    _, prep_ms, state_ms = kda.kernel_times()
    kda.kernel_timing(False)
    ms = e0.elapsed_time(e1) / steps
    flops = prefill_flops_per_token_head(d) * T * H
    out = {"tokens": T, "sequences": N, "heads": H, "head_dim": d, "ms_per_step": ms,
           "tokens_per_s": T / (ms * 1e-3), "algorithmic_tflops": flops / (ms * 1e-3) / 1e12,
           "frac_of_measured_bf16": flops / (ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
           "kernels_ms": {"chunk_prep": prep_ms, "state_pass": state_ms}, "steps": steps,
           "warmup": warmup}
    if gated:
        out["output_gate"] = "o <- o / sqrt(mean o^2 + 1e-5) * w * sigmoid(gate), fused into the state pass"
    del q, k, v, alpha, b, o, ws, gate
    torch.cuda.empty_cache()
    return out


def decode_bytes(N, H, d, esz=2):
    """Algorithmic bytes of one decode step: state read+write, conv state r/w, token in, o out."""
    state = 2 * N * H * d * d * 4
    conv = 2 * N * 3 * 3 * H * d * esz
    tok = N * H * (3 * d * esz + d * esz + esz) + N * H * d * esz
    return state + conv + tok


# ---------------------------------------------------------------- CPU oracle timing

def cpu_baseline(seconds: float = 15.0, tokens: int = None):
    """Time the fp64 oracle on host cores, tokens/s counting every head.  Default: whole
    sequences of the prefill workload (8192 tokens x 32 heads each), as many as fit in
    about `seconds` of wall time (at least one, at most all four); with `tokens`: the first
    `tokens` tokens of sequence 0 (the reference arm's per-step sample)."""
    from gated_delta_rule_70_b200 import workloads as W
    from oracle import oracle

    s = W.spec("prefill_4x8k")
    params = W.make_params(s)
    S0_all = W.make_initial_state(s).astype(np.float64)
    L = s.seq_lens[0]
    f_par = {kk: W.as_f64(vv) for kk, vv in params.items()}

    def run_seq(n, t1, nthreads=0):
        tok = W.make_tokens(s, n * L, n * L + t1)
        f = {kk: W.as_f64(vv) for kk, vv in tok.items()}
        t0 = time.perf_counter()
        _, _, _, used = oracle.forward([0, t1], s.H, s.d, f["q"], f["k"], f["v"], f_par["conv_w"],
                                       f["alpha"], f["b"], f_par["A_log"], f_par["dt_bias"],
                                       state0=S0_all[n:n + 1], nthreads=nthreads)
        return time.perf_counter() - t0, used

    if tokens is not None:
        dt, used = run_seq(0, tokens)
        return {"value": tokens / dt, "unit": "tokens/s", "cores": int(used), "kind": "oracle",
                "sample": "sequence 0 of prefill B=4 T=8192 H=32 d=128: first %d tokens, all 32 heads, "
                          "fp64 C oracle, %d threads over heads, %.1f s" % (tokens, used, dt)}
    total, done, used = 0.0, 0, 1
    for n in range(s.num_seqs):
        dt, used = run_seq(n, L)
        total += dt
        done += 1
        if total >= seconds:
            break
    one_t = 512
    one_dt, _ = run_seq(0, one_t, nthreads=1)
    dec = cpu_decode_baseline()
    return {"value": done * L / total, "unit": "tokens/s", "cores": int(used), "kind": "oracle",
            "sample": "%d of the 4 sequences of prefill B=4 T=8192 H=32 d=128 (%d tokens x 32 heads), "
                      "fp64 C oracle, %d threads over heads, %.1f s" % (done, done * L, used, total),
            "one_core": {"value": one_t / one_dt, "unit": "tokens/s", "cores": 1,
                         "sample": "first %d tokens of sequence 0, all 32 heads, 1 thread, %.1f s"
                                   % (one_t, one_dt)},
            "decode": dec}


def cpu_decode_baseline(seqs: int = 32, steps: int = 4):
    """The fp64 oracle on a bounded sample of the decode workload (256 sequences x 32 heads,
    d=128): its first ``seqs`` sequences, all heads, ``steps`` decode steps from an N(0, 0.02)
    state and conv history (the cost does not depend on their values).  Tokens/s counts one
    token per sequence per step, as the GPU decode figure does."""
    from gated_delta_rule_70_b200 import workloads as W
    from oracle import oracle

    sd = W.spec("decode_256")
    H, d = sd.H, sd.d
    par = {kk: W.as_f64(vv) for kk, vv in W.make_params(sd).items()}
    rng = np.random.default_rng(0)
    state = 0.02 * rng.standard_normal((seqs, H, d, d))
    conv = W.as_f64(W.bf16_bits(rng.standard_normal((seqs, 3, 3 * H * d)).astype(np.float32)))
    total = 0.0
    for i in range(steps):
        x = {kk: W.as_f64(vv)[:seqs] for kk, vv in W.make_decode_step(sd, i).items()}
        t0 = time.perf_counter()
        _, state, conv = oracle.decode_step(H, d, state, conv, x["q"], x["k"], x["v"], x["alpha"],
                                            x["b"], par["conv_w"], par["A_log"], par["dt_bias"])
        total += time.perf_counter() - t0
    return {"value": seqs * steps / total, "unit": "tokens/s", "cores": int(os.cpu_count() or 1),
            "kind": "oracle",
            "sample": "decode 256 seqs x 32 heads, d=128: first %d sequences, all heads, %d steps, "
                      "fp64 C oracle, threads over heads, %.2f s" % (seqs, steps, total)}


def run_reference(args, rank):
    if rank != 0:
        return None
    from oracle import oracle
    oracle.build()
    per_step_tokens = args.ref_tokens
    for _ in range(args.warmup):
        cpu_baseline(tokens=max(64, per_step_tokens // 4))
    t0 = time.perf_counter()
    samples = [cpu_baseline(tokens=per_step_tokens) for _ in range(args.steps)]
    dt = time.perf_counter() - t0
    value = per_step_tokens * args.steps / dt
    cb = dict(samples[-1])
    cb["value"] = value
    return {
        "impl": "reference",
        "metric": "KDA prefill tokens/s and % bf16 TC peak; decode state GB/s vs HBM peak",
        "value": value, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "prefill B=4 T=8192 H=32 d=128 (oracle sample: sequence 0, "
                               "first %d tokens, all heads)" % per_step_tokens,
                   "global_batch": 4, "seq_len": 8192, "parallelism": "host threads over heads"},
        "cpu_baseline": cb,
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-tokens", type=int, default=1024)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--batch", type=int, default=4,
                    help="prefill sequences (the measured workload is 4; smaller only for profiling)")
    ap.add_argument("--only", choices=["all", "prefill", "prologue", "decode"], default="all",
                    help="profiling runs: one part alone (the JSON line is not a bench result)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the long (1x262144) and varlen (32 sequences) prefill workloads")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    from gated_delta_rule_70_b200 import dist as kdist
    rank, world, local_rank = kdist.world_info(os.environ)
    if args.impl == "reference":
        line = run_reference(args, rank)
        if line is not None:
            print(json.dumps(line), flush=True)
        return 0

    import torch
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local_rank))
    try:
        line = run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
