"""GPU parity at the full workload sizes, in the launch configuration the bench
times, against the fp64 oracle threaded over the host's cores.

  prefill 4 x 8192 x 32    every (sequence, head): o and final state
  varlen 32 sequences      every (sequence, head): o and final state
  decode 256 x 32          every (sequence, head): the T = 1024 prefill that seeds
                           the state, then o of all 64 decode steps and the state after
  long 1 x 262144 x 32     heads 0-1 on the first 16384 tokens (o; the final state by a
                           GPU prefill of that prefix), plus the split identity at any
                           size: prefill(all) == prefill(second half) seeded with
                           prefill(first half)

Tolerance: max relative L2 per (sequence, head) <= 1e-2 for bf16 I/O.  Each test
prints its largest per-pair errors.
"""

import numpy as np
import pytest
import torch

from gated_delta_rule_70_b200 import kda
from gated_delta_rule_70_b200 import workloads as W
from oracle import oracle

pytestmark = [pytest.mark.gpu, pytest.mark.slow]
TOL = 1e-2


def rel(x, ref):
    return float(np.linalg.norm(x - ref) / np.linalg.norm(ref))


def upload(inp):
    return {k: W.to_device(v) for k, v in inp.items()}


def run(s, d, cu=None, S0=None, conv0=None):
    return kda.prefill(d["q"], d["k"], d["v"], d["conv_w"], d["alpha"], d["b"], d["A_log"],
                       d["dt_bias"], initial_state=S0, cu_seqlens=cu, initial_conv_state=conv0,
                       num_seqs=s.num_seqs, check=True)


def oracle_seqs(s, inp, seqs, t_end=None, S0=None, heads=None):
    """The oracle on sequences `seqs` (all heads, or `heads`), threaded over (sequence, head).
    Returns (o [tokens, H', d], final state [len(seqs), H', d, d], final conv, local cu)."""
    cu = s.cu_seqlens
    D = s.d
    hs = list(range(s.H)) if heads is None else list(heads)
    rows, lens = [], []
    for n in seqs:
        a = int(cu[n])
        z = int(cu[n + 1]) if t_end is None else a + t_end
        rows.append(np.arange(a, z))
        lens.append(z - a)
    r = np.concatenate(rows)
    cols = np.concatenate([np.arange(h * D, (h + 1) * D) for h in hs])
    f = lambda x: W.as_f64(np.ascontiguousarray(x))
    lcu = np.concatenate([[0], np.cumsum(lens)])
    s0 = None if S0 is None else f(S0[seqs][:, hs])
    o, s1, c1, _ = oracle.forward(
        lcu, len(hs), D, f(inp["q"][r][:, cols]), f(inp["k"][r][:, cols]), f(inp["v"][r][:, cols]),
        f(inp["conv_w"][:, cols]), f(inp["alpha"][r][:, hs]), f(inp["b"][r][:, hs]),
        f(inp["A_log"][hs]), f(inp["dt_bias"][hs]), state0=s0, nthreads=0)
    return o, s1, c1, lcu


def check_all_pairs(s, inp, o, fs, batch):
    """Every (sequence, head) of the workload against the oracle, `batch` sequences at a time."""
    cu = s.cu_seqlens
    og = o.float().cpu().numpy()
    sg = fs.cpu().numpy()
    worst_o = worst_s = 0.0
    for b0 in range(0, s.num_seqs, batch):
        seqs = list(range(b0, min(s.num_seqs, b0 + batch)))
        o_ref, s_ref, _, lcu = oracle_seqs(s, inp, seqs, S0=inp.get("S0"))
        for i, n in enumerate(seqs):
            a = int(cu[n])
            for h in range(s.H):
                e_o = rel(og[a:a + lcu[i + 1] - lcu[i], h], o_ref[lcu[i]:lcu[i + 1], h])
                e_s = rel(sg[n, h], s_ref[i, h])
                assert e_o <= TOL, ("o", n, h, e_o)
                assert e_s <= TOL, ("state", n, h, e_s)
                worst_o, worst_s = max(worst_o, e_o), max(worst_s, e_s)
    print("\n%s: %d (sequence, head) pairs, max rel-L2 o %.3e, final state %.3e"
          % (s.name, s.num_seqs * s.H, worst_o, worst_s))
    return worst_o, worst_s


def test_prefill_4x8k_every_pair():
    s = W.spec("prefill_4x8k")
    inp = W.make_inputs(s)
    d = upload(inp)
    o, fs, _ = run(s, d, S0=d["S0"])
    torch.cuda.synchronize()
    del d
    check_all_pairs(s, inp, o, fs, batch=1)


def test_varlen_32_every_pair():
    s = W.spec("varlen_32")
    inp = W.make_inputs(s)
    d = upload(inp)
    o, fs, _ = run(s, d, cu=d["cu_seqlens"], S0=d["S0"])
    torch.cuda.synchronize()
    del d
    check_all_pairs(s, inp, o, fs, batch=8)


def test_long_256k_prefix_and_split():
    s = W.spec("long_256k")
    inp = W.make_inputs(s)
    d = upload(inp)
    o, fs, fc = run(s, d)
    torch.cuda.synchronize()
    # o on heads 0-1 over the first 16384 tokens against the oracle on that prefix
    P = 16384
    o_ref, s_ref, _, _ = oracle_seqs(s, inp, [0], t_end=P, heads=[0, 1])
    og = o.float().cpu().numpy()
    for i, h in enumerate((0, 1)):
        assert rel(og[:P, h], o_ref[:, i]) <= TOL
    # final state at the prefix: a GPU prefill of the 16384-token prefix vs the oracle
    sp = W.Spec("prefix", "bf16", [P], H=s.H, d=s.d, seed=s.seed, alpha_mu=s.alpha_mu)
    dp = {k: (v[:P] if k in ("q", "k", "v", "alpha", "b") else v) for k, v in d.items()}
    _, fsp, _ = run(sp, dp)
    torch.cuda.synchronize()
    for i, h in enumerate((0, 1)):
        assert rel(fsp[0, h].cpu().numpy(), s_ref[0, i]) <= TOL
    # any size: prefill(all) == prefill(second half) seeded with prefill(first half)
    half = s.total_tokens // 2
    s1 = W.Spec("h1", "bf16", [half], H=s.H, d=s.d, seed=s.seed)
    d1 = {k: (v[:half] if k in ("q", "k", "v", "alpha", "b") else v) for k, v in d.items()}
    d2 = {k: (v[half:].contiguous() if k in ("q", "k", "v", "alpha", "b") else v) for k, v in d.items()}
    o1, st1, cs1 = run(s1, d1)
    o2, st2, _ = run(s1, d2, S0=st1, conv0=cs1)
    torch.cuda.synchronize()
    og = o.float()
    for h in range(0, s.H, 5):
        assert rel(o2[:, h].float().cpu().numpy(), og[half:, h].cpu().numpy()) <= TOL
        assert rel(st2[0, h].cpu().numpy(), fs[0, h].cpu().numpy()) <= TOL


def test_decode_256_every_pair():
    s = W.spec("decode_256")
    inp = W.make_inputs(s)
    d = upload(inp)
    o, st, cs = run(s, d)
    del d
    steps = 64
    xs = [W.make_decode_step(s, i) for i in range(steps)]
    outs = []
    for x in xs:
        dx = upload(x)
        outs.append(kda.decode_step(dx["q"], dx["k"], dx["v"], dx["alpha"], dx["b"],
                                    W.to_device(inp["conv_w"]), W.to_device(inp["A_log"]),
                                    W.to_device(inp["dt_bias"]), st, cs).float().cpu().numpy())
    torch.cuda.synchronize()
    og_pre = o.float().cpu().numpy()
    sg = st.cpu().numpy()
    D, H = s.d, s.H
    f = lambda x: W.as_f64(np.ascontiguousarray(x))
    par = {k: f(inp[k]) for k in ("conv_w", "A_log", "dt_bias")}
    worst_pre = worst_o = worst_s = 0.0
    batch = 16
    for b0 in range(0, s.num_seqs, batch):
        seqs = list(range(b0, b0 + batch))
        o_ref, S, C, lcu = oracle_seqs(s, inp, seqs)   # the T = 1024 prefill that seeds decode
        for i, n in enumerate(seqs):
            for h in range(H):
                e = rel(og_pre[n * 1024:(n + 1) * 1024, h], o_ref[lcu[i]:lcu[i + 1], h])
                assert e <= TOL, ("prefill o", n, h, e)
                worst_pre = max(worst_pre, e)
        got, want = [], []
        for t, x in enumerate(xs):
            o_t, S, C = oracle.decode_step(H, D, S, C, f(x["q"][seqs]), f(x["k"][seqs]),
                                           f(x["v"][seqs]), f(x["alpha"][seqs]), f(x["b"][seqs]),
                                           par["conv_w"], par["A_log"], par["dt_bias"])
            got.append(outs[t][seqs])
            want.append(o_t)
        got, want = np.stack(got, axis=1), np.stack(want, axis=1)   # [seq, step, H, D]
        for i, n in enumerate(seqs):
            for h in range(H):
                e_o = rel(got[i, :, h], want[i, :, h])
                e_s = rel(sg[n, h], S[i, h])
                assert e_o <= TOL, ("decode o", n, h, e_o)
                assert e_s <= TOL, ("state", n, h, e_s)
                worst_o, worst_s = max(worst_o, e_o), max(worst_s, e_s)
    print("\ndecode_256: %d (sequence, head) pairs, max rel-L2 seeding prefill o %.3e, "
          "decode o (64 steps) %.3e, state after %.3e" % (s.num_seqs * H, worst_pre, worst_o, worst_s))
