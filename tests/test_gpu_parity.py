"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Metric (per sequence n and head h): ||x_gpu - x_ref||_2 / ||x_ref||_2 over
(t, d_v) for o and over (d_k, d_v) for the final state; the maximum over all
(n, h) must stay within 1e-2 for bf16 I/O (fp32 accumulation) and 1e-4 in the
fp32 test mode.  Small cases span several 64-token chunks and a ragged tail and
run the oracle on everything; full-size workloads run the GPU in the launch
configuration the bench times and check sampled (sequence, head) pairs, which
the oracle computes one by one.
"""

import numpy as np
import pytest
import torch

from gated_delta_rule_70_b200 import kda
from gated_delta_rule_70_b200 import workloads as W
from oracle import oracle

pytestmark = pytest.mark.gpu

TOL = {"bf16": 1e-2, "fp32": 1e-4}


def _dev(arr):
    return W.to_device(arr)


def gpu_prefill(s: W.Spec, inp: dict, conv0=None, want_conv=True, neg=False, flags=0):
    cu = _dev(inp["cu_seqlens"]) if s.varlen else None
    o, fs, fc = kda.prefill(_dev(inp["q"]), _dev(inp["k"]), _dev(inp["v"]), _dev(inp["conv_w"]),
                            _dev(inp["alpha"]), _dev(inp["b"]), _dev(inp["A_log"]),
                            _dev(inp["dt_bias"]), initial_state=_dev(inp["S0"]), cu_seqlens=cu,
                            initial_conv_state=_dev(conv0), num_seqs=s.num_seqs,
                            lower_bound=s.lower_bound, l2norm_eps=s.eps, scale=s.scale,
                            negative_eigenvalues=neg, want_conv_state=want_conv, check=True,
                            flags=flags)
    torch.cuda.synchronize()
    return o, fs, fc


def f64_inputs(inp):
    return {k: W.as_f64(v) for k, v in inp.items() if k != "cu_seqlens"}


def oracle_prefill(s: W.Spec, inp: dict, conv0=None, neg=False):
    f = f64_inputs(inp)
    return oracle.forward(inp["cu_seqlens"], s.H, s.d, f["q"], f["k"], f["v"], f["conv_w"],
                          f["alpha"], f["b"], f["A_log"], f["dt_bias"], state0=f["S0"],
                          conv0=W.as_f64(conv0), lower_bound=s.lower_bound, eps=s.eps,
                          scale=s.scale, negative_eigenvalues=neg)


def rel_l2(x, ref):
    den = np.linalg.norm(ref)
    num = np.linalg.norm(x - ref)
    if den == 0.0:
        return num
    return num / den


def max_pair_err(o_gpu, o_ref, cu, H):
    worst = 0.0
    for n in range(len(cu) - 1):
        a, z = int(cu[n]), int(cu[n + 1])
        if z == a:
            continue
        for h in range(H):
            worst = max(worst, rel_l2(o_gpu[a:z, h], o_ref[a:z, h]))
    return worst


def max_state_err(s_gpu, s_ref):
    N, H = s_ref.shape[:2]
    return max(rel_l2(s_gpu[n, h], s_ref[n, h]) for n in range(N) for h in range(H))


def check_prefill(s: W.Spec, conv0=None, neg=False, flags=0):
    inp = W.make_inputs(s)
    o, fs, fc = gpu_prefill(s, inp, conv0, neg=neg, flags=flags)
    o_ref, s_ref, c_ref, _ = oracle_prefill(s, inp, conv0, neg=neg)
    tol = TOL[s.io_dtype]
    eo = max_pair_err(W.from_device(o), o_ref, inp["cu_seqlens"], s.H)
    es = max_state_err(W.from_device(fs), s_ref)
    assert eo <= tol, "o rel-L2 %.3g > %.0e" % (eo, tol)
    assert es <= tol, "final_state rel-L2 %.3g > %.0e" % (es, tol)
    # conv history is a copy of raw inputs: bit-exact
    np.testing.assert_array_equal(W.from_device(fc), c_ref)
    return eo, es


# ------------------------------------------------------------------ prologue

@pytest.mark.parametrize("io,d,lens,varlen", [("bf16", 128, [1, 2, 17, 70], True),
                                              ("fp32", 64, [33, 5], True),
                                              ("bf16", 128, [40, 40], False),
                                              ("fp32", 128, [19], False)])
def test_prologue_parity(io, d, lens, varlen):
    s = W.small("pro", lens, H=3, d=d, io_dtype=io, seed=7, varlen=varlen)
    inp = W.make_inputs(s)
    rng = np.random.default_rng(3)
    conv0 = W._store(rng.standard_normal((s.num_seqs, 3, 3 * s.H * d)).astype(np.float32), io)
    cu = _dev(inp["cu_seqlens"]) if varlen else None
    qn, kn, vc, g, beta, _ = kda.prologue(_dev(inp["q"]), _dev(inp["k"]), _dev(inp["v"]),
                                       _dev(inp["conv_w"]), _dev(inp["alpha"]), _dev(inp["b"]),
                                       _dev(inp["A_log"]), _dev(inp["dt_bias"]), cu_seqlens=cu,
                                       initial_conv_state=_dev(conv0), num_seqs=s.num_seqs)
    torch.cuda.synchronize()
    f = f64_inputs(inp)
    ref = oracle.prologue(inp["cu_seqlens"], s.H, d, f["q"], f["k"], f["v"], f["conv_w"],
                          f["alpha"], f["b"], f["A_log"], f["dt_bias"], conv0=W.as_f64(conv0))
    rt = 2.0 ** -8 if io == "bf16" else 2e-6     # bf16 outputs carry one rounding
    for got, want in zip((qn, kn, vc), ref[:3]):
        np.testing.assert_allclose(W.from_device(got), want, rtol=rt, atol=rt * 0.05)
    np.testing.assert_allclose(W.from_device(g), ref[3], rtol=2e-6, atol=1e-6)
    np.testing.assert_allclose(W.from_device(beta), ref[4], rtol=2e-6, atol=1e-7)


def test_prologue_parity_large_activations():
    """q, k, v scaled by 40: most conv outputs sit where the SiLU's tanh has saturated (x/2 well
    past 9), on both signs; outputs still match the oracle elementwise at one bf16 rounding, and
    the fused prologue of the prefill (its own SiLU) matches through the whole recurrence."""
    s = W.small("pro_big", [70, 33], H=2, d=128, seed=8, varlen=True)
    inp = W.make_inputs(s)
    for name in ("q", "k", "v"):
        inp[name] = W._store(W.bf16_to_f32(inp[name]) * np.float32(40.0), "bf16")
    qn, kn, vc, g, beta, _ = kda.prologue(_dev(inp["q"]), _dev(inp["k"]), _dev(inp["v"]),
                                       _dev(inp["conv_w"]), _dev(inp["alpha"]), _dev(inp["b"]),
                                       _dev(inp["A_log"]), _dev(inp["dt_bias"]),
                                       cu_seqlens=_dev(inp["cu_seqlens"]), num_seqs=s.num_seqs)
    torch.cuda.synchronize()
    f = f64_inputs(inp)
    ref = oracle.prologue(inp["cu_seqlens"], s.H, s.d, f["q"], f["k"], f["v"], f["conv_w"],
                          f["alpha"], f["b"], f["A_log"], f["dt_bias"])
    rt = 2.0 ** -8
    for got, want in zip((qn, kn, vc), ref[:3]):
        np.testing.assert_allclose(W.from_device(got), want, rtol=rt, atol=rt * 0.05 * 40)
    # the prefill's fused prologue on the same inputs, against the oracle's whole recurrence
    o, st, _ = gpu_prefill(s, inp)
    o_ref, s_ref, _, _ = oracle_prefill(s, inp)
    assert max_pair_err(W.from_device(o), o_ref, s.cu_seqlens, s.H) <= TOL["bf16"]
    assert max_state_err(W.from_device(st), s_ref) <= TOL["bf16"]


# ------------------------------------------------------------------ prefill, small

def test_prefill_tiny_fp32_workload():
    """The fp32 test-mode workload exactly (B=1, T=256, H=2, d=64): 1e-4."""
    check_prefill(W.spec("tiny_fp32"))


@pytest.mark.parametrize("lens,H,seed", [([200, 200], 4, 11), ([64], 2, 12), ([1], 2, 13),
                                         ([3, 130], 2, 14)])
def test_prefill_bf16_dense(lens, H, seed):
    s = W.small("dense", lens, H=H, d=128, seed=seed, s0_std=0.02)
    if len(set(lens)) > 1:
        s.varlen = True
    check_prefill(s)


def test_prefill_bf16_varlen_edges():
    """Empty, 1-token, exactly-one-chunk, chunk+1 and multi-chunk sequences packed together."""
    s = W.small("varlen", [1, 3, 64, 65, 0, 130, 17], H=2, d=128, seed=15, s0_std=0.02,
                varlen=True)
    check_prefill(s)


@pytest.mark.parametrize("varlen", [True, False])
def test_prefill_all_sequences_empty(varlen):
    """Zero tokens in the whole batch: no arithmetic, so the final state and the conv history
    are the initial ones bit for bit (zeros when none is given)."""
    s = W.small("empty", [0, 0, 0], H=2, d=128, seed=30, s0_std=0.02, varlen=varlen)
    inp = W.make_inputs(s)
    conv0 = W._store(np.random.default_rng(6).standard_normal((3, 3, 3 * 2 * 128)).astype(np.float32),
                     "bf16")
    o, fs, fc = gpu_prefill(s, inp, conv0)
    o_ref, s_ref, c_ref, _ = oracle_prefill(s, inp, conv0)
    assert o.numel() == 0 and o_ref.size == 0
    np.testing.assert_array_equal(W.from_device(fs), s_ref)
    np.testing.assert_array_equal(W.from_device(fc), c_ref)
    cu = _dev(inp["cu_seqlens"]) if varlen else None
    _, fs0, fc0 = kda.prefill(_dev(inp["q"]), _dev(inp["k"]), _dev(inp["v"]), _dev(inp["conv_w"]),
                              _dev(inp["alpha"]), _dev(inp["b"]), _dev(inp["A_log"]),
                              _dev(inp["dt_bias"]), cu_seqlens=cu, num_seqs=3, check=True)
    torch.cuda.synchronize()
    assert not W.from_device(fs0).any() and not W.from_device(fc0).any()


def test_prefill_bf16_slow_decay():
    """alpha ~ N(-2, 1): the slow-decay distribution of the long-context workload."""
    s = W.small("slow", [300], H=2, d=128, seed=16, alpha_mu=-2.0)
    check_prefill(s)


def test_prefill_fp32_varlen_with_conv_history():
    s = W.small("fp32v", [5, 70, 2], H=2, d=64, io_dtype="fp32", seed=17, s0_std=0.02,
                varlen=True)
    conv0 = W._store(np.random.default_rng(4).standard_normal((3, 3, 3 * 2 * 64)).astype(np.float32),
                     "fp32")
    check_prefill(s, conv0)


def test_prefill_bf16_varlen_with_conv_history():
    """The tensor-core path's first chunks take the caller's conv history (fused prologue)."""
    s = W.small("bf16v", [5, 70, 2, 130], H=2, d=128, seed=24, s0_std=0.02, varlen=True)
    conv0 = W._store(np.random.default_rng(5).standard_normal((4, 3, 3 * 2 * 128)).astype(np.float32),
                     "bf16")
    check_prefill(s, conv0)


def test_prefill_bf16_continuation():
    """prefill(T1) then prefill(T2) from its final state and conv history == prefill(T1 + T2)."""
    H, d, T1, T2 = 2, 128, 150, 97
    s = W.small("cont", [T1 + T2], H=H, d=d, seed=25, s0_std=0.02)
    inp = W.make_inputs(s)
    o_all, s_all, c_all = gpu_prefill(s, inp)
    part = lambda a, z: {k: (v[a:z] if k in ("q", "k", "v", "alpha", "b") else v) for k, v in inp.items()}
    s1 = W.small("cont", [T1], H=H, d=d, seed=25, s0_std=0.02)
    o1, st1, cs1 = gpu_prefill(s1, part(0, T1))
    p2 = part(T1, T1 + T2)
    o2, st2, cs2 = kda.prefill(_dev(p2["q"]), _dev(p2["k"]), _dev(p2["v"]), _dev(p2["conv_w"]),
                               _dev(p2["alpha"]), _dev(p2["b"]), _dev(p2["A_log"]), _dev(p2["dt_bias"]),
                               initial_state=st1, initial_conv_state=cs1, num_seqs=1, check=True)
    torch.cuda.synchronize()
    o_cat = np.concatenate([W.from_device(o1), W.from_device(o2)])
    o_ref, s_ref, c_ref, _ = oracle_prefill(s, inp)
    for h in range(H):
        assert rel_l2(o_cat[:, h], o_ref[:, h]) <= TOL["bf16"]
        assert rel_l2(o_cat[:, h], W.from_device(o_all)[:, h]) <= TOL["bf16"]
    assert max_state_err(W.from_device(st2), s_ref) <= TOL["bf16"]
    np.testing.assert_array_equal(W.from_device(cs2), c_ref)


def test_recurrence_entry_bf16():
    """kda_prologue + kda_recurrence (chunk_prep on prepared inputs) against the oracle."""
    s = W.small("rec", [130, 64, 3], H=2, d=128, seed=26, s0_std=0.02, varlen=True)
    inp = W.make_inputs(s)
    cu = _dev(inp["cu_seqlens"])
    qn, kn, vc, g, beta, _ = kda.prologue(_dev(inp["q"]), _dev(inp["k"]), _dev(inp["v"]),
                                       _dev(inp["conv_w"]), _dev(inp["alpha"]), _dev(inp["b"]),
                                       _dev(inp["A_log"]), _dev(inp["dt_bias"]), cu_seqlens=cu,
                                       num_seqs=s.num_seqs)
    o, fs = kda.recurrence(qn, kn, vc, g, beta, _dev(inp["S0"]), cu_seqlens=cu, num_seqs=s.num_seqs)
    torch.cuda.synchronize()
    o_ref, s_ref, _, _ = oracle_prefill(s, inp)
    assert max_pair_err(W.from_device(o), o_ref, inp["cu_seqlens"], s.H) <= TOL["bf16"]
    assert max_state_err(W.from_device(fs), s_ref) <= TOL["bf16"]


@pytest.mark.parametrize("lower_bound", [-5.5, -8.0, -10.0, -12.0])
def test_prefill_bf16_saturated_gates(lower_bound):
    """Gates pinned at the lower bound.  Down to -10 the tensor-core path runs (its split
    decay factors span at most 8 gates: within 2^{+-116}); -12 runs the token kernel."""
    s = W.small("sat", [200], H=2, d=128, seed=27, alpha_mu=3.0, s0_std=0.02)
    s.lower_bound = lower_bound
    check_prefill(s)


@pytest.mark.parametrize("alpha_mu", [100.0, -100.0])
def test_prefill_bf16_extreme_gate_inputs(alpha_mu):
    """alpha + dt_bias far beyond where exp overflows (every gate at the lower bound) or
    underflows (no decay): the kernels' base-2 softplus must agree with the oracle's."""
    s = W.small("xgate", [150], H=2, d=128, seed=31, alpha_mu=alpha_mu, s0_std=0.02)
    check_prefill(s)


def test_prefill_in_place_state():
    """final_state may be the same buffer as initial_state."""
    s = W.small("inplace", [100, 100], H=2, d=128, seed=18, s0_std=0.02)
    inp = W.make_inputs(s)
    st = _dev(inp["S0"]).clone()
    o, fs, _ = kda.prefill(_dev(inp["q"]), _dev(inp["k"]), _dev(inp["v"]), _dev(inp["conv_w"]),
                           _dev(inp["alpha"]), _dev(inp["b"]), _dev(inp["A_log"]),
                           _dev(inp["dt_bias"]), initial_state=st, num_seqs=2, final_state=st, check=True)
    o_ref, s_ref, _, _ = oracle_prefill(s, inp)
    assert max_state_err(W.from_device(st), s_ref) <= TOL["bf16"]
    assert max_pair_err(W.from_device(o), o_ref, inp["cu_seqlens"], s.H) <= TOL["bf16"]


def test_bad_cu_seqlens_is_reported():
    s = W.small("bad", [10, 10, 10], H=2, d=128, seed=19, varlen=True)
    inp = W.make_inputs(s)
    inp["cu_seqlens"] = np.array([0, 12, 5, 30], dtype=np.int32)    # decreasing
    with pytest.raises(kda.KdaError) as e:
        gpu_prefill(s, inp)
    assert e.value.status == kda.KDA_ERR_INVALID_ARGUMENT
    inp["cu_seqlens"] = np.array([0, 10, 20, 29], dtype=np.int32)   # wrong total
    with pytest.raises(kda.KdaError):
        gpu_prefill(s, inp)
    # the context is still healthy afterwards
    check_prefill(W.small("after", [20], H=2, d=128, seed=20))


# ------------------------------------------------------------------ decode

def _decode_inputs(s: W.Spec, step):
    return W.make_decode_step(s, step)


@pytest.mark.parametrize("H,N,T1,neg", [(3, 5, 70, False), (16, 40, 20, False), (3, 4, 30, True),
                                        (16, 40, 20, True)])
def test_decode_parity_and_handoff(H, N, T1, neg):
    """prefill(T1) -> decode steps on GPU vs the oracle.  H=3 takes the per-item kernel;
    H=16 with 640 items takes the persistent one, several items per CTA around its ring.
    neg: beta = 2 sigmoid(b) in the prefill and every step."""
    d, steps = 128, 4
    s = W.small("dec", [T1] * N, H=H, d=d, seed=21, s0_std=0.02)
    inp = W.make_inputs(s)
    o, st, cs = gpu_prefill(s, inp, neg=neg)
    f = f64_inputs(inp)
    o_ref, s_ref, c_ref, _ = oracle_prefill(s, inp, neg=neg)
    for step in range(steps):
        x = _decode_inputs(s, step)
        o_t = kda.decode_step(_dev(x["q"]), _dev(x["k"]), _dev(x["v"]), _dev(x["alpha"]),
                              _dev(x["b"]), _dev(inp["conv_w"]), _dev(inp["A_log"]),
                              _dev(inp["dt_bias"]), st, cs, negative_eigenvalues=neg)
        xf = {k: W.as_f64(v) for k, v in x.items()}
        o_r, s_ref, c_ref = oracle.decode_step(H, d, s_ref, c_ref, xf["q"], xf["k"], xf["v"],
                                               xf["alpha"], xf["b"], f["conv_w"], f["A_log"],
                                               f["dt_bias"], negative_eigenvalues=neg)
        torch.cuda.synchronize()
        og = W.from_device(o_t)
        worst = max(rel_l2(og[n, h], o_r[n, h]) for n in range(N) for h in range(H))
        assert worst <= TOL["bf16"], (step, worst)
        np.testing.assert_array_equal(W.from_device(cs), c_ref)
    assert max_state_err(W.from_device(st), s_ref) <= TOL["bf16"]


def test_decode_fp32_d64():
    H, d, N = 2, 64, 3
    s = W.small("dec32", [9] * N, H=H, d=d, io_dtype="fp32", seed=22, s0_std=0.1)
    inp = W.make_inputs(s)
    o, st, cs = gpu_prefill(s, inp)
    f = f64_inputs(inp)
    _, s_ref, c_ref, _ = oracle_prefill(s, inp)
    x = _decode_inputs(s, 0)
    o_t = kda.decode_step(_dev(x["q"]), _dev(x["k"]), _dev(x["v"]), _dev(x["alpha"]), _dev(x["b"]),
                          _dev(inp["conv_w"]), _dev(inp["A_log"]), _dev(inp["dt_bias"]), st, cs)
    xf = {k: W.as_f64(v) for k, v in x.items()}
    o_r, s_r, c_r = oracle.decode_step(H, d, s_ref, c_ref, xf["q"], xf["k"], xf["v"], xf["alpha"],
                                       xf["b"], f["conv_w"], f["A_log"], f["dt_bias"])
    torch.cuda.synchronize()
    og = W.from_device(o_t)
    assert max(rel_l2(og[n, h], o_r[n, h]) for n in range(N) for h in range(H)) <= TOL["fp32"]
    assert max_state_err(W.from_device(st), s_r) <= TOL["fp32"]


def test_prefill_plus_decode_equals_long_prefill_gpu():
    """The state hand-off on the GPU alone: prefill(T1) + T2 decode steps vs prefill(T1 + T2)."""
    H, d, T1, T2 = 2, 128, 100, 6
    s = W.small("handoff", [T1 + T2], H=H, d=d, seed=23, s0_std=0.02)
    inp = W.make_inputs(s)
    o_long, s_long, _ = gpu_prefill(s, inp)
    s1 = W.small("handoff", [T1], H=H, d=d, seed=23, s0_std=0.02)
    cut = {k: (v[:T1] if k in ("q", "k", "v", "alpha", "b") else v) for k, v in inp.items()}
    cut["cu_seqlens"] = np.array([0, T1], dtype=np.int32)
    o1, st, cs = gpu_prefill(s1, cut)
    outs = [W.from_device(o1)]
    for t in range(T1, T1 + T2):
        o_t = kda.decode_step(_dev(inp["q"][t:t + 1]), _dev(inp["k"][t:t + 1]), _dev(inp["v"][t:t + 1]),
                              _dev(inp["alpha"][t:t + 1]), _dev(inp["b"][t:t + 1]),
                              _dev(inp["conv_w"]), _dev(inp["A_log"]), _dev(inp["dt_bias"]), st, cs)
        outs.append(W.from_device(o_t))
    torch.cuda.synchronize()
    o_cat = np.concatenate(outs)
    ol = W.from_device(o_long)
    for h in range(H):
        assert rel_l2(o_cat[:, h], ol[:, h]) <= TOL["bf16"]
    assert max_state_err(W.from_device(st), W.from_device(s_long)) <= TOL["bf16"]


# ------------------------------------------------------------------ negative eigenvalues

@pytest.mark.parametrize("io,d,lens", [("bf16", 128, [1, 70, 200]), ("fp32", 64, [33, 90]),
                                       ("fp32", 128, [65])])
def test_prefill_negative_eigenvalues(io, d, lens):
    """beta = 2 sigmoid(b) (kda_allow_negative_eigenvalues): the bf16 chunk path and the
    fp32 token kernel against the switched oracle."""
    s = W.small("neg", lens, H=3, d=d, io_dtype=io, seed=41, s0_std=0.02, varlen=len(lens) > 1)
    check_prefill(s, neg=True)


def test_prologue_negative_eigenvalues_beta():
    s = W.small("negpro", [9, 30], H=2, d=128, io_dtype="bf16", seed=42)
    inp = W.make_inputs(s)
    out = kda.prologue(_dev(inp["q"]), _dev(inp["k"]), _dev(inp["v"]), _dev(inp["conv_w"]),
                       _dev(inp["alpha"]), _dev(inp["b"]), _dev(inp["A_log"]), _dev(inp["dt_bias"]),
                       cu_seqlens=_dev(inp["cu_seqlens"]), num_seqs=s.num_seqs,
                       negative_eigenvalues=True)
    torch.cuda.synchronize()
    f = f64_inputs(inp)
    ref = oracle.prologue(inp["cu_seqlens"], s.H, s.d, f["q"], f["k"], f["v"], f["conv_w"],
                          f["alpha"], f["b"], f["A_log"], f["dt_bias"], negative_eigenvalues=True)
    np.testing.assert_allclose(W.from_device(out[4]), ref[4], rtol=1e-5, atol=1e-6)
    assert float(W.from_device(out[4]).max()) > 1.0   # the doubled range is in use


# ------------------------------------------------------------------ output epilogue

@pytest.mark.parametrize("io,d,lens", [("bf16", 128, [1, 70, 200]), ("bf16", 128, [64, 64]),
                                       ("fp32", 64, [33, 90]), ("fp32", 128, [65])])
def test_prefill_output_gate(io, d, lens):
    """o <- rmsnorm(o) * w * sigmoid(gate) fused into the store: the bf16 state pass (its
    gate-tile warp, fp32 staging) and the token kernel, against the oracle's epilogue."""
    s = W.small("og", lens, H=3, d=d, io_dtype=io, seed=43, s0_std=0.02, varlen=len(set(lens)) > 1)
    inp = W.make_inputs(s)
    G = W.make_output_gate(s, s.total_tokens)
    cu = _dev(inp["cu_seqlens"]) if s.varlen else None
    o, fs, _ = kda.prefill(_dev(inp["q"]), _dev(inp["k"]), _dev(inp["v"]), _dev(inp["conv_w"]),
                           _dev(inp["alpha"]), _dev(inp["b"]), _dev(inp["A_log"]), _dev(inp["dt_bias"]),
                           initial_state=_dev(inp["S0"]), cu_seqlens=cu, num_seqs=s.num_seqs,
                           out_gate=_dev(G["gate"]), o_norm_weight=_dev(G["o_norm_weight"]),
                           o_norm_eps=1e-5, check=True)
    torch.cuda.synchronize()
    f = f64_inputs(inp)
    o_ref, s_ref, _, _ = oracle.forward(inp["cu_seqlens"], s.H, s.d, f["q"], f["k"], f["v"],
                                        f["conv_w"], f["alpha"], f["b"], f["A_log"], f["dt_bias"],
                                        state0=f["S0"], out_gate=W.as_f64(G["gate"]),
                                        o_norm_weight=W.as_f64(G["o_norm_weight"]), o_norm_eps=1e-5)
    tol = TOL[io]
    eo = max_pair_err(W.from_device(o), o_ref, inp["cu_seqlens"], s.H)
    assert eo <= tol, "gated o rel-L2 %.3g > %.0e" % (eo, tol)
    assert max_state_err(W.from_device(fs), s_ref) <= tol


@pytest.mark.parametrize("H,N", [(3, 5), (16, 40)])
def test_decode_output_gate(H, N):
    """The epilogue in both decode kernels (H=3: per item; H=16 x 40: the persistent ring)."""
    d, T1, steps = 128, 20, 3
    s = W.small("ogdec", [T1] * N, H=H, d=d, seed=44, s0_std=0.02)
    inp = W.make_inputs(s)
    o, st, cs = gpu_prefill(s, inp)
    f = f64_inputs(inp)
    _, s_ref, c_ref, _ = oracle_prefill(s, inp)
    wgt = W.make_output_gate(s, N)["o_norm_weight"]
    for step in range(steps):
        x = _decode_inputs(s, step)
        gate = W.make_output_gate(s, N, tag=step + 1)["gate"]
        o_t = kda.decode_step(_dev(x["q"]), _dev(x["k"]), _dev(x["v"]), _dev(x["alpha"]),
                              _dev(x["b"]), _dev(inp["conv_w"]), _dev(inp["A_log"]),
                              _dev(inp["dt_bias"]), st, cs, out_gate=_dev(gate),
                              o_norm_weight=_dev(wgt))
        xf = {k: W.as_f64(v) for k, v in x.items()}
        o_r, s_ref, c_ref = oracle.decode_step(H, d, s_ref, c_ref, xf["q"], xf["k"], xf["v"],
                                               xf["alpha"], xf["b"], f["conv_w"], f["A_log"],
                                               f["dt_bias"], out_gate=W.as_f64(gate),
                                               o_norm_weight=W.as_f64(wgt))
        torch.cuda.synchronize()
        og = W.from_device(o_t)
        worst = max(rel_l2(og[n, h], o_r[n, h]) for n in range(N) for h in range(H))
        assert worst <= TOL["bf16"], (step, worst)
    assert max_state_err(W.from_device(st), s_ref) <= TOL["bf16"]


# ------------------------------------------------------------------ state snapshots

@pytest.mark.parametrize("io,d,lens,every,cap", [("bf16", 128, [64 * 5 + 7, 128, 300, 64, 0], 1, 6),
                                                 ("bf16", 128, [64 * 6, 200], 2, 3),
                                                 ("bf16", 128, [64 * 6], 2, 2),
                                                 ("fp32", 64, [150, 64], 1, 3)])
def test_prefill_state_snapshots(io, d, lens, every, cap):
    """Snapshot j = the state after (j + 1) * 64 * every tokens of each sequence (the state
    pass on the chunk path, the token kernel in fp32); slots past a sequence or past the
    capacity stay untouched."""
    s = W.small("snap", lens, H=2, d=d, io_dtype=io, seed=45, s0_std=0.02, varlen=len(set(lens)) > 1)
    inp = W.make_inputs(s)
    cu = _dev(inp["cu_seqlens"]) if s.varlen else None
    snaps = torch.full((s.num_seqs, cap, s.H, d, d), float("nan"), dtype=torch.float32, device="cuda")
    o, fs, _ = kda.prefill(_dev(inp["q"]), _dev(inp["k"]), _dev(inp["v"]), _dev(inp["conv_w"]),
                           _dev(inp["alpha"]), _dev(inp["b"]), _dev(inp["A_log"]), _dev(inp["dt_bias"]),
                           initial_state=_dev(inp["S0"]), cu_seqlens=cu, num_seqs=s.num_seqs,
                           snapshots=snaps, snapshot_every=every, check=True)
    torch.cuda.synchronize()
    f = f64_inputs(inp)
    ref = oracle.snapshots(inp["cu_seqlens"], s.H, d, 64 * every, cap, f["q"], f["k"], f["v"],
                           f["conv_w"], f["alpha"], f["b"], f["A_log"], f["dt_bias"], state0=f["S0"])
    got = W.from_device(snaps)
    tol = TOL[io]
    for n in range(s.num_seqs):
        for j in range(cap):
            if np.isnan(ref[n, j]).all():
                assert np.isnan(got[n, j]).all(), (n, j)   # not written
            else:
                for h in range(s.H):
                    e = rel_l2(got[n, j, h], ref[n, j, h])
                    assert e <= tol, (n, j, h, e)
    # the plain outputs are unchanged by asking for snapshots
    o_ref, s_ref, _, _ = oracle_prefill(s, inp)
    assert max_pair_err(W.from_device(o), o_ref, inp["cu_seqlens"], s.H) <= tol
    assert max_state_err(W.from_device(fs), s_ref) <= tol


# ------------------------------------------------------------------ multi-token decode

@pytest.mark.parametrize("io,H,N,T,gated", [("bf16", 3, 5, 2, False), ("bf16", 16, 40, 4, False),
                                            ("bf16", 8, 6, 3, True), ("fp32", 2, 3, 4, False),
                                            ("bf16", 64, 2, 16, True), ("bf16", 8, 3, 1, False)])
def test_decode_multi(io, H, N, T, gated):
    """T tokens per sequence in one call (speculative-token verification): o, the state and
    conv state after the T tokens and the state after each token, against the oracle run
    over those T tokens from the same state and conv history.  Two calls in a row.  bf16
    with H a multiple of 8 runs the persistent multi-token kernel, here up to its limits
    (16 tokens, 64 heads: 95 bulk copies per item; T = 1 with per-token states)."""
    d = 128
    s = W.small("dmulti", [24] * N, H=H, d=d, io_dtype=io, seed=46, s0_std=0.02)
    inp = W.make_inputs(s)
    o, st, cs = gpu_prefill(s, inp)
    f = f64_inputs(inp)
    _, s_ref, c_ref, _ = oracle_prefill(s, inp)
    wgt = W.make_output_gate(s, N)["o_norm_weight"] if gated else None
    for call in range(2):
        xs = [_decode_inputs(s, call * T + t) for t in range(T)]
        x = {k: np.ascontiguousarray(np.stack([xx[k] for xx in xs], axis=1)) for k in xs[0]}  # [N, T, ...]
        gate = W.make_output_gate(s, N * T, tag=call + 1)["gate"].reshape(N, T, H, d) if gated else None
        steps = torch.full((N, T, H, d, d), float("nan"), dtype=torch.float32, device="cuda")
        o_t = kda.decode_multi(_dev(x["q"]), _dev(x["k"]), _dev(x["v"]), _dev(x["alpha"]),
                               _dev(x["b"]), _dev(inp["conv_w"]), _dev(inp["A_log"]),
                               _dev(inp["dt_bias"]), st, cs, step_states=steps,
                               out_gate=_dev(gate) if gated else None,
                               o_norm_weight=_dev(wgt) if gated else None)
        torch.cuda.synchronize()
        cu = np.arange(0, N * T + 1, T)
        flat = lambda a, tail: W.as_f64(a).reshape((N * T,) + tail)
        fx = dict(q=flat(x["q"], (H * d,)), k=flat(x["k"], (H * d,)), v=flat(x["v"], (H * d,)),
                  alpha=flat(x["alpha"], (H, d)), b=flat(x["b"], (H,)))
        kw = dict(out_gate=W.as_f64(gate).reshape(N * T, H, d), o_norm_weight=W.as_f64(wgt)) if gated else {}
        o_r, s_new, c_new, _ = oracle.forward(cu, H, d, fx["q"], fx["k"], fx["v"], f["conv_w"],
                                              fx["alpha"], fx["b"], f["A_log"], f["dt_bias"],
                                              state0=s_ref, conv0=c_ref, **kw)
        st_r = oracle.snapshots(cu, H, d, 1, T, fx["q"], fx["k"], fx["v"], f["conv_w"], fx["alpha"],
                                fx["b"], f["A_log"], f["dt_bias"], state0=s_ref, conv0=c_ref)
        tol = TOL[io]
        og = W.from_device(o_t).reshape(N * T, H, d)
        worst = max(rel_l2(og[i, h], o_r[i, h]) for i in range(N * T) for h in range(H))
        assert worst <= tol, (call, worst)
        gs = W.from_device(steps)
        for t in range(T):
            assert max_state_err(gs[:, t], st_r[:, t]) <= tol, (call, t)
        s_ref, c_ref = s_new, c_new
        assert max_state_err(W.from_device(st), s_ref) <= tol
        np.testing.assert_array_equal(W.from_device(cs), c_ref)


# ------------------------------------------------------------------ time-segmented schedule

def test_prefill_time_segments_gated():
    """Dense batches with few (sequence, head) chains and at least 256 chunks per sequence
    run chunk_prep and the state pass in time segments of 128 chunks on two streams, the
    state carried between segments through final_state.  Two sequences of 16428 tokens
    (3 segments, the last one a single ragged 44-token chunk), an initial state and the
    output epilogue, against the oracle on everything."""
    s = W.small("seg", [16428, 16428], H=2, d=128, seed=61, s0_std=0.02, varlen=False)
    inp = W.make_inputs(s)
    G = W.make_output_gate(s, s.total_tokens)
    o, fs, fc = kda.prefill(_dev(inp["q"]), _dev(inp["k"]), _dev(inp["v"]), _dev(inp["conv_w"]),
                            _dev(inp["alpha"]), _dev(inp["b"]), _dev(inp["A_log"]), _dev(inp["dt_bias"]),
                            initial_state=_dev(inp["S0"]), num_seqs=s.num_seqs,
                            out_gate=_dev(G["gate"]), o_norm_weight=_dev(G["o_norm_weight"]),
                            o_norm_eps=1e-5, check=True)
    torch.cuda.synchronize()
    f = f64_inputs(inp)
    o_ref, s_ref, c_ref, _ = oracle.forward(inp["cu_seqlens"], s.H, s.d, f["q"], f["k"], f["v"],
                                            f["conv_w"], f["alpha"], f["b"], f["A_log"], f["dt_bias"],
                                            state0=f["S0"], out_gate=W.as_f64(G["gate"]),
                                            o_norm_weight=W.as_f64(G["o_norm_weight"]), o_norm_eps=1e-5)
    eo = max_pair_err(W.from_device(o), o_ref, inp["cu_seqlens"], s.H)
    es = max_state_err(W.from_device(fs), s_ref)
    assert eo <= TOL["bf16"], "o rel-L2 %.3g" % eo
    assert es <= TOL["bf16"], "final_state rel-L2 %.3g" % es
    np.testing.assert_array_equal(W.from_device(fc), c_ref)


def test_prefill_time_segments_snapshots():
    """Snapshots every 4096 tokens of a 16448-token sequence (257 chunks: time segments
    [0, 128), [128, 256), [256, 257)): those after chunks 128 and 256 end a segment and
    are stored as its final state, the others are stored between chunks."""
    every, cap = 64, 5
    s = W.small("segsnap", [16448], H=2, d=128, seed=62, s0_std=0.02, varlen=False)
    inp = W.make_inputs(s)
    snaps = torch.full((1, cap, s.H, 128, 128), float("nan"), dtype=torch.float32, device="cuda")
    o, fs, _ = kda.prefill(_dev(inp["q"]), _dev(inp["k"]), _dev(inp["v"]), _dev(inp["conv_w"]),
                           _dev(inp["alpha"]), _dev(inp["b"]), _dev(inp["A_log"]), _dev(inp["dt_bias"]),
                           initial_state=_dev(inp["S0"]), num_seqs=1, snapshots=snaps, snapshot_every=every, check=True)
    torch.cuda.synchronize()
    f = f64_inputs(inp)
    ref = oracle.snapshots(inp["cu_seqlens"], s.H, 128, 64 * every, cap, f["q"], f["k"], f["v"],
                           f["conv_w"], f["alpha"], f["b"], f["A_log"], f["dt_bias"], state0=f["S0"])
    got = W.from_device(snaps)
    for j in range(cap):
        if np.isnan(ref[0, j]).all():
            assert np.isnan(got[0, j]).all(), j
        else:
            for h in range(s.H):
                e = rel_l2(got[0, j, h], ref[0, j, h])
                assert e <= TOL["bf16"], (j, h, e)


@pytest.mark.parametrize("n_seqs", [40, 2100])
def test_prefill_bf16_many_varlen_sequences(n_seqs):
    """Many sequences in one varlen batch, empty ones among them: the state pass runs its
    (sequence, head) chains longest first up to 2048 sequences (a ranked order of the chunk
    counts) and in sequence order beyond; both must match the oracle.

    Lengths are drawn from [16, 100), the varlen workload's lower clip being 16: over the 1 to
    7 rows of a shorter sequence the per-(sequence, head) relative L2 of o is ill-conditioned
    where q.k is nearly orthogonal, and the bf16 rounding of q, k, v after the prologue alone
    (shared by every bf16 path: the tensor-core kernels and the token loop gave the same
    error, 3.7e-2, on such a 2-token sequence) can exceed 1e-2 there."""
    rng = np.random.default_rng(90 + n_seqs)
    lens = [int(x) for x in rng.integers(16, 100, n_seqs)]
    lens[3] = lens[n_seqs // 2] = 0
    s = W.small("many", lens, H=2, d=128, io_dtype="bf16", seed=91, s0_std=0.02, varlen=True)
    check_prefill(s)
