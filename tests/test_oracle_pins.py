"""Pins for the fp64 oracle: every check here is independent of the oracle's code.

The oracle restates the KDA forward pass from the AliceAI-Foundation KDA
write-up ("二、KDA 线性注意力" section: per-token loop, gate formula, causal conv
kernel 4 / padding 3 / no bias + SiLU, L2-normalised q/k) and the
Ling-3.0-flash-VL config table (kda_lower_bound -5.0).  These tests pin it to
things fixed by the mathematics or by library routines:

* recurrence      -> brute-force unrolled matrix product (dense numpy algebra)
* delta rule      -> retrieval identity with beta=1, g=0, unit key
* decay / gate    -> beta=0 closed form, lower-bound e^{-5n} closed form,
                     a hand-computed scalar gate, the alpha -> -inf limit
* prologue        -> torch Conv1d (groups=channels, padding 3, truncated),
                     scipy expit / numpy logaddexp, unit norms
* state hand-off  -> prefill(T1) + T2 decode steps == prefill(T1 + T2)
* varlen packing  -> packed run == separate runs (bitwise)
"""

import numpy as np
import pytest
import scipy.special as sp
import torch

from oracle import oracle


def _rng(seed):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------- recurrence

def _brute_force(q, k, v, g, beta, S0):
    """S_t = P(t,0) S0 + sum_s P(t,s) beta_s k_s v_s^T with A_t = (I - beta_t k_t k_t^T) diag(e^{g_t}),
    P(t,s) = A_t A_{t-1} ... A_{s+1};  o_t = S_t^T q_t."""
    T, D = q.shape
    A = [(np.eye(D) - beta[t] * np.outer(k[t], k[t])) @ np.diag(np.exp(g[t])) for t in range(T)]

    def P(t, s):
        M = np.eye(D)
        for r in range(s + 1, t + 1):
            M = A[r] @ M
        return M

    outs, S = [], None
    for t in range(T):
        S = P(t, -1) @ S0 + sum(P(t, s) @ (beta[s] * np.outer(k[s], v[s])) for s in range(t + 1))
        outs.append(S.T @ q[t])
    return np.stack(outs), S


@pytest.mark.parametrize("T,D,seed", [(1, 2, 0), (3, 3, 1), (8, 4, 2), (7, 4, 3)])
def test_recurrence_matches_unrolled_product(T, D, seed):
    r = _rng(seed)
    q, k, v = r.standard_normal((3, T, 1, D))
    g = -r.uniform(0.0, 2.0, (T, 1, D))
    beta = r.uniform(0.05, 0.95, (T, 1))
    S0 = r.standard_normal((1, 1, D, D))          # non-symmetric: a transposed S fails
    o, S = oracle.recurrence([0, T], q, k, v, g, beta, S0)
    o_ref, S_ref = _brute_force(q[:, 0], k[:, 0], v[:, 0], g[:, 0], beta[:, 0], S0[0, 0])
    np.testing.assert_allclose(o[:, 0], o_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(S[0, 0], S_ref, rtol=0, atol=1e-12)


def test_recurrence_scale_multiplies_output_only():
    r = _rng(5)
    T, D = 5, 3
    q, k, v = r.standard_normal((3, T, 1, D))
    g = -r.uniform(0, 1, (T, 1, D))
    beta = r.uniform(0, 1, (T, 1))
    o1, S1 = oracle.recurrence([0, T], q, k, v, g, beta, None, scale=1.0)
    o2, S2 = oracle.recurrence([0, T], q, k, v, g, beta, None, scale=0.25)
    np.testing.assert_allclose(o2, 0.25 * o1, rtol=1e-14, atol=0)
    np.testing.assert_array_equal(S1, S2)


def test_delta_rule_retrieval_identity():
    """beta=1, g=0, unit key: reading with q = k right after the write returns v."""
    r = _rng(7)
    T, D = 6, 8
    k = r.standard_normal((T, 1, D))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = r.standard_normal((T, 1, D))
    g = np.zeros((T, 1, D))
    beta = np.ones((T, 1))
    S0 = r.standard_normal((1, 1, D, D))
    o, _ = oracle.recurrence([0, T], k.copy(), k, v, g, beta, S0)
    np.testing.assert_allclose(o, v, rtol=0, atol=1e-12)


def test_beta_zero_only_decays():
    r = _rng(8)
    T, D = 5, 4
    q, k, v = r.standard_normal((3, T, 1, D))
    g = -r.uniform(0, 3, (T, 1, D))
    S0 = r.standard_normal((1, 1, D, D))
    o, S = oracle.recurrence([0, T], q, k, v, g, np.zeros((T, 1)), S0)
    Gam = np.cumsum(g[:, 0], axis=0)                    # [T, D]
    for t in range(T):
        St = np.exp(Gam[t])[:, None] * S0[0, 0]
        np.testing.assert_allclose(o[t, 0], St.T @ q[t, 0], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(S[0, 0], np.exp(Gam[-1])[:, None] * S0[0, 0], rtol=1e-12)


# ---------------------------------------------------------------- prologue

def _prologue_inputs(seed, lens, H, D, conv_std=0.5):
    r = _rng(seed)
    T = sum(lens)
    HD = H * D
    return dict(
        cu=np.concatenate([[0], np.cumsum(lens)]).astype(np.int64),
        q=r.standard_normal((T, HD)), k=r.standard_normal((T, HD)), v=r.standard_normal((T, HD)),
        conv_w=r.standard_normal((3, HD, 4)) * conv_std,
        alpha=r.standard_normal((T, H, D)), b=r.standard_normal((T, H)),
        A_log=np.log(r.uniform(1, 16, H)), dt_bias=r.uniform(-1, 1, (H, D)))


def _torch_conv_silu(x, w):
    """nn.Conv1d(C, C, groups=C, kernel_size=4, padding=3, bias=False) on [T, C], output truncated to T, then SiLU."""
    T, C = x.shape
    xt = torch.from_numpy(x.T[None].copy())                        # [1, C, T]
    wt = torch.from_numpy(w[:, None, :].copy())                    # [C, 1, 4]
    y = torch.nn.functional.conv1d(xt, wt, padding=3, groups=C)[0, :, :T].T.numpy()
    return y * sp.expit(y)


def test_prologue_matches_torch_conv1d_and_scipy():
    H, D, lens = 2, 8, [11, 5, 2]
    I = _prologue_inputs(11, lens, H, D)
    qn, kn, vc, g, beta = oracle.prologue(I["cu"], H, D, I["q"], I["k"], I["v"], I["conv_w"],
                                          I["alpha"], I["b"], I["A_log"], I["dt_bias"])
    eps = 1e-6
    for n in range(len(lens)):
        a, z = I["cu"][n], I["cu"][n + 1]
        for blk, (name, got) in enumerate((("q", qn), ("k", kn), ("v", vc))):
            y = _torch_conv_silu(I[name][a:z], I["conv_w"][blk])      # [L, H*D]
            y = y.reshape(z - a, H, D)
            if name != "v":
                y = y / np.sqrt((y * y).sum(-1, keepdims=True) + eps)
            np.testing.assert_allclose(got[a:z], y, rtol=1e-12, atol=1e-14)
    x = I["alpha"] + I["dt_bias"][None]
    g_ref = np.maximum(-np.exp(I["A_log"])[None, :, None] * np.logaddexp(0.0, x), -5.0)
    np.testing.assert_allclose(g, g_ref, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(beta, sp.expit(I["b"]), rtol=1e-14)


def test_prologue_unit_norms():
    H, D = 3, 16
    I = _prologue_inputs(12, [40], H, D)
    qn, kn, vc, _, _ = oracle.prologue(I["cu"], H, D, I["q"], I["k"], I["v"], I["conv_w"],
                                       I["alpha"], I["b"], I["A_log"], I["dt_bias"])
    for x in (qn, kn):
        nrm = np.linalg.norm(x, axis=-1)
        np.testing.assert_allclose(nrm, 1.0, atol=1e-5)   # eps=1e-6 inside the root
    assert not np.allclose(np.linalg.norm(vc, axis=-1), 1.0)


def test_gate_closed_forms():
    """A_log = ln 2, alpha + dt_bias = 0 -> g = -2 ln 2; alpha -> +inf -> g = -5 exactly;
    alpha -> -inf -> g -> 0 from below."""
    H, D = 1, 4
    I = _prologue_inputs(13, [3], H, D)
    I["A_log"] = np.array([np.log(2.0)])
    I["dt_bias"] = np.array([[0.0, 0.0, 0.5, -0.5]])
    I["alpha"] = np.array([[[0.0, 1e4, -0.5, 0.5]], [[-1e4, 0.0, 0.0, 0.0]], [[3.0, 3.0, 3.0, 3.0]]])
    _, _, _, g, _ = oracle.prologue(I["cu"], H, D, I["q"], I["k"], I["v"], I["conv_w"],
                                    I["alpha"], I["b"], I["A_log"], I["dt_bias"])
    assert abs(g[0, 0, 0] - (-2.0 * np.log(2.0))) < 1e-15
    assert g[0, 0, 1] == -5.0
    assert abs(g[0, 0, 2] - (-2.0 * np.log(2.0))) < 1e-15
    assert abs(g[0, 0, 3] - (-2.0 * np.log(2.0))) < 1e-15
    assert -1e-300 < g[1, 0, 0] <= 0.0
    # 2 * softplus(3 + 0.5) = 7.06 > 5: clamped; 2 * softplus(2.5) = 5.16: clamped; 2*softplus(3)=6.1: clamped
    assert np.all(g[2, 0] == -5.0)


def test_lower_bound_decay_closed_form():
    """k = 0 (zero raw inputs) and alpha -> +inf: after n steps S = e^{-5n} S0."""
    H, D, n = 2, 4, 6
    I = _prologue_inputs(14, [n], H, D)
    for name in ("q", "k", "v"):
        I[name] = np.zeros_like(I[name])
    I["alpha"] = np.full_like(I["alpha"], 1e4)
    S0 = _rng(15).standard_normal((1, H, D, D))
    o, S1, _, _ = oracle.forward(I["cu"], H, D, I["q"], I["k"], I["v"], I["conv_w"], I["alpha"],
                                 I["b"], I["A_log"], I["dt_bias"], state0=S0)
    np.testing.assert_allclose(S1, np.exp(-5.0 * n) * S0, rtol=1e-12)
    assert np.all(o == 0.0)


# ---------------------------------------------------------------- composition

# ---------------------------------------------------------------- negative eigenvalues
# The kda_allow_negative_eigenvalues switch (AliceAI-Foundation KDA write-up, section
# "二": with it off, beta is not multiplied by 2 and stays in (0, 1)): beta = 2 sigmoid(b).

def test_negative_eigenvalues_beta_is_twice_sigmoid():
    """The prologue's beta doubles; q, k, v and g do not change."""
    H, D, lens = 2, 8, [7, 3]
    I = _prologue_inputs(31, lens, H, D)
    args = (I["cu"], H, D, I["q"], I["k"], I["v"], I["conv_w"], I["alpha"], I["b"], I["A_log"],
            I["dt_bias"])
    plain = oracle.prologue(*args)
    neg = oracle.prologue(*args, negative_eigenvalues=True)
    for x, y in zip(plain[:4], neg[:4]):
        np.testing.assert_array_equal(x, y)
    np.testing.assert_allclose(neg[4], 2.0 * sp.expit(I["b"]), rtol=1e-14)


def test_negative_eigenvalues_write_is_a_householder_reflection():
    """beta = 2 (b -> +inf), no decay (alpha -> -inf), unit key (eps = 0), v = 0: one
    write maps S to (I - 2 k k^T) S, the reflection through the plane normal to k,
    whose eigenvalue along k is -1."""
    H, D = 1, 6
    I = _prologue_inputs(32, [1], H, D)
    I["b"][:] = 50.0          # sigmoid -> 1 in fp64
    I["alpha"][:] = -800.0    # softplus -> 0, g = 0
    I["v"][:] = 0.0
    S0 = _rng(33).standard_normal((1, H, D, D))
    o, S1, _, _ = oracle.forward(I["cu"], H, D, I["q"], I["k"], I["v"], I["conv_w"], I["alpha"],
                                 I["b"], I["A_log"], I["dt_bias"], state0=S0, eps=0.0,
                                 negative_eigenvalues=True)
    # the unit key, from the conv + SiLU + norm of token 0 (only the newest tap sees it)
    y = I["k"][0] * I["conv_w"][1][:, 3]
    k = y * sp.expit(y)
    k /= np.linalg.norm(k)
    R = np.eye(D) - 2.0 * np.outer(k, k)
    np.testing.assert_allclose(S1[0, 0], R @ S0[0, 0], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(k @ S1[0, 0], -(k @ S0[0, 0]), rtol=1e-12, atol=1e-13)
    # without the switch the same write is a projection: k^T S' = 0
    _, S1p, _, _ = oracle.forward(I["cu"], H, D, I["q"], I["k"], I["v"], I["conv_w"], I["alpha"],
                                  I["b"], I["A_log"], I["dt_bias"], state0=S0, eps=0.0)
    np.testing.assert_allclose(k @ S1p[0, 0], 0.0, atol=1e-13)


def test_negative_eigenvalues_equal_plain_run_with_rescaled_b():
    """For b < 0, 2 sigmoid(b) < 1 is itself a sigmoid: the switched run equals the plain
    run on b' = logit(2 sigmoid(b))."""
    H, D, lens = 2, 8, [9, 5]
    I = _prologue_inputs(34, lens, H, D)
    I["b"] = -np.abs(I["b"]) - 0.1
    S0 = _rng(35).standard_normal((2, H, D, D)) * 0.1
    common = (I["cu"], H, D, I["q"], I["k"], I["v"], I["conv_w"], I["alpha"])
    o1, S1, _, _ = oracle.forward(*common, I["b"], I["A_log"], I["dt_bias"], state0=S0,
                                  negative_eigenvalues=True)
    b2 = sp.logit(2.0 * sp.expit(I["b"]))
    o2, S2, _, _ = oracle.forward(*common, b2, I["A_log"], I["dt_bias"], state0=S0)
    np.testing.assert_allclose(o1, o2, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(S1, S2, rtol=1e-10, atol=1e-12)


def test_recurrence_with_beta_above_one_matches_unrolled_product():
    """beta in (1, 2): the transition has a negative eigenvalue; the product form still holds."""
    r = _rng(36)
    T, D = 6, 4
    q, k, v = (r.standard_normal((T, 1, D)) for _ in range(3))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    g = -r.uniform(0, 1, (T, 1, D))
    beta = r.uniform(1.05, 1.95, (T, 1))
    S0 = r.standard_normal((1, 1, D, D))
    o, S = oracle.recurrence([0, T], q, k, v, g, beta, S0)
    o_ref, S_ref = _brute_force(q[:, 0], k[:, 0], v[:, 0], g[:, 0], beta[:, 0], S0[0, 0])
    np.testing.assert_allclose(o[:, 0], o_ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(S[0, 0], S_ref, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- output epilogue
# o_norm then sigmoid output gating (write-up sections "二" and "三"):
# properties that hold for an RMS norm with a per-channel weight followed by a sigmoid gate.

def _gated(I, H, D, S0, gate, w, eps=0.0, scale=1.0):
    return oracle.forward(I["cu"], H, D, I["q"], I["k"], I["v"], I["conv_w"], I["alpha"], I["b"],
                          I["A_log"], I["dt_bias"], state0=S0, scale=scale, out_gate=gate,
                          o_norm_weight=w, o_norm_eps=eps)


def test_output_gate_unit_rms_and_direction():
    """w = 1, gate -> +inf, eps = 0: each head's output has RMS exactly 1 over its D
    channels and points the way the plain output does; the state is untouched."""
    H, D, lens = 2, 8, [6, 3]
    I = _prologue_inputs(51, lens, H, D)
    S0 = _rng(52).standard_normal((2, H, D, D))
    T = sum(lens)
    og, S1g, _, _ = _gated(I, H, D, S0, np.full((T, H, D), 60.0), np.ones(D))
    op, S1p, _, _ = oracle.forward(I["cu"], H, D, I["q"], I["k"], I["v"], I["conv_w"], I["alpha"],
                                   I["b"], I["A_log"], I["dt_bias"], state0=S0)
    np.testing.assert_allclose(np.sqrt((og * og).mean(-1)), 1.0, rtol=1e-12)
    cos = (og * op).sum(-1) / np.linalg.norm(og, axis=-1) / np.linalg.norm(op, axis=-1)
    np.testing.assert_allclose(cos, 1.0, rtol=1e-12)
    np.testing.assert_array_equal(S1g, S1p)


def test_output_gate_is_a_sigmoid():
    """sigmoid(x) + sigmoid(-x) = 1 and sigmoid(0) = 1/2, elementwise in the gate."""
    H, D, lens = 2, 8, [7]
    I = _prologue_inputs(53, lens, H, D)
    S0 = _rng(54).standard_normal((1, H, D, D))
    w = _rng(55).uniform(0.5, 1.5, D)
    g = _rng(56).standard_normal((7, H, D)) * 2.0
    o_pos, _, _, _ = _gated(I, H, D, S0, g, w, eps=1e-5)
    o_neg, _, _, _ = _gated(I, H, D, S0, -g, w, eps=1e-5)
    o_inf, _, _, _ = _gated(I, H, D, S0, np.full_like(g, 60.0), w, eps=1e-5)
    o_zero, _, _, _ = _gated(I, H, D, S0, np.zeros_like(g), w, eps=1e-5)
    np.testing.assert_allclose(o_pos + o_neg, o_inf, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(o_zero, 0.5 * o_inf, rtol=1e-13, atol=1e-15)


def test_output_gate_acts_channel_by_channel():
    """A one-hot gate (+60 on channel m, -60 elsewhere) keeps channel m of the fully open
    output and closes the rest (sigmoid(-60) ~ 1e-26)."""
    H, D, lens = 2, 8, [4]
    I = _prologue_inputs(65, lens, H, D)
    S0 = _rng(66).standard_normal((1, H, D, D))
    w = _rng(67).uniform(0.5, 1.5, D)
    o_inf, _, _, _ = _gated(I, H, D, S0, np.full((4, H, D), 60.0), w, eps=1e-5)
    for m in (0, 3, D - 1):
        g = np.full((4, H, D), -60.0)
        g[..., m] = 60.0
        o_m, _, _, _ = _gated(I, H, D, S0, g, w, eps=1e-5)
        np.testing.assert_allclose(o_m[..., m], o_inf[..., m], rtol=1e-14)
        others = np.delete(o_m, m, axis=-1)
        assert np.abs(others).max() <= 1e-20 * np.abs(o_inf).max()


def test_output_gate_weight_is_per_channel():
    H, D, lens = 1, 8, [5]
    I = _prologue_inputs(57, lens, H, D)
    S0 = _rng(58).standard_normal((1, H, D, D))
    g = _rng(59).standard_normal((5, H, D))
    w = _rng(60).uniform(-2, 2, D)
    o_w, _, _, _ = _gated(I, H, D, S0, g, w, eps=1e-5)
    o_1, _, _, _ = _gated(I, H, D, S0, g, np.ones(D), eps=1e-5)
    np.testing.assert_allclose(o_w, o_1 * w, rtol=1e-13, atol=1e-15)


def test_output_gate_eps_inside_the_mean_square():
    """o scales with `scale`; the norm is homogeneous when eps scales with the mean
    square: out(scale c, eps c^2) == out(scale 1, eps), and eps = 0 makes it scale-free."""
    H, D, lens = 2, 8, [6]
    I = _prologue_inputs(61, lens, H, D)
    S0 = _rng(62).standard_normal((1, H, D, D)) * 0.1
    g = _rng(63).standard_normal((6, H, D))
    w = _rng(64).uniform(0.5, 1.5, D)
    c = 7.0
    a, _, _, _ = _gated(I, H, D, S0, g, w, eps=0.3, scale=1.0)
    b_, _, _, _ = _gated(I, H, D, S0, g, w, eps=0.3 * c * c, scale=c)
    np.testing.assert_allclose(a, b_, rtol=1e-12, atol=1e-14)
    z1, _, _, _ = _gated(I, H, D, S0, g, w, eps=0.0, scale=1.0)
    zc, _, _, _ = _gated(I, H, D, S0, g, w, eps=0.0, scale=c)
    np.testing.assert_allclose(z1, zc, rtol=1e-12, atol=1e-14)
    assert not np.allclose(a, z1, rtol=1e-3)   # the eps in use does matter at this size


def test_forward_equals_prologue_then_recurrence():
    H, D, lens = 2, 8, [9, 4]
    I = _prologue_inputs(16, lens, H, D)
    S0 = _rng(17).standard_normal((2, H, D, D)) * 0.1
    o, S1, _, _ = oracle.forward(I["cu"], H, D, I["q"], I["k"], I["v"], I["conv_w"], I["alpha"],
                                 I["b"], I["A_log"], I["dt_bias"], state0=S0)
    qn, kn, vc, g, beta = oracle.prologue(I["cu"], H, D, I["q"], I["k"], I["v"], I["conv_w"],
                                          I["alpha"], I["b"], I["A_log"], I["dt_bias"])
    o2, S2 = oracle.recurrence(I["cu"], qn, kn, vc, g, beta, S0)
    np.testing.assert_allclose(o, o2, rtol=0, atol=1e-14)
    np.testing.assert_allclose(S1, S2, rtol=0, atol=1e-14)


@pytest.mark.parametrize("T1,T2", [(7, 5), (1, 4), (2, 1), (0, 3)])
def test_prefill_then_decode_equals_long_prefill(T1, T2):
    H, D = 2, 8
    I = _prologue_inputs(18, [T1 + T2], H, D)
    S0 = _rng(19).standard_normal((1, H, D, D)) * 0.1
    args = lambda a, z: (I["q"][a:z], I["k"][a:z], I["v"][a:z], I["conv_w"], I["alpha"][a:z],
                         I["b"][a:z], I["A_log"], I["dt_bias"])
    o_long, S_long, C_long, _ = oracle.forward([0, T1 + T2], H, D, *args(0, T1 + T2), state0=S0)
    o1, S, C, _ = oracle.forward([0, T1], H, D, *args(0, T1), state0=S0)
    outs = [o1]
    for t in range(T1, T1 + T2):
        q, k, v, w, al, b, A, dt = args(t, t + 1)
        o_t, S, C = oracle.decode_step(H, D, S, C, q, k, v, al, b, w, A, dt)
        outs.append(o_t)
    np.testing.assert_allclose(np.concatenate(outs), o_long, rtol=0, atol=1e-12)
    np.testing.assert_allclose(S, S_long, rtol=0, atol=1e-12)
    np.testing.assert_array_equal(C, C_long)


def test_final_conv_state_holds_last_three_raw_tokens():
    H, D = 2, 4
    I = _prologue_inputs(20, [6, 2], H, D)
    _, _, C, _ = oracle.forward(I["cu"], H, D, I["q"], I["k"], I["v"], I["conv_w"], I["alpha"],
                                I["b"], I["A_log"], I["dt_bias"])
    raw = np.concatenate([I["q"], I["k"], I["v"]], axis=1)            # [T, 3*H*D]
    np.testing.assert_array_equal(C[0], raw[3:6])
    np.testing.assert_array_equal(C[1, 0], 0.0)                        # history before a 2-token sequence
    np.testing.assert_array_equal(C[1, 1:], raw[6:8])


def test_varlen_equals_separate_sequences():
    H, D, lens = 2, 8, [5, 1, 12, 3]
    I = _prologue_inputs(21, lens, H, D)
    S0 = _rng(22).standard_normal((len(lens), H, D, D)) * 0.1
    o, S1, C1, _ = oracle.forward(I["cu"], H, D, I["q"], I["k"], I["v"], I["conv_w"], I["alpha"],
                                  I["b"], I["A_log"], I["dt_bias"], state0=S0)
    cu = I["cu"]
    for n in range(len(lens)):
        a, z = cu[n], cu[n + 1]
        o_n, S_n, C_n, _ = oracle.forward([0, z - a], H, D, I["q"][a:z], I["k"][a:z], I["v"][a:z],
                                          I["conv_w"], I["alpha"][a:z], I["b"][a:z], I["A_log"],
                                          I["dt_bias"], state0=S0[n:n + 1])
        np.testing.assert_array_equal(o[a:z], o_n)
        np.testing.assert_array_equal(S1[n], S_n[0])
        np.testing.assert_array_equal(C1[n], C_n[0])


def test_thread_count_does_not_change_results():
    H, D, lens = 4, 8, [10, 7]
    I = _prologue_inputs(23, lens, H, D)
    a = oracle.forward(I["cu"], H, D, I["q"], I["k"], I["v"], I["conv_w"], I["alpha"], I["b"],
                       I["A_log"], I["dt_bias"], nthreads=1)
    b = oracle.forward(I["cu"], H, D, I["q"], I["k"], I["v"], I["conv_w"], I["alpha"], I["b"],
                       I["A_log"], I["dt_bias"], nthreads=5)
    for x, y in zip(a[:3], b[:3]):
        np.testing.assert_array_equal(x, y)
