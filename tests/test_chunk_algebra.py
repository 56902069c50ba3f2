"""The chunked form of the prefill kernels (tests/chunk_model.py), in fp64, against the
oracle's token loop; and the exponent ranges its split decay factors stay in.

CPU only.  The prepared inputs are drawn directly (unit-norm q and k, gates in
[lower_bound, 0], beta in (0, 1)), since the factorisation starts after the prologue.
"""

import numpy as np
import pytest

from oracle import oracle
from tests import chunk_model as CM


def prepared(lens, H, d, lb, seed, gate_lo=None):
    rng = np.random.default_rng(seed)
    T = int(sum(lens))
    unit = lambda x: x / np.linalg.norm(x, axis=-1, keepdims=True)
    q = unit(rng.standard_normal((T, H, d)))
    k = unit(rng.standard_normal((T, H, d)))
    v = rng.standard_normal((T, H, d))
    lo = lb if gate_lo is None else gate_lo
    g = rng.uniform(lo, 0.0, (T, H, d))
    g[rng.random((T, H, d)) < 0.05] = lb    # some gates sit on the bound
    beta = rng.uniform(0.05, 1.0, (T, H))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    S0 = 0.1 * rng.standard_normal((len(lens), H, d, d))
    return cu, q, k, v, g, beta, S0


def rel(x, ref):
    return np.linalg.norm(x - ref) / max(np.linalg.norm(ref), 1e-300)


@pytest.mark.parametrize("lens,lb,seed", [([150, 64, 1, 0, 70], -5.0, 0),
                                          ([200], -10.0, 1),
                                          ([65, 127], -0.5, 2)])
def test_chunked_form_equals_token_loop(lens, lb, seed):
    """Chunks, sub-block references, T = (I + A_kk)^-1, W, U and the inter-chunk update
    reproduce the per-token recurrence (ragged tails, an empty and a one-token sequence)."""
    cu, q, k, v, g, beta, S0 = prepared(lens, H=2, d=16, lb=lb, seed=seed)
    o_ref, s_ref = oracle.recurrence(cu, q, k, v, g, beta, state0=S0)
    o, s = CM.chunked_forward(cu, q, k, v, g, beta, state0=S0)
    assert rel(o, o_ref) < 1e-10
    assert rel(s, s_ref) < 1e-10


@pytest.mark.parametrize("mistake", ["no_block_constant", "kk_diagonal", "beta_after_T"])
def test_chunked_form_comparison_catches_a_planted_mistake(mistake):
    """The comparison is not vacuous: an R row of an earlier block without its block constant,
    A_kk with its diagonal, or beta applied after T each break the agreement.  (Any reference
    m_I used consistently on both sides is exact: it only moves the exponent ranges.)"""
    cu, q, k, v, g, beta, S0 = prepared([130], H=1, d=8, lb=-2.0, seed=3)
    o_ref, _ = oracle.recurrence(cu, q, k, v, g, beta, state0=S0)
    o, _ = CM.chunked_forward(cu, q, k, v, g, beta, state0=S0, mistake=mistake)
    assert rel(o, o_ref) > 1e-3


@pytest.mark.parametrize("lb", [-5.0, -5.5, -8.0, -10.0])
def test_split_factors_stay_in_fp32_normal_range(lb):
    """Every L and R factor the kernels exponentiate spans at most 8 gates: |log2| <=
    8 |lb| log2 e (2^+-116 at the path's limit of -10), so none overflows fp32 or drops
    below its normal range (2^-126), where the special-function exponential flushes to 0."""
    rng = np.random.default_rng(4)
    d = 8
    g = np.full((CM.CH, d), lb)               # the worst case: every gate on the bound
    g[:, ::2] = rng.uniform(lb, 0.0, (CM.CH, d // 2))
    x = np.ones((CM.CH, d))
    *_, exps = CM.chunk_factors(x, x, x, g, np.full(CM.CH, 0.5))
    worst = max(np.max(e) for e in exps), min(np.min(e) for e in exps)
    bound = 8 * abs(lb) * CM.LOG2E + 1e-9
    assert worst[0] <= bound
    L_exp, Rd_exp = exps[0], exps[1]
    assert np.min(L_exp) >= -bound and np.min(Rd_exp) >= -bound
    assert bound < 126.0 or lb < -10.0


def test_block_start_reference_would_leave_the_normal_range():
    """Why the reference sits mid-block: from the block's start a factor spans 16 gates,
    and at gates of -5.5 the last token's factor falls below 2^-126."""
    span_from_start = 16 * 5.5 * CM.LOG2E
    span_mid = 8 * 5.5 * CM.LOG2E
    assert span_from_start > 126.0 > span_mid


@pytest.mark.parametrize("sb", [8, 32, 64])
def test_chunked_form_holds_for_other_sub_block_lengths(sb):
    """The factorisation is exact for any sub-block length; only the exponent ranges move."""
    cu, q, k, v, g, beta, S0 = prepared([150], H=1, d=8, lb=-5.0, seed=5)
    o_ref, s_ref = oracle.recurrence(cu, q, k, v, g, beta, state0=S0)
    o, s = CM.chunked_forward(cu, q, k, v, g, beta, state0=S0, sb=sb)
    assert rel(o, o_ref) < 1e-10 and rel(s, s_ref) < 1e-10


@pytest.mark.parametrize("lb,fits", [(-5.0, True), (-5.45, True), (-5.5, False)])
def test_32_token_sub_blocks_fit_only_near_the_default_bound(lb, fits):
    """With 32-token sub-blocks a factor spans up to 16 gates: inside fp32's normal range
    (|log2| < 126) at the default bound of -5 and just above it, outside from -5.5."""
    g = np.full((CM.CH, 4), lb)
    x = np.ones((CM.CH, 4))
    *_, exps = CM.chunk_factors(x, x, x, g, np.full(CM.CH, 0.5), sb=32)
    span = max(np.max(np.abs(exps[0])), np.max(np.abs(exps[1])))
    assert (span < 126.0) == fits



def _emulated_errors(s, sites=True, sb=CM.SB):
    """Largest per-(sequence, head) rel-L2 error of o and of the final state when the chunked
    form rounds to bf16 at ``sites`` (all of the kernels' bf16 points by default), against
    the oracle, on a workload's own inputs."""
    from gated_delta_rule_70_b200 import workloads as W
    inp = W.make_inputs(s)
    f = {k: W.as_f64(v) for k, v in inp.items() if k != "cu_seqlens"}
    cu = inp["cu_seqlens"]
    qn, kn, vc, g, beta = oracle.prologue(cu, s.H, s.d, f["q"], f["k"], f["v"], f["conv_w"],
                                          f["alpha"], f["b"], f["A_log"], f["dt_bias"],
                                          lower_bound=s.lower_bound)
    o_ref, s_ref = oracle.recurrence(cu, qn, kn, vc, g, beta, state0=f["S0"])
    o, st = CM.chunked_forward(cu, qn, kn, vc, g, beta, state0=f["S0"], bf16=sites, sb=sb)
    eo = max(rel(o[cu[n]:cu[n + 1], h], o_ref[cu[n]:cu[n + 1], h])
             for n in range(len(cu) - 1) for h in range(s.H) if cu[n + 1] > cu[n])
    es = max(rel(st[n, h], s_ref[n, h]) for n in range(len(cu) - 1) for h in range(s.H))
    return eo, es


@pytest.mark.parametrize("lens,H,seed,alpha_mu,lb,varlen", [
    ([150, 70], 2, 5, 0.0, -5.0, True),      # the smoke check's inputs
    ([200, 200], 4, 11, 0.0, -5.0, False),
    ([300], 2, 16, -2.0, -5.0, False),       # slow decay
    ([200], 2, 27, 3.0, -10.0, False),       # gates at a lower bound of -10
])
def test_bf16_rounding_points_fit_the_tolerance(lens, H, seed, alpha_mu, lb, varlen):
    """The precision design: rounding to bf16 wherever the kernels hold bf16 (q, k, v after
    the prologue, the MMA operands, T diag(beta), the record, the state's MMA copy, D and o)
    costs between 1e-3 and 6e-3 of the oracle's o and final state, inside the 1e-2 bar with
    room for the fp32 accumulation and the special-function approximations on top."""
    from gated_delta_rule_70_b200 import workloads as W
    s = W.small("emu", lens, H=H, d=128, seed=seed, s0_std=0.02, alpha_mu=alpha_mu,
                varlen=varlen)
    s.lower_bound = lb
    eo, es = _emulated_errors(s)
    assert 1e-3 < eo < 6e-3, eo
    assert 1e-3 < es < 6e-3, es


def test_each_bf16_site_alone_costs_about_one_rounding():
    """No single rounding site is amplified by the factorisation: each alone stays below
    3e-3 (bf16's unit roundoff is 2^-9 = 2e-3), and every site changes something."""
    from gated_delta_rule_70_b200 import workloads as W
    s = W.small("emu1", [200, 200], H=2, d=128, seed=11, s0_std=0.02)
    for site in CM.SITES:
        eo, es = _emulated_errors(s, [site])
        assert max(eo, es) < 3e-3, (site, eo, es)
        assert max(eo, es) > 1e-6, (site, eo, es)


@pytest.mark.parametrize("alpha_mu", [0.0, 3.0])
def test_32_token_sub_blocks_keep_the_precision_budget(alpha_mu):
    """At the default bound, 32-token sub-blocks round at the same sites with the same
    budget (alpha_mu = 3 puts most gates on the bound of -5)."""
    from gated_delta_rule_70_b200 import workloads as W
    s = W.small("emu32", [200, 70], H=2, d=128, seed=28, s0_std=0.02, alpha_mu=alpha_mu)
    e16 = _emulated_errors(s)
    e32 = _emulated_errors(s, sb=32)
    assert max(e32) < 6e-3
    assert max(e32) < 1.1 * max(e16)



def test_blocked_inverse_is_exact():
    """The blocked form of T = (I + A)^-1 (16 x 16 diagonal inverses, then the blocks next to the
    diagonal, then the 32 x 32 halves) is the inverse, in fp64."""
    rng = np.random.default_rng(6)
    A = np.tril(rng.standard_normal((CM.CH, CM.CH)) * 0.3, -1)
    assert np.abs(CM.blocked_inverse(A) - np.linalg.inv(np.eye(CM.CH) + A)).max() < 1e-12


def _collinear_keys(rho, seed=0, d=128, T=256):
    """Prepared inputs whose keys share one direction (spread rho around it), slow decay."""
    rng = np.random.default_rng(seed)
    unit = lambda x: x / np.linalg.norm(x, axis=-1, keepdims=True)
    base = rng.standard_normal(d)
    k = unit(base[None, None, :] + rho * rng.standard_normal((T, 1, d)))
    q = unit(rng.standard_normal((T, 1, d)))
    v = rng.standard_normal((T, 1, d))
    g = rng.uniform(-0.1, 0.0, (T, 1, d))
    beta = rng.uniform(0.5, 1.0, (T, 1))
    S0 = 0.02 * rng.standard_normal((1, 1, d, d))
    return [0, T], q, k, v, g, beta, S0


def _errs(cu, q, k, v, g, beta, S0, **kw):
    o_ref, s_ref = oracle.recurrence(cu, q, k, v, g, beta, state0=S0)
    o, s = CM.chunked_forward(cu, q, k, v, g, beta, state0=S0, **kw)
    return rel(o, o_ref), rel(s, s_ref)


@pytest.mark.parametrize("solve", ["blocked_tf32", "blocked_tf32_trunc", "blocked_bf16"])
@pytest.mark.parametrize("rho", [10.0, 0.5])
def test_blocked_solve_on_tensor_cores_keeps_the_budget(solve, rho):
    """The solve's products with tf32 operands (rounded, or truncated as chunk_prep's warp-level
    tensor-core products read fp32 data) or even bf16 ones, with wide accumulation, add next to
    nothing to the bf16 design's error, for independent keys and for strongly correlated ones."""
    x = _collinear_keys(rho)
    base = _errs(*x, bf16=True)
    got = _errs(*x, bf16=True, solve=solve)
    assert max(got) < 1.1 * max(base), (got, base)


def test_collinear_keys_amplify_every_rounding_site():
    """A design property, not a tolerance: when the keys share a direction (mean |k_i . k_j|
    about 0.96) the system I + A_kk is worse conditioned and the bf16 design's error grows by
    about 2.5x, spread over the sites (leaving any one of them wide removes ~10 %).  The
    workloads draw independent keys, where it is 4-5e-3."""
    x_ind, x_col = _collinear_keys(10.0), _collinear_keys(0.2)
    e_ind = max(_errs(*x_ind, bf16=True))
    e_col = max(_errs(*x_col, bf16=True))
    assert 1.5 * e_ind < e_col < 2e-2
    for site in ("T_b", "D", "qkv"):
        without = max(_errs(*x_col, bf16=[s for s in CM.SITES if s != site]))
        assert without > 0.75 * e_col, (site, without, e_col)


@pytest.mark.parametrize("sb,mistake,ok", [(16, None, True), (32, None, True),
                                           (32, "sb32_full_constant", False)])
def test_earlier_block_rows_survive_fp32_flush_at_saturated_gates(sb, mistake, ok):
    """With every gate on the bound (-5) the constant between the two 32-token blocks'
    references spans 32 gates, 2^-231, and flushes to zero in fp32, while the factors it
    multiplies reach 2^+-115: a row of block 1 against block 0 would lose entries worth
    e^-5 q.k.  Taken as its root (16 gates) applied twice it survives; with 16-token blocks
    the constant spans 16 gates and needs no split."""
    cu, q, k, v, g, beta, S0 = prepared([128], H=1, d=8, lb=-5.0, seed=9, gate_lo=-5.0)
    o_ref, s_ref = oracle.recurrence(cu, q, k, v, g, beta, state0=S0)
    o, s = CM.chunked_forward(cu, q, k, v, g, beta, state0=S0, sb=sb, flush=True, mistake=mistake)
    err = max(rel(o, o_ref), rel(s, s_ref))
    if ok:
        assert err < 1e-10
    else:
        assert err > 1e-3
