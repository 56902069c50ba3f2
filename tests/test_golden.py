"""The oracle against stored fixtures (tests/golden/): a worked example of the per-token loop and
gate / beta closed forms computed by hand, and a regression record of the oracle's own outputs.

CPU only.  Each fixture file states its source passage in its header.
"""

import importlib.util
import math
import os

import numpy as np
import pytest

from oracle import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as fh:
        for line in fh:
            line = line.split("#", 1)[0].split()
            if line:
                yield line[0], line[1:]


def test_hand_worked_recurrence():
    """Three tokens of the loop, d = 2, dyadic values: o after each token and the final state."""
    d, S0, toks, want_o, want_S = None, None, [], [], None
    for kind, x in _rows("hand_recurrence.txt"):
        if kind == "d":
            d = int(x[0])
        elif kind == "S0":
            S0 = np.array(x, dtype=np.float64).reshape(1, 1, d, d)
        elif kind == "token":
            toks.append(np.array(x, dtype=np.float64))
        elif kind == "expect_o":
            want_o.append(np.array(x, dtype=np.float64))
        elif kind == "expect_S":
            want_S = np.array(x, dtype=np.float64).reshape(d, d)
    T = len(toks)
    tok = np.stack(toks)                     # decay(d) k(d) v(d) beta q(d)
    g = np.log(tok[:, 0:d]).reshape(T, 1, d)
    k = tok[:, d:2 * d].reshape(T, 1, d)
    v = tok[:, 2 * d:3 * d].reshape(T, 1, d)
    beta = tok[:, 3 * d].reshape(T, 1)
    q = tok[:, 3 * d + 1:4 * d + 1].reshape(T, 1, d)
    o, S = oracle.recurrence([0, T], q, k, v, g, beta, state0=S0)
    np.testing.assert_allclose(o[:, 0], np.stack(want_o), rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(S[0, 0], want_S, rtol=1e-14, atol=1e-14)


def test_gate_and_beta_closed_forms():
    gates = [list(map(float, x)) for kind, x in _rows("gate_closed_forms.txt") if kind == "gate"]
    betas = [list(map(float, x)) for kind, x in _rows("gate_closed_forms.txt") if kind == "beta"]
    assert gates and betas and len({r[3] for r in gates}) == 1
    H, D = len(gates), 1
    z = lambda *shape: np.zeros(shape)
    A_log = np.array([r[0] for r in gates])
    alpha = np.array([r[1] for r in gates]).reshape(1, H, D)
    dt_bias = np.array([r[2] for r in gates]).reshape(H, D)
    _, _, _, g, _ = oracle.prologue([0, 1], H, D, z(1, H * D), z(1, H * D), z(1, H * D),
                                    z(3, H * D, 4), alpha, z(1, H), A_log, dt_bias,
                                    lower_bound=gates[0][3])
    for h, r in enumerate(gates):
        assert math.isclose(g[0, h, 0], r[4], rel_tol=1e-14, abs_tol=1e-30), (r, g[0, h, 0])
    Hb = len(betas)
    b = np.array([r[0] for r in betas]).reshape(1, Hb)
    _, _, _, _, beta = oracle.prologue([0, 1], Hb, D, z(1, Hb * D), z(1, Hb * D), z(1, Hb * D),
                                       z(3, Hb * D, 4), z(1, Hb, D), b, z(Hb), z(Hb, D))
    for h, r in enumerate(betas):
        assert math.isclose(beta[0, h], r[1], rel_tol=1e-15), (r, beta[0, h])


def _fixture_module():
    spec = importlib.util.spec_from_file_location(
        "make_oracle_fixture", os.path.join(GOLDEN, "make_oracle_fixture.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_oracle_matches_its_stored_record():
    """An unintended change to the oracle's arithmetic moves these values; an intended one
    regenerates the file (tests/golden/make_oracle_fixture.py) with its justification."""
    stored = {(kind, int(x[0]), int(x[1]), int(x[2])): float(x[3])
              for kind, x in _rows("oracle_tiny_fp32.txt")}
    now = {(kind, a, b_, c): val for kind, a, b_, c, val in _fixture_module().compute()}
    assert stored.keys() == now.keys()
    for key, val in stored.items():
        assert math.isclose(now[key], val, rel_tol=1e-12, abs_tol=1e-15), (key, now[key], val)


@pytest.mark.parametrize("name", ["hand_recurrence.txt", "gate_closed_forms.txt",
                                  "oracle_tiny_fp32.txt"])
def test_every_fixture_states_its_source(name):
    with open(os.path.join(GOLDEN, name)) as fh:
        head = "".join(fh.readline() for _ in range(8))
    assert "#" in head and ("section" in head or "oracle" in head)
