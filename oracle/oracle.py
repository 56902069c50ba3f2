"""Python face of the fp64 KDA oracle -- TEST INFRASTRUCTURE ONLY.

The oracle is a plain CPU implementation of the Kimi Delta Attention forward
pass (``kda_oracle.c``), written token by token from the AliceAI-Foundation KDA
write-up ("二、KDA 线性注意力": the per-token loop, the gate formula, the kernel-4
causal conv with SiLU, L2-normalised q/k) and the Ling-3.0-flash-VL config
table (kda_lower_bound = -5.0).  Only the tests, ``__graft_entry__.smoke()`` and
the bench's CPU-baseline leg may use it; the product library never does.

Every function here is pinned by the ``-m "not gpu"`` tests in
``tests/test_oracle_pins.py`` against checks that do not reuse its code:
a brute-force unrolled product of the recurrence, the delta-rule retrieval
identity, the lower-bound decay closed form, numpy/scipy convolution and
special functions, unit norms, prefill+decode == long prefill, and
varlen == separate sequences.

Inputs are fp64 numpy arrays (use ``workloads.as_f64`` on stored bf16/fp32
inputs so the oracle sees exactly the values the GPU reads).
"""

from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with plain -O2 (no fast-math) into oracle/liboracle.so."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _bind(lib):
    D = ctypes.POINTER(ctypes.c_double)
    I = ctypes.POINTER(ctypes.c_int64)
    i64, f64 = ctypes.c_int64, ctypes.c_double
    lib.kda_oracle_forward.argtypes = [i64, I, i64, i64, D, D, D, D, D, D, D, D, D, D,
                                       f64, f64, f64, ctypes.c_int, D, D, f64, D, D, D, ctypes.c_int]
    lib.kda_oracle_forward.restype = ctypes.c_int
    lib.kda_oracle_prologue.argtypes = [i64, I, i64, i64, D, D, D, D, D, D, D, D, D,
                                        f64, f64, ctypes.c_int, D, D, D, D, D, ctypes.c_int]
    lib.kda_oracle_prologue.restype = ctypes.c_int
    lib.kda_oracle_recurrence.argtypes = [i64, I, i64, i64, D, D, D, D, D, D, f64, D, D]
    lib.kda_oracle_recurrence.restype = ctypes.c_int
    return lib


def swap_library(path: Optional[str]):
    """Point this module at another build of the oracle (a planted-mistake copy in
    the mutation tests); ``None`` restores the real one.  Returns the previous handle."""
    global _lib
    prev = _lib
    _lib = None if path is None else _bind(ctypes.CDLL(path))
    return prev


def _load():
    global _lib
    if _lib is None:
        _lib = _bind(ctypes.CDLL(build()))
    return _lib


def _p(a: Optional[np.ndarray]):
    if a is None:
        return None
    assert a.dtype == np.float64 and a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _f(a) -> Optional[np.ndarray]:
    return None if a is None else np.ascontiguousarray(a, dtype=np.float64)


def _cu(cu_seqlens) -> np.ndarray:
    return np.ascontiguousarray(cu_seqlens, dtype=np.int64)


def forward(cu_seqlens, H: int, D: int, q, k, v, conv_w, alpha, b, A_log, dt_bias,
            state0=None, conv0=None, lower_bound: float = -5.0, eps: float = 1e-6,
            scale: float = 1.0, nthreads: int = 0, negative_eigenvalues: bool = False,
            out_gate=None, o_norm_weight=None, o_norm_eps: float = 1e-5
            ) -> Tuple[np.ndarray, np.ndarray, np.ndarray, int]:
    """Prefill over packed sequences.  Returns (o [T,H,D], final_state [N,H,D,D],
    final_conv_state [N,3,3*H*D], threads used).  ``negative_eigenvalues``: beta =
    2 sigmoid(b) (the kda_allow_negative_eigenvalues switch, section "二").  ``out_gate``
    [T,H,D] with ``o_norm_weight`` [D]: the output epilogue o <- rmsnorm(o) * w * sigmoid(gate)."""
    cu = _cu(cu_seqlens)
    N, T = len(cu) - 1, int(cu[-1])
    q, k, v, conv_w, alpha, b = map(_f, (q, k, v, conv_w, alpha, b))
    A_log, dt_bias, state0, conv0 = map(_f, (A_log, dt_bias, state0, conv0))
    out_gate, o_norm_weight = _f(out_gate), _f(o_norm_weight)
    if (out_gate is None) != (o_norm_weight is None):
        raise ValueError("out_gate and o_norm_weight go together")
    o = np.zeros((T, H, D))
    s1 = np.zeros((N, H, D, D))
    c1 = np.zeros((N, 3, 3 * H * D))
    used = _load().kda_oracle_forward(
        N, cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), H, D,
        _p(q), _p(k), _p(v), _p(conv_w), _p(alpha), _p(b), _p(A_log), _p(dt_bias),
        _p(state0), _p(conv0), lower_bound, eps, scale, int(negative_eigenvalues), _p(out_gate),
        _p(o_norm_weight), o_norm_eps, _p(o), _p(s1), _p(c1), nthreads)
    return o, s1, c1, used


def prologue(cu_seqlens, H: int, D: int, q, k, v, conv_w, alpha, b, A_log, dt_bias,
             conv0=None, lower_bound: float = -5.0, eps: float = 1e-6, nthreads: int = 0,
             negative_eigenvalues: bool = False):
    """Prepared per-token inputs: (qn, kn, vc [T,H,D], g [T,H,D], beta [T,H])."""
    cu = _cu(cu_seqlens)
    N, T = len(cu) - 1, int(cu[-1])
    q, k, v, conv_w, alpha, b = map(_f, (q, k, v, conv_w, alpha, b))
    A_log, dt_bias, conv0 = map(_f, (A_log, dt_bias, conv0))
    qn, kn, vc, g = (np.zeros((T, H, D)) for _ in range(4))
    beta = np.zeros((T, H))
    _load().kda_oracle_prologue(
        N, cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), H, D,
        _p(q), _p(k), _p(v), _p(conv_w), _p(alpha), _p(b), _p(A_log), _p(dt_bias),
        _p(conv0), lower_bound, eps, int(negative_eigenvalues), _p(qn), _p(kn), _p(vc), _p(g),
        _p(beta), nthreads)
    return qn, kn, vc, g, beta


def recurrence(cu_seqlens, q, k, v, g, beta, state0=None, scale: float = 1.0):
    """The token recurrence on prepared inputs q, k, v, g [T,H,D], beta [T,H]."""
    cu = _cu(cu_seqlens)
    q, k, v, g, beta, state0 = map(_f, (q, k, v, g, beta, state0))
    T, H, D = q.shape
    N = len(cu) - 1
    o = np.zeros((T, H, D))
    s1 = np.zeros((N, H, D, D))
    _load().kda_oracle_recurrence(
        N, cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), H, D,
        _p(q), _p(k), _p(v), _p(g), _p(beta), _p(state0), scale, _p(o), _p(s1))
    return o, s1


def decode_step(H: int, D: int, state, conv_state, q, k, v, alpha, b, conv_w, A_log,
                dt_bias, lower_bound: float = -5.0, eps: float = 1e-6, scale: float = 1.0,
                nthreads: int = 0, negative_eigenvalues: bool = False, out_gate=None,
                o_norm_weight=None, o_norm_eps: float = 1e-5):
    """One token per sequence (q, k, v [N, H*D], alpha [N,H,D], b [N,H]) on top of
    (state [N,H,D,D], conv_state [N,3,3*H*D]).  Returns (o [N,H,D], state', conv_state')."""
    N = np.asarray(state).shape[0]
    cu = np.arange(N + 1, dtype=np.int64)
    o, s1, c1, _ = forward(cu, H, D, q, k, v, conv_w, alpha, b, A_log, dt_bias,
                           state0=state, conv0=conv_state, lower_bound=lower_bound,
                           eps=eps, scale=scale, nthreads=nthreads,
                           negative_eigenvalues=negative_eigenvalues, out_gate=out_gate,
                           o_norm_weight=o_norm_weight, o_norm_eps=o_norm_eps)
    return o, s1, c1


def snapshots(cu_seqlens, H: int, D: int, every: int, cap: int, q, k, v, conv_w, alpha, b, A_log,
              dt_bias, state0=None, conv0=None, **kw):
    """State snapshots aligned to each sequence start: snap[n, j] (j < cap) is the final state
    of the first (j + 1) * every tokens of sequence n, by definition; slots past the sequence
    are NaN.  Composed from ``forward`` on those prefixes (no arithmetic of its own)."""
    cu = _cu(cu_seqlens)
    N = len(cu) - 1
    q, k, v, alpha, b = map(_f, (q, k, v, alpha, b))
    out = np.full((N, cap, H, D, D), np.nan)
    for n in range(N):
        a, z = int(cu[n]), int(cu[n + 1])
        for j in range(min(cap, (z - a) // every)):
            t = a + (j + 1) * every
            s0 = None if state0 is None else np.ascontiguousarray(np.asarray(state0)[n:n + 1])
            c0 = None if conv0 is None else np.ascontiguousarray(np.asarray(conv0)[n:n + 1])
            _, s1, _, _ = forward([0, t - a], H, D, q[a:t], k[a:t], v[a:t], conv_w, alpha[a:t],
                                  b[a:t], A_log, dt_bias, state0=s0, conv0=c0, **kw)
            out[n, j] = s1[0]
    return out


def pair_inputs(f64: dict, H: int, D: int, cu, n: int, h: int, t_end: Optional[int] = None):
    """Slice packed fp64 inputs down to one (sequence n, head h) pair (H = 1), optionally
    keeping only the first t_end tokens of the sequence."""
    a = int(cu[n])
    z = int(cu[n + 1]) if t_end is None else a + t_end
    sl = lambda x: np.ascontiguousarray(x[a:z, h * D:(h + 1) * D])
    out = dict(q=sl(f64["q"]), k=sl(f64["k"]), v=sl(f64["v"]),
               conv_w=np.ascontiguousarray(f64["conv_w"][:, h * D:(h + 1) * D, :]),
               alpha=np.ascontiguousarray(f64["alpha"][a:z, h:h + 1, :]),
               b=np.ascontiguousarray(f64["b"][a:z, h:h + 1]),
               A_log=np.ascontiguousarray(f64["A_log"][h:h + 1]),
               dt_bias=np.ascontiguousarray(f64["dt_bias"][h:h + 1]))
    S0 = f64.get("S0")
    out["state0"] = None if S0 is None else np.ascontiguousarray(S0[n:n + 1, h:h + 1])
    return out, z - a


def forward_pair(f64: dict, H: int, D: int, cu, n: int, h: int, t_end: Optional[int] = None,
                 lower_bound: float = -5.0, eps: float = 1e-6, scale: float = 1.0):
    """Oracle prefill of one (sequence, head) pair: (o [L, D], final_state [D, D])."""
    P, L = pair_inputs(f64, H, D, cu, n, h, t_end)
    o, s1, _, _ = forward([0, L], 1, D, P["q"], P["k"], P["v"], P["conv_w"], P["alpha"], P["b"],
                          P["A_log"], P["dt_bias"], state0=P["state0"], lower_bound=lower_bound,
                          eps=eps, scale=scale, nthreads=1)
    return o[:, 0], s1[0, 0]
