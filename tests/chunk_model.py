"""A plain fp64 numpy model of the chunked form the tensor-core kernels compute.

Test infrastructure, not the oracle: the oracle runs the per-token loop of the
AliceAI-Foundation KDA write-up ("二、KDA 线性注意力"); this model re-associates that loop
over 64-token chunks the way the prefill kernels do, so that a CPU test can hold the
factorisation itself against the oracle, independently of any GPU.

Per chunk (length <= 64, padded with zero tokens and zero gates), per key channel c:

  Gamma_t      = sum_{s <= t} g_s                         (cumulative gate, kept in base 2)
  m_I          = Gamma after token 16 I + 7                (reference of 16-token block I)
  L_t          = x_t 2^{Gamma_t - m_I(t)}                  (x = q or k)
  R^(I)_s      = k_s 2^{m_I - Gamma_s}, built for s in an earlier block J as
                 (k_s 2^{m_J - Gamma_s}) 2^{m_I - m_J}
  A_qk[t, s]   = L_q,t . R^(I(t))_s          (s <= t)
  A_kk[t, s]   = beta_t L_k,t . R^(I(t))_s   (s < t)
  T            = (I + A_kk)^{-1}
  W            = T diag(beta) (K 2^Gamma),   U = T diag(beta) V

and across chunks, with S the [d_k, d_v] state:

  D = U - W S;   O = (Q 2^Gamma) S + A_qk D;   S <- diag(2^{Gamma_C}) S + (K 2^{Gamma_C - Gamma})^T D.
"""

from __future__ import annotations

import numpy as np

from gated_delta_rule_70_b200 import workloads as W

CH = 64   # chunk length
SB = 16   # sub-block length
LOG2E = 1.4426950408889634


def block_refs(G2: np.ndarray, sb: int = SB) -> np.ndarray:
    """References m_I [64 / sb, d_k] of a padded 64-token chunk's base-2 cumulative gate
    G2 [64, d_k]: Gamma after the middle token of each sb-token block."""
    return np.stack([G2[sb * I + sb // 2 - 1] for I in range(CH // sb)])


# where the kernels hold bf16 values (each a separate rounding site of the emulation)
SITES = ("qkv", "LR", "A_qk", "T_b", "W", "U", "Qt", "Kh", "S_copy", "D", "o")


def _bf16(x):
    """Round to bf16 (nearest even), back in fp64."""
    return W.bf16_to_f32(W.bf16_bits(np.asarray(x, dtype=np.float32))).astype(np.float64)


def _tf32(x):
    """Round to tf32 (10 explicit mantissa bits, nearest with ties away from zero, as the
    conversion to tf32 does), back in fp64."""
    u = np.asarray(x, dtype=np.float32).copy().view(np.uint32)
    u = (u + np.uint32(0x1000)) & np.uint32(0xFFFFE000)
    return u.view(np.float32).astype(np.float64)


def _tf32_trunc(x):
    """tf32 as the warp-level tensor-core path reads an fp32 operand: the low 13 mantissa bits
    dropped (toward zero), back in fp64."""
    u = np.asarray(x, dtype=np.float32).copy().view(np.uint32) & np.uint32(0xFFFFE000)
    return u.view(np.float32).astype(np.float64)


def _flush(x):
    """fp32's flush to zero below its normal range (2^-126), which the special-function
    exponential applies to its results."""
    x = np.asarray(x, dtype=np.float64)
    return np.where(np.abs(x) < 2.0 ** -126, 0.0, x)


def blocked_inverse(A, tf32: bool = False, bf16: bool = False, tf32_trunc: bool = False):
    """(I + A)^{-1} for a strictly lower-triangular 64 x 64 A, by blocks: the 16 x 16 diagonal
    blocks' inverses D_i by substitution, then T_ij = -D_i (A_ij D_j) for the blocks next to the
    diagonal, then the 32 x 32 halves T_21 = -T_2 (A_21 T_1).  Every product there is a small
    dense matrix product (tensor-core shaped); ``tf32`` (or ``bf16``) rounds their operands to
    that type and keeps the accumulation wide."""
    r = _tf32 if tf32 else (_bf16 if bf16 else (_tf32_trunc if tf32_trunc else (lambda x: x)))
    n = A.shape[0]
    T = np.zeros_like(A)
    for i in range(0, n, 16):
        T[i:i + 16, i:i + 16] = np.linalg.inv(np.eye(16) + A[i:i + 16, i:i + 16])
    for j in (0, 32):
        i = j + 16
        X = r(A[i:i + 16, j:j + 16]) @ r(T[j:j + 16, j:j + 16])
        T[i:i + 16, j:j + 16] = -(r(T[i:i + 16, i:i + 16]) @ r(X))
    X = r(A[32:, :32]) @ r(T[:32, :32])
    T[32:, :32] = -(r(T[32:, 32:]) @ r(X))
    return T


def _rounder(bf16):
    """bf16: False (no rounding), True (every site) or a collection of SITES names ->
    site -> rounding function."""
    on = set(SITES) if bf16 is True else set(bf16 or ())
    assert on <= set(SITES), on - set(SITES)
    return lambda site: _bf16 if site in on else (lambda x: x)


def chunk_factors(q, k, v, g, beta, mistake=None, sb: int = SB, bf16=False, solve: str = "direct",
                  flush: bool = False):
    """One padded chunk (q, k, v [64, d], g [64, d_k] natural-log gates, beta [64]) ->
    (A_qk, W, U, Q 2^Gamma, K 2^{Gamma_C - Gamma}, 2^{Gamma_C}, the log2 exponents of every
    L and R factor taken).  ``mistake`` plants one plausible error, for the test that shows
    the comparison with the oracle catches it.  ``sb`` is the sub-block length (32 in the
    kernels at gate bounds >= -5.02, else 16).  ``bf16`` rounds where the kernels hold bf16: the MMA operands L and R, T diag(beta),
    and the record's A_qk, W, U, Q 2^Gamma and K 2^{Gamma_C - Gamma}; A_kk, T, the gates and
    2^{Gamma_C} stay wide (fp32 in the kernels, fp64 here).  A collection of SITES names
    rounds at those sites only.  ``solve``: "direct" (a plain inverse), "blocked",
    "blocked_tf32", "blocked_tf32_trunc" (the kernels' form) or "blocked_bf16"
    (``blocked_inverse``).  ``flush`` applies fp32's flush
    to zero below 2^-126 to the exponentials and the R rows of earlier blocks, as the
    kernels' arithmetic does; with 32-token blocks the earlier block's constant is then
    taken as its root applied twice (the constant itself spans 32 gates, the root 16), as
    the kernel does, unless ``mistake == "sb32_full_constant"``."""
    rb = _rounder(bf16)
    G2 = np.cumsum(g * LOG2E, axis=0)
    m = block_refs(G2, sb)
    blk = np.arange(CH) // sb
    L_exp = G2 - m[blk]                       # exponent of every L factor
    Lq = rb("LR")(q * np.exp2(L_exp))
    Lk = rb("LR")(k * np.exp2(L_exp))
    Rd_exp = m[blk] - G2                      # the diagonal-block R factor
    Rd = k * np.exp2(Rd_exp)
    exps = [L_exp, Rd_exp]
    A_qk = np.zeros((CH, CH))
    A_kk = np.zeros((CH, CH))
    for I in range(CH // sb):
        rows = slice(sb * I, sb * (I + 1))
        R = np.zeros((CH, k.shape[1]))
        for J in range(I + 1):
            cols = slice(sb * J, sb * (J + 1))
            c_exp = m[I] - m[J]               # <= 0: the later block's constant
            if mistake == "no_block_constant":
                c_exp = np.zeros_like(c_exp)
            exps.append(np.broadcast_to(c_exp, (1, k.shape[1])))
            if not flush:
                R[cols] = rb("LR")(Rd[cols] * np.exp2(c_exp))
            elif sb == 32 and J < I and mistake != "sb32_full_constant":
                ch = _flush(np.exp2(c_exp / 2))
                R[cols] = rb("LR")(_flush(_flush(_flush(Rd[cols]) * ch) * ch))
            else:
                R[cols] = rb("LR")(_flush(_flush(Rd[cols]) * _flush(np.exp2(c_exp))))
        A_qk[rows] = Lq[rows] @ R.T
        A_kk[rows] = beta[rows, None] * (Lk[rows] @ R.T)
    t = np.arange(CH)
    A_qk *= t[:, None] >= t[None, :]
    A_kk *= (t[:, None] >= t[None, :]) if mistake == "kk_diagonal" else (t[:, None] > t[None, :])
    A_qk = rb("A_qk")(A_qk)
    if solve == "direct":
        T = np.linalg.inv(np.eye(CH) + A_kk)
    else:
        T = blocked_inverse(A_kk, tf32=solve == "blocked_tf32", bf16=solve == "blocked_bf16",
                            tf32_trunc=solve == "blocked_tf32_trunc")
    Kt = rb("LR")(k * np.exp2(G2))
    if mistake == "beta_after_T":
        W = beta[:, None] * (T @ Kt)
        U = beta[:, None] * (T @ v)
    else:
        Tb = rb("T_b")(T * beta[None, :])            # T diag(beta)
        W = rb("W")(Tb @ Kt)
        U = rb("U")(Tb @ v)
    Qt = rb("Qt")(q * np.exp2(G2))
    Kh = rb("Kh")(k * np.exp2(G2[-1] - G2))
    return A_qk, W, U, Qt, Kh, np.exp2(G2[-1]), exps


def chunked_forward(cu_seqlens, q, k, v, g, beta, state0=None, mistake=None, sb: int = SB,
                    bf16=False, solve: str = "direct", flush: bool = False):
    """The chunked form over packed prepared inputs (q, k, v, g [T, H, d], beta [T, H]) ->
    (o [T, H, d], final state [N, H, d, d]), the same contract as the oracle's recurrence.
    ``bf16`` also rounds q, k, v, the state's copy that the MMAs read, D (after U is added)
    and o, as the kernels do; the state itself stays wide."""
    rb = _rounder(bf16)
    q, k, v = rb("qkv")(q), rb("qkv")(k), rb("qkv")(v)
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    T, H, d = q.shape
    N = len(cu) - 1
    o = np.zeros((T, H, d))
    s1 = np.zeros((N, H, d, d))
    for n in range(N):
        a, z = int(cu[n]), int(cu[n + 1])
        for h in range(H):
            S = np.zeros((d, d)) if state0 is None else np.array(state0[n, h], dtype=np.float64)
            for c0 in range(a, z, CH):
                c1 = min(c0 + CH, z)
                L = c1 - c0
                pad = lambda x: np.concatenate([x, np.zeros((CH - L,) + x.shape[1:])])
                A_qk, W, U, Qt, Kh, eGC, _ = chunk_factors(
                    pad(q[c0:c1, h]), pad(k[c0:c1, h]), pad(v[c0:c1, h]), pad(g[c0:c1, h]),
                    pad(beta[c0:c1, h]), mistake, sb, bf16, solve, flush)
                Sb = rb("S_copy")(S)
                D = rb("D")(U - W @ Sb)
                O = Qt @ Sb + A_qk @ D
                o[c0:c1, h] = rb("o")(O[:L])
                S = eGC[:, None] * S + Kh.T @ D
            s1[n, h] = S
    return o, s1
