"""Seeded synthetic inputs for the Kimi Delta Attention (KDA) forward pass.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic, so the CPU oracle and the CUDA path can both consume what
it produces without sharing any computation.

Workloads (value distributions as the KDA write-ups state them for the
AliceAI-Foundation KDA layer, "二、KDA 线性注意力" section, and the Ling-3.0-flash-VL
config table):

* ``tiny_fp32``   fp32 I/O, B=1, T=256, H=2, d=64, zero initial state
* ``prefill_4x8k`` bf16 I/O, B=4, T=8192, H=32, d=128, S0 ~ N(0, 0.02)
* ``long_256k``   bf16 I/O, B=1, T=262144, H=32, d=128, zero S0, alpha ~ N(-2, 1)
* ``varlen_32``   bf16 I/O, 32 packed sequences, lengths round(lognormal(7.5, 1))
                  clipped to [16, 32768], per-sequence S0 ~ N(0, 0.02)
* ``decode_256``  256 sequences, H=32, d=128: a T=1024 prefill seeds the state,
                  then 64 single-token steps

Common distributions: q, k, v ~ N(0, 1) (pre-conv), conv_w ~ N(0, 0.5) with
shape [3, H*d, 4] (q | k | v channel blocks), alpha ~ N(0, 1), dt_bias ~ U(-1, 1)
per (head, dim), A_log = ln U(1, 16) per head, b ~ N(0, 1).  N(mu, s) takes s as
the standard deviation.  Workload i is drawn with seed i.

Token-indexed tensors are drawn in blocks of ``BLOCK`` tokens, each block from
its own generator keyed by (seed, tensor, block).  Any token range can then be
regenerated on its own, which lets a test rebuild a slice of a 262144-token
input for the oracle without holding the whole thing.

bf16 values are produced by round-to-nearest-even from fp32 draws and are
returned as raw uint16 bit patterns; ``as_f64`` widens them exactly.
"""

from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional

import numpy as np

BLOCK = 4096

_TAGS = {"q": 1, "k": 2, "v": 3, "alpha": 4, "b": 5, "conv_w": 6, "A_log": 7,
         "dt_bias": 8, "S0": 9, "lens": 10, "step": 11, "gate": 12, "o_norm_w": 13}


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round finite fp32 values to bf16 (nearest, ties to even); return the uint16 bits.
    In uint32: the largest finite pattern plus 0x8000 stays below 2**32."""
    u = np.array(x, dtype=np.float32, copy=True).view(np.uint32)
    lsb = u >> 16
    lsb &= 1
    lsb += 0x7FFF
    u += lsb
    u >>= 16
    return u.astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32."""
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def as_f64(arr: Optional[np.ndarray]) -> Optional[np.ndarray]:
    """Exact fp64 view of a stored input (bf16 bits or fp32 values)."""
    if arr is None:
        return None
    if arr.dtype == np.uint16:
        return bf16_to_f32(arr).astype(np.float64)
    return np.asarray(arr, dtype=np.float64)


@dataclasses.dataclass
class Spec:
    """Shape and distribution parameters of one synthetic workload."""
    name: str
    io_dtype: str              # "bf16" or "fp32"
    seq_lens: List[int]        # one entry per sequence
    H: int
    d: int
    seed: int
    alpha_mu: float = 0.0
    s0_std: float = 0.0        # 0 => zero initial state
    varlen: bool = False       # pass cu_seqlens (packed) rather than dense [B, T]
    lower_bound: float = -5.0
    eps: float = 1e-6
    scale: float = 1.0

    @property
    def num_seqs(self) -> int:
        return len(self.seq_lens)

    @property
    def total_tokens(self) -> int:
        return int(sum(self.seq_lens))

    @property
    def cu_seqlens(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.seq_lens)]).astype(np.int32)


def varlen_lengths(seed: int, n: int = 32, mu: float = 7.5, sigma: float = 1.0,
                   lo: int = 16, hi: int = 32768) -> List[int]:
    rng = np.random.default_rng([seed, _TAGS["lens"]])
    lens = np.clip(np.round(rng.lognormal(mu, sigma, size=n)), lo, hi).astype(np.int64)
    return [int(x) for x in lens]


def spec(name: str) -> Spec:
    """The named workloads (see module docstring)."""
    if name == "tiny_fp32":
        return Spec(name, "fp32", [256], H=2, d=64, seed=0)
    if name == "prefill_4x8k":
        return Spec(name, "bf16", [8192] * 4, H=32, d=128, seed=1, s0_std=0.02)
    if name == "long_256k":
        return Spec(name, "bf16", [262144], H=32, d=128, seed=2, alpha_mu=-2.0)
    if name == "varlen_32":
        return Spec(name, "bf16", varlen_lengths(3), H=32, d=128, seed=3, s0_std=0.02,
                    varlen=True)
    if name == "decode_256":
        return Spec(name, "bf16", [1024] * 256, H=32, d=128, seed=4)
    raise KeyError(name)


WORKLOADS = ["tiny_fp32", "prefill_4x8k", "long_256k", "varlen_32", "decode_256"]


def _store(x: np.ndarray, io_dtype: str) -> np.ndarray:
    return bf16_bits(x) if io_dtype == "bf16" else np.ascontiguousarray(x, dtype=np.float32)


def _token_tensor(s: Spec, tag: str, t0: int, t1: int, width: int, mu: float = 0.0,
                  std: float = 1.0, store: Optional[str] = None) -> np.ndarray:
    """Rows [t0, t1) of a [total_tokens, width] N(mu, std) tensor, drawn blockwise (blocks in
    parallel threads; each block has its own generator, so the result does not depend on the
    thread count).  ``store`` = "bf16" returns bf16 bits, else fp32 values."""
    import concurrent.futures
    out = np.empty((t1 - t0, width), dtype=np.uint16 if store == "bf16" else np.float32)
    if t1 <= t0:
        return out
    b0, b1 = t0 // BLOCK, (t1 - 1) // BLOCK

    def one(blk):
        rng = np.random.default_rng([s.seed, _TAGS[tag], blk])
        lo, hi = blk * BLOCK, min((blk + 1) * BLOCK, s.total_tokens)
        block = rng.standard_normal((hi - lo, width), dtype=np.float32)
        if std != 1.0:
            block *= np.float32(std)
        if mu != 0.0:
            block += np.float32(mu)
        a, z = max(lo, t0), min(hi, t1)
        part = block[a - lo:z - lo]
        out[a - t0:z - t0] = bf16_bits(part) if store == "bf16" else part

    nblk = b1 - b0 + 1
    if nblk == 1:
        one(b0)
    else:
        import os
        with concurrent.futures.ThreadPoolExecutor(max_workers=min(nblk, os.cpu_count() or 1)) as ex:
            list(ex.map(one, range(b0, b1 + 1)))
    return out


def make_params(s: Spec) -> Dict[str, np.ndarray]:
    """Per-layer parameters: conv_w [3, H*d, 4] (io dtype), A_log [H], dt_bias [H, d] (fp32)."""
    HD = s.H * s.d
    rng = np.random.default_rng([s.seed, _TAGS["conv_w"]])
    conv_w = rng.standard_normal((3, HD, 4), dtype=np.float32) * np.float32(0.5)
    rng = np.random.default_rng([s.seed, _TAGS["A_log"]])
    A_log = np.log(rng.uniform(1.0, 16.0, size=s.H)).astype(np.float32)
    rng = np.random.default_rng([s.seed, _TAGS["dt_bias"]])
    dt_bias = rng.uniform(-1.0, 1.0, size=(s.H, s.d)).astype(np.float32)
    return {"conv_w": _store(conv_w, s.io_dtype), "A_log": A_log, "dt_bias": dt_bias}


def make_tokens(s: Spec, t0: int = 0, t1: Optional[int] = None) -> Dict[str, np.ndarray]:
    """Token-indexed inputs for packed rows [t0, t1): q, k, v [T, H*d], alpha [T, H, d], b [T, H]."""
    t1 = s.total_tokens if t1 is None else t1
    HD = s.H * s.d
    st = s.io_dtype
    out = {}
    for tag in ("q", "k", "v"):
        out[tag] = _token_tensor(s, tag, t0, t1, HD, store=st)
    out["alpha"] = _token_tensor(s, "alpha", t0, t1, HD, mu=s.alpha_mu,
                                 store=st).reshape(t1 - t0, s.H, s.d)
    out["b"] = _token_tensor(s, "b", t0, t1, s.H, store=st)
    return out


def make_initial_state(s: Spec) -> Optional[np.ndarray]:
    """fp32 [N, H, d, d] initial states, or None when the workload starts from zero."""
    if s.s0_std == 0.0:
        return None
    rng = np.random.default_rng([s.seed, _TAGS["S0"]])
    return (rng.standard_normal((s.num_seqs, s.H, s.d, s.d), dtype=np.float32)
            * np.float32(s.s0_std))


def make_inputs(s: Spec) -> Dict[str, np.ndarray]:
    """Everything a prefill over the whole workload consumes."""
    out = make_params(s)
    out.update(make_tokens(s))
    out["S0"] = make_initial_state(s)
    out["cu_seqlens"] = s.cu_seqlens
    return out


def make_decode_step(s: Spec, step: int) -> Dict[str, np.ndarray]:
    """One fresh token per sequence for decode step ``step``: q, k, v [N, H*d], alpha [N, H, d], b [N, H]."""
    N, HD = s.num_seqs, s.H * s.d
    rng = np.random.default_rng([s.seed, _TAGS["step"], step])
    q = rng.standard_normal((N, HD), dtype=np.float32)
    k = rng.standard_normal((N, HD), dtype=np.float32)
    v = rng.standard_normal((N, HD), dtype=np.float32)
    alpha = rng.standard_normal((N, s.H, s.d), dtype=np.float32)
    if s.alpha_mu != 0.0:
        alpha += np.float32(s.alpha_mu)
    b = rng.standard_normal((N, s.H), dtype=np.float32)
    return {k_: _store(v_, s.io_dtype) for k_, v_ in
            (("q", q), ("k", k), ("v", v), ("alpha", alpha), ("b", b))}


def make_output_gate(s: Spec, rows: int, tag: int = 0) -> Dict[str, np.ndarray]:
    """Inputs of the output epilogue: gate ~ N(0,1) [rows, H, d] in the io dtype (rows =
    the workload's tokens, or its sequences for a decode step; ``tag`` tells steps apart)
    and the o_norm weight ~ U(0.5, 1.5) [d] fp32."""
    rng = np.random.default_rng([s.seed, _TAGS["gate"], tag])
    gate = rng.standard_normal((rows, s.H, s.d), dtype=np.float32)
    w = np.random.default_rng([s.seed, _TAGS["o_norm_w"]]).uniform(0.5, 1.5, s.d).astype(np.float32)
    return {"gate": _store(gate, s.io_dtype), "o_norm_weight": w}


def small(name: str, seq_lens: List[int], H: int, d: int, io_dtype: str = "bf16",
          seed: int = 100, s0_std: float = 0.0, alpha_mu: float = 0.0,
          varlen: bool = False) -> Spec:
    """A reduced workload with the same distributions, for parity tests the oracle finishes quickly."""
    return Spec(name, io_dtype, list(seq_lens), H=H, d=d, seed=seed, s0_std=s0_std,
                alpha_mu=alpha_mu, varlen=varlen)


def to_device(arr: Optional[np.ndarray], device="cuda"):
    """Upload a stored input (bf16 bits -> torch.bfloat16, fp32 -> float32, int32 as is)."""
    import torch
    if arr is None:
        return None
    if arr.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(arr).view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(arr)).to(device)


def from_device(t) -> np.ndarray:
    """fp64 copy of a device tensor (bf16/fp32)."""
    import torch
    return t.detach().to(torch.float64).cpu().numpy()
