"""kda_prefill_noalloc: the prefill for callers that cannot allocate device memory.

Some embedders cannot give the library a workspace (they own all device memory
and lend only inputs and outputs, or run where cudaMalloc is not allowed).
kda_prefill_noalloc keeps the prologue's intermediates in a fixed library-owned
device array instead.  This test calls it through the C ABI twice in a row
(different inputs and dtypes, so the second call sees the first call's leftover
scratch contents) and checks each result against kda_prefill on the same
inputs and against the fp64 oracle, with the parity tolerance the other tests
use (max relative L2 per (sequence, head) 1e-2 for bf16, 1e-4 in fp32).  It also
checks the size limit at its edge: on the tensor-core path (bf16, d = 128) the
scratch holds one 74,752-byte record per 64-token chunk and head, so at 32
heads 896 tokens (14 chunks) fit in the 32 MiB and 960 tokens (15 chunks) are
refused.

This file is named so that pytest collects it last.
"""

import ctypes

import numpy as np
import pytest
import torch

from gated_delta_rule_70_b200 import kda
from gated_delta_rule_70_b200 import workloads as W
from oracle import oracle

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 32 << 20   # KDA_NOALLOC_SCRATCH_BYTES in include/kda.h


def _lib():
    lib = kda.load_library()
    P = ctypes.c_void_p
    lib.kda_prefill_noalloc.argtypes = [ctypes.POINTER(kda.Shape)] + [P] * 14 + [P]
    lib.kda_prefill_noalloc.restype = ctypes.c_int
    return lib


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc(s, d):
    shape = kda.make_shape(s.num_seqs, s.total_tokens if s.varlen else s.seq_lens[0], s.H, s.d,
                           d["q"].dtype)
    T, H, D, N = s.total_tokens, s.H, s.d, s.num_seqs
    o = torch.full((T, H, D), float("nan"), dtype=d["q"].dtype, device="cuda")
    fs = torch.full((N, H, D, D), float("nan"), dtype=torch.float32, device="cuda")
    fc = torch.empty((N, 3, 3 * H * D), dtype=d["q"].dtype, device="cuda")
    st = _lib().kda_prefill_noalloc(
        ctypes.byref(shape), _p(d["q"]), _p(d["k"]), _p(d["v"]), _p(d["conv_w"]), _p(d["alpha"]),
        _p(d["b"]), _p(d["A_log"]), _p(d["dt_bias"]), _p(d.get("S0")), None,
        _p(d["cu_seqlens"]) if s.varlen else None, _p(o), _p(fs), _p(fc),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st, o, fs, fc


def _rel_max(a, b, cu, H):
    a, b = a.double().cpu().numpy(), b.double().cpu().numpy()
    worst = 0.0
    for n in range(len(cu) - 1):
        lo, hi = int(cu[n]), int(cu[n + 1])
        for h in range(H):
            den = np.linalg.norm(b[lo:hi, h])
            if hi > lo:
                worst = max(worst, np.linalg.norm(a[lo:hi, h] - b[lo:hi, h]) / max(den, 1e-30))
    return worst


@pytest.mark.parametrize("first", ["bf16", "fp32"])
def test_noalloc_matches_prefill_twice_in_a_row(first):
    specs = [W.small("na1", [150, 70], H=2, d=128, io_dtype="bf16", seed=61, s0_std=0.02, varlen=True),
             W.small("na2", [96, 96, 96], H=3, d=64, io_dtype="fp32", seed=62, s0_std=0.02)]
    if first == "fp32":
        specs = specs[::-1]
    for s in specs:
        inp = W.make_inputs(s)
        d = {k: W.to_device(v) for k, v in inp.items()}
        st, o, fs, fc = _noalloc(s, d)
        assert st == kda.KDA_OK, kda.status_string(st)
        o_ref, fs_ref, fc_ref = kda.prefill(d["q"], d["k"], d["v"], d["conv_w"], d["alpha"], d["b"],
                                            d["A_log"], d["dt_bias"], initial_state=d["S0"],
                                            cu_seqlens=d["cu_seqlens"] if s.varlen else None,
                                            num_seqs=s.num_seqs, check=True)
        torch.cuda.synchronize()
        tol = 1e-2 if s.io_dtype == "bf16" else 1e-4
        cu = s.cu_seqlens
        assert _rel_max(o, o_ref, cu, s.H) <= tol
        for n in range(s.num_seqs):
            for h in range(s.H):
                a, b = fs[n, h].double().cpu().numpy(), fs_ref[n, h].double().cpu().numpy()
                assert np.linalg.norm(a - b) / np.linalg.norm(b) <= tol
        assert torch.equal(fc, fc_ref)
        # and against the oracle itself
        f = {k: W.as_f64(v) for k, v in inp.items() if k != "cu_seqlens"}
        o_or, s_or, _, _ = oracle.forward(cu, s.H, s.d, f["q"], f["k"], f["v"], f["conv_w"],
                                          f["alpha"], f["b"], f["A_log"], f["dt_bias"],
                                          state0=f["S0"])
        assert _rel_max(o, torch.from_numpy(o_or), cu, s.H) <= tol
        fs64 = fs.double().cpu().numpy()
        for n in range(s.num_seqs):
            for h in range(s.H):
                assert np.linalg.norm(fs64[n, h] - s_or[n, h]) / np.linalg.norm(s_or[n, h]) <= tol


def test_noalloc_size_limit_at_its_edge():
    # 960 tokens x 32 heads: 15 chunk records per head, beyond the scratch: refused before any
    # launch (the pointers are never read)
    shape = kda.make_shape(1, 960, 32, 128, torch.bfloat16)
    x = torch.zeros(256, dtype=torch.uint8, device="cuda")
    P = _p(x)
    st = _lib().kda_prefill_noalloc(ctypes.byref(shape), P, P, P, P, P, P, P, P, None, None, None,
                                    P, P, None, None)
    assert st == kda.KDA_ERR_WORKSPACE
    # 896 tokens x 32 heads: 14 records per head, fits; the result matches kda_prefill
    s = W.small("na_edge", [896], H=32, d=128, io_dtype="bf16", seed=63, s0_std=0.02)
    inp = W.make_inputs(s)
    d = {k: W.to_device(v) for k, v in inp.items()}
    st, o, fs, _ = _noalloc(s, d)
    assert st == kda.KDA_OK, kda.status_string(st)
    o_ref, fs_ref, _ = kda.prefill(d["q"], d["k"], d["v"], d["conv_w"], d["alpha"], d["b"],
                                   d["A_log"], d["dt_bias"], initial_state=d["S0"], num_seqs=1,
                                   check=True)
    torch.cuda.synchronize()
    assert _rel_max(o, o_ref, s.cu_seqlens, s.H) <= 1e-2
    a, b = fs.double().cpu().numpy(), fs_ref.double().cpu().numpy()
    for h in range(s.H):
        assert np.linalg.norm(a[0, h] - b[0, h]) / np.linalg.norm(b[0, h]) <= 1e-2
