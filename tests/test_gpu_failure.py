"""Failure detection without a GPU fault.

A call made with KDA_FLAG_TEST_EXPIRE_WAITS has every bounded device-side wait
give up at its first check (no data race is needed to make that happen: the
limit is zero polls).  Each kernel family must then stop issuing work, wait out
the copies and tensor-core operations it had already started (with the normal
limit), free its tensor memory and return, and the call's status word must
report the timeout -- chunk preparation and the state pass each with their own
bit.  Nothing faults and the context stays usable: the next ordinary call on
the same device, from the same inputs, matches the fp64 oracle.

Tolerance: max relative L2 per (sequence, head) <= 1e-2 (bf16 I/O).
"""

import numpy as np
import pytest
import torch

from gated_delta_rule_70_b200 import kda
from gated_delta_rule_70_b200 import workloads as W
from oracle import oracle

pytestmark = pytest.mark.gpu
TOL = 1e-2
EXPIRE = kda.KDA_FLAG_TEST_EXPIRE_WAITS


def rel(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def _prefill(s, d, ws, flags=0, segments=True):
    return kda.prefill(d["q"], d["k"], d["v"], d["conv_w"], d["alpha"], d["b"], d["A_log"],
                       d["dt_bias"], initial_state=d["S0"],
                       cu_seqlens=d["cu_seqlens"] if s.varlen else None, num_seqs=s.num_seqs,
                       workspace=ws, flags=flags, segments=segments)


def _oracle_check(s, inp, o, fs):
    f = {k: W.as_f64(v) for k, v in inp.items() if k != "cu_seqlens"}
    o_ref, s_ref, _, _ = oracle.forward(inp["cu_seqlens"], s.H, s.d, f["q"], f["k"], f["v"],
                                        f["conv_w"], f["alpha"], f["b"], f["A_log"], f["dt_bias"],
                                        state0=f.get("S0"))
    og, sg = W.from_device(o), W.from_device(fs)
    cu = inp["cu_seqlens"]
    worst = 0.0
    for n in range(s.num_seqs):
        for h in range(s.H):
            if cu[n + 1] > cu[n]:
                worst = max(worst, rel(og[cu[n]:cu[n + 1], h], o_ref[cu[n]:cu[n + 1], h]))
            worst = max(worst, rel(sg[n, h], s_ref[n, h]))
    assert worst <= TOL, worst
    return worst


@pytest.mark.parametrize("case", ["varlen", "segmented"])
def test_prefill_waits_expire_then_recover(case):
    if case == "varlen":   # one launch of chunk_prep and of the state pass
        s = W.small("fail_varlen", [200, 130, 64], H=2, d=128, seed=71, s0_std=0.02, varlen=True)
    else:                  # dense, 260 chunks: time segments on the side stream
        s = W.small("fail_seg", [260 * 64], H=2, d=128, seed=72, s0_std=0.02)
    inp = W.make_inputs(s)
    d = {k: W.to_device(v) for k, v in inp.items()}
    shape = kda.make_shape(s.num_seqs, s.total_tokens if s.varlen else s.seq_lens[0], s.H, s.d,
                           torch.bfloat16)
    ws = torch.empty(kda.prefill_workspace_size(shape, s.varlen), dtype=torch.uint8, device="cuda")
    word = ws[:4].view(torch.int32)

    _prefill(s, d, ws, flags=EXPIRE)
    assert kda.device_status(word) == kda.KDA_ERR_TIMEOUT
    bits = int(word.item())
    assert bits & kda.KDA_STATUS_TIMEOUT_PREP, hex(bits)
    assert bits & kda.KDA_STATUS_TIMEOUT_STATE, hex(bits)
    assert not bits & kda.KDA_STATUS_BAD_CU_SEQLENS, hex(bits)

    # the same workspace, an ordinary call: clean status and oracle parity
    o, fs, _ = _prefill(s, d, ws)
    assert kda.device_status(word) == kda.KDA_OK
    _oracle_check(s, inp, o, fs)
    if case == "segmented":   # the segmented schedule computes exactly the one-launch result
        o1, fs1, _ = _prefill(s, d, ws, segments=False)
        torch.cuda.synchronize()
        assert torch.equal(o, o1) and torch.equal(fs, fs1)


@pytest.mark.parametrize("ntok", [1, 2])
def test_decode_waits_expire_then_recover(ntok):
    # 16 sequences x 8 heads: bf16, d = 128, H a multiple of 8 -> the TMA decode kernels
    s = W.small("fail_dec", [70] * 16, H=8, d=128, seed=73)
    inp = W.make_inputs(s)
    d = {k: W.to_device(v) for k, v in inp.items()}
    _, st, cs = kda.prefill(d["q"], d["k"], d["v"], d["conv_w"], d["alpha"], d["b"], d["A_log"],
                            d["dt_bias"], num_seqs=s.num_seqs, check=True)
    xs = [W.make_decode_step(s, i) for i in range(ntok)]
    dx = {k: W.to_device(np.stack([x[k] for x in xs], axis=1)) for k in xs[0]}
    st0, cs0 = st.clone(), cs.clone()
    status = torch.full((4,), -1, dtype=torch.int32, device="cuda")
    steps = torch.empty((s.num_seqs, ntok, s.H, s.d, s.d), dtype=torch.float32, device="cuda")

    def call(flags):
        if ntok == 1:
            return kda.decode_step(dx["q"][:, 0].contiguous(), dx["k"][:, 0].contiguous(),
                                   dx["v"][:, 0].contiguous(), dx["alpha"][:, 0].contiguous(),
                                   dx["b"][:, 0].contiguous(), d["conv_w"], d["A_log"],
                                   d["dt_bias"], st, cs, status=status[:1], flags=flags)
        return kda.decode_multi(dx["q"], dx["k"], dx["v"], dx["alpha"], dx["b"], d["conv_w"],
                                d["A_log"], d["dt_bias"], st, cs, step_states=steps,
                                status=status[:1], flags=flags)

    call(EXPIRE)
    assert kda.device_status(status[:1]) == kda.KDA_ERR_TIMEOUT
    assert int(status[0].item()) & kda.KDA_STATUS_TIMEOUT_DECODE

    st.copy_(st0)
    cs.copy_(cs0)
    o = call(0)
    assert kda.device_status(status[:1]) == kda.KDA_OK
    assert int(status[1].item()) == -1   # the call zeroes its own word only

    # oracle: prefill then the decode token(s)
    f = {k: W.as_f64(v) for k, v in inp.items() if k != "cu_seqlens"}
    _, S, C, _ = oracle.forward(inp["cu_seqlens"], s.H, s.d, f["q"], f["k"], f["v"], f["conv_w"],
                                f["alpha"], f["b"], f["A_log"], f["dt_bias"])
    og = W.from_device(o).reshape(s.num_seqs, ntok, s.H, s.d)
    worst = 0.0
    for t, x in enumerate(xs):
        xf = {k: W.as_f64(v) for k, v in x.items()}
        o_ref, S, C = oracle.decode_step(s.H, s.d, S, C, xf["q"], xf["k"], xf["v"], xf["alpha"],
                                         xf["b"], f["conv_w"], f["A_log"], f["dt_bias"])
        for n in range(s.num_seqs):
            for h in range(s.H):
                worst = max(worst, rel(og[n, t, h], o_ref[n, h]))
    sg = W.from_device(st)
    for n in range(s.num_seqs):
        for h in range(s.H):
            worst = max(worst, rel(sg[n, h], S[n, h]))
    assert worst <= TOL, worst
