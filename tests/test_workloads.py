"""The seeded input generator: bf16 rounding, slice determinism, workload shapes."""

import numpy as np
import torch

from gated_delta_rule_70_b200 import workloads as W


def test_bf16_rounding_matches_torch():
    x = np.random.default_rng(0).standard_normal(200000).astype(np.float32) * 3
    x[:5] = [1.0, 1.00390625, 1.01171875, -3.0000001, 65504.0]
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(W.bf16_bits(x), ref)
    np.testing.assert_array_equal(W.bf16_to_f32(ref), torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_token_slices_are_regenerable():
    s = W.small("slice", [5000, 4000], H=2, d=64, seed=9)
    full = W.make_tokens(s)
    part = W.make_tokens(s, 4090, 8100)
    for k in full:
        np.testing.assert_array_equal(part[k], full[k][4090:8100])


def test_named_workloads():
    s = W.spec("prefill_4x8k")
    assert (s.num_seqs, s.total_tokens, s.H, s.d, s.io_dtype) == (4, 32768, 32, 128, "bf16")
    s = W.spec("varlen_32")
    assert s.num_seqs == 32 and all(16 <= L <= 32768 for L in s.seq_lens) and s.varlen
    s = W.spec("long_256k")
    assert s.total_tokens == 262144 and s.alpha_mu == -2.0 and s.s0_std == 0.0
    s = W.spec("tiny_fp32")
    assert (s.io_dtype, s.H, s.d, s.total_tokens) == ("fp32", 2, 64, 256)
    p = W.make_params(W.spec("tiny_fp32"))
    assert p["conv_w"].shape == (3, 128, 4) and p["dt_bias"].shape == (2, 64)
    assert np.all((p["A_log"] >= 0) & (p["A_log"] <= np.log(16.0)))
