"""The chunkwise algebra on the GPU in fp32 (the fp32 test mode).

Off the tensor-core path (fp32 I/O, head_dim 64) the recurrence runs as the same
64-token chunk factorisation the tensor-core kernels use -- in-chunk cumulative
gate, 16-token sub-blocks with mid-block references for the split decay factors,
A_qk / A_kk, the unit-lower-triangular solve for W and U, then the state step --
but with fp32 operands and accurate exponentials.  These tests hold it to the
fp32 tolerance against the fp64 oracle (max relative L2 per (sequence, head)
<= 1e-4; 1e-2 for bf16 I/O), next to the token-by-token CUDA-core loop that
KDA_FLAG_TOKEN_RECURRENCE selects, on the fp32 workload (B=1, T=256, H=2, d=64)
and on ragged, long, saturated-gate and d=128 cases.
"""

import pytest

from gated_delta_rule_70_b200 import kda
from gated_delta_rule_70_b200 import workloads as W

from tests.test_gpu_parity import check_prefill

pytestmark = pytest.mark.gpu
TOKEN = kda.KDA_FLAG_TOKEN_RECURRENCE


@pytest.mark.parametrize("flags", [0, TOKEN], ids=["chunked", "token_loop"])
def test_tiny_fp32_workload_both_paths(flags):
    eo, es = check_prefill(W.spec("tiny_fp32"), flags=flags)
    print("\ntiny_fp32 (%s): max rel-L2 o %.2e, final state %.2e"
          % ("token loop" if flags else "chunked", eo, es))


@pytest.mark.parametrize("d,lens,H", [(64, [1, 63, 64, 65, 130], 3), (128, [200, 17], 2),
                                      (64, [1000], 2)])
def test_fp32_chunked_ragged_and_long(d, lens, H):
    check_prefill(W.small("c32", lens, H=H, d=d, io_dtype="fp32", seed=81, s0_std=0.02,
                          varlen=len(lens) > 1))


@pytest.mark.parametrize("lower_bound", [-8.0, -10.0])
def test_fp32_chunked_saturated_gates(lower_bound):
    # alpha far above zero saturates every gate at the bound: the split factors reach
    # e^{+-8 |lower_bound|}, the range the sub-block references are sized for
    s = W.small("c32sat", [150, 70], H=2, d=64, io_dtype="fp32", seed=82, s0_std=0.02,
                alpha_mu=20.0, varlen=True)
    s.lower_bound = lower_bound
    check_prefill(s)


def test_bf16_d64_chunked():
    check_prefill(W.small("c16", [129, 40], H=2, d=64, io_dtype="bf16", seed=83, s0_std=0.02,
                          varlen=True))
