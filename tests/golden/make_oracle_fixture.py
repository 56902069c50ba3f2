"""Writes oracle_tiny_fp32.txt: sampled outputs of the fp64 oracle on the fp32 test-mode
workload (B=1, T=256, H=2, d=64, seed 0).  It calls only the oracle and the seeded input
generator, never the CUDA library.  tests/test_golden.py re-runs the oracle and compares, so an
unintended change to the oracle's arithmetic shows up; an intended one regenerates this file
and names the passage that justifies it in its commit message.

    python tests/golden/make_oracle_fixture.py
"""

import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from gated_delta_rule_70_b200 import workloads as W  # noqa: E402
from oracle import oracle  # noqa: E402

# (token, head, value channel) of o, and (head, key channel, value channel) of the final state
O_SAMPLES = [(0, 0, 0), (1, 1, 5), (63, 0, 17), (64, 1, 40), (127, 0, 63), (200, 1, 1), (255, 0, 31),
             (255, 1, 62)]
S_SAMPLES = [(0, 0, 0), (0, 5, 9), (1, 63, 63), (1, 20, 33), (0, 40, 2)]


def compute():
    s = W.spec("tiny_fp32")
    inp = W.make_inputs(s)
    f = {k: W.as_f64(v) for k, v in inp.items() if k != "cu_seqlens"}
    o, st, _, _ = oracle.forward(inp["cu_seqlens"], s.H, s.d, f["q"], f["k"], f["v"], f["conv_w"],
                                 f["alpha"], f["b"], f["A_log"], f["dt_bias"], state0=f["S0"])
    rows = [("o", t, h, j, o[t, h, j]) for t, h, j in O_SAMPLES]
    rows += [("S", h, i, j, st[0, h, i, j]) for h, i, j in S_SAMPLES]
    rows += [("o_norm", h, -1, -1, float(np.linalg.norm(o[:, h]))) for h in range(s.H)]
    rows += [("S_norm", h, -1, -1, float(np.linalg.norm(st[0, h]))) for h in range(s.H)]
    return rows


def main():
    lines = ["# Written by tests/golden/make_oracle_fixture.py from the fp64 oracle alone (workload",
             "# tiny_fp32: B=1, T=256, H=2, d=64, zero initial state, seed 0).  Columns: kind, three",
             "# indices (-1 where unused), value.  o[t, h, j]; S[h, i, j] of sequence 0; norms per head."]
    lines += ["%s %d %d %d %.17g" % r for r in compute()]
    with open(os.path.join(HERE, "oracle_tiny_fp32.txt"), "w") as fh:
        fh.write("\n".join(lines) + "\n")


if __name__ == "__main__":
    main()
