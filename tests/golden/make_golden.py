"""Write the stored expected outputs under tests/golden/ from the oracle.

Calls only ``oracle`` and the seeded input generator; nothing here comes from
the CUDA path.  Run from the repository root:

    python tests/golden/make_golden.py
"""
from __future__ import annotations

import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from reduce_residual_add_b200.inputs import WORKLOADS, as_u16, make_inputs  # noqa: E402

HEADER = """# Oracle outputs for the small workload c1_small: W=2 partials, T=8, H=64,
# bf16, partials and residual N(0,1) (seed 0), gamma U(0.5,1.5), eps=1e-6,
# weight_bias=0, pattern all-reduce + residual + RMSNorm.
# Defined by vllm.models.common.ops.fused_allreduce_rms_norm (docstring:
# (normed_output, new_residual) = norm(all_reduce(hidden_states), residual)).
# Written by tests/golden/make_golden.py from the fp64 oracle only.
# One line per row: 64 bf16 patterns in hex.
"""


def write_c1(path: str) -> None:
    wl = WORKLOADS["c1_small"]
    inp = make_inputs(wl)
    r = oracle.fused([as_u16(p) for p in inp["partials"]], as_u16(inp["residual"]),
                     as_u16(inp["gamma"]), wl.dtype, wl.eps, wl.weight_bias, wl.pattern)
    with open(path, "w") as f:
        f.write(HEADER)
        for key in ("residual_out", "norm_out"):
            f.write("[%s]\n" % key)
            for row in r[key]:
                f.write(" ".join("%04x" % int(v) for v in row) + "\n")


def read_fixture(path: str) -> dict:
    out, key = {}, None
    for line in open(path):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        if line.startswith("["):
            key = line[1:-1]
            out[key] = []
            continue
        out[key].append([int(x, 16) for x in line.split()])
    return out


if __name__ == "__main__":
    write_c1(os.path.join(HERE, "c1_small_oracle.txt"))
    print("wrote", os.path.join(HERE, "c1_small_oracle.txt"))
