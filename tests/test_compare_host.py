"""The parity helper's tolerance rule, on the CPU with the oracle only.

The GPU tests compare against the oracle with exact accumulation; where the
pages' fp32 accumulation is not exact (a rounded running sum followed by
cancellation) an element may instead match the oracle with fp32
accumulation.  This checks that rule both ways: the fp32-accumulation
outputs pass against the exact reference (through the fallback, which the
statistics count), and a 2-ulp error planted anywhere else still fails."""
from __future__ import annotations

import numpy as np
import pytest

from gpu_util import compare, run_oracle
from reduce_residual_add_b200.inputs import random_inputs

# an input set known to hold one cancellation element (row 2394, column 3897):
# four of its five values cancel exactly and the fifth is 5.5e-8
INP = dict(W=4, T=3000, H=8192, dtype="bf16", seed=901, partial_sigma=0.25, residual_sigma=0.25)


@pytest.fixture(scope="module")
def case():
    inp = random_inputs(**INP)
    rows = list(range(2390, 2400))
    ref = run_oracle(inp, "bf16", 1e-6, 0.5, 2, row_list=rows)
    acc = run_oracle(inp, "bf16", 1e-6, 0.5, 2, row_list=rows, acc32=True)
    return ref, acc, rows


def test_fp32_accumulation_result_passes_through_the_fallback(case):
    ref, acc, rows = case
    assert acc["residual_out"][2394, 3897] != ref["residual_out"][2394, 3897]
    st = compare(acc, ref, "bf16", rows=rows)
    assert st["residual_out"][2] == 1 and st["norm_out"][2] == 1


def test_an_error_outside_the_cancellation_elements_still_fails(case):
    ref, acc, rows = case
    bad = {k: (None if v is None or k.startswith("_") else v.copy()) for k, v in acc.items()}
    bad["norm_out"][2391, 100] = (int(bad["norm_out"][2391, 100]) + 2) & 0xFFFF
    with pytest.raises(AssertionError):
        compare(bad, ref, "bf16", rows=rows)
    # ... and so does an error at the cancellation element beyond 1 ulp of
    # the fp32-accumulation reference
    bad2 = {k: (None if v is None or k.startswith("_") else v.copy()) for k, v in acc.items()}
    bad2["residual_out"][2394, 3897] = (int(bad2["residual_out"][2394, 3897]) + 2) & 0xFFFF
    with pytest.raises(AssertionError):
        compare(bad2, ref, "bf16", rows=rows)
