"""What the d = 128 chunk kernel's fp16 operands cost, measured on the CPU.

The kernel rounds every tensor-core operand to fp16 once (state, residuals, T,
AT, gains; K and Q are exact in fp16).  The float64 model of those roundings
(tests/operand_rounding_model.py) runs a layer-length head against the same
model without rounding; the normwise error must stay well inside the 3e-3
budget for bf16 inputs (measured: at most 6e-4 over 8192 tokens).  The
retired bf16 hi/lo form is kept as the comparison: about 1e-5.
"""

import numpy as np
import pytest

from delta_rule_recurrent_scan_b200.workloads import WORKLOADS, make_scan_inputs
from operand_rounding_model import chunk_scan_rounded


def _err(x, y):
    return float(np.abs(x - y).max() / np.abs(y).max())


@pytest.mark.parametrize("variant,name", [("delta", "gdn_d128"), ("kalman_diag", "kalman_diag_d128")])
def test_fp16_operands_stay_inside_the_bf16_budget(variant, name):
    w = WORKLOADS[name]
    x = make_scan_inputs(w, seed=0, B=1, H=1, L=2048)
    args = [x[n][0, 0].double().numpy() for n in ("q", "k", "v", "beta", "a", "r")]
    exact = chunk_scan_rounded(variant, *args, w.qn, "exact")
    f16 = chunk_scan_rounded(variant, *args, w.qn, "f16")
    pair = chunk_scan_rounded(variant, *args, w.qn, "bf16_pair")
    for got, ref in zip(f16, exact):
        assert _err(got, ref) < 1e-3
    for got, ref in zip(pair, exact):
        assert _err(got, ref) < 5e-5
    # the model is not trivially exact: fp16 costs clearly more than the pairs
    assert _err(f16[0], exact[0]) > 10 * _err(pair[0], exact[0])
