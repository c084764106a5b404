"""The device failure path on the GPU, without a fault.

A kernel's bounded wait on a barrier that nothing completes runs out, records the
timeout in the device failure word and returns; la_check_status reports it once and
clears it, and the context keeps working: a prefill right after it is checked against
the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from parity_util import TOL, f64, slice_rel_err

pytestmark = pytest.mark.gpu


def test_bounded_wait_timeout_is_reported_and_the_device_survives():
    import gated_delta_rule_attention_b200 as la
    la.library()
    la.check_status()                                   # nothing pending
    la.selftest_wait_timeout()
    with pytest.raises(la.LaError, match="TIMEOUT"):
        la.check_status()
    la.check_status()                                   # reported once, then cleared
    w = W.Workload("after", 2, torch.bfloat16, B=1, H=2, T=130, dk=128, dv=128, seed=55,
                   qk_l2norm=True, gate="softplus", beta=True)
    inp = W.prefill_inputs(w, device="cuda")
    o, S, _ = la.prefill(inp["q"], inp["k"], inp["v"], mode=2, gate=inp["gate"], beta=inp["beta"])
    la.check_status()
    ro, rS, _ = oracle.prefill(2, f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["gate"]),
                               f64(inp["beta"]))
    assert slice_rel_err(f64(o), ro) < TOL[torch.bfloat16]
    assert slice_rel_err(f64(S), rS) < TOL[torch.bfloat16]
