"""GPU parity of the constant-decay (RetNet) mode against the oracle.

Mode 4 runs the scalar-gate kernels with one fixed gate per head (gate [H], read once per
head instead of per token).  Checked against the oracle's mode 4 on the tensor-core path
(bf16, d = 128: one pass, the segmented passes, an initial state), the CUDA-core path
(fp32, d = 64), packed sequences and the decode step; tolerance as for the other modes.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from parity_util import TOL, f64, slice_rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def la():
    import gated_delta_rule_attention_b200 as m
    m.library()
    return m


def wl(dtype, d, B, H, T, seed=400):
    return W.Workload("retnet", W.MODE_RETNET, dtype, B=B, H=H, T=T, dk=d, dv=d, seed=seed,
                      qk_scale=1 / np.sqrt(d), gate="retnet")


@pytest.mark.parametrize("dtype,d,B,H,T,ws,init", [
    (torch.bfloat16, 128, 2, 3, 300, None, False),     # one pass
    (torch.bfloat16, 128, 1, 4, 3000, "auto", False),  # segmented: local + outputs passes
    (torch.bfloat16, 128, 1, 4, 3000, "auto", True),   # segmented with a start state
    (torch.float32, 64, 2, 3, 150, None, True),
])
def test_retnet_prefill_matches_oracle(la, dtype, d, B, H, T, ws, init):
    w = wl(dtype, d, B, H, T)
    inp = W.prefill_inputs(w, device="cuda", init_state_std=0.05 if init else 0.0)
    assert inp["gate"].shape == (H,)
    o, S, _ = la.prefill(inp["q"], inp["k"], inp["v"], mode=la.MODE_RETNET, gate=inp["gate"],
                         state=inp["state0"].clone() if init else None, init_state=init,
                         workspace=ws if ws else None)
    la.check_status()
    ro, rS, _ = oracle.prefill(oracle.MODE_RETNET, f64(inp["q"]), f64(inp["k"]), f64(inp["v"]),
                               f64(inp["gate"]), None, f64(inp["state0"]) if init else None)
    assert slice_rel_err(f64(o), ro) < TOL[dtype]
    assert slice_rel_err(f64(S), rS) < TOL[dtype]


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 64)])
def test_retnet_varlen_and_decode(la, dtype, d):
    w = wl(dtype, d, 1, 3, 0, seed=401)
    lengths = [70, 0, 130, 5]
    inp = W.varlen_inputs(w, lengths, device="cuda")
    o, S, _ = la.prefill_varlen(inp["q"], inp["k"], inp["v"], inp["cu"], mode=la.MODE_RETNET,
                                gate=inp["gate"])
    la.check_status()
    cu = [int(x) for x in inp["cu"].tolist()]
    ro, rS, _ = oracle.prefill_packed(oracle.MODE_RETNET, f64(inp["q"]), f64(inp["k"]), f64(inp["v"]),
                                      cu, f64(inp["gate"]))
    for s in range(len(lengths)):
        a, b = cu[s], cu[s + 1]
        if b > a:
            assert slice_rel_err(f64(o[:, a:b]), ro[:, a:b], lead=1) < TOL[dtype]
    assert slice_rel_err(f64(S), rS) < TOL[dtype]
    # one decode step per sequence from the packed final states
    g = torch.Generator(device="cuda").manual_seed(7)
    N, H = len(lengths), 3
    q1 = (torch.randn(N, H, d, generator=g, device="cuda") / np.sqrt(d)).to(dtype)
    k1 = (torch.randn(N, H, d, generator=g, device="cuda") / np.sqrt(d)).to(dtype)
    v1 = torch.randn(N, H, d, generator=g, device="cuda").to(dtype)
    od, S2, _ = la.decode_step(q1, k1, v1, mode=la.MODE_RETNET, state=S.clone(), gate=inp["gate"])
    la.check_status()
    rod, rS2, _ = oracle.decode_step(oracle.MODE_RETNET, f64(q1), f64(k1), f64(v1), f64(inp["gate"]),
                                     None, f64(S))
    assert slice_rel_err(f64(od), rod, lead=1) < TOL[dtype]
    assert slice_rel_err(f64(S2), rS2) < TOL[dtype]
