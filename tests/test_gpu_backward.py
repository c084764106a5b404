"""GPU parity of the prefill's backward pass (``la_prefill_backward``) against the fp64
reverse-mode oracle (``oracle/backward.py``).

Scalar gates (mode 1, with and without a gate tensor) and the constant per-head decay
(mode 4), both head sizes and I/O dtypes, sequences of one token, of exactly one and
several chunks of 32 with a ragged tail, with and without an initial state and a
final-state cotangent.  Tolerance per (batch, head) slice, max|x - r| / max|r|: 2e-3 for
fp32 I/O, 2e-2 for bf16 I/O, for dq, dk, dv, the gate gradient and dS_0.
"""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import backward as ob
from parity_util import TOL, f64, slice_rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def la():
    import gated_delta_rule_attention_b200 as m
    m.library()
    return m


def _case(mode, dtype, d, T, gate, seed, B=2, H=2):
    w = W.Workload("bwd", mode, dtype, B=B, H=H, T=T, dk=d, dv=d, seed=seed,
                   qk_scale=1 / np.sqrt(d), gate=gate, gate_shift=-2.0)
    inp = W.prefill_inputs(w, device="cuda", init_state_std=0.1)
    g = torch.Generator(device="cuda").manual_seed(seed + 1)
    dO = torch.randn(B, H, T, d, generator=g, device="cuda").to(dtype)
    dST = torch.randn(B, H, d, d, generator=g, device="cuda") * 0.1
    return inp, dO, dST


@pytest.mark.parametrize("mode,gate", [(1, "softplus"), (1, "none"), (4, "retnet")])
@pytest.mark.parametrize("dtype,d", [(torch.float32, 64), (torch.bfloat16, 128), (torch.float32, 128)])
@pytest.mark.parametrize("T", [1, 32, 100])
@pytest.mark.parametrize("with_state", [False, True])
def test_backward_matches_oracle(la, mode, gate, dtype, d, T, with_state):
    inp, dO, dST = _case(mode, dtype, d, T, gate, seed=10 * T + d + mode)
    S0 = inp["state0"] if with_state else None
    dS = dST if with_state else None
    dq, dk, dv, dg, dS0 = la.prefill_backward(inp["q"], inp["k"], inp["v"], dO, mode=mode,
                                              gate=inp["gate"], state0=S0, dstate=dS,
                                              need_dstate0=with_state)
    la.check_status()
    g = lambda t: None if t is None else f64(t)
    rq, rk, rv, rg, rS0 = ob.prefill_backward(mode, g(inp["q"]), g(inp["k"]), g(inp["v"]), g(inp["gate"]),
                                              g(dO), g(S0), g(dS))
    tol = TOL[dtype]
    for name, x, r in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
        e = slice_rel_err(f64(x), r)
        assert e < tol, f"{name}: {e:.3e}"
    if mode == 1 and gate != "none":
        e = slice_rel_err(f64(dg), rg)
        assert e < tol, f"dgate: {e:.3e}"
    else:
        assert dg is None
    if with_state:
        e = slice_rel_err(f64(dS0), rS0)
        assert e < tol, f"dS0: {e:.3e}"


def test_backward_argument_checks(la):
    inp, dO, _ = _case(4, torch.float32, 64, 10, "retnet", seed=3)
    with pytest.raises(la.LaError):   # mode 4 keeps its gates fixed: no gate gradient
        lib = la.library()
        import ctypes
        n = lib.la_backward_workspace_size(4, 2, 2, 10, 64, 64)
        ws = torch.empty(n, dtype=torch.uint8, device="cuda")
        p = lambda t: ctypes.c_void_p(t.data_ptr())
        dg = torch.empty(2, 2, 10, device="cuda")
        x = [torch.empty_like(inp["q"]) for _ in range(3)]
        st = lib.la_prefill_backward(4, 0, 2, 2, 10, 64, 64, p(inp["q"]), p(inp["k"]), p(inp["v"]),
                                     p(inp["gate"]), None, p(dO), None, p(x[0]), p(x[1]), p(x[2]),
                                     p(dg), None, p(ws), n, None)
        la._check(st, "la_prefill_backward")


def test_backward_full_size_sampled(la):
    """The benchmark's backward workload (mode 1, B4 H16 T4096, d = 128, bf16) in its launch
    configuration, checked on sampled heads: the oracle runs on each head alone."""
    w = W.BACKWARD_CONFIGS["gated_bwd_bf16_b4h16t4096"]
    inp = W.prefill_inputs(w, device="cuda")
    g = torch.Generator(device="cuda").manual_seed(w.seed + 1)
    dO = torch.randn(w.B, w.H, w.T, w.dv, generator=g, device="cuda").to(w.dtype)
    dq, dk, dv, dg, _ = la.prefill_backward(inp["q"], inp["k"], inp["v"], dO, mode=1, gate=inp["gate"])
    la.check_status()
    for b, h in [(0, 0), (3, 15)]:
        sl = lambda t: f64(t[b:b + 1, h:h + 1])
        rq, rk, rv, rg, _ = ob.prefill_backward(1, sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(inp["gate"]),
                                                sl(dO))
        for name, x, r in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv), ("dgate", dg, rg)):
            e = slice_rel_err(sl(x), r)
            assert e < TOL[w.dtype], f"{name} head ({b},{h}): {e:.3e}"


@pytest.mark.parametrize("dk,dv", [(64, 64), (64, 128), (128, 64)])
@pytest.mark.parametrize("T", [1, 33, 300])
@pytest.mark.parametrize("with_state", [False, True])
def test_backward_bf16_head_sizes(la, dk, dv, T, with_state):
    """bf16 I/O runs the state scans and the per-chunk kernel: every head-size pair they are
    built for, ragged tails, one and many chunks."""
    B, H = 2, 2
    w = W.Workload("bwd", 1, torch.bfloat16, B=B, H=H, T=T, dk=dk, dv=dv, seed=7 * T + dk + dv,
                   qk_scale=1 / np.sqrt(dk), gate="softplus", gate_shift=-2.0)
    inp = W.prefill_inputs(w, device="cuda", init_state_std=0.1)
    g = torch.Generator(device="cuda").manual_seed(T + 3)
    dO = torch.randn(B, H, T, dv, generator=g, device="cuda").to(torch.bfloat16)
    dST = torch.randn(B, H, dv, dk, generator=g, device="cuda") * 0.1
    S0 = inp["state0"] if with_state else None
    dS = dST if with_state else None
    dq, dk_, dv_, dg, dS0 = la.prefill_backward(inp["q"], inp["k"], inp["v"], dO, mode=1, gate=inp["gate"],
                                                state0=S0, dstate=dS, need_dstate0=with_state)
    la.check_status()
    f = lambda t: None if t is None else f64(t)
    rq, rk, rv, rg, rS0 = ob.prefill_backward(1, f(inp["q"]), f(inp["k"]), f(inp["v"]), f(inp["gate"]),
                                              f(dO), f(S0), f(dS))
    tol = TOL[torch.bfloat16]
    for name, x, r in (("dq", dq, rq), ("dk", dk_, rk), ("dv", dv_, rv), ("dgate", dg, rg)):
        e = slice_rel_err(f64(x), r)
        assert e < tol, f"{name}: {e:.3e}"
    if with_state:
        e = slice_rel_err(f64(dS0), rS0)
        assert e < tol, f"dS0: {e:.3e}"
