"""Argument checks of the C ABI that need device memory: buffers a call writes must not
overlap one another or what it reads (la.h: o must not overlap q, k, v or the state).

Every rejected call returns LA_ERR_INVALID_ARG before any launch; a call with disjoint
buffers right after each rejection still succeeds.
"""
import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu

INVALID = 1


@pytest.fixture(scope="module")
def la():
    import gated_delta_rule_attention_b200 as m
    m.library()
    return m


def _raises_invalid(fn):
    import gated_delta_rule_attention_b200 as m
    with pytest.raises(m.LaError) as e:
        fn()
    assert e.value.status == INVALID


@pytest.mark.parametrize("mode", [0, 2])
def test_prefill_rejects_overlapping_outputs(la, mode):
    w = W.Workload("ov", mode, torch.bfloat16, B=1, H=2, T=64, dk=128, dv=128, seed=3,
                   qk_l2norm=(mode == 2), gate="none" if mode == 0 else "softplus", beta=(mode == 2))
    inp = W.prefill_inputs(w, device="cuda")
    q, k, v, g, b = (inp[x] for x in ("q", "k", "v", "gate", "beta"))
    st = torch.empty(1, 2, 128, 128, device="cuda")
    z = torch.empty(1, 2, 128, device="cuda") if mode == 0 else None
    call = lambda **kw: la.prefill(**{**dict(q=q, k=k, v=v, mode=mode, gate=g, beta=b, state=st, z=z,
                                             init_state=False), **kw})
    _raises_invalid(lambda: call(o=q))                       # o aliases q
    # o carved out of the state buffer
    o_in_state = st.view(-1).view(torch.bfloat16)[: 2 * 64 * 128].view(1, 2, 64, 128)
    _raises_invalid(lambda: call(o=o_in_state))
    # inputs may alias one another (they are only read): k = v is a valid call
    call(o=torch.empty_like(v), k=v)
    o, S, _ = call()
    la.check_status()
    assert torch.isfinite(o.float()).all()


def test_decode_rejects_state_over_inputs(la):
    N, H = 2, 2
    q = torch.randn(N, H, 128, device="cuda", dtype=torch.bfloat16)
    k = torch.randn(N, H, 128, device="cuda", dtype=torch.bfloat16)
    v = torch.randn(N, H, 128, device="cuda", dtype=torch.bfloat16)
    g = torch.rand(N, H, device="cuda")
    b = torch.rand(N, H, device="cuda")
    st = torch.zeros(N, H, 128, 128, device="cuda")
    _raises_invalid(lambda: la.decode_step(q, k, v, mode=2, state=st, gate=g, beta=b, o=q))
    o_in_state = st.view(-1)[: N * H * 64].view(torch.bfloat16).view(N, H, 128)
    _raises_invalid(lambda: la.decode_step(q, k, v, mode=2, state=st, gate=g, beta=b, o=o_in_state))
    o, S, _ = la.decode_step(q, k, v, mode=2, state=st, gate=g, beta=b)
    la.check_status()
    assert torch.isfinite(o.float()).all()


def test_varlen_rejects_output_over_offsets(la):
    H, T = 2, 100
    lengths = [40, 60]
    w = W.Workload("ovl", 2, torch.bfloat16, B=1, H=H, T=T, dk=128, dv=128, seed=4, qk_l2norm=True,
                   gate="softplus", beta=True)
    inp = W.varlen_inputs(w, lengths, device="cuda")
    st = torch.empty(2, H, 128, 128, device="cuda")
    call = lambda **kw: la.prefill_varlen(**{**dict(q=inp["q"], k=inp["k"], v=inp["v"], cu_seqlens=inp["cu"],
                                                    mode=2, gate=inp["gate"], beta=inp["beta"], state=st,
                                                    init_state=False), **kw})
    _raises_invalid(lambda: call(o=inp["v"]))
    o, S, _ = call()
    la.check_status()
    assert torch.isfinite(o.float()).all()


def test_two_streams_get_their_own_workspace(la):
    """The automatic segment workspace is per (device, stream): two calls that run
    concurrently on two streams do not share scratch, and both match the single-stream
    result."""
    w = W.Workload("ws2", 1, torch.bfloat16, B=1, H=4, T=4096, dk=128, dv=128, seed=9,
                   qk_scale=0.09, gate="softplus", gate_shift=-3.0)
    assert la.workspace_size(1, torch.bfloat16, 1, 4, 4096, 128, 128) > 0
    inp = W.prefill_inputs(w, device="cuda")
    o_ref, S_ref, _ = la.prefill(inp["q"], inp["k"], inp["v"], mode=1, gate=inp["gate"])
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    outs = []
    for _ in range(3):
        for s in streams:
            with torch.cuda.stream(s):
                outs.append(la.prefill(inp["q"], inp["k"], inp["v"], mode=1, gate=inp["gate"], stream=s))
    torch.cuda.synchronize()
    la.check_status()
    for o, S, _ in outs:
        assert torch.equal(o, o_ref) and torch.equal(S, S_ref)
