"""GPU parity of packed variable-length prefill (``la_prefill_varlen``) against the oracle.

Each sequence of the packed batch is checked against the recurrent form run on that
sequence alone (``oracle.prefill_packed``), outputs and final state, per (sequence,
head) slice with the tolerance of the dense prefill (2e-2 bf16, 2e-3 fp32 I/O).  The
length mixes put sequence ends inside, at, and just past chunk boundaries, with empty
and one-token sequences; the tensor-core path (bf16, d = 128, modes 0-2) and the
CUDA-core path (fp32, d = 64, and mode 3) are both covered, with and without start
states, plus a bad offsets table (clamped and reported, nothing out of bounds), the
longest-first schedule of the outputs passes (ties, more than 128 sequences) and the
serving-batch workload the benchmark times, on sampled sequences.
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


def seq_err(x, r, cu):
    """max over (sequence, head) of max|x - r| / max|r| on [H, T, d] arrays."""
    worst = 0.0
    for s in range(len(cu) - 1):
        a, b = cu[s], cu[s + 1]
        if b > a:
            worst = max(worst, slice_rel_err(x[:, a:b], r[:, a:b], lead=1))
    return worst


def base(mode, dtype, d, seed=200):
    return W.Workload(f"v{mode}", mode, dtype, B=1, H=3, T=0, dk=d, dv=d, seed=seed,
                      qk_scale=1 / np.sqrt(d), qk_l2norm=(mode >= 2),
                      gate="none" if mode == 0 else "softplus", beta=(mode >= 2))


LENGTHS = [65, 0, 1, 64, 130, 63, 200, 2]


@pytest.mark.parametrize("init", [False, True])
@pytest.mark.parametrize("mode,dtype,d", [
    (0, torch.bfloat16, 128), (1, torch.bfloat16, 128), (2, torch.bfloat16, 128),
    (3, torch.bfloat16, 128), (0, torch.float32, 64), (2, torch.float32, 64), (3, torch.float32, 64),
])
def test_varlen_matches_oracle(la, mode, dtype, d, init):
    w = base(mode, dtype, d)
    inp = W.varlen_inputs(w, LENGTHS, device="cuda", init_state_std=0.05 if init else 0.0)
    cu = [int(x) for x in inp["cu"].tolist()]
    N = len(LENGTHS)
    z0 = (torch.rand(N, w.H, d, device="cuda") + 1.0) if (mode == 0 and init) else None
    state = inp["state0"].clone()
    z = None if z0 is None else z0.clone()
    o, S, zo = la.prefill_varlen(inp["q"], inp["k"], inp["v"], inp["cu"], mode=mode, gate=inp["gate"],
                                 beta=inp["beta"], state=state, z=z, init_state=init)
    la.check_status()
    g = lambda t: None if t is None else f64(t)
    ro, rS, rz = oracle.prefill_packed(mode, g(inp["q"]), g(inp["k"]), g(inp["v"]), cu, g(inp["gate"]),
                                       g(inp["beta"]), g(inp["state0"]) if init else None, g(z0))
    tol = TOL[dtype]
    assert seq_err(f64(o), ro, cu) < tol
    assert slice_rel_err(f64(S), rS) < tol
    if mode == 0:
        assert slice_rel_err(f64(zo), rz) < tol
    # the empty sequence keeps its start state (zero without one)
    np.testing.assert_allclose(f64(S[1]), f64(inp["state0"][1]) if init else 0.0, rtol=0, atol=0)


def test_varlen_equals_separate_dense_calls(la):
    """The packed call and one la_prefill per sequence run the same kernel arithmetic."""
    w = base(2, torch.bfloat16, 128, seed=300)
    inp = W.varlen_inputs(w, [100, 64, 300], device="cuda")
    cu = [int(x) for x in inp["cu"].tolist()]
    o, S, _ = la.prefill_varlen(inp["q"], inp["k"], inp["v"], inp["cu"], mode=2, gate=inp["gate"],
                                beta=inp["beta"])
    for s in range(3):
        a, b = cu[s], cu[s + 1]
        sl = lambda t: t[:, a:b][None].contiguous()
        od, Sd, _ = la.prefill(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), mode=2, gate=sl(inp["gate"]),
                               beta=sl(inp["beta"]), workspace=None)
        torch.cuda.synchronize()
        assert torch.equal(o[:, a:b], od[0]), f"sequence {s}: outputs differ"
        assert torch.equal(S[s], Sd[0])


@pytest.mark.parametrize("lengths", [
    [64] * 5 + [1] * 3 + [200, 65] + [64] * 4,          # ties: equal lengths keep index order
    [(37 * i) % 150 for i in range(130)],               # more than 128 sequences: launch order
])
def test_varlen_longest_first_schedule(la, lengths):
    """The outputs passes take packed sequences longest first (ties by index), ranking them in
    every warp, up to 128 sequences, and in launch order beyond: each sequence's outputs and
    final state are still its own (bit for bit against the call on the sequences in reverse
    order, whose schedule differs), and match the oracle on sampled sequences."""
    w = base(2, torch.bfloat16, 128, seed=302)
    inp = W.varlen_inputs(w, lengths, device="cuda")
    cu = [int(x) for x in inp["cu"].tolist()]
    o, S, _ = la.prefill_varlen(inp["q"], inp["k"], inp["v"], inp["cu"], mode=2, gate=inp["gate"],
                                beta=inp["beta"])
    la.check_status()
    # the same sequences packed in reverse order
    N = len(lengths)
    rev = list(range(N))[::-1]
    cat = lambda t: torch.cat([t[:, cu[s]:cu[s + 1]] for s in rev], dim=1).contiguous()
    rcu = torch.tensor(np.concatenate([[0], np.cumsum([lengths[s] for s in rev])]), dtype=torch.int32,
                       device="cuda")
    o2, S2, _ = la.prefill_varlen(cat(inp["q"]), cat(inp["k"]), cat(inp["v"]), rcu, mode=2,
                                  gate=cat(inp["gate"]), beta=cat(inp["beta"]))
    la.check_status()
    rc = [int(x) for x in rcu.tolist()]
    for j, s in enumerate(rev):
        assert torch.equal(o[:, cu[s]:cu[s + 1]], o2[:, rc[j]:rc[j + 1]]), f"sequence {s}"
        assert torch.equal(S[s], S2[j]), f"state {s}"
    g = lambda t: f64(t)
    pick = [s for s in (0, 5, 8, N - 1) if lengths[s] > 0][:3]
    for s in pick:
        a, b = cu[s], cu[s + 1]
        sub = lambda t: t[:, a:b]
        ro, rS, _ = oracle.prefill_packed(2, g(sub(inp["q"])), g(sub(inp["k"])), g(sub(inp["v"])), [0, b - a],
                                          g(sub(inp["gate"])), g(sub(inp["beta"])), None, None)
        assert seq_err(f64(o[:, a:b]), ro, [0, b - a]) < TOL[torch.bfloat16], f"sequence {s}"
        assert slice_rel_err(f64(S[s:s + 1]), rS) < TOL[torch.bfloat16], f"state {s}"


def test_varlen_bad_offsets_are_reported(la):
    w = base(1, torch.bfloat16, 128, seed=301)
    inp = W.varlen_inputs(w, [70, 70], device="cuda")
    bad = torch.tensor([0, 90, 10_000], dtype=torch.int32, device="cuda")   # past T = 140
    la.prefill_varlen(inp["q"], inp["k"], inp["v"], bad, mode=1, gate=inp["gate"])
    with pytest.raises(la.LaError, match="INVALID_ARG"):
        la.check_status()
    la.check_status()   # cleared


def test_varlen_serving_batch_sampled(la):
    """The benchmark's packed batch (64 sequences of 75..6305 tokens, Gated DeltaNet,
    bf16, H = 16, d = 128) in its launch configuration, checked on sampled sequences
    (the shortest, the longest, and two in between)."""
    vw = W.VARLEN_CONFIGS["gdn_varlen_bf16_n64h16"]
    L = vw.lengths()
    inp = W.varlen_inputs(vw.base, L, device="cuda")
    o, S, _ = la.prefill_varlen(inp["q"], inp["k"], inp["v"], inp["cu"], mode=2, gate=inp["gate"],
                                beta=inp["beta"])
    la.check_status()
    cu = [int(x) for x in inp["cu"].tolist()]
    order = np.argsort(L)
    for s in [int(order[0]), int(order[-1]), int(order[len(L) // 2]), 5]:
        a, b = cu[s], cu[s + 1]
        for h in (0, 11):
            sl = lambda t: f64(t[h, a:b])[None, None]
            ro, rS, _ = oracle.prefill(2, sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(inp["gate"]),
                                       sl(inp["beta"]))
            assert slice_rel_err(f64(o[h, a:b])[None], ro[0], lead=1) < TOL[torch.bfloat16]
            assert slice_rel_err(f64(S[s, h])[None], rS[0, 0][None], lead=1) < TOL[torch.bfloat16]


def test_serving_chain_conv_prefill_decode(la):
    """A packed serving step end to end: the short convolution over packed projections
    (SiLU, q/k L2 norm), the packed Gated DeltaNet prefill from per-sequence start states,
    then one decode step per sequence from the states it wrote -- against the oracle
    chain on the same bf16 intermediates."""
    from oracle import conv as oconv
    lengths = [40, 1, 97, 64]
    N, H, d, width = len(lengths), 2, 128, 4
    T = sum(lengths)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int32, device="cuda")
    ys, refs = [], []
    for i in range(3):
        x, w, _ = W.conv_inputs(1, T, H * d, width, torch.bfloat16, seed=500 + i, device="cuda",
                                window=False)
        y, _ = la.short_conv_varlen(x[0], w, cu, heads=H, silu=True, l2norm=(i < 2))
        ys.append(y)
        refs.append(oconv.short_conv_packed(f64(x[0]), f64(w), cu.tolist(), None, H=H, silu=True,
                                            l2norm=(i < 2))[0])
    for y, r in zip(ys, refs):
        assert slice_rel_err(f64(y), r, lead=1) < 8e-3
    g = torch.Generator(device="cuda").manual_seed(9)
    gate = torch.sigmoid(torch.randn(H, T, generator=g, device="cuda") + 3.0)
    beta = torch.sigmoid(torch.randn(H, T, generator=g, device="cuda"))
    S0 = torch.randn(N, H, d, d, generator=g, device="cuda") * 0.05
    o, S, _ = la.prefill_varlen(*ys, cu, mode=2, gate=gate, beta=beta, state=S0.clone())
    la.check_status()
    ro, rS, _ = oracle.prefill_packed(2, f64(ys[0]), f64(ys[1]), f64(ys[2]), cu.tolist(), f64(gate),
                                      f64(beta), f64(S0))
    assert seq_err(f64(o), ro, cu.tolist()) < TOL[torch.bfloat16]
    assert slice_rel_err(f64(S), rS) < TOL[torch.bfloat16]
    # one decode step per sequence from the packed final states
    q1, k1, v1 = (torch.nn.functional.normalize(torch.randn(N, H, d, generator=g, device="cuda"), dim=-1)
                  .to(torch.bfloat16) for _ in range(3))
    a1 = torch.sigmoid(torch.randn(N, H, generator=g, device="cuda") + 3.0)
    b1 = torch.sigmoid(torch.randn(N, H, generator=g, device="cuda"))
    od, S2, _ = la.decode_step(q1, k1, v1, mode=2, state=S.clone(), gate=a1, beta=b1)
    la.check_status()
    rod, rS2, _ = oracle.decode_step(2, f64(q1), f64(k1), f64(v1), f64(a1), f64(b1), f64(S))
    assert slice_rel_err(f64(od), rod, lead=1) < TOL[torch.bfloat16]
    assert slice_rel_err(f64(S2), rS2) < TOL[torch.bfloat16]
