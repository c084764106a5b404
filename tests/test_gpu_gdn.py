"""GPU parity of the single-pass gated-delta prefill against the fp64 oracle.

Dense gated-delta calls with 16 to 37 head rows take the single-pass kernel that splits
each head's d_v rows over four CTAs; these cases pin it element by element: ragged tails
and chunk edges, one token, weak decay and no gate (the carried state dominates), strong
decay, beta near 0 and 1, an initial state, split prefill followed by decode steps, and
agreement with the segmented kernels (8 head rows).  Tolerance: max relative error per
(batch, head) slice of 2e-2 (bf16 I/O).
"""
import itertools

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from parity_util import TOL, f64, oracle_prefill_slices, pick, slice_rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def la():
    import gated_delta_rule_attention_b200 as m
    m.library()
    return m


def gdn(T, B=1, H=16, gate="softplus", shift=0.0, seed=500):
    return W.Workload("gdn", 2, torch.bfloat16, B=B, H=H, T=T, dk=128, dv=128, seed=seed,
                      qk_scale=1 / np.sqrt(128), qk_l2norm=True, gate=gate, gate_shift=shift,
                      beta=True)


def check(la, w, inp, init=False, heads=None):
    """Both variants: the single pass (no workspace) and the two-pass variant (pass 1 forms
    every chunk's A, T diag(b), T diag(b g) into the workspace)."""
    if heads is None:
        heads = list(itertools.product(range(w.B), range(w.H)))
    ro, rS, _ = oracle_prefill_slices(2, inp, heads, init_state=init)
    for ws in (None, "auto"):
        state = inp["state0"].clone()
        o, S, _ = la.prefill(inp["q"], inp["k"], inp["v"], mode=2, gate=inp["gate"],
                             beta=inp["beta"], state=state, init_state=init, workspace=ws)
        la.check_status()
        eo = slice_rel_err(pick(o, heads), ro, lead=1)
        eS = slice_rel_err(pick(S, heads), rS, lead=1)
        assert eo <= TOL[torch.bfloat16] and eS <= TOL[torch.bfloat16], (ws, eo, eS)
    tol = TOL[torch.bfloat16]
    assert eo <= tol, f"output rel err {eo:.3e} > {tol}"
    assert eS <= tol, f"state rel err {eS:.3e} > {tol}"
    return eo, eS


@pytest.mark.parametrize("T", [1, 2, 63, 64, 65, 127, 128, 200, 333])
def test_single_pass_lengths(la, T):
    w = gdn(T)
    check(la, w, W.prefill_inputs(w, device="cuda"))


@pytest.mark.parametrize("gate,shift", [("softplus", -4.0), ("none", 0.0), ("softplus", 3.0)])
def test_single_pass_decay_regimes(la, gate, shift):
    """a ~ 0.98 and a = 1 make the state of earlier chunks dominate; a ~ 0.05 forgets fast."""
    w = gdn(1000, B=2, H=8, gate=gate, shift=shift, seed=501)
    check(la, w, W.prefill_inputs(w, device="cuda"))


def test_single_pass_initial_state(la):
    w = gdn(150, B=2, H=8, shift=-3.0, seed=502)
    check(la, w, W.prefill_inputs(w, device="cuda", init_state_std=0.05), init=True)


def test_single_pass_large_initial_state_weak_decay(la):
    """A large start state kept by weak decay: the state path carries the output."""
    w = gdn(300, B=1, H=16, shift=-5.0, seed=503)
    check(la, w, W.prefill_inputs(w, device="cuda", init_state_std=1.0), init=True)


@pytest.mark.parametrize("beta_shift", [-8.0, 8.0])
def test_single_pass_beta_extremes(la, beta_shift):
    """beta -> 0 (pure decay of the state) and beta -> 1 (full overwrite along k)."""
    w = gdn(200, B=1, H=16, shift=-2.0, seed=504)
    inp = W.prefill_inputs(w, device="cuda", init_state_std=0.1)
    inp["beta"] = torch.sigmoid(torch.logit(inp["beta"].clamp(1e-6, 1 - 1e-6)) + beta_shift).contiguous()
    check(la, w, inp, init=True)


def test_single_pass_split_then_decode(la):
    """prefill(T1); prefill(T2) from that state; decode steps == the oracle over the whole."""
    w = gdn(190, B=1, H=16, shift=-3.0, seed=505)
    inp = W.prefill_inputs(w, device="cuda")
    T1, T2 = 77, 100
    sl = lambda t, a, b: t[:, :, a:b].contiguous()
    o1, S, _ = la.prefill(sl(inp["q"], 0, T1), sl(inp["k"], 0, T1), sl(inp["v"], 0, T1), mode=2,
                          gate=sl(inp["gate"], 0, T1), beta=sl(inp["beta"], 0, T1), workspace=None)
    o2, S, _ = la.prefill(sl(inp["q"], T1, T1 + T2), sl(inp["k"], T1, T1 + T2),
                          sl(inp["v"], T1, T1 + T2), mode=2, gate=sl(inp["gate"], T1, T1 + T2),
                          beta=sl(inp["beta"], T1, T1 + T2), state=S, init_state=True,
                          workspace=None)
    outs = [o1, o2]
    for t in range(T1 + T2, w.T):
        o, S, _ = la.decode_step(inp["q"][:, :, t].contiguous(), inp["k"][:, :, t].contiguous(),
                                 inp["v"][:, :, t].contiguous(), state=S, mode=2,
                                 gate=inp["gate"][:, :, t].contiguous(),
                                 beta=inp["beta"][:, :, t].contiguous())
        outs.append(o[:, :, None])
    la.check_status()
    o = torch.cat(outs, dim=2)
    heads = list(itertools.product(range(w.B), range(w.H)))
    ro, rS, _ = oracle_prefill_slices(2, inp, heads)
    assert slice_rel_err(pick(o, heads), ro, lead=1) <= TOL[torch.bfloat16]
    assert slice_rel_err(pick(S, heads), rS, lead=1) <= TOL[torch.bfloat16]


def test_single_pass_matches_segmented_path(la):
    """16 head rows through the single-pass kernel equal the same heads as two calls of 8
    head rows, which take the segmented kernels (local, transition, combine, outputs)."""
    w = gdn(1500, B=1, H=16, shift=-1.0, seed=506)
    inp = W.prefill_inputs(w, device="cuda")
    # 16 head rows: the two-pass variant's per-chunk factors (24 KB a chunk); 8: segments
    assert la.workspace_size(2, torch.bfloat16, 1, 16, w.T, 128, 128) == 16 * ((w.T + 63) // 64) * 24576
    assert la.workspace_size(2, torch.bfloat16, 1, 8, w.T, 128, 128) > 0
    o, S, _ = la.prefill(inp["q"], inp["k"], inp["v"], mode=2, gate=inp["gate"], beta=inp["beta"])
    for h in (0, 8):
        sl = lambda t: t[:, h:h + 8].contiguous()
        o2, S2, _ = la.prefill(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), mode=2, gate=sl(inp["gate"]),
                               beta=sl(inp["beta"]))
        assert slice_rel_err(f64(o[:, h:h + 8]), f64(o2)) <= TOL[torch.bfloat16]
        assert slice_rel_err(f64(S[:, h:h + 8]), f64(S2)) <= TOL[torch.bfloat16]
    la.check_status()
