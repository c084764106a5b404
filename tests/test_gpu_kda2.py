"""GPU parity of the two-pass KDA prefill (mode 3) against the fp64 oracle.

Dense KDA calls (bf16, d = 128) with 16 to 37 head rows and a workspace take the two-pass
variant: pass 1 writes one record per chunk (A, T diag(b), Q o Gam, W = T diag(b)(K o Gam),
K o 2^(lam_L - lam) and Gam_L, the per-channel decays of "The delta rule and Gated
DeltaNet" moved into the operands) and the gated-delta chain kernel carries the state with
a per-row decay.  Without a workspace, or with a gate tensor the bulk copies cannot read
(not 16-byte aligned), the same call takes the segmented kernels.  Checked here against the
oracle's recurrence, per (batch, head) slice to the bf16 tolerance: ragged tails and chunk
edges, one token, weak and strong decay, gates far below the Gram products' floor, a large
initial state that the gates must erase, no gate, 16 to 37 head rows, and the fallbacks.
"""
import itertools

import numpy as np
import pytest
import torch

import workloads as W
from parity_util import TOL, f64, oracle_prefill_slices, pick, slice_rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def la():
    import gated_delta_rule_attention_b200 as m
    m.library()
    return m


def kda(T, B=1, H=16, gate="softplus", shift=0.0, seed=600):
    return W.Workload("kda", 3, torch.bfloat16, B=B, H=H, T=T, dk=128, dv=128, seed=seed,
                      qk_scale=1 / np.sqrt(128), qk_l2norm=True, gate=gate, gate_shift=shift,
                      beta=True)


def run(la, inp, init, workspace="auto", gate=None):
    """One call; returns o, S and the number of kernel launches it made."""
    state = inp["state0"].clone()
    la.launch_timing(True)
    try:
        o, S, _ = la.prefill(inp["q"], inp["k"], inp["v"], mode=3,
                             gate=inp["gate"] if gate is None else gate, beta=inp["beta"],
                             state=state, init_state=init, workspace=workspace)
        torch.cuda.synchronize()
        n = len(la.launch_times())
    finally:
        la.launch_timing(False)
    la.check_status()
    return o, S, n


def check(la, w, inp, init=False, heads=None, both=True):
    """The two-pass variant (default workspace: two launches) and, with `both`, the
    segmented kernels (no workspace), each against the oracle."""
    if heads is None:
        heads = list(itertools.product(range(w.B), range(w.H)))
    ro, rS, _ = oracle_prefill_slices(3, inp, heads, init_state=init)
    tol = TOL[torch.bfloat16]
    for ws in (("auto", None) if both else ("auto",)):
        o, S, n = run(la, inp, init, workspace=ws)
        if ws == "auto":
            assert n == 2, f"two-pass variant expected (2 launches), got {n}"
        eo = slice_rel_err(pick(o, heads), ro, lead=1)
        eS = slice_rel_err(pick(S, heads), rS, lead=1)
        assert eo <= tol, f"workspace {ws}: output rel err {eo:.3e} > {tol}"
        assert eS <= tol, f"workspace {ws}: state rel err {eS:.3e} > {tol}"


@pytest.mark.parametrize("T", [1, 2, 63, 64, 65, 127, 200, 333])
def test_kda2_lengths(la, T):
    w = kda(T)
    check(la, w, W.prefill_inputs(w, device="cuda"))


@pytest.mark.parametrize("shift", [-3.0, 0.0, 4.0])
def test_kda2_decay_regimes_with_state(la, shift):
    """Weak decay (a near 0.95), the default recipe, strong decay (a near 0.02), all with an
    initial state."""
    w = kda(150, shift=shift, seed=601)
    check(la, w, W.prefill_inputs(w, device="cuda", init_state_std=0.05), init=True)


@pytest.mark.parametrize("shift", [6.0, 9.0])
def test_kda2_gates_below_the_gram_floor(la, shift):
    """Gates near 0.0025 and down to 1e-4 and below: the diagonal blocks of the Gram products
    bound each log2 gate at -7.5 (pair weights across such a gate are already below 0.0055);
    every state-facing factor takes the gates as given."""
    w = kda(200, shift=shift, seed=602)
    inp = W.prefill_inputs(w, device="cuda", init_state_std=0.05)
    if shift == 9.0:
        assert float(inp["gate"].min()) < 1e-4
    check(la, w, inp, init=True, both=False)


@pytest.mark.parametrize("shift", [4.0, 9.0])
def test_kda2_large_initial_state_is_forgotten(la, shift):
    """An initial state of std 10 under gates below 0.02: every output must show it decayed
    by the exact per-channel products, which a floor on the state-facing factors would not."""
    w = kda(160, shift=shift, seed=603)
    check(la, w, W.prefill_inputs(w, device="cuda", init_state_std=10.0), init=True, both=False)


def test_kda2_no_gate(la):
    """a = 1 in every channel: the delta rule alone, the state carried unscaled."""
    w = kda(260, gate="none", seed=604)
    check(la, w, W.prefill_inputs(w, device="cuda", init_state_std=0.05), init=True)


@pytest.mark.parametrize("B,H", [(2, 8), (1, 37), (4, 5)])
def test_kda2_head_rows(la, B, H):
    """16, 37 (148 CTAs) and 20 head rows, ragged length."""
    w = kda(100, B=B, H=H, seed=605)
    check(la, w, W.prefill_inputs(w, device="cuda", init_state_std=0.05), init=True, both=False)


def test_kda2_unaligned_gate_takes_segmented_kernels(la):
    """A gate tensor 4 bytes off a 16-byte boundary (allowed by the interface) cannot feed the
    bulk copies: the call falls back to the segmented kernels, with the same results."""
    w = kda(130, seed=606)
    inp = W.prefill_inputs(w, device="cuda", init_state_std=0.05)
    g = inp["gate"]
    buf = torch.empty(g.numel() + 1, device="cuda", dtype=torch.float32)
    gu = buf[1:].view(g.shape)
    gu.copy_(g)
    assert gu.data_ptr() % 16 != 0
    o, S, n = run(la, inp, True, gate=gu)
    assert n != 2
    heads = list(itertools.product(range(w.B), range(w.H)))
    ro, rS, _ = oracle_prefill_slices(3, inp, heads, init_state=True)
    assert slice_rel_err(pick(o, heads), ro, lead=1) <= TOL[torch.bfloat16]
    assert slice_rel_err(pick(S, heads), rS, lead=1) <= TOL[torch.bfloat16]


def test_kda2_split_sequence_continues(la):
    """Two calls carrying the state equal one call over the whole sequence."""
    w = kda(300, seed=607)
    inp = W.prefill_inputs(w, device="cuda")
    o, S, _ = run(la, inp, False)
    cut = 137
    first = {k: (v[:, :, :cut].contiguous() if k in ("q", "k", "v", "gate", "beta") else v) for k, v in inp.items()}
    second = {k: (v[:, :, cut:].contiguous() if k in ("q", "k", "v", "gate", "beta") else v) for k, v in inp.items()}
    oa, Sa, _ = run(la, first, False)
    second["state0"] = Sa
    ob, Sb, _ = run(la, second, True)
    assert slice_rel_err(f64(torch.cat([oa, ob], dim=2)), f64(o)) <= TOL[torch.bfloat16]
    assert slice_rel_err(f64(Sb), f64(S)) <= TOL[torch.bfloat16]
