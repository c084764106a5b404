"""GPU parity at the full workload sizes, in the launch configuration the benchmark times.

The CUDA path runs the whole workload (every batch entry and head, the same
``prefill`` / ``decode_step`` call with the library's default chunk and workspace that
``bench.py`` times); the fp64 oracle recomputes a sample of (batch, head) slices over
the full sequence, and every output and final-state element of those slices is
compared.  Tolerance: per-slice max relative error 2e-2 (bf16 I/O) / 2e-3 (fp32 I/O).
"""
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


def _check_prefill(la, w, heads):
    inp = W.prefill_inputs(w, device="cuda")
    o, S, z = la.prefill(inp["q"], inp["k"], inp["v"], mode=w.mode, gate=inp["gate"],
                         beta=inp["beta"], chunk=w.chunk)
    la.check_status()
    assert torch.isfinite(o.float()).all() and torch.isfinite(S).all()
    ro, rS, rz = oracle_prefill_slices(w.mode, inp, heads)
    tol = TOL[w.dtype]
    eo = slice_rel_err(pick(o, heads), ro, lead=1)
    eS = slice_rel_err(pick(S, heads), rS, lead=1)
    assert eo <= tol, f"{w.name}: output rel err {eo:.3e}"
    assert eS <= tol, f"{w.name}: state rel err {eS:.3e}"
    if w.mode == 0:
        assert slice_rel_err(pick(z, heads), rz, lead=1) <= tol
    return eo, eS


def test_elu1_f32_small_every_head(la):
    w = W.CONFIGS["elu1_f32_small"]
    _check_prefill(la, w, [(b, h) for b in range(w.B) for h in range(w.H)])


def test_elu1_bf16_b4h16t4096_sampled(la):
    _check_prefill(la, W.CONFIGS["elu1_bf16_b4h16t4096"], [(0, 0), (1, 7), (2, 11), (3, 15)])


def test_gated_bf16_b8h16t8192_sampled(la):
    _check_prefill(la, W.CONFIGS["gated_bf16_b8h16t8192"], [(0, 0), (3, 5), (7, 15)])


def test_gdn_bf16_b2h16t32768_sampled(la):
    _check_prefill(la, W.CONFIGS["gdn_bf16_b2h16t32768"], [(0, 0), (1, 9), (1, 15)])


def test_kda_bf16_b2h16t32768_sampled(la):
    _check_prefill(la, W.CONFIGS["kda_bf16_b2h16t32768"], [(0, 0), (1, 15)])


@pytest.mark.parametrize("name", ["gated_bf16_b8h16t8192", "gdn_bf16_b2h16t32768",
                                  "kda_bf16_b2h16t32768"])
def test_full_size_weak_decay_state_path(la, name):
    """At the configs' own gate distribution the state decays by ~e^-50 per chunk, so
    the carried state barely matters; a ~0.98 gate at the same sizes (fewer heads)
    makes the segment chaining and the carried state dominate."""
    w = W.variant(W.CONFIGS[name], B=1, H=4, gate_shift=-4.0)
    _check_prefill(la, w, [(0, 0), (0, 3)])


@pytest.mark.parametrize("name", ["gdn_decode_n256h32", "kda_decode_n256h32"])
def test_decode_n256h32_sampled(la, name):
    w = W.CONFIGS[name]
    steps = 12
    inp = W.decode_inputs(w, steps=steps, device="cuda")
    S = inp["state0"].clone()
    o = torch.empty(w.B, w.H, w.dv, device="cuda", dtype=w.dtype)
    seqs = [0, 77, 255]
    Sr = f64(inp["state0"][seqs])
    for t in range(steps):
        la.decode_step(inp["q"][t], inp["k"][t], inp["v"][t], mode=w.mode, state=S,
                       gate=inp["gate"][t], beta=inp["beta"][t], o=o)
        ro, Sr, _ = oracle.decode_step(w.mode, f64(inp["q"][t][seqs]), f64(inp["k"][t][seqs]),
                                       f64(inp["v"][t][seqs]), f64(inp["gate"][t][seqs]),
                                       f64(inp["beta"][t][seqs]), Sr)
        la.check_status()
        assert slice_rel_err(f64(o[seqs]), ro) <= TOL[w.dtype], t
    assert slice_rel_err(f64(S[seqs]), Sr) <= TOL[w.dtype]


def _decode_oracle(mode, inp, seqs):
    """The oracle over the decode steps of the listed sequences: the same tokens as one
    recurrent prefill from the seeded state gives every step's output and the final state.
    Returns (o [n, H, steps, d_v], S [n, H, d_v, d_k])."""
    sel = lambda t: None if t is None else f64(t[:, seqs].movedim(0, 2).contiguous())
    o, S, _ = oracle.prefill(mode, sel(inp["q"]), sel(inp["k"]), sel(inp["v"]), sel(inp["gate"]),
                             sel(inp["beta"]), f64(inp["state0"][seqs]))
    return o, S


@pytest.mark.parametrize("shift", [0.0, -4.0])
def test_decode_n256h32_1000_steps(la, shift):
    """The configured decode workload over its full length: 1000 sequential
    ``decode_step`` calls on 256 sequences x 32 heads (the launch the benchmark times).
    Every step's output of 16 sequences is compared with the oracle; at the configured
    gates also the final state of all 256 sequences.  With weak decay (a ~ 0.98) the state
    carries ~50 steps of history, so rounding in the fp32 state could accumulate there."""
    w = W.variant(W.CONFIGS["gdn_decode_n256h32"], gate_shift=shift)
    steps = w.T
    assert steps == 1000
    inp = W.decode_inputs(w, steps=steps, device="cuda")
    S = inp["state0"].clone()
    o = torch.empty(w.B, w.H, w.dv, device="cuda", dtype=w.dtype)
    seqs = list(range(0, w.B, 16))
    outs = torch.empty(len(seqs), w.H, steps, w.dv, device="cuda", dtype=w.dtype)
    for t in range(steps):
        la.decode_step(inp["q"][t], inp["k"][t], inp["v"][t], mode=w.mode, state=S,
                       gate=inp["gate"][t], beta=inp["beta"][t], o=o)
        outs[:, :, t] = o[seqs]
    la.check_status()
    ro, rS = _decode_oracle(w.mode, inp, seqs)
    assert slice_rel_err(f64(outs), ro) <= TOL[w.dtype]
    assert slice_rel_err(f64(S[seqs]), rS) <= TOL[w.dtype]
    if shift == 0.0:
        for g in range(0, w.B, 32):
            grp = list(range(g, g + 32))
            _, rS = _decode_oracle(w.mode, inp, grp)
            assert slice_rel_err(f64(S[grp]), rS) <= TOL[w.dtype], g


@pytest.mark.parametrize("mode", [0, 1, 2])
def test_segmented_equals_single_pass(la, mode):
    """The workspace (parallel segments chained by the combine kernel) and the
    single-pass run agree with each other and with the oracle."""
    w = W.Workload("seg", mode, torch.bfloat16, B=1, H=3, T=3000, dk=128, dv=128, seed=31,
                   qk_scale=1 / np.sqrt(128), qk_l2norm=(mode == 2),
                   gate="none" if mode == 0 else "softplus", gate_shift=-4.0, beta=(mode == 2))
    assert la.workspace_size(mode, torch.bfloat16, 1, 3, 3000, 128, 128) > 0
    inp = W.prefill_inputs(w, device="cuda", init_state_std=0.05)
    z0 = torch.rand(1, 3, 128, device="cuda") + 1 if mode == 0 else None
    outs = []
    for ws in ("auto", None):
        st = inp["state0"].clone()
        z = None if z0 is None else z0.clone()
        o, S, zz = la.prefill(inp["q"], inp["k"], inp["v"], mode=mode, gate=inp["gate"],
                              beta=inp["beta"], state=st, z=z, init_state=True, workspace=ws)
        la.check_status()
        outs.append((o.float(), S, zz))
    heads = [(0, h) for h in range(3)]
    ro, rS, rz = oracle_prefill_slices(mode, inp, heads, init_state=True, z0=z0)
    for o, S, zz in outs:
        assert slice_rel_err(pick(o, heads), ro, lead=1) <= TOL[w.dtype]
        assert slice_rel_err(pick(S, heads), rS, lead=1) <= TOL[w.dtype]
