"""GPU parity of the fused convolution + gated-delta prefill (``la_prefill_conv``).

The short causal convolution of the lesson page's section "Hybrids of 2025: Qwen3-Next and
Kimi Linear" runs inside the loads of the Gated DeltaNet prefill ("The delta rule and
Gated DeltaNet").  Checked here:

* against the fp64 oracle chain, ``oracle.conv.short_conv`` for q, k, v, then
  ``oracle.prefill`` in mode 2 on the bf16 convolution outputs the attention sees: the
  convolution outputs element by element (the tolerance of the stand-alone convolution
  tests), the outputs o and the final state S by the prefill tolerance, the carried
  windows exactly (they are copies);
* against the unfused path on the same kernels, bit for bit: three ``la_short_conv``
  calls and ``la_prefill`` with a workspace (the two-pass gated-delta kernels, which the
  library selects when 4 B H lies in [64, 148]) give identical y, o and S;
* widths 1 to 4, with and without SiLU and the norm, with and without a carried window
  and an initial state, ragged and short sequences (T = 1, T < 64, T not a multiple of
  64), and the arguments the entry point refuses.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from oracle import conv as oconv
from parity_util import TOL, f64, slice_rel_err

pytestmark = pytest.mark.gpu

BF = torch.bfloat16


@pytest.fixture(scope="module")
def la():
    import gated_delta_rule_attention_b200 as m
    m.library()
    return m


def close(y, ref, silu):
    """The stand-alone convolution tests' bound: one bf16 rounding of an fp32 result (2^-8
    relative), plus 2^-10 max|r| when the sigmoid comes from tanh.approx (else 1e-5)."""
    y = f64(y)
    ref = np.asarray(ref)
    atol = (2.0 ** -10 if silu else 1e-5) * max(np.abs(ref).max(), 1e-30)
    bad = np.abs(y - ref) > 2.0 ** -8 * np.abs(ref) + atol
    assert not bad.any(), f"{bad.sum()} of {bad.size} outside tolerance; max err {np.abs(y - ref).max():.3e}"


def inputs(B, T, H, width, seed, window=True):
    C = H * 128
    xs = [W.conv_inputs(B, T, C, width, BF, seed=seed + i, device="cuda", window=window) for i in range(3)]
    gen = torch.Generator(device="cuda").manual_seed(seed + 9)
    gate = torch.sigmoid(torch.randn(B, H, T, generator=gen, device="cuda") + 3.0)
    beta = torch.sigmoid(torch.randn(B, H, T, generator=gen, device="cuda"))
    win = torch.stack([w for (_, _, w) in xs]) if window and width > 1 else None
    return xs, win, gate, beta


CASES = [  # (B, T, H, width)
    (1, 1, 2, 4), (1, 3, 2, 4), (2, 63, 2, 4), (1, 64, 1, 4), (2, 70, 2, 4), (1, 200, 3, 4),
    (1, 130, 2, 3), (2, 129, 1, 2), (1, 77, 2, 1),
]


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("window", [False, True])
def test_fused_matches_oracle(la, case, window):
    B, T, H, width = case
    xs, win, gate, beta = inputs(B, T, H, width, seed=11 * T + width, window=window)
    o, S, y, wout = la.prefill_conv(*(x for x, _, _ in xs), *(w for _, w, _ in xs), heads=H, gate=gate,
                                    beta=beta, window=win)
    la.check_status()
    refs = []
    for i, (x, w, _) in enumerate(xs):
        r, rw = oconv.short_conv(f64(x), f64(w), None if win is None else f64(win[i]), H=H, silu=True,
                                 l2norm=(i < 2))
        close(y[i], r, True)
        if width > 1:
            np.testing.assert_array_equal(f64(wout[i]), rw)
        refs.append(r)
    ro, rS, _ = oracle.prefill(2, f64(y[0]), f64(y[1]), f64(y[2]), f64(gate), f64(beta))
    assert slice_rel_err(f64(o), ro) < TOL[BF]
    assert slice_rel_err(f64(S), rS) < TOL[BF]


@pytest.mark.parametrize("flags", [(True, True, True), (False, False, False), (True, False, False),
                                   (False, True, True), (True, True, False)])
def test_fused_flags_and_initial_state(la, flags):
    qk_silu, qk_l2, v_silu = flags
    B, T, H, width = 1, 150, 2, 4
    xs, win, gate, beta = inputs(B, T, H, width, seed=5)
    S0 = torch.randn(B, H, 128, 128, device="cuda") * 0.05
    o, S, y, _ = la.prefill_conv(*(x for x, _, _ in xs), *(w for _, w, _ in xs), heads=H, gate=gate,
                                 beta=beta, window=win, qk_silu=qk_silu, qk_l2norm=qk_l2, v_silu=v_silu,
                                 state=S0.clone())
    la.check_status()
    for i, (x, w, _) in enumerate(xs):
        silu = v_silu if i == 2 else qk_silu
        r, _ = oconv.short_conv(f64(x), f64(w), f64(win[i]), H=H, silu=silu, l2norm=(qk_l2 and i < 2))
        close(y[i], r, silu)
    if not qk_l2:
        return   # unnormalised keys make the delta rule's I - b k k^T expand: only y is compared
    ro, rS, _ = oracle.prefill(2, f64(y[0]), f64(y[1]), f64(y[2]), f64(gate), f64(beta), state=f64(S0))
    assert slice_rel_err(f64(o), ro) < TOL[BF]
    assert slice_rel_err(f64(S), rS) < TOL[BF]


@pytest.mark.parametrize("T", [256, 1000])
def test_fused_equals_unfused_bit_for_bit(la, T):
    """Same kernels, same arithmetic: B H = 16 selects the two-pass gated-delta kernels for
    la_prefill with a workspace too."""
    B, H, width = 1, 16, 4
    xs, win, gate, beta = inputs(B, T, H, width, seed=T)
    o, S, y, wout = la.prefill_conv(*(x for x, _, _ in xs), *(w for _, w, _ in xs), heads=H, gate=gate,
                                    beta=beta, window=win)
    ys, wos = [], []
    for i, (x, w, _) in enumerate(xs):
        yi, wi = la.short_conv(x, w, heads=H, window=win[i], silu=True, l2norm=(i < 2))
        ys.append(yi)
        wos.append(wi)
    o2, S2, _ = la.prefill(*ys, mode=la.MODE_GATED_DELTA, gate=gate, beta=beta)
    la.check_status()
    for i in range(3):
        assert torch.equal(y[i], ys[i]), f"y[{i}]"
        assert torch.equal(wout[i], wos[i]), f"window[{i}]"
    assert torch.equal(o, o2)
    assert torch.equal(S, S2)


def test_fused_split_sequence_continues(la):
    """Two calls carrying the windows and the state equal one call over the whole sequence."""
    B, T, H, width, cut = 2, 190, 2, 4, 77
    xs, win, gate, beta = inputs(B, T, H, width, seed=3)
    args = dict(heads=H)
    x3, w3 = [x for x, _, _ in xs], [w for _, w, _ in xs]
    o, S, _, wout = la.prefill_conv(*x3, *w3, gate=gate, beta=beta, window=win, **args)
    oa, Sa, _, wa = la.prefill_conv(*(x[:, :cut].contiguous() for x in x3), *w3, gate=gate[..., :cut].contiguous(),
                                    beta=beta[..., :cut].contiguous(), window=win, **args)
    ob, Sb, _, wb = la.prefill_conv(*(x[:, cut:].contiguous() for x in x3), *w3,
                                    gate=gate[..., cut:].contiguous(), beta=beta[..., cut:].contiguous(),
                                    window=wa.clone(), state=Sa, **args)
    la.check_status()
    assert torch.equal(wb, wout)
    both = torch.cat([oa, ob], dim=2)
    assert slice_rel_err(f64(both), f64(o)) < TOL[BF]
    assert slice_rel_err(f64(Sb), f64(S)) < TOL[BF]


def test_fused_refuses_bad_arguments(la):
    B, T, H, width = 1, 64, 2, 4
    xs, win, gate, beta = inputs(B, T, H, width, seed=1)
    x3, w3 = [x for x, _, _ in xs], [w for _, w, _ in xs]
    with pytest.raises(la.LaError):   # the window updated in place is refused here
        la.prefill_conv(*x3, *w3, heads=H, gate=gate, beta=beta, window=win, window_out=win)
    n = B * T * H * 128
    buf = torch.zeros(4 * n, dtype=BF, device="cuda")
    xq = buf[:n].view(B, T, H * 128)
    xq.copy_(x3[0])
    with pytest.raises(la.LaError):   # y over an input
        la.prefill_conv(xq, *x3[1:], *w3, heads=H, gate=gate, beta=beta, y=buf[:3 * n].view(3, B, H, T, 128))


def test_fused_full_size_sampled(la):
    """The benchmark's layer workload in its launch configuration (B2 H16 T32768): the fused
    call equals the separate calls bit for bit, the convolution outputs match the oracle on
    sampled token ranges, and sampled heads' outputs and final states match the oracle's
    recurrence on the convolved q, k, v."""
    lw = W.LAYER_CONFIGS["gdn_layer_fused_bf16_b2h16t32768"]
    cw, pw = lw.conv, lw.prefill
    B, H, T = cw.B, cw.H, cw.T
    xs = [W.conv_inputs(B, T, H * 128, cw.width, cw.dtype, seed=cw.seed + 10 * i, device="cuda", window=False)
          for i in range(3)]
    inp = W.prefill_inputs(pw, device="cuda")
    gate, beta = inp["gate"], inp["beta"]
    del inp
    x3, w3 = [x for x, _, _ in xs], [w for _, w, _ in xs]
    o, S, y, wout = la.prefill_conv(*x3, *w3, heads=H, gate=gate, beta=beta)
    ys = [la.short_conv(x3[i], w3[i], heads=H, silu=True, l2norm=(i < 2))[0] for i in range(3)]
    o2, S2, _ = la.prefill(*ys, mode=la.MODE_GATED_DELTA, gate=gate, beta=beta)
    la.check_status()
    for i in range(3):
        assert torch.equal(y[i], ys[i]), f"y[{i}]"
    assert torch.equal(o, o2) and torch.equal(S, S2)
    for i in range(3):
        np.testing.assert_array_equal(f64(wout[i]), f64(x3[i][:, -3:]))
    for b, t0, n in [(0, 0, 40), (1, 17000, 33), (1, T - 50, 50)]:
        for i in range(3):
            win = x3[i][b:b + 1, t0 - 3:t0] if t0 >= 3 else None
            ref, _ = oconv.short_conv(f64(x3[i][b:b + 1, t0:t0 + n]), f64(w3[i]), None if win is None else f64(win),
                                      H=H, silu=True, l2norm=(i < 2))
            close(y[i][b:b + 1, :, t0:t0 + n], ref, True)
    for b, h in [(0, 3), (1, 12)]:
        sl = lambda t: f64(t[b:b + 1, h:h + 1])
        ro, rS, _ = oracle.prefill(2, sl(y[0]), sl(y[1]), sl(y[2]), sl(gate), sl(beta))
        assert slice_rel_err(sl(o), ro) < TOL[BF], f"o head ({b},{h})"
        assert slice_rel_err(sl(S), rS) < TOL[BF], f"S head ({b},{h})"
