"""GPU parity of the short causal convolution prologue against the fp64 oracle.

``la_short_conv`` / ``la_short_conv_step`` through the C ABI against ``oracle.conv`` on
seeded inputs: every width, both head sizes and dtypes, with and without SiLU, the L2
norm and a carried window, sequences shorter than the window, one thread run, several
runs with a ragged tail, the window updated in place, decode steps continuing a
prefill, the prologue feeding the Gated DeltaNet prefill, and the full-size workload in
the benchmark's launch configuration on sampled token ranges.

Tolerance, element by element: |y - r| <= rtol |r| + atol with rtol = 2^-8 for bf16
output (one rounding of an fp32 result: at most 2^-9 relative) and 1e-5 for fp32, and
atol = 1e-5 max|r| for the fp32 sum of width products.  With SiLU and bf16 output the
kernel's sigmoid comes from the tanh.approx instruction (absolute error below 2^-11,
so at most |u| 2^-12 on the output): atol is then 2^-10 max|r|.  The carried window is
a copy of inputs and must match exactly.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from oracle import conv as oconv
from parity_util import TOL, f64, slice_rel_err

pytestmark = pytest.mark.gpu

RTOL = {torch.bfloat16: 2.0 ** -8, torch.float32: 1e-5}


@pytest.fixture(scope="module")
def la():
    import gated_delta_rule_attention_b200 as m
    m.library()
    return m


def close(y, ref, dtype, silu=False):
    y = f64(y)
    ref = np.asarray(ref)
    atol = (2.0 ** -10 if (silu and dtype == torch.bfloat16) else 1e-5) * max(np.abs(ref).max(), 1e-30)
    bad = np.abs(y - ref) > RTOL[dtype] * np.abs(ref) + atol
    assert not bad.any(), (f"{bad.sum()} of {bad.size} outside tolerance; max abs err "
                           f"{np.abs(y - ref).max():.3e}")


CASES = [  # (B, T, H, d, width): one run, several runs with ragged tails, odd lengths
    (2, 1, 3, 64, 4), (2, 2, 3, 64, 4), (1, 3, 2, 128, 4), (2, 37, 3, 64, 4),
    (2, 100, 2, 128, 4), (3, 64, 1, 64, 3), (2, 70, 2, 128, 2), (1, 45, 2, 64, 1),
    (1, 129, 2, 128, 4), (2, 200, 3, 64, 4), (1, 9, 1, 128, 4),
]


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("silu,l2", [(False, False), (True, False), (False, True), (True, True)])
def test_conv_matches_oracle(la, dtype, case, silu, l2):
    B, T, H, d, width = case
    x, w, win = W.conv_inputs(B, T, H * d, width, dtype, seed=T * 7 + width, device="cuda")
    y, wout = la.short_conv(x, w, heads=H, window=win if width > 1 else None, silu=silu, l2norm=l2)
    torch.cuda.synchronize()
    ref, rwin = oconv.short_conv(f64(x), f64(w), f64(win) if width > 1 else None, H=H,
                                 silu=silu, l2norm=l2)
    close(y, ref, dtype, silu)
    np.testing.assert_array_equal(f64(wout), rwin)


@pytest.mark.parametrize("T", [5, 33, 200])
def test_conv_zero_window_and_in_place_window(la, T):
    B, H, d, width = 2, 2, 128, 4
    x, w, win = W.conv_inputs(B, T, H * d, width, torch.bfloat16, seed=T, device="cuda")
    y0, _ = la.short_conv(x, w, heads=H, silu=True, l2norm=True)
    ref0, _ = oconv.short_conv(f64(x), f64(w), None, H=H, silu=True, l2norm=True)
    close(y0, ref0, torch.bfloat16, True)
    keep = win.clone()
    y1, wout = la.short_conv(x, w, heads=H, window=win, window_out=win, silu=True, l2norm=True)
    torch.cuda.synchronize()
    assert wout.data_ptr() == win.data_ptr()
    ref1, rwin = oconv.short_conv(f64(x), f64(w), f64(keep), H=H, silu=True, l2norm=True)
    close(y1, ref1, torch.bfloat16, True)
    np.testing.assert_array_equal(f64(win), rwin)


def test_conv_empty_sequence_copies_the_window(la):
    x, w, win = W.conv_inputs(2, 0, 256, 4, torch.bfloat16, seed=3, device="cuda")
    y, wout = la.short_conv(x, w, heads=2, window=win)
    torch.cuda.synchronize()
    assert y.shape == (2, 2, 0, 128)
    np.testing.assert_array_equal(f64(wout), f64(win))
    _, wz = la.short_conv(x, w, heads=2)
    torch.cuda.synchronize()
    assert float(wz.abs().max()) == 0.0


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_conv_step_continues_the_prefill(la, dtype):
    B, T, H, d, width = 3, 21, 2, 64, 4
    x, w, win = W.conv_inputs(B, T + 5, H * d, width, dtype, seed=11, device="cuda")
    _, cur = la.short_conv(x[:, :T].contiguous(), w, heads=H, window=win, silu=True, l2norm=True)
    ref, _ = oconv.short_conv(f64(x), f64(w), f64(win), H=H, silu=True, l2norm=True)
    for t in range(T, T + 5):
        yt = la.short_conv_step(x[:, t].contiguous(), w, cur, heads=H, silu=True, l2norm=True)
        torch.cuda.synchronize()
        close(yt, ref[:, :, t], dtype, True)
    np.testing.assert_array_equal(f64(cur), f64(x[:, -3:]))


def test_conv_prologue_feeds_the_gated_delta_prefill(la):
    """x -> conv (SiLU, q/k L2 norm) -> Gated DeltaNet prefill, against the oracle chain."""
    B, T, H, d, width = 2, 150, 2, 128, 4
    dt = torch.bfloat16
    xs = [W.conv_inputs(B, T, H * d, width, dt, seed=40 + i, device="cuda", window=False)
          for i in range(3)]
    ys = [la.short_conv(x, w, heads=H, silu=True, l2norm=(i < 2))[0] for i, (x, w, _) in enumerate(xs)]
    gen = torch.Generator(device="cuda").manual_seed(5)
    gate = torch.sigmoid(torch.randn(B, H, T, generator=gen, device="cuda") + 3.0)
    beta = torch.sigmoid(torch.randn(B, H, T, generator=gen, device="cuda"))
    o, S, _ = la.prefill(*ys, mode=la.MODE_GATED_DELTA, gate=gate, beta=beta)
    torch.cuda.synchronize()
    refs = [oconv.short_conv(f64(x), f64(w), None, H=H, silu=True, l2norm=(i < 2))[0]
            for i, (x, w, _) in enumerate(xs)]
    # the attention sees the bf16 outputs of the convolution, as on the GPU
    for y, r in zip(ys, refs):
        close(y, r, dt, True)
    ro, rS, _ = oracle.prefill(2, f64(ys[0]), f64(ys[1]), f64(ys[2]), f64(gate), f64(beta))
    assert slice_rel_err(f64(o), ro) < TOL[dt]
    assert slice_rel_err(f64(S), rS) < TOL[dt]


def test_conv_full_size_sampled(la):
    """The benchmark's workload and launch (B2 H16 T32768, d = 128, bf16, SiLU + L2 norm),
    checked on sampled token ranges: the oracle runs on each range with the three tokens
    before it as the carried window."""
    cw = W.CONV_CONFIGS["conv_bf16_b2h16t32768"]
    C = cw.H * cw.dk
    x, w, _ = W.conv_inputs(cw.B, cw.T, C, cw.width, cw.dtype, seed=cw.seed, device="cuda",
                            window=False)
    y, wout = la.short_conv(x, w, heads=cw.H, silu=True, l2norm=True)
    torch.cuda.synchronize()
    for b, t0, n in [(0, 0, 40), (1, 4093, 70), (0, 17000, 33), (1, cw.T - 50, 50)]:
        win = x[b:b + 1, t0 - 3:t0] if t0 >= 3 else None
        ref, _ = oconv.short_conv(f64(x[b:b + 1, t0:t0 + n]), f64(w),
                                  None if win is None else f64(win), H=cw.H, silu=True, l2norm=True)
        close(y[b:b + 1, :, t0:t0 + n], ref, cw.dtype, True)
    np.testing.assert_array_equal(f64(wout), f64(x[:, -3:]))


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("lengths", [[65, 0, 1, 64, 130, 63, 200, 2], [5], [0, 0, 3], [300, 1, 1, 70]])
@pytest.mark.parametrize("with_window", [False, True])
def test_conv_varlen_matches_oracle(la, dtype, lengths, with_window):
    H, d, width = 2, 128 if dtype == torch.bfloat16 else 64, 4
    C = H * d
    T = sum(lengths)
    x, w, _ = W.conv_inputs(1, T, C, width, dtype, seed=T + len(lengths), device="cuda", window=False)
    x = x[0]
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int32, device="cuda")
    win = None
    if with_window:
        win = torch.randn(len(lengths), width - 1, C, device="cuda").to(dtype)
    keep = None if win is None else win.clone()
    y, wout = la.short_conv_varlen(x, w, cu, heads=H, window=win, window_out=win, silu=True,
                                   l2norm=True)
    la.check_status()
    ry, rw = oconv.short_conv_packed(f64(x), f64(w), cu.tolist(), None if keep is None else f64(keep),
                                     H=H, silu=True, l2norm=True)
    if T:
        close(y, ry, dtype, True)
    np.testing.assert_array_equal(f64(wout), rw)


def test_conv_varlen_bad_offsets_are_reported(la):
    x, w, _ = W.conv_inputs(1, 100, 256, 4, torch.bfloat16, seed=1, device="cuda", window=False)
    bad = torch.tensor([0, 60, 40, 500], dtype=torch.int32, device="cuda")
    la.short_conv_varlen(x[0], w, bad, heads=2)
    with pytest.raises(la.LaError, match="INVALID_ARG"):
        la.check_status()
