"""Pins for the fp64 oracle of the short causal convolution (``oracle/conv.py``).

The convolution is tied to library routines and closed forms rather than to itself:
numpy's full convolution per channel, the unit-tap special cases (identity and a pure
delay), linearity, the split-sequence continuation through the carried window, the
decode step against the prefill, and the closed forms of SiLU and the L2 row norm.
"""
import importlib.util
import os

import numpy as np
import pytest


def _load_conv():
    # A test that plants a mistake in a copy of oracle/conv.py points this at the copy,
    # to check that these pins catch it.
    path = os.environ.get("LA_ORACLE_CONV_OVERRIDE")
    if not path:
        from oracle import conv as mod
        return mod
    spec = importlib.util.spec_from_file_location("conv_mutant", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


conv = _load_conv()


def _inputs(seed, B=2, T=37, H=3, d=8, width=4):
    r = np.random.default_rng(seed)
    C = H * d
    return r.normal(size=(B, T, C)), r.normal(size=(C, width)), r.normal(size=(B, width - 1, C))


@pytest.mark.parametrize("width", [1, 2, 3, 4])
def test_matches_numpy_convolve_per_channel(width):
    x, w, win = _inputs(1, width=width)
    y, _ = conv.short_conv(x, w, win, H=3)
    B, T, C = x.shape
    for b in range(B):
        for c in range(C):
            seq = np.concatenate([win[b, :, c], x[b, :, c]])
            # np.convolve flips its second argument: tap width-1 multiplies the newest input
            ref = np.convolve(seq, w[c, ::-1], mode="full")[width - 1:width - 1 + T]
            h, dd = divmod(c, C // 3)
            np.testing.assert_allclose(y[b, h, :, dd], ref, rtol=1e-12, atol=1e-12)


def test_unit_taps_identity_and_delay():
    x, _, _ = _inputs(2)
    C = x.shape[2]
    ident = np.zeros((C, 4)); ident[:, 3] = 1.0
    y, _ = conv.short_conv(x, ident, None, H=1)
    np.testing.assert_array_equal(y[:, 0], x)
    delay = np.zeros((C, 4)); delay[:, 0] = 1.0
    y, _ = conv.short_conv(x, delay, None, H=1)
    np.testing.assert_array_equal(y[:, 0, 3:], x[:, :-3])
    np.testing.assert_array_equal(y[:, 0, :3], 0.0)      # zero window: nothing before x_0


def test_window_feeds_the_first_tokens():
    x, w, win = _inputs(3)
    y0, _ = conv.short_conv(x, w, None, H=3)
    y1, _ = conv.short_conv(x, w, win, H=3)
    np.testing.assert_array_equal(y1[:, :, 3:], y0[:, :, 3:])   # only t < width-1 change
    assert np.abs(y1[:, :, :3] - y0[:, :, :3]).max() > 1e-3


def test_linear_in_x_and_in_w():
    x, w, win = _inputs(4)
    x2, w2, _ = _inputs(5)
    ya, _ = conv.short_conv(x, w, win, H=3)
    yb, _ = conv.short_conv(x2, w, win * 0, H=3)
    yab, _ = conv.short_conv(x + x2, w, win, H=3)
    np.testing.assert_allclose(yab, ya + yb, rtol=1e-12, atol=1e-12)
    yw, _ = conv.short_conv(x, w + w2, win, H=3)
    yw2, _ = conv.short_conv(x, w2, win, H=3)
    np.testing.assert_allclose(yw, ya + yw2, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("split", [1, 2, 5, 36])
def test_split_sequence_continues_through_the_window(split):
    x, w, win = _inputs(6)
    y, wout = conv.short_conv(x, w, win, H=3, silu=True, l2norm=True)
    ya, wa = conv.short_conv(x[:, :split], w, win, H=3, silu=True, l2norm=True)
    yb, wb = conv.short_conv(x[:, split:], w, wa, H=3, silu=True, l2norm=True)
    np.testing.assert_allclose(np.concatenate([ya, yb], axis=2), y, rtol=1e-13, atol=1e-13)
    np.testing.assert_array_equal(wb, wout)
    np.testing.assert_array_equal(wout, x[:, -3:])


def test_short_sequence_window_keeps_old_rows():
    x, w, win = _inputs(7, T=2)
    _, wout = conv.short_conv(x, w, win, H=3)
    np.testing.assert_array_equal(wout[:, 0], win[:, 2])
    np.testing.assert_array_equal(wout[:, 1:], x)


def test_decode_steps_equal_the_prefill():
    x, w, win = _inputs(8, T=9)
    y, wout = conv.short_conv(x, w, win, H=3, silu=True, l2norm=True)
    cur = win
    for t in range(x.shape[1]):
        yt, cur = conv.short_conv_step(x[:, t], w, cur, H=3, silu=True, l2norm=True)
        np.testing.assert_allclose(yt, y[:, :, t], rtol=1e-13, atol=1e-13)
    np.testing.assert_array_equal(cur, wout)


def test_silu_closed_form():
    C = 5
    ident = np.zeros((C, 4)); ident[:, 3] = 1.0
    x = np.array([[[0.0, 1.0, -1.0, 30.0, -30.0]]])
    y, _ = conv.short_conv(x, ident, None, H=1, silu=True)
    e = np.exp(1.0)
    expect = [0.0, e / (1 + e), -1 / (1 + e), 30.0, 0.0]
    np.testing.assert_allclose(y[0, 0, 0], expect, rtol=1e-12, atol=1e-11)


def test_l2norm_gives_unit_rows_with_the_same_direction():
    x, w, win = _inputs(9)
    y, _ = conv.short_conv(x, w, win, H=3)
    yn, _ = conv.short_conv(x, w, win, H=3, l2norm=True)
    norms = np.linalg.norm(y, axis=-1, keepdims=True)
    np.testing.assert_allclose(yn, y / np.sqrt(norms ** 2 + conv.L2_EPS), rtol=1e-12)
    np.testing.assert_allclose(np.linalg.norm(yn, axis=-1), 1.0, atol=1e-6)
    # a 3-4-5 row: exact direction, norm 1 up to eps
    C = 2
    ident = np.zeros((C, 1)); ident[:, 0] = 1.0
    z, _ = conv.short_conv(np.array([[[3.0, 4.0]]]), ident, None, H=1, l2norm=True)
    np.testing.assert_allclose(z[0, 0, 0], [0.6, 0.8], rtol=1e-7)
    zero, _ = conv.short_conv(np.zeros((1, 1, 2)), ident, None, H=1, l2norm=True)
    np.testing.assert_array_equal(zero, 0.0)


def test_heads_are_normalised_separately():
    C, H = 4, 2
    ident = np.zeros((C, 4)); ident[:, 3] = 1.0
    x = np.array([[[3.0, 4.0, 0.0, 2.0]]])
    y, _ = conv.short_conv(x, ident, None, H=H, l2norm=True)
    np.testing.assert_allclose(y[0, :, 0], [[0.6, 0.8], [0.0, 1.0]], rtol=1e-6)


def test_packed_equal_lengths_match_the_batched_call():
    x, w, win = _inputs(12, B=3, T=11)
    y, wout = conv.short_conv(x, w, win, H=3, silu=True, l2norm=True)
    B, T, C = x.shape
    cu = np.arange(B + 1) * T
    py, pw = conv.short_conv_packed(x.reshape(B * T, C), w, cu, win, H=3, silu=True, l2norm=True)
    np.testing.assert_allclose(py, np.concatenate(list(y), axis=1), rtol=1e-13, atol=1e-13)
    np.testing.assert_array_equal(pw, wout)


def test_packed_sequences_do_not_mix():
    """A sequence's first outputs see only its own window, never the previous sequence's
    last tokens; an empty sequence passes its window through."""
    r = np.random.default_rng(13)
    C, width = 8, 4
    cu = np.array([0, 5, 5, 12])
    x = r.normal(size=(12, C))
    w = r.normal(size=(C, width))
    py, pw = conv.short_conv_packed(x, w, cu, None, H=1)
    alone, _ = conv.short_conv(x[5:12][None], w, None, H=1)
    np.testing.assert_array_equal(py[:, 5:12], alone[0])
    np.testing.assert_array_equal(pw[1], 0.0)
    win = r.normal(size=(3, width - 1, C))
    _, pw2 = conv.short_conv_packed(x, w, cu, win, H=1)
    np.testing.assert_array_equal(pw2[1], win[1])
    np.testing.assert_array_equal(pw2[2], x[9:12])
