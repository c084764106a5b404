"""fp64 oracle of the short causal convolution prologue -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may
import this module; the product path never does.

The lesson page "Linear attention and hybrids", section "Hybrids of 2025: Qwen3-Next and
Kimi Linear", says that Gated DeltaNet (and KDA) layers put a short causal depthwise
convolution over time, kernel width 4, in front of the queries, keys and values: each
token is mixed with the three before it.  The page fixes nothing else, so this module
takes the plainest reading (every item is a reading, listed with the others):

* depthwise: channel c of the output sees only channel c of the input, with its own
  ``width`` taps w[c, 0..width-1] and no bias;
* causal, with tap ``width-1`` on the current token:
  u_t[c] = sum_i w[c, i] * x_{t-(width-1)+i}[c], where x_{-1}, x_{-2}, ... are the
  ``width-1`` tokens of the carried window (zero when there is none);
* the carried window after a call is the last ``width-1`` rows of [window; x], so that
  splitting a sequence into two calls gives the same result as one call;
* an optional SiLU, u * sigmoid(u), and an optional L2 normalisation of every head's
  row, u / sqrt(sum u^2 + eps) with eps = 1e-6 (the page names neither: SiLU is the
  activation the models it names apply after this convolution, and the row norm is the
  L2-normalised q and k of the Gated DeltaNet workload; eps keeps a zero row finite);
* the input is token-major [B, T, H*d] (a projection's output), the output head-major
  [B, H, T, d] (the attention's input layout).

Everything is computed in fp64 on the exact values the GPU receives.
"""
from __future__ import annotations

import numpy as np

L2_EPS = 1e-6


def _f64(x):
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def short_conv(x, w, window=None, H=1, silu=False, l2norm=False):
    """Causal depthwise convolution over time of a whole sequence per batch row.

    x: [B, T, C] with C = H * d; w: [C, width]; window: [B, width-1, C] (the inputs
    before x_0, oldest first) or None for zeros.
    Returns (y [B, H, T, d], window_out [B, width-1, C]), fp64.
    """
    x, w = _f64(x), _f64(w)
    B, T, C = x.shape
    width = w.shape[1]
    if w.shape != (C, width) or C % H:
        raise ValueError("shape mismatch")
    win = np.zeros((B, width - 1, C)) if window is None else _f64(window)
    if win.shape != (B, width - 1, C):
        raise ValueError("window shape mismatch")
    full = np.concatenate([win, x], axis=1)            # [B, width-1+T, C]
    u = np.zeros((B, T, C))
    for i in range(width):                              # tap i reads token t-(width-1)+i
        u += w[:, i] * full[:, i:i + T, :]
    y = _activate(u, H, silu, l2norm)
    d = C // H
    y = y.reshape(B, T, H, d).transpose(0, 2, 1, 3).copy()
    return y, full[:, T:, :].copy()


def short_conv_step(x, w, window, H=1, silu=False, l2norm=False):
    """One token per sequence: x [N, C], window [N, width-1, C].

    Returns (y [N, H, d], window_new [N, width-1, C]); the inputs are not modified.
    """
    x, w, win = _f64(x), _f64(w), _f64(window)
    y, win_new = short_conv(x[:, None, :], w, win, H, silu, l2norm)
    return y[:, :, 0, :], win_new


def short_conv_packed(x, w, cu, window=None, H=1, silu=False, l2norm=False):
    """Packed variable-length sequences: sequence s = tokens cu[s] .. cu[s+1] of the packed
    axis, each convolved on its own with its own carried window.

    x: [T, C]; window: [N, width-1, C] or None (zeros).  Returns (y [H, T, d],
    window_out [N, width-1, C]).
    """
    x, w = _f64(x), _f64(w)
    T, C = x.shape
    width = w.shape[1]
    cu = [int(c) for c in np.asarray(cu).reshape(-1)]
    N = len(cu) - 1
    y = np.zeros((H, T, C // H))
    wout = np.zeros((N, width - 1, C))
    for s in range(N):
        a, b = cu[s], cu[s + 1]
        win = None if window is None else _f64(window)[s][None]
        ys, ws = short_conv(x[a:b][None], w, win, H, silu, l2norm)
        y[:, a:b] = ys[0]
        wout[s] = ws[0]
    return y, wout


def _activate(u, H, silu, l2norm):
    if silu:
        u = u / (1.0 + np.exp(-u))
    if l2norm:
        B, T, C = u.shape
        r = u.reshape(B, T, H, C // H)
        r = r / np.sqrt((r * r).sum(axis=-1, keepdims=True) + L2_EPS)
        u = r.reshape(B, T, C)
    return u
