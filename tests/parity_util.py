"""Helpers shared by the GPU parity tests: error metric, tolerances, oracle on slices."""
import numpy as np
import torch

import oracle

# Max relative error allowed (per (batch, head) slice: max|x - r| / max|r|), by I/O dtype.
TOL = {torch.float32: 2e-3, torch.bfloat16: 2e-2}


def f64(t):
    """Exact upcast of a torch tensor (any device, bf16/fp32) to a numpy fp64 array."""
    return t.detach().to("cpu", torch.float64).numpy()


def slice_rel_err(x, ref, lead=2):
    """max over the leading `lead` dims of  max|x - ref| / max|ref|  within each slice."""
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert x.shape == ref.shape, (x.shape, ref.shape)
    if x.size == 0:
        return 0.0
    n = int(np.prod(x.shape[:lead]))
    xs = x.reshape(n, -1)
    rs = ref.reshape(n, -1)
    scale = np.abs(rs).max(axis=1)
    scale = np.where(scale > 0, scale, 1.0)
    return float((np.abs(xs - rs).max(axis=1) / scale).max())


def oracle_prefill_slices(mode, inp, heads, init_state=False, z0=None):
    """Run the oracle on the listed (b, h) pairs of a prefill input dict.

    Returns (o [n, T, dv], S [n, dv, dk], z [n, dk] or None) for the n listed heads."""
    sel = lambda t: None if t is None else np.stack([f64(t[b, h]) for b, h in heads])[None]
    o, S, z = oracle.prefill(mode, sel(inp["q"]), sel(inp["k"]), sel(inp["v"]), sel(inp["gate"]),
                             sel(inp["beta"]), sel(inp["state0"]) if init_state else None,
                             sel(z0) if z0 is not None else None)
    return o[0], S[0], (None if z is None else z[0])


def pick(t, heads):
    return np.stack([f64(t[b, h]) for b, h in heads])
