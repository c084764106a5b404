"""fp64 oracle of the prefill's backward pass (scalar-gate modes) -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may
import this module; the product path never does.

The lesson page "Linear attention and hybrids" (section "Three forms of one computation"
and its table of the forms) names the chunked form as the one used for training on long
texts; training needs the backward pass, for which the page gives no formulas.  The
gradients are defined here as the plain derivatives of the
recurrent form of section "Memory must forget: decay and gates",

    S_t = a_t S_{t-1} + v_t k_t^T,   o_t = S_t q_t,   S_0 given (or zero),

of the scalar L = sum_t do_t . o_t + <dS_T, S_T>_F for given output and final-state
cotangents do, dS_T.  They are computed by PyTorch's reverse-mode differentiation of that
recurrence, written out token by token in fp64 on the CPU (a library primitive used as a
step), and the tests pin them to finite differences.  Mode 4 (one constant gate per head)
takes the gate as a fixed hyperparameter: no gate gradient.
"""
from __future__ import annotations

import numpy as np
import torch

MODE_GATED = 1
MODE_RETNET = 4


def _t(x):
    return None if x is None else torch.as_tensor(np.asarray(x, dtype=np.float64))


def recurrence(q, k, v, a, S0):
    """The recurrent form over [B, H, T, d] tensors; a: [B, H, T] (None: 1).
    Returns (o [B, H, T, d_v], S_T [B, H, d_v, d_k])."""
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    S = S0 if S0 is not None else torch.zeros(B, H, dv, dk, dtype=q.dtype)
    outs = []
    for t in range(T):
        S = S if a is None else a[:, :, t, None, None] * S
        S = S + v[:, :, t, :, None] * k[:, :, t, None, :]
        outs.append(torch.einsum("bhij,bhj->bhi", S, q[:, :, t]))
    o = torch.stack(outs, dim=2) if T else torch.zeros(B, H, 0, dv, dtype=q.dtype)
    return o, S


def prefill_backward(mode, q, k, v, gate, do, S0=None, dS_T=None):
    """Gradients of L = sum(do * o) + <dS_T, S_T> for the recurrent form.

    q, k: [B,H,T,d_k]; v, do: [B,H,T,d_v]; gate: [B,H,T] (mode 1; None: a = 1) or [H]
    (mode 4); S0, dS_T: [B,H,d_v,d_k] or None.
    Returns (dq, dk, dv, dgate or None, dS0 or None), fp64 numpy arrays.
    """
    q, k, v, do = (_t(x).clone().requires_grad_(True) if i < 3 else _t(x)
                   for i, x in enumerate((q, k, v, do)))
    B, H, T, _ = q.shape
    g = _t(gate)
    need_dg = mode == MODE_GATED and g is not None
    if g is not None:
        g = g.clone().requires_grad_(need_dg)
        a = g if mode == MODE_GATED else g.reshape(1, H, 1).expand(B, H, T)
    else:
        a = None
    s0 = None if S0 is None else _t(S0).clone().requires_grad_(True)
    o, ST = recurrence(q, k, v, a, s0)
    L = (o * do).sum()
    if dS_T is not None:
        L = L + (ST * _t(dS_T)).sum()
    inputs = [q, k, v] + ([g] if need_dg else []) + ([s0] if s0 is not None else [])
    grads = torch.autograd.grad(L, inputs, allow_unused=True)
    grads = [torch.zeros_like(x) if gr is None else gr for x, gr in zip(inputs, grads)]
    dq, dk, dv = (x.detach().numpy() for x in grads[:3])
    rest = grads[3:]
    dg = rest.pop(0).detach().numpy() if need_dg else None
    ds0 = rest.pop(0).detach().numpy() if s0 is not None else None
    return dq, dk, dv, dg, ds0
