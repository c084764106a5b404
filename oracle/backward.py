"""fp64 oracle of the prefill's backward pass -- TEST INFRASTRUCTURE ONLY.

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

The delta-rule modes (``delta_backward``) differentiate the recurrences of the lesson page
"Delta rule and Gated DeltaNet" in the same way: Gated DeltaNet (mode 2)

    S_t = a_t S_{t-1} (I - b_t k_t k_t^T) + b_t v_t k_t^T,

and Kimi Delta Attention (mode 3), where the scalar a_t becomes the diagonal matrix
Diag(a_t) of a per-channel gate a_t in R^{d_k}:

    S_t = S_{t-1} Diag(a_t) (I - b_t k_t k_t^T) + b_t v_t k_t^T,

both read as o_t = S_t q_t (update, then read).  The delta rate b_t is an input like the
others and gets its own gradient.
"""
from __future__ import annotations

import numpy as np
import torch

MODE_GATED = 1
MODE_GATED_DELTA = 2
MODE_KDA = 3
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


def delta_recurrence(mode, q, k, v, a, beta, S0):
    """The delta-rule recurrence over [B, H, T, d] tensors, token by token.

    a: [B, H, T] (mode 2) or [B, H, T, d_k] (mode 3), None for a = 1; beta: [B, H, T].
    Returns (o [B, H, T, d_v], S_T [B, H, d_v, d_k])."""
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    S = S0 if S0 is not None else torch.zeros(B, H, dv, dk, dtype=q.dtype)
    outs = []
    for t in range(T):
        if a is not None:
            # decay first: a_t S_{t-1} (mode 2) or S_{t-1} Diag(a_t) (mode 3, columns)
            S = S * (a[:, :, t, None, :] if mode == MODE_KDA else a[:, :, t, None, None])
        kt, b = k[:, :, t], beta[:, :, t, None, None]
        Sk = torch.einsum("bhij,bhj->bhi", S, kt)               # (decayed S) k_t
        S = S - b * Sk[..., :, None] * kt[..., None, :] + b * v[:, :, t, :, None] * kt[..., None, :]
        outs.append(torch.einsum("bhij,bhj->bhi", S, q[:, :, t]))
    o = torch.stack(outs, dim=2) if T else torch.zeros(B, H, 0, dv, dtype=q.dtype)
    return o, S


def delta_backward(mode, q, k, v, gate, beta, do, S0=None, dS_T=None):
    """Gradients of L = sum(do * o) + <dS_T, S_T> for the delta-rule recurrence.

    q, k: [B,H,T,d_k]; v, do: [B,H,T,d_v]; gate: [B,H,T] (mode 2) or [B,H,T,d_k] (mode 3),
    None for a = 1; beta: [B,H,T]; S0, dS_T: [B,H,d_v,d_k] or None.
    Returns (dq, dk, dv, dgate or None, dbeta, dS0 or None), fp64 numpy arrays.
    """
    assert mode in (MODE_GATED_DELTA, MODE_KDA)
    q, k, v, b = (_t(x).clone().requires_grad_(True) for x in (q, k, v, beta))
    g = _t(gate)
    if g is not None:
        g = g.clone().requires_grad_(True)
    s0 = None if S0 is None else _t(S0).clone().requires_grad_(True)
    o, ST = delta_recurrence(mode, q, k, v, g, b, s0)
    L = (o * _t(do)).sum()
    if dS_T is not None:
        L = L + (_t(dS_T) * ST).sum()
    inputs = [q, k, v, b] + ([g] if g is not None else []) + ([s0] if s0 is not None else [])
    grads = torch.autograd.grad(L, inputs, allow_unused=True)
    grads = [torch.zeros_like(x) if gr is None else gr for x, gr in zip(inputs, grads)]
    dq, dk, dv, db = (x.detach().numpy() for x in grads[:4])
    rest = grads[4:]
    dg = rest.pop(0).detach().numpy() if g is not None else None
    ds0 = rest.pop(0).detach().numpy() if s0 is not None else None
    return dq, dk, dv, dg, db, ds0
