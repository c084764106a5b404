"""Pins for the delta-rule gradients of the fp64 backward oracle (``delta_backward`` in
``oracle/backward.py``, modes 2 and 3).

The gradients come from reverse-mode differentiation of the recurrence; these tests tie
them to things other than that machinery:

* the recurrence itself equals the pinned C oracle (modes 2 and 3);
* central finite differences of the loss, every input, tiny sizes;
* b = 0 closed form: the state only decays, S_t = S_0 Diag(g_t) with the running gate
  product g_t, so every gradient is a finite sum written out by hand below;
* a = 1 closed form: with b = 1 and orthonormal keys the delta rule never corrects
  (S_{t-1} k_t = 0), so o_t = sum_{j<=t} (q_t . k_j) v_j and dq, dv, db and da have sums of
  the linear-attention kind;
* d_k = 1 reduction: the Gated DeltaNet update becomes the scalar-gate one with gate
  a_t (1 - b_t k_t^2) and value b_t v_t, so its gradients follow from the separately
  pinned mode-1 gradients by the chain rule;
* channel-uniform Kimi gates reproduce the Gated DeltaNet gradients (the gate gradient
  summed over channels).
"""
import importlib.util
import os

import numpy as np
import pytest
import torch

import oracle


def _load_backward():
    # A test that plants a mistake in a copy of oracle/backward.py points this at the copy.
    path = os.environ.get("LA_ORACLE_BACKWARD_OVERRIDE")
    if not path:
        from oracle import backward as mod
        return mod
    spec = importlib.util.spec_from_file_location("backward_mutant", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


ob = _load_backward()


def _inputs(seed, mode, B=1, H=2, T=7, dk=3, dv=2, gate_lo=0.3):
    r = np.random.default_rng(seed)
    q, k = r.normal(size=(B, H, T, dk)), r.normal(size=(B, H, T, dk))
    k = k / np.linalg.norm(k, axis=-1, keepdims=True)
    v, do = r.normal(size=(B, H, T, dv)), r.normal(size=(B, H, T, dv))
    a = r.uniform(gate_lo, 1.0, size=(B, H, T) + ((dk,) if mode == 3 else ()))
    b = r.uniform(0.1, 0.9, size=(B, H, T))
    S0 = r.normal(size=(B, H, dv, dk))
    dST = r.normal(size=(B, H, dv, dk))
    return q, k, v, a, b, do, S0, dST


def _loss(mode, q, k, v, a, b, S0, do, dST):
    t = lambda x: None if x is None else torch.as_tensor(x)
    o, ST = ob.delta_recurrence(mode, t(q), t(k), t(v), t(a), t(b), t(S0))
    L = float((o * torch.as_tensor(do)).sum())
    if dST is not None:
        L += float((ST * torch.as_tensor(dST)).sum())
    return L


@pytest.mark.parametrize("mode", [2, 3])
@pytest.mark.parametrize("with_state", [False, True])
def test_recurrence_is_the_pinned_c_oracle(mode, with_state):
    q, k, v, a, b, _, S0, _ = _inputs(11, mode, B=2, H=3, T=10, dk=4, dv=3)
    if not with_state:
        S0 = None
    o, ST = ob.delta_recurrence(mode, *(None if x is None else torch.as_tensor(x) for x in (q, k, v, a, b, S0)))
    ro, rS, _ = oracle.prefill(mode, q, k, v, a, b, S0)
    np.testing.assert_allclose(o.numpy(), ro, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(ST.numpy(), rS, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("mode", [2, 3])
@pytest.mark.parametrize("with_state", [False, True])
def test_gradients_match_finite_differences(mode, with_state):
    q, k, v, a, b, do, S0, dST = _inputs(1 + mode, mode)
    if not with_state:
        S0 = dST = None
    dq, dk, dv, da, db, dS0 = ob.delta_backward(mode, q, k, v, a, b, do, S0, dST)
    args = dict(q=q, k=k, v=v, a=a, b=b, S0=S0)
    grads = dict(q=dq, k=dk, v=dv, a=da, b=db, S0=dS0)
    h = 1e-6
    r = np.random.default_rng(7)
    for name in ["q", "k", "v", "a", "b"] + (["S0"] if with_state else []):
        x = args[name]
        for _ in range(8):
            idx = tuple(r.integers(0, n) for n in x.shape)
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            num = (_loss(mode, **{**args, name: xp}, do=do, dST=dST)
                   - _loss(mode, **{**args, name: xm}, do=do, dST=dST)) / (2 * h)
            assert abs(grads[name][idx] - num) <= 1e-6 * max(1.0, abs(num)), (name, idx, grads[name][idx], num)


@pytest.mark.parametrize("mode", [2, 3])
def test_zero_rate_closed_form(mode):
    """b = 0: S_t = S_0 Diag(g_t), g_t = prod_{s<=t} a_s (per channel in mode 3), so
    o_t = S_0 (g_t * q_t),  dq_t = g_t * (S_0^T do_t),  dk = dv = 0,
    dS_0 = sum_t do_t (g_t * q_t)^T + dS_T Diag(g_T),
    dL/da_t = (1 / a_t) [sum_{u>=t} g_u * q_u * (S_0^T do_u) + g_T * colsum(dS_T * S_0)],
    dL/db_t = (G_t k_t) . (v_t - S_0 (g_t * k_t)) with
    G_t = sum_{u>=t} do_u (q_u * g_u / g_t)^T + dS_T Diag(g_T / g_t)."""
    q, k, v, a, _, do, S0, dST = _inputs(21, mode, T=6, dk=4, dv=3)
    b = np.zeros(q.shape[:3])
    dq, dk, dv, da, db, dS0 = ob.delta_backward(mode, q, k, v, a, b, do, S0, dST)
    T, dk_ = q.shape[2], q.shape[3]
    for h in range(q.shape[1]):
        Q, K, V, dO, S, dS = q[0, h], k[0, h], v[0, h], do[0, h], S0[0, h], dST[0, h]
        A = a[0, h] if mode == 3 else np.repeat(a[0, h][:, None], dk_, axis=1)   # [T, d_k]
        g = np.cumprod(A, axis=0)
        np.testing.assert_allclose(dq[0, h], g * (dO @ S), rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(dk[0, h], 0.0, atol=1e-12)
        np.testing.assert_allclose(dv[0, h], 0.0, atol=1e-12)
        np.testing.assert_allclose(dS0[0, h], dO.T @ (g * Q) + dS * g[-1], rtol=1e-11, atol=1e-12)
        per_u = g * Q * (dO @ S)                                      # [T, d_k]
        tail = np.flip(np.cumsum(np.flip(per_u, 0), 0), 0) + g[-1] * (dS * S).sum(0)
        dA = tail / A
        want_da = dA if mode == 3 else dA.sum(1)
        np.testing.assert_allclose(da[0, h], want_da, rtol=1e-10, atol=1e-11)
        for t in range(T):
            G = sum(np.outer(dO[u], Q[u] * g[u] / g[t]) for u in range(t, T)) + dS * (g[-1] / g[t])
            want = (G @ K[t]) @ (V[t] - S @ (g[t] * K[t]))
            assert abs(db[0, h, t] - want) <= 1e-10 * max(1.0, abs(want)), (t, db[0, h, t], want)


@pytest.mark.parametrize("mode", [2, 3])
def test_unit_gate_orthonormal_keys_closed_form(mode):
    """a = 1, b = 1, orthonormal keys, S_0 = 0: S_{t-1} k_t = 0, so S_t = sum_{j<=t} v_j k_j^T
    and with P_tj = q_t . k_j, R_tj = do_t . v_j (j <= t):
    dq_t = sum_{j<=t} R_tj k_j,  dv_j = sum_{t>=j} P_tj do_t,
    dL/db_t = sum_{u>=t} P_ut R_ut,
    dL/da_t = sum_{u>=t} sum_{j<t} P_uj R_uj  (mode 2).
    In mode 3 the gate of channel c also scales the correction term, and the state
    cotangent G_t is projected off k_{t+1} .. k_u; channel c of the gate gradient is
    dL/da_tc = sum_{u>=t} sum_{j<t} R_uj k_jc (q_uc - sum_{s=t}^{u} P_us k_sc),
    whose sum over channels is the mode-2 value (the keys are orthonormal)."""
    r = np.random.default_rng(31)
    T, dk, dv = 5, 6, 3
    Kb = np.linalg.qr(r.normal(size=(dk, dk)))[0][:T]               # orthonormal rows
    q = r.normal(size=(1, 1, T, dk))
    k = Kb[None, None]
    v, do = r.normal(size=(1, 1, T, dv)), r.normal(size=(1, 1, T, dv))
    a = np.ones((1, 1, T) + ((dk,) if mode == 3 else ()))
    b = np.ones((1, 1, T))
    dq, dk_, dv_, da, db, _ = ob.delta_backward(mode, q, k, v, a, b, do)
    Q, K, V, dO = q[0, 0], k[0, 0], v[0, 0], do[0, 0]
    m = np.tril(np.ones((T, T)))
    P, R = m * (Q @ K.T), m * (dO @ V.T)
    np.testing.assert_allclose(dq[0, 0], R @ K, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(dv_[0, 0], P.T @ dO, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(db[0, 0], (P * R).sum(0), rtol=1e-11, atol=1e-12)
    if mode == 2:
        want = np.array([sum(P[u, j] * R[u, j] for u in range(t, T) for j in range(t)) for t in range(T)])
    else:
        want = np.array([[sum(R[u, j] * K[j, c] * (Q[u, c] - sum(P[u, s] * K[s, c] for s in range(t, u + 1)))
                               for u in range(t, T) for j in range(t))
                          for c in range(dk)] for t in range(T)])
        want2 = np.array([sum(P[u, j] * R[u, j] for u in range(t, T) for j in range(t)) for t in range(T)])
        np.testing.assert_allclose(want.sum(1), want2, rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(da[0, 0], want, rtol=1e-10, atol=1e-11)


@pytest.mark.parametrize("with_state", [False, True])
def test_one_channel_reduces_to_the_scalar_gate_mode(with_state):
    """d_k = 1: S_t = a_t (1 - b_t k_t^2) S_{t-1} + (b_t v_t) k_t is mode 1 with gate
    a'_t = a_t (1 - b_t k_t^2) and value v'_t = b_t v_t.  By the chain rule
    dv = b dv', da = (1 - b k^2) da', db = -a k^2 da' + v . dv', dk = dk' - 2 a b k da'."""
    q, k, v, a, b, do, S0, dST = _inputs(41, 2, B=2, H=2, T=8, dk=1, dv=3)
    k = np.random.default_rng(42).normal(size=k.shape)               # any scalar key
    if not with_state:
        S0 = dST = None
    dq, dk, dv, da, db, dS0 = ob.delta_backward(2, q, k, v, a, b, do, S0, dST)
    k2 = k[..., 0] ** 2
    a1 = a * (1 - b * k2)
    v1 = b[..., None] * v
    dq1, dk1, dv1, da1, dS01 = ob.prefill_backward(1, q, k, v1, a1, do, S0, dST)
    np.testing.assert_allclose(dq, dq1, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(dv, b[..., None] * dv1, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(da, (1 - b * k2) * da1, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(db, -a * k2 * da1 + (v * dv1).sum(-1), rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(dk[..., 0], dk1[..., 0] - 2 * a * b * k[..., 0] * da1, rtol=1e-10, atol=1e-11)
    if with_state:
        np.testing.assert_allclose(dS0, dS01, rtol=1e-11, atol=1e-12)


def test_uniform_channel_gates_reproduce_gated_deltanet():
    q, k, v, a, b, do, S0, dST = _inputs(51, 2, B=1, H=2, T=9, dk=4, dv=3)
    a3 = np.repeat(a[..., None], 4, axis=-1)
    r2 = ob.delta_backward(2, q, k, v, a, b, do, S0, dST)
    r3 = ob.delta_backward(3, q, k, v, a3, b, do, S0, dST)
    for i in (0, 1, 2, 4, 5):
        np.testing.assert_allclose(r3[i], r2[i], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(r3[3].sum(-1), r2[3], rtol=1e-11, atol=1e-12)


def test_no_gate_means_unit_gate():
    q, k, v, a, b, do, S0, dST = _inputs(61, 2, T=5)
    r_none = ob.delta_backward(2, q, k, v, None, b, do, S0, dST)
    r_one = ob.delta_backward(2, q, k, v, np.ones_like(a), b, do, S0, dST)
    assert r_none[3] is None
    for i in (0, 1, 2, 4, 5):
        np.testing.assert_allclose(r_none[i], r_one[i], rtol=1e-13, atol=1e-13)
