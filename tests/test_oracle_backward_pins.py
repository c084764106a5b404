"""Pins for the fp64 backward oracle (``oracle/backward.py``).

The gradients come from reverse-mode differentiation of the recurrent form; they are tied
to things other than that machinery: the forward recurrence itself equals the pinned C
oracle, central finite differences of the loss (every input, tiny sizes), the closed form
of the ungated case, and the decay identity that the CUDA kernel uses,
d log a_t = sum_{u >= t} (q_u . dq_u - k_u . dk_u) (plus <dS_T, S_T> at the last token),
which follows from differentiating the decay mask exp(lam_s - lam_j).
"""
import importlib.util
import os

import numpy as np
import pytest
import torch

import oracle


def _load_backward():
    # A test that plants a mistake in a copy of oracle/backward.py points this at the copy,
    # to check that these pins catch it.
    path = os.environ.get("LA_ORACLE_BACKWARD_OVERRIDE")
    if not path:
        from oracle import backward as mod
        return mod
    spec = importlib.util.spec_from_file_location("backward_mutant", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


ob = _load_backward()


def _inputs(seed, B=1, H=2, T=7, dk=3, dv=2):
    r = np.random.default_rng(seed)
    q, k = r.normal(size=(B, H, T, dk)), r.normal(size=(B, H, T, dk))
    v, do = r.normal(size=(B, H, T, dv)), r.normal(size=(B, H, T, dv))
    a = 1 / (1 + np.exp(r.normal(size=(B, H, T))))
    S0 = r.normal(size=(B, H, dv, dk))
    dST = r.normal(size=(B, H, dv, dk))
    return q, k, v, do, a, S0, dST


def _loss(q, k, v, a, S0, do, dST):
    t = lambda x: None if x is None else torch.as_tensor(x)
    o, ST = ob.recurrence(t(q), t(k), t(v), t(a), t(S0))
    L = float((o * torch.as_tensor(do)).sum())
    if dST is not None:
        L += float((ST * torch.as_tensor(dST)).sum())
    return L


@pytest.mark.parametrize("with_state", [False, True])
def test_gradients_match_finite_differences(with_state):
    q, k, v, do, a, S0, dST = _inputs(1)
    if not with_state:
        S0 = dST = None
    dq, dk, dv, da, dS0 = ob.prefill_backward(1, q, k, v, a, do, S0, dST)
    h = 1e-6
    args = dict(q=q, k=k, v=v, a=a, S0=S0)
    grads = dict(q=dq, k=dk, v=dv, a=da, S0=dS0)
    r = np.random.default_rng(5)
    for name in ["q", "k", "v", "a"] + (["S0"] if with_state else []):
        x = args[name]
        for _ in range(6):
            idx = tuple(r.integers(0, n) for n in x.shape)
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            fp = _loss(**{**args, name: xp}, do=do, dST=dST)
            fm = _loss(**{**args, name: xm}, do=do, dST=dST)
            num = (fp - fm) / (2 * h)
            assert abs(grads[name][idx] - num) <= 1e-6 * max(1.0, abs(num)), (name, idx)


def test_ungated_closed_form():
    """a = 1, S0 = 0: o_t = sum_{j<=t} (q_t . k_j) v_j, so
    dv_j = sum_{t>=j} (q_t . k_j) do_t and dq_t = sum_{j<=t} (do_t . v_j) k_j."""
    q, k, v, do, _, _, _ = _inputs(2, T=6)
    dq, dk, dv, _, _ = ob.prefill_backward(1, q, k, v, None, do)
    T = q.shape[2]
    m = np.tril(np.ones((T, T)))
    for h in range(q.shape[1]):
        Q, K, V, dO = q[0, h], k[0, h], v[0, h], do[0, h]
        np.testing.assert_allclose(dv[0, h], (m * (Q @ K.T)).T @ dO, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(dq[0, h], (m * (dO @ V.T)) @ K, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(dk[0, h], (m * (dO @ V.T)).T @ Q, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("with_state", [False, True])
def test_gate_gradient_decay_identity(with_state):
    q, k, v, do, a, S0, dST = _inputs(3, T=9)
    if not with_state:
        S0 = dST = None
    dq, dk, dv, da, _ = ob.prefill_backward(1, q, k, v, a, do, S0, dST)
    dlam = (q * dq).sum(-1) - (k * dk).sum(-1)                   # [B, H, T]
    if dST is not None:
        _, ST = ob.recurrence(*(torch.as_tensor(x) for x in (q, k, v, a, S0)))
        dlam[..., -1] += (dST * ST.numpy()).sum((-1, -2))
    dloga = np.flip(np.cumsum(np.flip(dlam, -1), -1), -1)         # suffix sums
    np.testing.assert_allclose(da * a, dloga, rtol=1e-10, atol=1e-10)


def test_retnet_mode_has_no_gate_gradient_and_matches_mode1():
    q, k, v, do, _, S0, dST = _inputs(4, B=2, H=3)
    gam = np.array([0.9, 0.5, 0.99])
    g1 = np.broadcast_to(gam.reshape(1, 3, 1), q.shape[:3]).copy()
    r4 = ob.prefill_backward(4, q, k, v, gam, do, S0, dST)
    r1 = ob.prefill_backward(1, q, k, v, g1, do, S0, dST)
    assert r4[3] is None
    for x, y in zip(r4[:3] + r4[4:], r1[:3] + r1[4:]):
        np.testing.assert_allclose(x, y, rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("with_state", [False, True])
def test_forward_recurrence_is_the_pinned_c_oracle(with_state):
    """The recurrence the gradients differentiate is the scalar-gate mode of the C oracle
    (pinned on its own to the page's worked examples and closed forms)."""
    q, k, v, _, a, S0, _ = _inputs(6, B=2, H=3, T=11)
    if not with_state:
        S0 = None
    o, ST = ob.recurrence(*(None if x is None else torch.as_tensor(x) for x in (q, k, v, a, S0)))
    ro, rS, _ = oracle.prefill(1, q, k, v, a, None, S0)
    np.testing.assert_allclose(o.numpy(), ro, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(ST.numpy(), rS, rtol=1e-12, atol=1e-12)
