"""GPU parity of the delta-rule backward pass (``la_prefill_backward_delta``) against the
fp64 reverse-mode oracle (``oracle/backward.py``, ``delta_backward``).

Gated DeltaNet (mode 2) and Kimi Delta Attention (mode 3); q and k L2-normalised rows as
the delta rule expects, b = sigmoid(N(0, 1)), gates a = exp(-softplus(x + shift)).
Sequences of one token, of exactly two chunks of 32, with a ragged tail, and 4096 tokens;
with and without an initial state and a final-state cotangent; ordinary, weak
(a ~ 0.99) and, for the per-channel gates, strong decay (a down to 1e-4).  Tolerance per
(batch, head) slice, max|x - r| / max|r|: 2e-3 for fp32 I/O, 2e-2 for bf16 I/O, for dq,
dk, dv, the gate gradient, the rate gradient and dS_0.
"""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import backward as ob
from parity_util import TOL, f64, slice_rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def la():
    import gated_delta_rule_attention_b200 as m
    m.library()
    return m


def _case(mode, dtype, dk, dv, T, shift, seed, B=1, H=2):
    w = W.Workload("dbwd", mode, dtype, B=B, H=H, T=T, dk=dk, dv=dv, seed=seed, qk_l2norm=True,
                   qk_scale=1.0, gate="softplus", gate_shift=shift, beta=True)
    inp = W.prefill_inputs(w, device="cuda", init_state_std=0.1)
    g = torch.Generator(device="cuda").manual_seed(seed + 1)
    dO = torch.randn(B, H, T, dv, generator=g, device="cuda").to(dtype)
    dST = torch.randn(B, H, dv, dk, generator=g, device="cuda") * 0.1
    return inp, dO, dST


def _compare(la, mode, dtype, inp, dO, S0, dS, use_gate=True, gate_as_log=False):
    gate = inp["gate"] if use_gate else None
    dq, dk, dv, dg, db, dS0 = la.prefill_backward_delta(inp["q"], inp["k"], inp["v"], dO, mode=mode,
                                                        beta=inp["beta"], gate=gate, state0=S0,
                                                        dstate=dS, need_dstate0=S0 is not None)
    la.check_status()
    g = lambda t: None if t is None else f64(t)
    ref = ob.delta_backward(mode, g(inp["q"]), g(inp["k"]), g(inp["v"]), g(gate), g(inp["beta"]),
                            g(dO), g(S0), g(dS))
    rq, rk, rv, rg, rb, rS0 = ref
    tol = TOL[dtype]
    errs = {}
    for name, x, r in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv), ("dbeta", db, rb)):
        errs[name] = slice_rel_err(f64(x), r)
    if use_gate and gate_as_log:
        a = f64(gate)
        errs["d log a"] = slice_rel_err(a * f64(dg), a * rg)
    elif use_gate:
        errs["dgate"] = slice_rel_err(f64(dg), rg)
    else:
        assert dg is None
    if S0 is not None:
        errs["dS0"] = slice_rel_err(f64(dS0), rS0)
    bad = {k: v for k, v in errs.items() if not v < tol}
    assert not bad, f"{bad} (tol {tol})"


@pytest.mark.parametrize("mode", [2, 3])
@pytest.mark.parametrize("dtype,dk,dv", [(torch.float32, 64, 64), (torch.float32, 128, 128),
                                         (torch.bfloat16, 128, 128), (torch.float32, 128, 64)])
@pytest.mark.parametrize("T", [1, 64, 200])
@pytest.mark.parametrize("with_state", [False, True])
def test_delta_backward_matches_oracle(la, mode, dtype, dk, dv, T, with_state):
    inp, dO, dST = _case(mode, dtype, dk, dv, T, -2.0, seed=7 * T + dk + dv + mode)
    S0 = inp["state0"] if with_state else None
    dS = dST if with_state else None
    _compare(la, mode, dtype, inp, dO, S0, dS)


@pytest.mark.parametrize("mode", [2, 3])
def test_delta_backward_weak_decay_long(la, mode):
    """4096 tokens (128 chunks) with a ~ 0.99: the carried cotangent and the chunk-start
    states travel far, so their error would accumulate."""
    inp, dO, dST = _case(mode, torch.float32, 128, 128, 4096, -5.0, seed=90 + mode, H=1)
    _compare(la, mode, torch.float32, inp, dO, inp["state0"], dST)


@pytest.mark.parametrize("mode", [2, 3])
def test_delta_backward_without_gate(la, mode):
    inp, dO, dST = _case(mode, torch.float32, 128, 128, 100, -2.0, seed=70 + mode)
    _compare(la, mode, torch.float32, inp, dO, inp["state0"], dST, use_gate=False)


@pytest.mark.parametrize("mode", [2, 3])
def test_delta_backward_strong_decay(la, mode):
    """Gates down to 1e-4 (shift +9): chunk log-gate spans far beyond fp32's exponent range,
    every decay factor taken as is.  The gate gradient is compared as d log a = a dL/da:
    dL/da_t = (d log a_t) / a_t, and d log a_t, a sum of O(1) terms that cancel down to
    O(a_t), carries an absolute fp32 rounding error that the division by a_t ~ 1e-4 scales
    up; d log a is the well-conditioned quantity (and the one a log-parameterised gate
    trains on)."""
    inp, dO, dST = _case(mode, torch.float32, 128, 128, 96, 9.0, seed=80 + mode)
    assert float(inp["gate"].min()) < 1e-3
    _compare(la, mode, torch.float32, inp, dO, inp["state0"], dST, gate_as_log=True)


def test_delta_backward_bf16_full_state_several_heads(la):
    inp, dO, dST = _case(2, torch.bfloat16, 128, 128, 333, -3.0, seed=5, B=2, H=3)
    _compare(la, 2, torch.bfloat16, inp, dO, inp["state0"], dST)


def test_delta_backward_outputs_are_optional(la):
    """dgate, dbeta and dS_0 may be omitted; the other gradients do not change."""
    inp, dO, dST = _case(2, torch.float32, 64, 64, 70, -2.0, seed=3)
    full = la.prefill_backward_delta(inp["q"], inp["k"], inp["v"], dO, mode=2, beta=inp["beta"],
                                     gate=inp["gate"], state0=inp["state0"], dstate=dST)
    part = la.prefill_backward_delta(inp["q"], inp["k"], inp["v"], dO, mode=2, beta=inp["beta"],
                                     gate=inp["gate"], state0=inp["state0"], dstate=dST,
                                     need_dgate=False, need_dstate0=False)
    la.check_status()
    assert part[3] is None and part[5] is None
    for a, b in zip(full[:3], part[:3]):
        assert torch.equal(a, b)


def test_delta_backward_full_size_sampled(la):
    """The bench's launch at full size (B2 H16 T32768, bf16, Gated DeltaNet) on sampled
    outputs the oracle computes one by one.  q enters only o_t = S_t q_t, so dq_t = S_t^T do_t
    with S_t the forward state (C oracle over the prefix); at the last token (no dS_T) the
    state cotangent is G_T = do_T q_T^T, so with u = G_T k_T:
    dv_T = b_T u,  db_T = u . (v_T - a_T S_{T-1} k_T)."""
    import oracle
    w = W.BACKWARD_CONFIGS["gdn_bwd_bf16_b2h16t32768"]
    inp = W.prefill_inputs(w, device="cuda")
    g = torch.Generator(device="cuda").manual_seed(w.seed + 1)
    dO = torch.randn(w.B, w.H, w.T, w.dv, generator=g, device="cuda").to(w.dtype)
    dq, dk, dv, dg, db, _ = la.prefill_backward_delta(inp["q"], inp["k"], inp["v"], dO, mode=2,
                                                      beta=inp["beta"], gate=inp["gate"])
    la.check_status()
    assert all(torch.isfinite(x.float()).all() for x in (dq, dk, dv, dg, db))
    tol = TOL[torch.bfloat16]
    T = w.T
    for b, h in ((0, 0), (1, 15)):
        f = lambda t, s=slice(None): t[b, h, s].detach().to("cpu", torch.float64).numpy()
        q, k, v, a, be = (f(inp[x]) for x in ("q", "k", "v", "gate", "beta"))
        do = f(dO)
        for t in (T // 2 - 1, T - 1):
            _, S_t, _ = oracle.prefill(2, q[None, None, :t + 1], k[None, None, :t + 1], v[None, None, :t + 1],
                                       a[None, None, :t + 1], be[None, None, :t + 1])
            want = S_t[0, 0].T @ do[t]
            got = f(dq)[t]
            assert np.abs(got - want).max() <= tol * np.abs(want).max(), (b, h, t)
        _, S_prev, _ = oracle.prefill(2, q[None, None, :T - 1], k[None, None, :T - 1], v[None, None, :T - 1],
                                      a[None, None, :T - 1], be[None, None, :T - 1])
        u = do[T - 1] * (q[T - 1] @ k[T - 1])
        want_dv = be[T - 1] * u
        got_dv = f(dv)[T - 1]
        assert np.abs(got_dv - want_dv).max() <= tol * np.abs(want_dv).max(), (b, h)
        want_db = u @ (v[T - 1] - a[T - 1] * (S_prev[0, 0] @ k[T - 1]))
        got_db = f(db)[T - 1]
        assert abs(got_db - want_db) <= tol * max(abs(want_db), np.abs(u).max() * np.abs(v[T - 1]).max()), \
            (b, h, got_db, want_db)


@pytest.mark.parametrize("mode", [2, 3])
def test_delta_backward_bf16_long(la, mode):
    """bf16 I/O over 4096 tokens (128 chunks): the gate gradient is a suffix sum within each
    chunk, but the carried cotangent and states cross all 128 chunks."""
    inp, dO, dST = _case(mode, torch.bfloat16, 128, 128, 4096, -3.0, seed=60 + mode, H=1)
    _compare(la, mode, torch.bfloat16, inp, dO, inp["state0"], dST)
