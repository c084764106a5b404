"""Pins for the fp64 oracle: printed values, closed forms, brute force, invariants.

Each test ties the C oracle (``oracle/la_oracle.c``) to something other than itself:
values the lesson page "Linear attention and hybrids" prints for worked examples
(``tests/golden/``), the page's claim that its three forms agree, closed forms of
special cases, and brute force on tiny inputs.  The set is chosen so that a dropped
term, a wrong sign, a swapped index or a transposed operand in any mode fails at
least one test (``test_pins_catch_planted_mistakes`` checks exactly that).
"""
import math
import os

import numpy as np
import pytest

import oracle
from oracle import forms

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.lstrip().startswith("#")]


def run1(mode, Q, K, V, gate=None, beta=None, S0=None, z0=None):
    """C oracle on one head (2-D arrays) -> (O [T,dv], S [dv,dk], z)."""
    Q, K, V = (np.asarray(x, dtype=np.float64) for x in (Q, K, V))
    g = None if gate is None else np.asarray(gate, dtype=np.float64)[None, None]
    b = None if beta is None else np.asarray(beta, dtype=np.float64)[None, None]
    st = None if S0 is None else np.asarray(S0, dtype=np.float64)[None, None]
    zz = None if z0 is None else np.asarray(z0, dtype=np.float64)[None, None]
    o, S, z = oracle.prefill(mode, Q[None, None], K[None, None], V[None, None], g, b, st, zz)
    return o[0, 0], S[0, 0], (None if z is None else z[0, 0])


def rng_inputs(seed, T, dk, dv, unit_keys=False):
    r = np.random.default_rng(seed)
    Q = r.normal(size=(T, dk))
    K = r.normal(size=(T, dk))
    V = r.normal(size=(T, dv))
    if unit_keys:
        K /= np.linalg.norm(K, axis=1, keepdims=True)
        Q /= np.linalg.norm(Q, axis=1, keepdims=True)
    a = 1.0 / (1.0 + np.exp(r.normal(size=T)))        # values in (0, 1)
    b = 1.0 / (1.0 + np.exp(-r.normal(size=T)))
    return Q, K, V, a, b


# ----------------------------------------------------------------------------------
# printed values of the page
# ----------------------------------------------------------------------------------

def _phi_through_oracle(x):
    """Recover phi(x) from the C oracle's mode 0: with d_k = d_v = 1, q_2 = 0 (phi = 1),
    k_1 = x, k_2 = 0 (phi = 1), v_1 = 1, v_2 = 0, the second output is
    phi(x) / (phi(x) + 1)."""
    o, _, _ = run1(0, [[0.0], [0.0]], [[x], [0.0]], [[1.0], [0.0]])
    r = o[1, 0]
    return r / (1.0 - r)


def test_feature_map_printed_values():
    for x, want, tol in _rows("feature_map.txt"):
        x, want, tol = float(x), float(want), float(tol)
        assert abs(forms.feature_map(x) - want) <= tol
        assert abs(_phi_through_oracle(x) - want) <= tol


def test_similarity_worked_example():
    g = {r[0]: [float(t) for t in r[1:]] for r in _rows("similarity_example.txt")}
    q, k, tol = np.array(g["q"]), np.array(g["k"]), g["tol"][0]
    assert np.allclose(forms.feature_map(q), g["phi_q"], atol=tol)
    assert np.allclose(forms.feature_map(k), g["phi_k"], atol=tol)
    assert abs(forms.feature_map(q) @ forms.feature_map(k) - g["sim"][0]) <= tol
    assert abs(math.exp(q @ k) - g["softmax"][0]) <= tol
    # Through the C oracle: token 1 has key k (weight w1 = phi(q).phi(k)), token 2 has
    # key 0 (phi = (1, 1), weight w2 = phi(q).(1, 1)); query q at step 2; values 1 and 0.
    o, _, _ = run1(0, [q, q], [k, [0.0, 0.0]], [[1.0], [0.0]])
    w1 = g["sim"][0]
    w2 = sum(g["phi_q"])
    assert abs(o[1, 0] - w1 / (w1 + w2)) <= 2e-3


def test_delta_rule_read_printed():
    g = {r[0]: [float(t) for t in r[1:]] for r in _rows("delta_rule_read.txt")}
    K = np.array([g["k"], g["k"]])
    V = np.array([g["v1"], g["v2"]])
    Q = K.copy()                               # read S k right after each write
    o_lin, S_lin, _ = run1(1, Q, K, V, gate=[1.0, 1.0])
    o_del, S_del, _ = run1(2, Q, K, V, gate=[1.0, 1.0], beta=[1.0, 1.0])
    assert np.array_equal(o_lin[1], g["linear"])
    assert np.array_equal(o_del[1], g["delta"])
    assert np.array_equal(o_del[0], g["v1"])       # beta = 1, unit key: reads back v_t
    assert np.array_equal(S_lin @ np.array(g["k"]), g["linear"])
    # also without a gate pointer (NULL gate means a = 1)
    o_del2, _, _ = run1(2, Q, K, V, beta=[1.0, 1.0])
    assert np.array_equal(o_del2, o_del)


def test_decay_mask_printed():
    rows = _rows("decay_mask_gamma09.txt")
    gamma = float(rows[0][1])
    max_diff = float(rows[1][1])
    D_print = np.array([[float(t) for t in r] for r in rows[3:]])
    T = D_print.shape[0]
    # O = ((Q K^T) * D) V with Q = ones, K = V = I gives O = D exactly.
    Q = np.ones((T, T))
    K = np.eye(T)
    V = np.eye(T)
    o, _, _ = run1(1, Q, K, V, gate=np.full(T, gamma))
    assert np.allclose(o, D_print, atol=5e-3)
    assert np.allclose(forms.decay_mask(np.full(T, gamma), T), D_print, atol=5e-3)
    # the page's recurrent-vs-parallel check on default_rng(0) inputs, fp64
    Qr, Kr, Vr = np.random.default_rng(0).normal(size=(3, 6, 4))
    o_rec, _, _ = run1(1, Qr, Kr, Vr, gate=np.full(6, gamma))
    o_par = forms.parallel_form(1, Qr, Kr, Vr, np.full(6, gamma))
    assert np.abs(o_rec - o_par).max() <= 100 * max_diff


def test_memory_capacity_table():
    rows = _rows("memory_capacity.txt")
    rng = np.random.default_rng(0)
    d = 32

    def cos_rows(a, b):
        return np.sum(a * b, axis=1) / np.linalg.norm(a, axis=1) / np.linalg.norm(b, axis=1)

    for n_s, lin_s, del_s, last_s in rows:
        n = int(n_s)
        K = rng.normal(size=(n, d))
        K /= np.linalg.norm(K, axis=1, keepdims=True)
        V = rng.normal(size=(n, d))
        _, S_lin, _ = run1(1, K, K, V, gate=np.ones(n))
        _, S_del, _ = run1(2, K, K, V, gate=np.ones(n), beta=np.ones(n))
        c_lin = cos_rows(K @ S_lin.T, V)
        c_del = cos_rows(K @ S_del.T, V)
        assert abs(c_lin.mean() - float(lin_s)) <= 5e-4, n
        assert abs(c_del.mean() - float(del_s)) <= 5e-4, n
        assert abs(c_del[-4:].mean() - float(last_s)) <= 5e-4, n


# ----------------------------------------------------------------------------------
# the three forms agree (brute force at T <= 64)
# ----------------------------------------------------------------------------------

@pytest.mark.parametrize("T", [1, 5, 17, 64])
def test_three_forms_agree_mode0(T):
    Q, K, V, _, _ = rng_inputs(10 + T, T, 4, 3)
    o, S, z = run1(0, Q, K, V)
    assert np.abs(o - forms.parallel_form(0, Q, K, V)).max() < 1e-12
    o_r, S_r, z_r = forms.recurrent_form(0, Q, K, V)
    assert np.abs(o - o_r).max() < 1e-12 and np.abs(S - S_r).max() < 1e-12
    assert np.abs(z - z_r).max() < 1e-12
    for C in (4, 16, 64):
        o_c, S_c, z_c = forms.chunked_form(0, Q, K, V, C)
        assert np.abs(o - o_c).max() < 1e-12 and np.abs(S - S_c).max() < 1e-11


@pytest.mark.parametrize("T", [1, 5, 17, 64])
def test_three_forms_agree_mode1(T):
    Q, K, V, a, _ = rng_inputs(20 + T, T, 5, 3)
    o, S, _ = run1(1, Q, K, V, gate=a)
    assert np.abs(o - forms.parallel_form(1, Q, K, V, a)).max() < 1e-12
    o_r, S_r, _ = forms.recurrent_form(1, Q, K, V, gate=a)
    assert np.abs(o - o_r).max() < 1e-12 and np.abs(S - S_r).max() < 1e-12
    for C in (4, 16, 64):
        o_c, S_c, _ = forms.chunked_form(1, Q, K, V, C, gate=a)
        assert np.abs(o - o_c).max() < 1e-12 and np.abs(S - S_c).max() < 1e-12


@pytest.mark.parametrize("T", [1, 5, 17, 64])
@pytest.mark.parametrize("weak_decay", [False, True])
def test_three_forms_agree_mode2(T, weak_decay):
    Q, K, V, a, b = rng_inputs(30 + T, T, 6, 4, unit_keys=True)
    if weak_decay:
        a = 0.98 + 0.02 * a
    S0 = np.random.default_rng(T).normal(size=(4, 6))
    o, S, _ = run1(2, Q, K, V, gate=a, beta=b, S0=S0)
    # literal Gated DeltaNet matrix form, token by token
    o_r, S_r, _ = forms.recurrent_form(2, Q, K, V, gate=a, beta=b, S0=S0)
    assert np.abs(o - o_r).max() < 1e-12 and np.abs(S - S_r).max() < 1e-12
    # the page gives no O(T^2) form for the delta rule: the chunked form with one
    # chunk (C = T) stands in for it, and C in {4, 16} is the chunked form
    for C in (T, 4, 16):
        o_c, S_c, _ = forms.chunked_form(2, Q, K, V, C, gate=a, beta=b, S0=S0)
        assert np.abs(o - o_c).max() < 1e-11 and np.abs(S - S_c).max() < 1e-11


def test_exercise_three_forms_and_state_shape():
    """The practice exercise: default_rng(0) Q, K, V of shape (6, 4), chunk 4."""
    Q, K, V = np.random.default_rng(0).normal(size=(3, 6, 4))
    o, S, z = run1(0, Q, K, V)
    assert np.allclose(forms.parallel_form(0, Q, K, V), o)
    assert np.allclose(forms.chunked_form(0, Q, K, V, 4)[0], o)
    assert S.shape == (4, 4) and z.shape == (4,)


# ----------------------------------------------------------------------------------
# closed forms and special cases
# ----------------------------------------------------------------------------------

def test_mode0_first_output_is_first_value_and_convexity():
    Q, K, V, _, _ = rng_inputs(1, 40, 8, 5)
    o, _, _ = run1(0, Q, K, V)
    assert np.allclose(o[0], V[0], rtol=0, atol=1e-14)
    for t in range(40):                       # convex combination of v_1..v_t
        assert np.all(o[t] <= V[:t + 1].max(axis=0) + 1e-12)
        assert np.all(o[t] >= V[:t + 1].min(axis=0) - 1e-12)


def test_mode0_equal_keys_give_prefix_mean():
    T = 30
    Q, _, V, _, _ = rng_inputs(2, T, 8, 5)
    K = np.tile(np.random.default_rng(3).normal(size=(1, 8)), (T, 1))
    o, _, _ = run1(0, Q, K, V)
    mean = np.cumsum(V, axis=0) / np.arange(1, T + 1)[:, None]
    assert np.abs(o - mean).max() < 1e-13


def test_mode1_ungated_is_brute_force_causal_sum():
    Q, K, V, _, _ = rng_inputs(4, 12, 5, 4)
    o, S, _ = run1(1, Q, K, V)                # NULL gate: a = 1
    ref = np.zeros_like(o)
    for i in range(12):
        for j in range(i + 1):
            ref[i] += (Q[i] @ K[j]) * V[j]
    assert np.abs(o - ref).max() < 1e-12
    assert np.abs(S - sum(np.outer(V[j], K[j]) for j in range(12))).max() < 1e-12


def test_mode1_constant_decay_closed_form():
    g = 0.7
    Q, K, V, _, _ = rng_inputs(5, 9, 4, 3)
    o, S, _ = run1(1, Q, K, V, gate=np.full(9, g))
    ref = np.zeros_like(o)
    for i in range(9):
        for j in range(i + 1):
            ref[i] += g ** (i - j) * (Q[i] @ K[j]) * V[j]
    assert np.abs(o - ref).max() < 1e-12
    assert np.abs(S - sum(g ** (8 - j) * np.outer(V[j], K[j]) for j in range(9))).max() < 1e-12


def test_mode2_identity_when_gate_one_beta_zero():
    Q, K, V, _, _ = rng_inputs(6, 20, 8, 6, unit_keys=True)
    S0 = np.random.default_rng(7).normal(size=(6, 8))
    o, S, _ = run1(2, Q, K, V, gate=np.ones(20), beta=np.zeros(20), S0=S0)
    assert np.array_equal(S, S0)
    assert np.abs(o - Q @ S0.T).max() < 1e-13


def test_mode2_beta_zero_only_decays():
    Q, K, V, a, _ = rng_inputs(8, 15, 8, 6, unit_keys=True)
    S0 = np.random.default_rng(9).normal(size=(6, 8))
    _, S, _ = run1(2, Q, K, V, gate=a, beta=np.zeros(15), S0=S0)
    assert np.abs(S - np.prod(a) * S0).max() < 1e-14


def test_mode2_orthonormal_keys_write_independently():
    d = 8
    Kb = np.linalg.qr(np.random.default_rng(11).normal(size=(d, d)))[0].T   # orthonormal rows
    r = np.random.default_rng(12)
    V = r.normal(size=(d, 5))
    b = r.uniform(0.1, 0.9, size=d)
    Q = r.normal(size=(d, d))
    _, S, _ = run1(2, Q, Kb, V, gate=np.ones(d), beta=b)
    ref = sum(b[t] * np.outer(V[t], Kb[t]) for t in range(d))
    assert np.abs(S - ref).max() < 1e-13


def test_mode2_equal_unit_keys_give_ema():
    T, d = 25, 6
    r = np.random.default_rng(13)
    k = r.normal(size=d)
    k /= np.linalg.norm(k)
    K = np.tile(k, (T, 1))
    V = r.normal(size=(T, 4))
    b = r.uniform(0.05, 0.95, size=T)
    S0 = r.normal(size=(4, d))
    Q = np.tile(k, (T, 1))                       # read along the key: o_t = S_t k
    o, _, _ = run1(2, Q, K, V, gate=np.ones(T), beta=b, S0=S0)
    m = S0 @ k
    for t in range(T):
        m = (1 - b[t]) * m + b[t] * V[t]
        assert np.abs(o[t] - m).max() < 1e-13


def test_mode2_contraction_bound():
    Q, K, V, a, b = rng_inputs(14, 50, 8, 5, unit_keys=True)
    S0 = np.random.default_rng(15).normal(size=(5, 8))
    S = S0
    for t in range(50):
        _, S_new, _ = run1(2, Q[t:t + 1], K[t:t + 1], V[t:t + 1], gate=a[t:t + 1],
                           beta=b[t:t + 1], S0=S)
        assert np.linalg.norm(S_new) <= a[t] * np.linalg.norm(S) + b[t] * np.linalg.norm(V[t]) + 1e-12
        S = S_new


# ----------------------------------------------------------------------------------
# structural invariants
# ----------------------------------------------------------------------------------

@pytest.mark.parametrize("mode", [0, 1, 2])
def test_state_shape_independent_of_length(mode):
    for T in (1, 10, 100):
        Q, K, V, a, b = rng_inputs(T, T, 7, 3, unit_keys=True)
        _, S, z = run1(mode, Q, K, V, gate=a, beta=b)
        assert S.shape == (3, 7)
        assert (z.shape == (7,)) if mode == 0 else z is None


@pytest.mark.parametrize("mode", [0, 1, 2])
def test_split_prefill_and_decode_continue_the_sequence(mode):
    T, T1 = 40, 23
    Q, K, V, a, b = rng_inputs(40 + mode, T, 6, 5, unit_keys=True)
    o, S, z = run1(mode, Q, K, V, gate=a, beta=b)
    o1, S1, z1 = run1(mode, Q[:T1], K[:T1], V[:T1], gate=a[:T1], beta=b[:T1])
    o2, S2, z2 = run1(mode, Q[T1:], K[T1:], V[T1:], gate=a[T1:], beta=b[T1:], S0=S1, z0=z1)
    assert np.abs(np.concatenate([o1, o2]) - o).max() < 1e-12
    assert np.abs(S2 - S).max() < 1e-12
    # prefill(T1) followed by decode steps == prefill(T)
    St, zt = S1[None, None], (None if z1 is None else z1[None, None])
    for t in range(T1, T):
        od, St, zt = oracle.decode_step(mode, Q[t][None, None], K[t][None, None], V[t][None, None],
                                        np.array([[a[t]]]), np.array([[b[t]]]), St, zt)
        assert np.abs(od[0, 0] - o[t]).max() < 1e-12
    assert np.abs(St[0, 0] - S).max() < 1e-12


@pytest.mark.parametrize("mode", [1, 2])
def test_linear_in_values_from_zero_state(mode):
    Q, K, V, a, b = rng_inputs(50, 30, 6, 4, unit_keys=True)
    V2 = np.random.default_rng(51).normal(size=V.shape)
    o1, S1, _ = run1(mode, Q, K, V, gate=a, beta=b)
    o2, S2, _ = run1(mode, Q, K, V2, gate=a, beta=b)
    o3, S3, _ = run1(mode, Q, K, 2.0 * V - 3.0 * V2, gate=a, beta=b)
    assert np.abs(o3 - (2 * o1 - 3 * o2)).max() < 1e-12
    assert np.abs(S3 - (2 * S1 - 3 * S2)).max() < 1e-12


@pytest.mark.parametrize("mode", [0, 1, 2])
def test_heads_and_batches_independent(mode):
    r = np.random.default_rng(60)
    B, H, T, dk, dv = 2, 3, 11, 5, 4
    q = r.normal(size=(B, H, T, dk))
    k = r.normal(size=(B, H, T, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = r.normal(size=(B, H, T, dv))
    a = r.uniform(0.3, 1.0, size=(B, H, T))
    b = r.uniform(0.0, 1.0, size=(B, H, T))
    o, S, z = oracle.prefill(mode, q, k, v, a, b)
    for bb in range(B):
        for hh in range(H):
            o1, S1, _ = run1(mode, q[bb, hh], k[bb, hh], v[bb, hh], gate=a[bb, hh], beta=b[bb, hh])
            assert np.array_equal(o[bb, hh], o1) and np.array_equal(S[bb, hh], S1)


def test_zero_length_sequence_keeps_state():
    S0 = np.random.default_rng(70).normal(size=(1, 1, 3, 4))
    o, S, _ = oracle.prefill(2, np.zeros((1, 1, 0, 4)), np.zeros((1, 1, 0, 4)),
                             np.zeros((1, 1, 0, 3)), np.zeros((1, 1, 0)), np.zeros((1, 1, 0)), S0)
    assert o.shape == (1, 1, 0, 3) and np.array_equal(S, S0)


def test_gate_zero_forgets_everything():
    """A gate of 0 erases the past (a document boundary)."""
    Q, K, V, a, b = rng_inputs(71, 10, 4, 3, unit_keys=True)
    a = a.copy()
    a[6] = 0.0
    for mode in (1, 2):
        o, S, _ = run1(mode, Q, K, V, gate=a, beta=b)
        o_tail, S_tail, _ = run1(mode, Q[6:], K[6:], V[6:], gate=a[6:], beta=b[6:])
        assert np.abs(o[6:] - o_tail).max() < 1e-14 and np.abs(S - S_tail).max() < 1e-14


# ----------------------------------------------------------------------------------
# Kimi Delta Attention (mode 3): the Gated DeltaNet update with Diag(a_t), one decay
# per channel of the memory (the d_k columns of S)
# ----------------------------------------------------------------------------------

def kda_inputs(seed, T, dk, dv):
    Q, K, V, _, b = rng_inputs(seed, T, dk, dv, unit_keys=True)
    r = np.random.default_rng(seed + 1000)
    a = 1.0 / (1.0 + np.exp(r.normal(size=(T, dk))))   # per-channel values in (0, 1)
    return Q, K, V, a, b


@pytest.mark.parametrize("T", [1, 5, 17, 64])
def test_three_forms_agree_mode3(T):
    """C oracle == literal per-token matrix form S Diag(a)(I - b k k^T) + b v k^T ==
    the per-channel chunked form derived for it (one chunk and C in {4, 16})."""
    Q, K, V, a, b = kda_inputs(80 + T, T, 6, 4)
    S0 = np.random.default_rng(T + 5).normal(size=(4, 6))
    o, S, _ = run1(3, Q, K, V, gate=a, beta=b, S0=S0)
    o_r, S_r, _ = forms.recurrent_form(3, Q, K, V, gate=a, beta=b, S0=S0)
    assert np.abs(o - o_r).max() < 1e-12 and np.abs(S - S_r).max() < 1e-12
    for C in (T, 4, 16):
        o_c, S_c, _ = forms.chunked_form(3, Q, K, V, C, gate=a, beta=b, S0=S0)
        assert np.abs(o - o_c).max() < 1e-11 and np.abs(S - S_c).max() < 1e-11


def test_mode3_uniform_channels_is_gated_deltanet():
    """Diag(a_t) with all channels equal to a_t is the scalar Gated DeltaNet gate."""
    Q, K, V, a, b = rng_inputs(90, 33, 8, 5, unit_keys=True)
    S0 = np.random.default_rng(91).normal(size=(5, 8))
    o2, S2, _ = run1(2, Q, K, V, gate=a, beta=b, S0=S0)
    o3, S3, _ = run1(3, Q, K, V, gate=np.repeat(a[:, None], 8, axis=1), beta=b, S0=S0)
    assert np.abs(o3 - o2).max() < 1e-13 and np.abs(S3 - S2).max() < 1e-13


def test_mode3_ungated_is_the_delta_rule():
    Q, K, V, _, b = rng_inputs(92, 21, 6, 4, unit_keys=True)
    o2, S2, _ = run1(2, Q, K, V, gate=None, beta=b)
    o3, S3, _ = run1(3, Q, K, V, gate=None, beta=b)
    assert np.array_equal(o3, o2) and np.array_equal(S3, S2)


def test_mode3_beta_zero_decays_each_channel():
    """b = 0 writes nothing: S_t = S_0 Diag(a_1 ... a_t), so column c of the state decays
    by its own product and o_t = S_0 Diag(prod) q_t."""
    Q, K, V, a, _ = kda_inputs(93, 12, 7, 4)
    S0 = np.random.default_rng(94).normal(size=(4, 7))
    o, S, _ = run1(3, Q, K, V, gate=a, beta=np.zeros(12), S0=S0)
    P = np.cumprod(a, axis=0)
    assert np.abs(S - S0 * P[-1][None, :]).max() < 1e-14
    assert np.abs(o - (Q * P) @ S0.T).max() < 1e-13


def test_mode3_closed_channel_keeps_only_fresh_writes():
    """A channel whose decay is 0 at every token holds only the latest write in it:
    column c of S_t is b_t (v_t - (M k_t)) k_t[c] with M the decayed old state."""
    Q, K, V, a, b = kda_inputs(95, 9, 5, 3)
    a = a.copy()
    a[:, 2] = 0.0
    _, S, _ = run1(3, Q, K, V, gate=a, beta=b)
    _, S8, _ = run1(3, Q[:8], K[:8], V[:8], gate=a[:8], beta=b[:8])
    M = S8 * a[8][None, :]
    col = b[8] * (V[8] - M @ K[8]) * K[8][2]
    assert np.abs(S[:, 2] - col).max() < 1e-13


def test_mode3_split_prefill_and_decode_continue():
    T, T1 = 30, 17
    Q, K, V, a, b = kda_inputs(96, T, 6, 5)
    o, S, _ = run1(3, Q, K, V, gate=a, beta=b)
    o1, S1, _ = run1(3, Q[:T1], K[:T1], V[:T1], gate=a[:T1], beta=b[:T1])
    o2, S2, _ = run1(3, Q[T1:], K[T1:], V[T1:], gate=a[T1:], beta=b[T1:], S0=S1)
    assert np.abs(np.concatenate([o1, o2]) - o).max() < 1e-12 and np.abs(S2 - S).max() < 1e-12
    St = S1[None, None]
    for t in range(T1, T):
        od, St, _ = oracle.decode_step(3, Q[t][None, None], K[t][None, None], V[t][None, None],
                                       a[t][None, None], np.array([[b[t]]]), St)
        assert np.abs(od[0, 0] - o[t]).max() < 1e-12
    assert np.abs(St[0, 0] - S).max() < 1e-12


def test_mode3_linear_in_values_from_zero_state():
    Q, K, V, a, b = kda_inputs(97, 25, 6, 4)
    V2 = np.random.default_rng(98).normal(size=V.shape)
    o1, S1, _ = run1(3, Q, K, V, gate=a, beta=b)
    o2, S2, _ = run1(3, Q, K, V2, gate=a, beta=b)
    o3, S3, _ = run1(3, Q, K, 2.0 * V - 3.0 * V2, gate=a, beta=b)
    assert np.abs(o3 - (2 * o1 - 3 * o2)).max() < 1e-12 and np.abs(S3 - (2 * S1 - 3 * S2)).max() < 1e-12


# ---- packed variable-length sequences
@pytest.mark.parametrize("mode", [0, 1, 2, 3])
def test_packed_equal_lengths_match_the_batched_call(mode):
    """N packed sequences of one length are the batch [N, H, L, d] of the dense call."""
    r = np.random.default_rng(70 + mode)
    N, H, L, dk, dv = 3, 2, 9, 4, 3
    q, k, v = r.normal(size=(N, H, L, dk)), r.normal(size=(N, H, L, dk)), r.normal(size=(N, H, L, dv))
    gshape = (N, H, L, dk) if mode == 3 else (N, H, L)
    gate = None if mode == 0 else 1 / (1 + np.exp(r.normal(size=gshape)))
    beta = 1 / (1 + np.exp(r.normal(size=(N, H, L)))) if mode >= 2 else None
    S0 = r.normal(size=(N, H, dv, dk)) * 0.1
    z0 = r.random(size=(N, H, dk)) + 1.0 if mode == 0 else None
    o, S, z = oracle.prefill(mode, q, k, v, gate, beta, S0, z0)
    pk = lambda x: None if x is None else np.concatenate(list(x), axis=1)   # [H, N*L, ..]
    cu = np.arange(N + 1) * L
    po, pS, pz = oracle.prefill_packed(mode, pk(q), pk(k), pk(v), cu, pk(gate), pk(beta), S0, z0)
    np.testing.assert_allclose(po, pk(o), rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(pS, S, rtol=1e-13, atol=1e-13)
    if mode == 0:
        np.testing.assert_allclose(pz, z, rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("mode", [1, 2, 3])
def test_packed_boundary_is_a_zero_gate(mode):
    """The page's document boundary: a gate a_t = 0 at the first token of a document
    forgets everything before it.  So one dense sequence with a = 0 at each boundary
    gives the packed result of the documents taken separately from zero states."""
    r = np.random.default_rng(80 + mode)
    H, T, dk, dv = 2, 23, 4, 3
    cu = np.array([0, 7, 8, 16, 23])
    q, k, v = r.normal(size=(H, T, dk)), r.normal(size=(H, T, dk)), r.normal(size=(H, T, dv))
    gshape = (H, T, dk) if mode == 3 else (H, T)
    gate = 1 / (1 + np.exp(r.normal(size=gshape)))
    beta = 1 / (1 + np.exp(r.normal(size=(H, T)))) if mode >= 2 else None
    po, pS, _ = oracle.prefill_packed(mode, q, k, v, cu, gate, beta)
    g0 = gate.copy()
    g0[:, cu[1:-1]] = 0.0
    o, S, _ = oracle.prefill(mode, q[None], k[None], v[None], g0[None],
                             None if beta is None else beta[None])
    np.testing.assert_allclose(po, o[0], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(pS[-1], S[0], rtol=1e-12, atol=1e-12)


def test_packed_empty_sequence_keeps_its_start_state():
    r = np.random.default_rng(90)
    H, dk, dv = 2, 4, 3
    cu = np.array([0, 5, 5, 9])
    q, k, v = r.normal(size=(H, 9, dk)), r.normal(size=(H, 9, dk)), r.normal(size=(H, 9, dv))
    S0 = r.normal(size=(3, H, dv, dk))
    _, pS, _ = oracle.prefill_packed(1, q, k, v, cu, None, None, S0)
    np.testing.assert_array_equal(pS[1], S0[1])
    _, pS0, _ = oracle.prefill_packed(1, q, k, v, cu)
    np.testing.assert_array_equal(pS0[1], 0.0)


# ---- constant decay per head (RetNet / Lightning): mode 4
def test_retnet_mode_matches_the_decay_mask_closed_form():
    """[decay/gates]: with a constant gamma the decay mask is D_ij = gamma^(i-j); per head
    o_t = sum_{j<=t} gamma_h^(t-j) (q_t . k_j) v_j and S_T = sum_j gamma_h^(T-1-j) v_j k_j^T."""
    r = np.random.default_rng(95)
    B, H, T, dk, dv = 2, 3, 13, 4, 5
    q, k, v = r.normal(size=(B, H, T, dk)), r.normal(size=(B, H, T, dk)), r.normal(size=(B, H, T, dv))
    gam = np.array([0.9, 0.5, 0.99])
    o, S, _ = oracle.prefill(oracle.MODE_RETNET, q, k, v, gam)
    t = np.arange(T)
    for h in range(H):
        D = np.where(t[:, None] >= t[None, :], gam[h] ** (t[:, None] - t[None, :]).clip(min=0), 0.0)
        for b in range(B):
            ref_o = (D * (q[b, h] @ k[b, h].T)) @ v[b, h]
            ref_S = (v[b, h].T * gam[h] ** (T - 1 - t)) @ k[b, h]
            np.testing.assert_allclose(o[b, h], ref_o, rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(S[b, h], ref_S, rtol=1e-12, atol=1e-12)
    # the decode step with the same constant gates continues the sequence
    od, Sd, _ = oracle.decode_step(oracle.MODE_RETNET, q[:, :, -1], k[:, :, -1], v[:, :, -1], gam, None,
                                   oracle.prefill(oracle.MODE_RETNET, q[:, :, :-1], k[:, :, :-1],
                                                  v[:, :, :-1], gam)[1])
    np.testing.assert_allclose(od, o[:, :, -1], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(Sd, S, rtol=1e-12, atol=1e-12)
