"""numpy fp64 restatements of the three forms of causal linear attention (tiny inputs).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).  These functions pin the C
oracle: the lesson page "Linear attention and hybrids" states that the parallel,
recurrent and chunked forms give the same output up to rounding (section "Three forms
of one computation"; its decay check in section "Practice" prints a max difference of
1.1e-15).  Every function works on ONE head: Q, K [T, d_k], V [T, d_v], gate/beta [T].

Citations (sections of that page, translated):
  [kernel trick]  "The kernel trick: removing softmax"    -- phi, S_i, z_i
  [three forms]   "Three forms of one computation"        -- parallel/recurrent/chunked
  [decay/gates]   "Memory must forget: decay and gates"   -- gamma, D mask, alpha_t gate
  [delta rule]    "The delta rule and Gated DeltaNet"     -- delta rule, Gated DeltaNet
"""
from __future__ import annotations

import numpy as np


def feature_map(x):
    """phi(x) = elu(x) + 1: x + 1 where x > 0, e^x elsewhere ([kernel trick])."""
    x = np.asarray(x, dtype=np.float64)
    return np.where(x > 0, x + 1.0, np.exp(np.minimum(x, 0.0)))


def decay_mask(gate, T):
    """D[i, j] = a_{j+1} * ... * a_i for j <= i (1 on the diagonal), 0 above it
    ([decay/gates]: the input-dependent gate; a constant gate gives gamma^(i-j))."""
    a = np.ones(T) if gate is None else np.asarray(gate, dtype=np.float64)
    D = np.zeros((T, T))
    for i in range(T):
        for j in range(i + 1):
            D[i, j] = np.prod(a[j + 1:i + 1])
    return D


def parallel_form(mode, Q, K, V, gate=None):
    """The O(T^2) masked-matrix form for modes 0 and 1.

    mode 0 ([three forms], parallel form): A = phi(Q) phi(K)^T, causal mask,
    row-normalised: o_i = (A_i V) / sum_j A_ij.
    mode 1 ([decay/gates]): O = ((Q K^T) * D) V with the decay mask D.
    """
    T = Q.shape[0]
    if mode == 0:
        A = feature_map(Q) @ feature_map(K).T
        A = np.tril(A)
        return (A @ V) / A.sum(axis=1, keepdims=True)
    if mode == 1:
        return ((Q @ K.T) * decay_mask(gate, T)) @ V
    raise ValueError("the page gives no O(T^2) form for the delta rule")


def recurrent_form(mode, Q, K, V, gate=None, beta=None, S0=None, z0=None):
    """Token-by-token recurrence (update, then read) in numpy.

    For mode 2 the Gated DeltaNet update of [delta rule] is evaluated literally with
    the d_k x d_k matrix (I - b_t k_t k_t^T): S_t = a_t S_{t-1} (I - b_t k k^T) + b_t v k^T.
    Mode 3 (Kimi Delta Attention) replaces a_t by the diagonal matrix Diag(a_t) (gate
    [T, d_k]): S_t = S_{t-1} Diag(a_t) (I - b_t k k^T) + b_t v k^T.
    Returns (O, S_T, z_T).
    """
    T, dk = Q.shape
    dv = V.shape[1]
    S = np.zeros((dv, dk)) if S0 is None else np.array(S0, dtype=np.float64)
    z = np.zeros(dk) if z0 is None else np.array(z0, dtype=np.float64)
    if mode == 3:
        a = np.ones((T, dk)) if gate is None else np.asarray(gate, dtype=np.float64)
    else:
        a = np.ones(T) if gate is None else np.asarray(gate, dtype=np.float64)
    O = np.zeros((T, dv))
    I = np.eye(dk)
    for t in range(T):
        if mode == 0:
            fk, fq = feature_map(K[t]), feature_map(Q[t])
            S = S + np.outer(V[t], fk)
            z = z + fk
            O[t] = (S @ fq) / (z @ fq)
        elif mode == 1:
            S = a[t] * S + np.outer(V[t], K[t])
            O[t] = S @ Q[t]
        elif mode == 3:
            b = beta[t]
            S = S @ np.diag(a[t]) @ (I - b * np.outer(K[t], K[t])) + b * np.outer(V[t], K[t])
            O[t] = S @ Q[t]
        else:
            b = beta[t]
            S = a[t] * S @ (I - b * np.outer(K[t], K[t])) + b * np.outer(V[t], K[t])
            O[t] = S @ Q[t]
    return O, S, (z if mode == 0 else None)


def chunked_form(mode, Q, K, V, C, gate=None, beta=None, S0=None, z0=None):
    """Chunked (block-parallel) form with blocks of C tokens; the last may be shorter.

    modes 0/1 follow [three forms] (chunked form): inside a block the masked C x C
    matrix, across blocks the state,
        O_b = [(phi(Q_b) phi(K_b)^T) * M] V_b + phi(Q_b) S_{b-1}^T,
        S_b = S_{b-1} + V_b^T phi(K_b)     (plus the same for the normaliser z),
    with the decay of [decay/gates] folded in for mode 1 (M -> D restricted to the
    block, the carried state decayed by the in-block gate products).

    mode 2 has no chunked form on the page (it only says one was found); this is the
    reading derived for it: within a block, with g_i = a_s ... a_i (inclusive) and
    D the in-block decay mask, the write vectors e_t = b_t (v_t - a_t S_{t-1} k_t)
    solve the unit lower-triangular system (I + L) E = diag(b) V - diag(b g) K S^T,
    L_ij = b_i D_ij (k_i . k_j) for j < i.  Then
        O = diag(g) Q S^T + ((Q K^T) * D) E,   S_new = g_last S + sum_j D_last,j e_j k_j^T.

    mode 3 (per-channel decay, gate [T, d_k]) is the same derivation with the in-block
    inclusive products G_i = a_s * ... * a_i taken per channel: the decay of a key j seen
    from row i is G_i / G_j channel by channel, so
        L_ij = b_i (k_i * G_i) . (k_j / G_j)  (j < i),   A_ij = (q_i * G_i) . (k_j / G_j)  (j <= i),
        (I + L) E = diag(b) V - diag(b) (K * G) S^T,
        O = (Q * G) S^T + A E,   S_new = S Diag(G_last) + E^T (K * G_last / G).
    Returns (O, S, z).
    """
    T, dk = Q.shape
    dv = V.shape[1]
    S = np.zeros((dv, dk)) if S0 is None else np.array(S0, dtype=np.float64)
    z = np.zeros(dk) if z0 is None else np.array(z0, dtype=np.float64)
    if mode == 3:
        a_all = np.ones((T, dk)) if gate is None else np.asarray(gate, dtype=np.float64)
    else:
        a_all = np.ones(T) if gate is None else np.asarray(gate, dtype=np.float64)
    O = np.zeros((T, dv))
    for s in range(0, T, C):
        e = min(s + C, T)
        L = e - s
        q, k, v, a = Q[s:e], K[s:e], V[s:e], a_all[s:e]
        if mode == 3:
            b = np.asarray(beta[s:e], dtype=np.float64)
            G = np.cumprod(a, axis=0)                      # [L, d_k] in-block channel products
            kg, kin = k * G, k / G
            Lm = np.tril(b[:, None] * (kg @ kin.T), -1)
            A = np.tril((q * G) @ kin.T)
            Tinv = np.linalg.inv(np.eye(L) + Lm)
            U, W = Tinv @ (b[:, None] * v), Tinv @ (b[:, None] * kg)
            E = U - W @ S.T
            O[s:e] = (q * G) @ S.T + A @ E
            S = S * G[-1][None, :] + E.T @ (k * (G[-1][None, :] / G))
            continue
        g = np.array([np.prod(a[:i + 1]) for i in range(L)])  # in-block inclusive gate products
        D = decay_mask(a, L)
        if mode == 0:
            fq, fk = feature_map(q), feature_map(k)
            A = np.tril(fq @ fk.T)
            num = A @ v + fq @ S.T
            den = A.sum(axis=1) + fq @ z
            O[s:e] = num / den[:, None]
            S = S + v.T @ fk
            z = z + fk.sum(axis=0)
        elif mode == 1:
            O[s:e] = g[:, None] * (q @ S.T) + ((q @ k.T) * D) @ v
            S = g[-1] * S + (D[-1][:, None] * v).T @ k
        else:
            b = np.asarray(beta[s:e], dtype=np.float64)
            Lm = np.tril(b[:, None] * D * (k @ k.T), -1)
            rhs_u = b[:, None] * v
            rhs_w = (b * g)[:, None] * k
            Tinv = np.linalg.inv(np.eye(L) + Lm)
            U, W = Tinv @ rhs_u, Tinv @ rhs_w
            E = U - W @ S.T
            O[s:e] = g[:, None] * (q @ S.T) + ((q @ k.T) * D) @ E
            S = g[-1] * S + (D[-1][:, None] * E).T @ k
    return O, S, (z if mode == 0 else None)
