"""fp64 CPU oracle for causal linear attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may
import this package.  The product path (``gated_delta_rule_attention_b200``) never
imports it, and this package imports nothing from the product.

Two parts:

* ``la_oracle.c`` -- the recurrent form in plain C, fp64, OpenMP over (batch, head).
  This is *the* oracle: it is the definition written out (the recurrent form of the
  lesson page "Linear attention and hybrids", section "Three forms of one
  computation", the decay of section "Memory must forget", and the Gated DeltaNet
  equation of section "The delta rule and Gated DeltaNet").
* ``forms.py`` -- numpy fp64 restatements of the parallel and chunked forms (and a
  literal per-token matrix form of the Gated DeltaNet update) for tiny inputs.  They
  exist to pin the C oracle to the page's claim that the three forms agree to
  rounding; they are not used to check GPU output.

Inputs are taken as the exact values the GPU receives (bf16/fp32 upcast to fp64).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "la_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

MODE_ELU1_NORM = 0
MODE_GATED = 1
MODE_GATED_DELTA = 2
MODE_KDA = 3
MODE_RETNET = 4   # mode 1 with one constant gate per head: gate [H]



def build(force: bool = False) -> str:
    """Compile ``la_oracle.c`` into ``liboracle.so`` (gcc, -O3, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O3", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-Wall",
               "-fno-fast-math", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            # A test that plants a mistake in a copy of la_oracle.c points this at the
            # planted build, to check that the pins catch it.
            path = os.environ.get("LA_ORACLE_LIB_OVERRIDE")
            if not path:
                path = build()
            lib = ctypes.CDLL(path)
            dp = ctypes.POINTER(ctypes.c_double)
            lib.oracle_prefill.argtypes = [ctypes.c_int, ctypes.c_long, ctypes.c_long, ctypes.c_long,
                                           ctypes.c_int, ctypes.c_int, dp, dp, dp, dp, dp, dp, dp, dp,
                                           ctypes.c_int, ctypes.c_int]
            lib.oracle_prefill.restype = ctypes.c_int
            lib.oracle_decode_step.argtypes = [ctypes.c_int, ctypes.c_long, ctypes.c_long,
                                               ctypes.c_int, ctypes.c_int, dp, dp, dp, dp, dp, dp,
                                               dp, dp, ctypes.c_int]
            lib.oracle_decode_step.restype = ctypes.c_int
            lib.oracle_max_threads.argtypes = []
            lib.oracle_max_threads.restype = ctypes.c_int
            _lib = lib
    return _lib


def _f64(x, shape=None):
    if x is None:
        return None
    a = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    if shape is not None and a.shape != tuple(shape):
        raise ValueError(f"expected shape {tuple(shape)}, got {a.shape}")
    return a


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def max_threads() -> int:
    """Threads the oracle's OpenMP loop uses by default."""
    return int(_load().oracle_max_threads())


def prefill(mode, q, k, v, gate=None, beta=None, state=None, z=None, nthreads=0):
    """Recurrent form over a whole sequence.

    q, k: [B,H,T,d_k]; v: [B,H,T,d_v]; gate, beta: [B,H,T] or None (mode 3: gate
    [B,H,T,d_k], one decay per channel);
    state: [B,H,d_v,d_k] initial state (None -> zero); z: [B,H,d_k] initial
    normaliser for mode 0 (None -> zero).
    Returns (o [B,H,T,d_v], S [B,H,d_v,d_k], z [B,H,d_k] or None), all fp64.
    """
    q = _f64(q)
    B, H, T, dk = q.shape
    if mode == MODE_RETNET:
        g = np.asarray(gate, dtype=np.float64).reshape(1, H, 1)
        mode, gate = 1, np.broadcast_to(g, (B, H, T)).copy()
    k = _f64(k, (B, H, T, dk))
    v = _f64(v)
    dv = v.shape[-1]
    if v.shape != (B, H, T, dv):
        raise ValueError("v shape mismatch")
    gate = _f64(gate, (B, H, T, dk) if mode == MODE_KDA else (B, H, T))
    beta = _f64(beta, (B, H, T))
    init = state is not None or (mode == 0 and z is not None)
    S = np.zeros((B, H, dv, dk)) if state is None else _f64(state, (B, H, dv, dk)).copy()
    zz = None
    if mode == 0:
        zz = np.zeros((B, H, dk)) if z is None else _f64(z, (B, H, dk)).copy()
    o = np.zeros((B, H, T, dv))
    rc = _load().oracle_prefill(int(mode), B, H, T, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(gate),
                                _ptr(beta), _ptr(S), _ptr(zz), _ptr(o), int(init), int(nthreads))
    if rc != 0:
        raise ValueError("oracle_prefill rejected its arguments")
    return o, S, zz


def decode_step(mode, q, k, v, gate, beta, state, z=None, nthreads=0):
    """One recurrent token for N sequences: q,k [N,H,d_k]; v [N,H,d_v]; gate, beta [N,H]
    (mode 3: gate [N,H,d_k]).

    Returns (o [N,H,d_v], S_new [N,H,d_v,d_k], z_new or None); inputs are not modified.
    """
    q = _f64(q)
    N, H, dk = q.shape
    if mode == MODE_RETNET:
        g = np.asarray(gate, dtype=np.float64).reshape(1, H)
        mode, gate = 1, np.broadcast_to(g, (N, H)).copy()
    k = _f64(k, (N, H, dk))
    v = _f64(v)
    dv = v.shape[-1]
    gate = _f64(gate, (N, H, dk) if mode == MODE_KDA else (N, H))
    beta = _f64(beta, (N, H))
    S = _f64(state, (N, H, dv, dk)).copy()
    zz = None
    if mode == 0:
        zz = np.zeros((N, H, dk)) if z is None else _f64(z, (N, H, dk)).copy()
    o = np.zeros((N, H, dv))
    rc = _load().oracle_decode_step(int(mode), N, H, dk, dv, _ptr(q), _ptr(k), _ptr(v),
                                    _ptr(gate), _ptr(beta), _ptr(S), _ptr(zz), _ptr(o),
                                    int(nthreads))
    if rc != 0:
        raise ValueError("oracle_decode_step rejected its arguments")
    return o, S, zz


def prefill_packed(mode, q, k, v, cu, gate=None, beta=None, state=None, z=None, nthreads=0):
    """Packed variable-length sequences: the recurrent form run on every sequence of the
    packed token axis on its own (sequence s = tokens cu[s] .. cu[s+1]).

    q, k: [H,T,d_k]; v: [H,T,d_v]; gate, beta: [H,T] (mode 3: gate [H,T,d_k]) or None;
    state: [N,H,d_v,d_k] start states (None -> zero); z: [N,H,d_k] (mode 0).
    Returns (o [H,T,d_v], S [N,H,d_v,d_k], z [N,H,d_k] or None), fp64.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    H, T, dk = q.shape
    dv = v.shape[-1]
    if mode == MODE_RETNET:
        g = np.asarray(gate, dtype=np.float64).reshape(H, 1)
        mode, gate = 1, np.broadcast_to(g, (H, T)).copy()
    cu = [int(x) for x in np.asarray(cu).reshape(-1)]
    N = len(cu) - 1
    o = np.zeros((H, T, dv))
    S = np.zeros((N, H, dv, dk))
    zz = np.zeros((N, H, dk)) if mode == 0 else None
    for s in range(N):
        a, b = cu[s], cu[s + 1]
        sl = lambda x: None if x is None else _f64(x)[:, a:b][None]
        st = None if state is None else _f64(state)[s][None]
        z0 = None if z is None else _f64(z)[s][None]
        if b > a:
            os_, Ss, zs = prefill(mode, sl(q), sl(k), sl(v), sl(gate), sl(beta), st, z0, nthreads)
            o[:, a:b] = os_[0]
            S[s] = Ss[0]
            if zz is not None:
                zz[s] = zs[0]
        else:   # no tokens: the state is the start state
            if state is not None:
                S[s] = _f64(state)[s]
            if zz is not None and z is not None:
                zz[s] = _f64(z)[s]
    return o, S, zz
