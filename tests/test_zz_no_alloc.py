"""la_prefill_noalloc: prefill for callers that cannot allocate device memory.

Some callers have no device allocator they may use (code inside another framework's
memory pool, processes that reserve all device memory up front).  The entry point
takes its scratch from a fixed 24 MiB array inside the library instead of a
caller-provided workspace.  These tests call it through the C ABI (ctypes) and check its
results against the regular la_prefill (given a torch-allocated workspace) and against
the fp64 oracle on sampled heads, on two calls in a row with different inputs: every
mode at a ragged length whose segment plan fits the array, a problem whose fastest plan
does not fit (a smaller plan runs), and one where no segmented plan fits (the single
pass runs).

This file is collected last so that a failure here cannot hide the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads as W
from parity_util import TOL, f64, oracle_prefill_slices, pick, slice_rel_err

LA_ERR_INVALID_ARG = 1
STATIC_BYTES = 24 << 20


def _lib():
    from gated_delta_rule_attention_b200 import build
    build.build()
    import gated_delta_rule_attention_b200 as la
    lib = la.library()
    vp, i, u = ctypes.c_void_p, ctypes.c_int, ctypes.c_uint
    lib.la_prefill_noalloc.argtypes = [i, i, i, i, i, i, i, vp, vp, vp, vp, vp, vp, vp, vp, i, u,
                                       vp]
    lib.la_prefill_noalloc.restype = i
    return la, lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def test_noalloc_accepts_what_prefill_accepts():
    """A problem whose smallest segment plan needs more than the array is not refused for
    its size: the host checks answer exactly as la_prefill's do (here: NULL tensors)."""
    la, lib = _lib()
    need = lib.la_prefill_workspace_size(2, 1, 1, 4, 65536, 128, 128, 0)
    assert need > STATIC_BYTES
    st = lib.la_prefill_noalloc(2, 1, 1, 4, 65536, 128, 128, *([None] * 8), 0, 0, None)
    assert st == LA_ERR_INVALID_ARG


def _run_both(la, lib, mode, B, H, T, seed, heads):
    """One call of each entry point on the same seeded inputs; returns nothing, asserts."""
    w = W.Workload("noalloc", mode, torch.bfloat16, B=B, H=H, T=T, dk=128, dv=128, seed=seed,
                   qk_scale=1 / np.sqrt(128), qk_l2norm=(mode >= 2),
                   gate="none" if mode == 0 else "softplus", gate_shift=-3.0, beta=(mode >= 2))
    inp = W.prefill_inputs(w, device="cuda", init_state_std=0.05)
    z0 = torch.rand(B, H, 128, device="cuda") + 1.0 if mode == 0 else None
    stream = torch.cuda.current_stream()
    # the existing entry point, with a torch-allocated workspace
    S_ref = inp["state0"].clone()
    z_ref = None if z0 is None else z0.clone()
    o_ref, S_ref, z_ref = la.prefill(inp["q"], inp["k"], inp["v"], mode=mode, gate=inp["gate"],
                                     beta=inp["beta"], state=S_ref, z=z_ref, init_state=True)
    la.check_status()
    # the no-alloc entry point through the C ABI
    S = inp["state0"].clone()
    z = None if z0 is None else z0.clone()
    o = torch.empty_like(o_ref)
    st = lib.la_prefill_noalloc(mode, 1, B, H, T, 128, 128, _ptr(inp["q"]), _ptr(inp["k"]),
                                _ptr(inp["v"]), _ptr(inp["gate"]), _ptr(inp["beta"]), _ptr(S),
                                _ptr(z), _ptr(o), 0, 1, ctypes.c_void_p(stream.cuda_stream))
    assert st == 0, lib.la_status_string(st)
    la.check_status()
    tol = TOL[torch.bfloat16]
    assert slice_rel_err(f64(o), f64(o_ref)) <= tol
    assert slice_rel_err(f64(S), f64(S_ref)) <= tol
    if mode == 0:
        assert slice_rel_err(f64(z), f64(z_ref)) <= tol
    # and against the oracle on the sampled heads
    ro, rS, rz = oracle_prefill_slices(mode, inp, heads, init_state=True, z0=z0)
    assert slice_rel_err(pick(o, heads), ro, lead=1) <= tol
    assert slice_rel_err(pick(S, heads), rS, lead=1) <= tol
    if mode == 0:
        assert slice_rel_err(pick(z, heads), rz, lead=1) <= tol


@pytest.mark.gpu
@pytest.mark.parametrize("mode", [0, 1, 2, 3])
def test_noalloc_matches_prefill_and_oracle_on_two_calls(mode):
    la, lib = _lib()
    B, H, T = 1, 4, 4000                   # a ragged last chunk (4000 = 62 x 64 + 32)
    need = la.workspace_size(mode, torch.bfloat16, B, H, T, 128, 128)
    assert 0 < need <= STATIC_BYTES        # the static array is really used
    for seed in (101, 202):                # two calls in a row, different inputs
        _run_both(la, lib, mode, B, H, T, seed, [(0, 0), (0, 3)])


@pytest.mark.gpu
def test_noalloc_runs_a_smaller_plan_when_the_fastest_does_not_fit():
    """KDA at B1 H32 T16384: the fastest segment plan needs 32 MiB, the smaller one fits."""
    la, lib = _lib()
    B, H, T = 1, 32, 16384
    assert la.workspace_size(3, torch.bfloat16, B, H, T, 128, 128) > STATIC_BYTES
    for seed in (303, 404):
        _run_both(la, lib, 3, B, H, T, seed, [(0, 5)])


@pytest.mark.gpu
def test_noalloc_runs_the_single_pass_when_no_plan_fits():
    """The gated delta rule at B1 H4 T65536: every segment plan needs more than 24 MiB, so
    the single pass (no workspace) runs."""
    la, lib = _lib()
    B, H, T = 1, 4, 65536
    assert la.workspace_size(2, torch.bfloat16, B, H, T, 128, 128) > STATIC_BYTES
    for seed in (505, 606):
        _run_both(la, lib, 2, B, H, T, seed, [(0, 1)])
