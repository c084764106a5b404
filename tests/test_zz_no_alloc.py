"""la_prefill_noalloc: prefill for callers that cannot allocate device memory.

Some callers have no device allocator they may use (code inside another framework's
memory pool, processes that reserve all device memory up front).  The entry point
takes its scratch from a fixed 24 MiB array inside the library instead of a
caller-provided workspace.  These tests call it through the C ABI (ctypes) and check
its results against the regular la_prefill (given a torch-allocated workspace) on two
calls in a row with different inputs, and that oversized problems are refused.

This file is collected last so that a failure here cannot hide the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads as W
from parity_util import TOL, f64, slice_rel_err

LA_ERR_UNSUPPORTED = 2
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


def test_noalloc_refuses_problems_beyond_its_buffer():
    la, lib = _lib()
    # gated delta rule, 4 heads of 65536 tokens: the segment plan needs > 24 MiB
    need = lib.la_prefill_workspace_size(2, 1, 1, 4, 65536, 128, 128, 0)
    assert need > STATIC_BYTES
    st = lib.la_prefill_noalloc(2, 1, 1, 4, 65536, 128, 128, *([None] * 8), 0, 0, None)
    assert st == LA_ERR_UNSUPPORTED


@pytest.mark.gpu
@pytest.mark.parametrize("mode", [2, 0, 1])
def test_noalloc_matches_prefill_on_two_calls(mode):
    la, lib = _lib()
    B, H, T = 1, 4, 4096
    need = la.workspace_size(mode, torch.bfloat16, B, H, T, 128, 128)
    assert 0 < need <= STATIC_BYTES        # the static buffer is really used
    stream = torch.cuda.current_stream()
    for seed in (101, 202):                # two calls in a row, different inputs
        w = W.Workload("noalloc", mode, torch.bfloat16, B=B, H=H, T=T, dk=128, dv=128, seed=seed,
                       qk_scale=1 / np.sqrt(128), qk_l2norm=(mode == 2),
                       gate="none" if mode == 0 else "softplus", gate_shift=-3.0,
                       beta=(mode == 2))
        inp = W.prefill_inputs(w, device="cuda", init_state_std=0.05)
        z0 = torch.rand(B, H, 128, device="cuda") + 1.0 if mode == 0 else None
        # the existing entry point, with a torch-allocated workspace
        S_ref = inp["state0"].clone()
        z_ref = None if z0 is None else z0.clone()
        o_ref, S_ref, z_ref = la.prefill(inp["q"], inp["k"], inp["v"], mode=mode,
                                         gate=inp["gate"], beta=inp["beta"], state=S_ref, z=z_ref,
                                         init_state=True)
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
