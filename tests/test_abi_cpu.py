"""The C-ABI library loads on a machine without a GPU and exports what include/la.h declares.

No compute call is made here: only symbol lookup, status strings, and argument checks
that the library answers on the host before touching the device.
"""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER_DIR = os.path.join(ROOT, "include")


@pytest.fixture(scope="module")
def lib():
    from gated_delta_rule_attention_b200 import build
    build.build()
    import gated_delta_rule_attention_b200 as la
    return la.library()


def declared_functions():
    names = []
    for fn in sorted(os.listdir(HEADER_DIR)):
        if fn.endswith(".h"):
            text = open(os.path.join(HEADER_DIR, fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"\b(la_[a-z0-9_]+)\s*\(", text)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("la_prefill", "la_decode_step", "la_check_status", "la_status_string",
                     "la_version", "la_prefill_workspace_size", "la_kernel_launches"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in include/ but not exported"
    from gated_delta_rule_attention_b200 import library_path
    out = subprocess.run(["nm", "-D", "--defined-only", library_path()], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\s[TW]\s+(la_[a-z0-9_]+)$", out, flags=re.M))
    assert set(declared_functions()) <= exported


def test_library_does_not_need_libcuda(lib):
    from gated_delta_rule_attention_b200 import library_path
    out = subprocess.run(["readelf", "-d", library_path()], capture_output=True, text=True,
                         check=True).stdout
    assert "libcuda.so" not in out


def test_status_strings_and_version(lib):
    for code, tag in enumerate(["LA_OK", "LA_ERR_INVALID_ARG", "LA_ERR_UNSUPPORTED",
                                "LA_ERR_CUDA", "LA_ERR_TIMEOUT"]):
        assert lib.la_status_string(code).decode().startswith(tag)
    assert lib.la_status_string(99).decode() == "unknown la_status_t"
    assert lib.la_version() >= 100


def _prefill(lib, mode=2, dtype=1, B=1, H=1, T=8, dk=128, dv=128, chunk=0, flags=0):
    null = None
    return lib.la_prefill(mode, dtype, B, H, T, dk, dv, null, null, null, null, null, null, null,
                          null, chunk, flags, null, 0, null)


def test_host_side_argument_checks(lib):
    INVALID, UNSUPPORTED = 1, 2
    assert _prefill(lib, mode=5) == INVALID
    assert _prefill(lib, mode=-1) == INVALID
    assert _prefill(lib, dtype=2) == INVALID
    assert _prefill(lib, B=0) == INVALID
    assert _prefill(lib, H=0) == INVALID
    assert _prefill(lib, T=-1) == INVALID
    assert _prefill(lib, flags=4) == INVALID
    assert _prefill(lib, chunk=-8) == INVALID
    assert _prefill(lib, dk=96) == UNSUPPORTED
    assert _prefill(lib, dv=256) == UNSUPPORTED
    # NULL tensors are rejected before any launch
    assert _prefill(lib) == INVALID
    assert lib.la_decode_step(2, 1, 0, 1, 128, 128, *([None] * 9)) == INVALID
    assert lib.la_decode_step(2, 1, 1, 1, 128, 32, *([None] * 9)) == UNSUPPORTED
    assert lib.la_decode_step(2, 1, 4, 2, 128, 128, *([None] * 9)) == INVALID


def test_workspace_size_query(lib):
    # bf16, d = 128: the tensor-core kernels; few heads and a long sequence -> segments
    assert lib.la_prefill_workspace_size(2, 1, 1, 8, 32768, 128, 128, 0) > 0
    assert lib.la_prefill_workspace_size(3, 1, 2, 16, 32768, 128, 128, 0) > 0
    # the gated delta rule with 16-37 head rows: the single-pass kernel, whose two-pass
    # variant keeps each chunk's A, T diag(b), T diag(b g) (3 x 8 KB) in the workspace
    assert lib.la_prefill_workspace_size(2, 1, 2, 16, 32768, 128, 128, 0) == 32 * 512 * 24576
    assert lib.la_prefill_workspace_size(2, 1, 1, 37, 32768, 128, 128, 0) == 37 * 512 * 24576
    assert lib.la_prefill_workspace_size(2, 1, 1, 38, 32768, 128, 128, 0) > 0
    # KDA with 16-37 head rows: the two-pass chain kernel's per-chunk records (A, T diag(b)
    # 8 KB each, Q o Gam, W, K o 2^(lam_L - lam) 16 KB each, Gam_L 512 B)
    assert lib.la_prefill_workspace_size(3, 1, 2, 16, 32768, 128, 128, 0) == 32 * 512 * 66048
    assert lib.la_prefill_workspace_size(3, 1, 1, 16, 65, 128, 128, 0) == 16 * 2 * 66048
    assert lib.la_prefill_workspace_size(1, 1, 8, 16, 8192, 128, 128, 0) == 0   # 128 heads
    assert lib.la_prefill_workspace_size(0, 0, 1, 2, 256, 64, 64, 0) == 0       # fp32 path
    assert lib.la_prefill_workspace_size(3, 1, 1, 1, 64, 128, 128, 0) == 0


def test_host_pointers_are_rejected(lib):
    """A host buffer is never handed to a kernel: the pointer check runs first."""
    import numpy as np
    buf = np.zeros(1 << 16, dtype=np.float32)
    p = buf.ctypes.data_as(ctypes.c_void_p)
    st = lib.la_decode_step(1, 0, 1, 1, 64, 64, p, p, p, None, None, p, None, p, None)
    assert st == 1


def test_launch_timing_without_launches(lib):
    """The timing hook answers without touching a device while nothing was launched."""
    import ctypes
    lib.la_launch_times.argtypes = [ctypes.c_void_p, ctypes.c_int]
    buf = (ctypes.c_float * 4)()
    assert lib.la_launch_timing(1) == 0
    assert lib.la_launch_times(ctypes.cast(buf, ctypes.c_void_p), 4) == 0
    assert lib.la_launch_times(None, 4) == -1
    assert lib.la_launch_times(ctypes.cast(buf, ctypes.c_void_p), -1) == -1
    assert lib.la_launch_timing(0) == 0
    assert lib.la_launch_times(ctypes.cast(buf, ctypes.c_void_p), 4) == 0


def test_short_conv_argument_checks(lib):
    INVALID, UNSUPPORTED = 1, 2
    n = [None] * 5

    def conv(dtype=1, B=1, T=8, H=2, d=128, width=4, flags=0):
        return lib.la_short_conv(dtype, B, T, H, d, width, *n, flags, None)

    assert conv(dtype=2) == INVALID
    assert conv(B=0) == INVALID
    assert conv(T=-1) == INVALID
    assert conv(width=0) == INVALID
    assert conv(width=5) == INVALID
    assert conv(flags=1) == INVALID        # LA_FLAG_INIT_STATE is not a conv flag
    assert conv(flags=8) == INVALID
    assert conv(d=96) == UNSUPPORTED
    assert conv() == INVALID               # NULL taps / tensors, before any launch
    assert conv(flags=2 | 4) == INVALID
    assert lib.la_short_conv_step(1, 0, 2, 128, 4, None, None, None, None, 0, None) == INVALID
    assert lib.la_short_conv_step(1, 1, 2, 96, 4, None, None, None, None, 0, None) == UNSUPPORTED
    assert lib.la_short_conv_step(1, 1, 2, 128, 4, None, None, None, None, 0, None) == INVALID


def test_prefill_varlen_argument_checks(lib):
    INVALID, UNSUPPORTED = 1, 2

    def call(mode=2, dtype=1, N=2, H=2, T=100, dk=128, dv=128, chunk=0, flags=0):
        return lib.la_prefill_varlen(mode, dtype, N, H, T, dk, dv, *([None] * 9), chunk, flags, None)

    assert call(mode=5) == INVALID
    assert call(dtype=3) == INVALID
    assert call(N=0) == INVALID
    assert call(H=0) == INVALID
    assert call(T=-1) == INVALID
    assert call(flags=2) == INVALID
    assert call(chunk=-1) == INVALID
    assert call(dk=96) == UNSUPPORTED
    assert call() == INVALID          # NULL cu_seqlens / tensors, before any launch
    assert call(T=0) == INVALID       # still needs the offsets and the state


def test_short_conv_varlen_argument_checks(lib):
    INVALID, UNSUPPORTED = 1, 2

    def call(dtype=1, N=2, T=10, H=2, d=128, width=4, flags=0):
        return lib.la_short_conv_varlen(dtype, N, T, H, d, width, *([None] * 6), flags, None)

    assert call(dtype=5) == INVALID
    assert call(N=0) == INVALID
    assert call(T=-1) == INVALID
    assert call(width=5) == INVALID
    assert call(flags=1) == INVALID
    assert call(d=32) == UNSUPPORTED
    assert call() == INVALID          # NULL offsets / taps, before any launch


def test_selftest_symbol_is_exported(lib):
    assert hasattr(lib, "la_selftest_wait_timeout")


def test_retnet_mode_needs_its_gate(lib):
    INVALID = 1
    # mode 4 without a gate is refused before anything else is looked at
    assert lib.la_decode_step(4, 1, 1, 1, 128, 128, *([None] * 9)) == INVALID
    assert lib.la_prefill_workspace_size(4, 1, 1, 16, 32768, 128, 128, 0) > 0   # the mode-1 plan
    assert lib.la_prefill_workspace_size(5, 1, 1, 16, 32768, 128, 128, 0) == 0


def test_prefill_backward_argument_checks(lib):
    INVALID, UNSUPPORTED = 1, 2

    def call(mode=1, dtype=1, B=1, H=2, T=64, dk=128, dv=128):
        return lib.la_prefill_backward(mode, dtype, B, H, T, dk, dv, *([None] * 13), 0, None)

    assert call(mode=2) == UNSUPPORTED     # the delta rule has its own entry point
    assert call(mode=7) == INVALID
    assert call(T=0) == INVALID
    assert call(dk=32) == UNSUPPORTED
    assert call() == INVALID               # NULL tensors, before any launch
    assert call(mode=4) == INVALID         # mode 4 needs its gate
    # 4 chunks: 9 [d_v, d_k] fp32-sized slots (states and cotangents) and dlam per (b, h)
    assert lib.la_backward_workspace_size(1, 2, 3, 100, 64, 64) == 4 * 2 * 3 * (9 * 64 * 64 + 100)
    # delta rule: chunk-start states (4 chunks of 32), fp32 dq, dk, dL/dlam and db
    BH, T, nch = 6, 100, 4
    assert lib.la_backward_workspace_size(2, 2, 3, T, 64, 64) == 4 * (BH * nch * 64 * 64 + 2 * BH * T * 64
                                                                      + BH * T + BH * T)
    assert lib.la_backward_workspace_size(3, 2, 3, T, 64, 64) == 4 * (BH * nch * 64 * 64 + 3 * BH * T * 64
                                                                      + BH * T)
    assert lib.la_backward_workspace_size(0, 2, 3, T, 64, 64) == 0


def test_prefill_backward_delta_argument_checks(lib):
    INVALID, UNSUPPORTED = 1, 2

    def call(mode=2, dtype=1, B=1, H=2, T=64, dk=128, dv=128):
        return lib.la_prefill_backward_delta(mode, dtype, B, H, T, dk, dv, *([None] * 15), 0, None)

    assert call(mode=1) == UNSUPPORTED     # scalar-gate modes: la_prefill_backward
    assert call(mode=4) == UNSUPPORTED
    assert call(mode=9) == INVALID
    assert call(T=0) == INVALID
    assert call(dk=96) == UNSUPPORTED
    assert call(dtype=5) == INVALID
    assert call() == INVALID               # NULL tensors, before any launch
    assert call(mode=3) == INVALID


def test_prefill_conv_argument_checks(lib):
    """la_prefill_conv refuses what it has no kernel for and malformed calls before any
    launch (no GPU needed: every check below fails before a pointer is used)."""
    INVALID, UNSUPPORTED = 1, 2

    def call(dtype=1, B=1, H=2, T=64, d=128, width=4, flags=0, fqk=6, fv=2):
        return lib.la_prefill_conv(dtype, B, H, T, d, width, *([None] * 8), fqk, fv, *([None] * 5),
                                   flags, None, 0, None)
    assert call(dtype=0) == UNSUPPORTED      # fp32: the fused path is bf16 only
    assert call(dtype=7) == INVALID
    assert call(d=64) == UNSUPPORTED
    assert call(d=96) == INVALID
    assert call(width=0) == INVALID
    assert call(width=5) == INVALID
    assert call(T=0) == INVALID
    assert call(flags=2) == INVALID
    assert call(fqk=8) == INVALID
    assert call() == INVALID                 # NULL tensors
    # the two-pass images: 3 x 8 KB per chunk of 64 tokens
    assert lib.la_prefill_conv_workspace_size(2, 16, 32768) == 32 * 512 * 24576
    assert lib.la_prefill_conv_workspace_size(1, 1, 65) == 2 * 24576
    assert lib.la_prefill_conv_workspace_size(0, 1, 64) == 0
