"""Causal linear attention for NVIDIA B200 (sm_100a): Python binding of liblinattn.

The compute path is the C ABI declared in ``include/la.h`` and implemented by the CUDA
kernels under ``csrc/``.  This module only marshals arguments (ctypes): it checks
shapes and dtypes, allocates outputs with torch when the caller does not pass them,
and forwards raw device pointers and the current CUDA stream.  Every step of the
method runs in the library's kernels; there is no Python or CPU fallback, and the
import fails loudly if the library is missing.

Four modes, named after the variants on the lesson page "Linear attention and hybrids":

* ``MODE_ELU1_NORM`` -- phi(x) = elu(x)+1 with the z normaliser (section "The kernel trick")
* ``MODE_GATED`` -- scalar decay gate a_t (section "Memory must forget: decay and gates")
* ``MODE_GATED_DELTA`` -- the Gated DeltaNet update (section "The delta rule and Gated DeltaNet")
* ``MODE_KDA`` -- Kimi Delta Attention, the same update with one decay per channel (gate
  [.., d_k] per token; same section)
* ``MODE_RETNET`` -- the constant decay of RetNet / Lightning attention: ``MODE_GATED`` with
  one fixed gate per head (gate [H]; section "Memory must forget: decay and gates")
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = ["MODE_ELU1_NORM", "MODE_GATED", "MODE_GATED_DELTA", "MODE_KDA", "MODE_RETNET", "FLAG_INIT_STATE", "LaError",
           "prefill", "prefill_varlen", "prefill_backward", "prefill_backward_delta", "decode_step", "short_conv", "short_conv_varlen", "short_conv_step", "prefill_conv", "check_status", "library",
           "library_path", "version", "kernel_launches", "workspace_size"]

MODE_ELU1_NORM = 0
MODE_GATED = 1
MODE_GATED_DELTA = 2
MODE_KDA = 3
MODE_RETNET = 4
FLAG_INIT_STATE = 1
CONV_SILU = 2
CONV_L2NORM = 4

LA_F32 = 0
LA_BF16 = 1
_STATUS = {0: "LA_OK", 1: "LA_ERR_INVALID_ARG", 2: "LA_ERR_UNSUPPORTED", 3: "LA_ERR_CUDA",
           4: "LA_ERR_TIMEOUT"}

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "liblinattn.so")
_lib = None


class LaError(RuntimeError):
    """A non-zero la_status_t from the library."""

    def __init__(self, status: int, where: str):
        self.status = status
        msg = library().la_status_string(status).decode()
        super().__init__(f"{where}: {msg}")


def library_path() -> str:
    return _LIB_PATH


def library():
    """Load liblinattn.so (ctypes).  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"liblinattn.so is not built ({_LIB_PATH}); run "
                          "`python -m gated_delta_rule_attention_b200.build`")
    lib = ctypes.CDLL(_LIB_PATH)
    vp, fp = ctypes.c_void_p, ctypes.c_void_p
    i, u = ctypes.c_int, ctypes.c_uint
    lib.la_prefill.argtypes = [i, i, i, i, i, i, i, vp, vp, vp, fp, fp, fp, fp, vp, i, u, vp,
                               ctypes.c_size_t, vp]
    lib.la_prefill.restype = i
    lib.la_decode_step.argtypes = [i, i, i, i, i, i, vp, vp, vp, fp, fp, fp, fp, vp, vp]
    lib.la_decode_step.restype = i
    lib.la_prefill_workspace_size.argtypes = [i, i, i, i, i, i, i, i]
    lib.la_prefill_workspace_size.restype = ctypes.c_size_t
    lib.la_check_status.argtypes = [vp]
    lib.la_check_status.restype = i
    lib.la_status_string.argtypes = [i]
    lib.la_status_string.restype = ctypes.c_char_p
    lib.la_version.argtypes = []
    lib.la_version.restype = i
    lib.la_kernel_launches.argtypes = []
    lib.la_kernel_launches.restype = ctypes.c_ulonglong
    lib.la_prefill_varlen.argtypes = [i, i, i, i, i, i, i, vp, vp, vp, vp, fp, fp, fp, fp, vp, i,
                                      u, vp]
    lib.la_prefill_varlen.restype = i
    lib.la_backward_workspace_size.argtypes = [i, i, i, i, i, i]
    lib.la_backward_workspace_size.restype = ctypes.c_size_t
    lib.la_prefill_backward.argtypes = [i, i, i, i, i, i, i, vp, vp, vp, fp, fp, vp, fp, vp, vp, vp,
                                        fp, fp, vp, ctypes.c_size_t, vp]
    lib.la_prefill_backward.restype = i
    lib.la_prefill_backward_delta.argtypes = [i, i, i, i, i, i, i, vp, vp, vp, fp, fp, fp, vp, fp, vp,
                                              vp, vp, fp, fp, fp, vp, ctypes.c_size_t, vp]
    lib.la_prefill_backward_delta.restype = i
    lib.la_short_conv.argtypes = [i, i, i, i, i, i, vp, fp, vp, vp, vp, u, vp]
    lib.la_short_conv.restype = i
    lib.la_short_conv_varlen.argtypes = [i, i, i, i, i, i, vp, vp, fp, vp, vp, vp, u, vp]
    lib.la_short_conv_varlen.restype = i
    lib.la_short_conv_step.argtypes = [i, i, i, i, i, vp, fp, vp, vp, u, vp]
    lib.la_short_conv_step.restype = i
    lib.la_prefill_conv_workspace_size.argtypes = [i, i, i]
    lib.la_prefill_conv_workspace_size.restype = ctypes.c_size_t
    lib.la_prefill_conv.argtypes = [i, i, i, i, i, i, vp, vp, vp, fp, fp, fp, vp, vp, u, u, vp, fp, fp,
                                    fp, vp, u, vp, ctypes.c_size_t, vp]
    lib.la_prefill_conv.restype = i
    lib.la_selftest_wait_timeout.argtypes = [vp]
    lib.la_selftest_wait_timeout.restype = i
    if hasattr(lib, "la_launch_timing"):   # diagnostic hook, absent from older builds
        lib.la_launch_timing.argtypes = [i]
        lib.la_launch_timing.restype = i
        lib.la_launch_times.argtypes = [ctypes.POINTER(ctypes.c_float), i]
        lib.la_launch_times.restype = i
    _lib = lib
    return lib


def version() -> int:
    return int(library().la_version())


def kernel_launches() -> int:
    """Kernels the library has enqueued in this process so far."""
    return int(library().la_kernel_launches())


def launch_timing(enable: bool) -> None:
    """Turn per-launch device timing on or off (la_launch_timing)."""
    _check(library().la_launch_timing(1 if enable else 0), "la_launch_timing")


def launch_times(max_n: int = 16) -> list:
    """Device durations (ms) of the launches of the last call, in launch order
    (la_launch_times); empty while timing is off."""
    buf = (ctypes.c_float * max_n)()
    n = library().la_launch_times(buf, max_n)
    if n < 0:
        raise RuntimeError("la_launch_times failed")
    return [float(buf[j]) for j in range(n)]


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _io_dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return LA_BF16
    if t.dtype == torch.float32:
        return LA_F32
    raise TypeError(f"q/k/v must be bfloat16 or float32, got {t.dtype}")


def _stream_handle(device: torch.device, stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream(device) if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(status: int, where: str):
    if status != 0:
        raise LaError(status, where)


def _need(t, shape, dtype, name):
    if t is None:
        raise ValueError(f"{name} is required")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _gate_shape(mode, lead, dk, H):
    """Shape of the gate tensor: per token, per channel in KDA, one per head in RetNet."""
    if mode == MODE_RETNET:
        return (H,)
    return (*lead, dk) if mode == MODE_KDA else tuple(lead)


_workspaces: dict = {}


def workspace_size(mode: int, dtype: torch.dtype, B: int, H: int, T: int, d_k: int, d_v: int,
                   chunk: int = 0) -> int:
    """Bytes of scratch ``la_prefill`` can use for these sizes (0 if none)."""
    dt = LA_BF16 if dtype == torch.bfloat16 else LA_F32
    return int(library().la_prefill_workspace_size(int(mode), dt, B, H, T, d_k, d_v, int(chunk)))


def _workspace(device: torch.device, nbytes: int, stream=None):
    """A scratch buffer for calls on one stream of one device (torch allocation), grown on
    demand and reused by later calls on that stream.  Calls on different streams never
    share a buffer, and each is allocated while its stream is current, so the caching
    allocator orders the reuse of a replaced buffer after that stream's work."""
    if nbytes <= 0:
        return None
    s = torch.cuda.current_stream(device) if stream is None else stream
    key = (device.index, s.cuda_stream)
    buf = _workspaces.get(key)
    if buf is None or buf.numel() < nbytes:
        with torch.cuda.stream(s):
            buf = torch.empty(nbytes, dtype=torch.uint8, device=device)
        _workspaces[key] = buf
    return buf


def prefill(q, k, v, *, mode: int, gate=None, beta=None, state=None, z=None, o=None,
            chunk: int = 0, init_state: bool | None = None, stream=None, workspace="auto"):
    """Chunked prefill over whole sequences (``la_prefill``).

    q, k: [B,H,T,d_k]; v: [B,H,T,d_v] (bf16 or fp32, one dtype); gate, beta: [B,H,T] fp32
    (``MODE_KDA``: gate [B,H,T,d_k]);
    state: [B,H,d_v,d_k] fp32 (read as S_0 when ``init_state``, default: when given);
    z: [B,H,d_k] fp32 (mode 0).  Returns (o, state, z).

    CUDA tensors run in place on the current stream.  If the inputs are CPU tensors they
    are copied to the current CUDA device, the call runs there, and the outputs are
    copied back to the CPU (the end-to-end path); the computation is still the kernel's.

    ``workspace``: "auto" (a per-stream scratch buffer of ``workspace_size`` bytes, kept for
    later calls), None (no scratch: the kernels' single-pass or smallest forms), or a uint8
    CUDA tensor.  The fastest forms can need a large one: the gated delta rule and KDA with
    16 to 37 head rows keep per-chunk factors (24 KB, KDA 66 048 bytes, per chunk and head
    row: 0.4 and 1.08 GB at B2 H16 T32768).
    """
    host = q.device.type == "cpu"
    if host:
        dev = torch.device("cuda", torch.cuda.current_device())
        move = (lambda t: None if t is None else t.to(dev, non_blocking=True))
        res = prefill(move(q), move(k), move(v), mode=mode, gate=move(gate), beta=move(beta),
                      state=move(state), z=move(z), o=None, chunk=chunk,
                      init_state=init_state if init_state is not None else state is not None,
                      stream=stream)
        back = tuple(None if t is None else t.to("cpu") for t in res)
        if o is not None:
            o.copy_(back[0])
            back = (o,) + back[1:]
        return back
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    dtype = _io_dtype(q)
    _need(q, (B, H, T, dk), dt, "q")
    _need(k, (B, H, T, dk), dt, "k")
    _need(v, (B, H, T, dv), dt, "v")
    if gate is not None:
        _need(gate, _gate_shape(mode, (B, H, T), dk, H), torch.float32, "gate")
    if beta is not None:
        _need(beta, (B, H, T), torch.float32, "beta")
    if init_state is None:
        init_state = state is not None
    if state is None:
        state = torch.empty(B, H, dv, dk, device=q.device, dtype=torch.float32)
    _need(state, (B, H, dv, dk), torch.float32, "state")
    if mode == MODE_ELU1_NORM:
        if z is None:
            if init_state:
                raise ValueError("mode 0 with init_state needs z")
            z = torch.empty(B, H, dk, device=q.device, dtype=torch.float32)
        _need(z, (B, H, dk), torch.float32, "z")
    if o is None:
        o = torch.empty(B, H, T, dv, device=q.device, dtype=dt)
    _need(o, (B, H, T, dv), dt, "o")
    if isinstance(workspace, str):
        ws = _workspace(q.device, workspace_size(mode, dt, B, H, T, dk, dv, chunk), stream) \
            if workspace == "auto" else None
    else:
        ws = workspace
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    st = library().la_prefill(int(mode), dtype, B, H, T, dk, dv, _ptr(q), _ptr(k), _ptr(v),
                              _ptr(gate), _ptr(beta), _ptr(state), _ptr(z), _ptr(o), int(chunk),
                              FLAG_INIT_STATE if init_state else 0, _ptr(ws), ws_bytes,
                              _stream_handle(q.device, stream))
    _check(st, "la_prefill")
    return o, state, (z if mode == MODE_ELU1_NORM else None)


def prefill_varlen(q, k, v, cu_seqlens, *, mode: int, gate=None, beta=None, state=None, z=None,
                   o=None, chunk: int = 0, init_state: bool | None = None, stream=None):
    """Prefill of N packed sequences (``la_prefill_varlen``).

    q, k: [H,T,d_k]; v: [H,T,d_v] with the N sequences packed along T; cu_seqlens: int32
    [N+1] on the device (sequence s = tokens cu[s]..cu[s+1]); gate, beta: [H,T] fp32
    (``MODE_KDA``: gate [H,T,d_k]); state: [N,H,d_v,d_k] fp32 (each sequence's start
    state when ``init_state``, default: when given); z: [N,H,d_k] (mode 0).
    Returns (o [H,T,d_v], state, z) with each sequence's final state in its slot.
    """
    H, T, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    dtype = _io_dtype(q)
    N = cu_seqlens.numel() - 1
    if N < 1:
        raise ValueError("cu_seqlens needs at least two entries")
    _need(cu_seqlens, (N + 1,), torch.int32, "cu_seqlens")
    _need(q, (H, T, dk), dt, "q")
    _need(k, (H, T, dk), dt, "k")
    _need(v, (H, T, dv), dt, "v")
    if gate is not None:
        _need(gate, _gate_shape(mode, (H, T), dk, H), torch.float32, "gate")
    if beta is not None:
        _need(beta, (H, T), torch.float32, "beta")
    if init_state is None:
        init_state = state is not None
    if state is None:
        state = torch.empty(N, H, dv, dk, device=q.device, dtype=torch.float32)
    _need(state, (N, H, dv, dk), torch.float32, "state")
    if mode == MODE_ELU1_NORM:
        if z is None:
            if init_state:
                raise ValueError("mode 0 with init_state needs z")
            z = torch.empty(N, H, dk, device=q.device, dtype=torch.float32)
        _need(z, (N, H, dk), torch.float32, "z")
    if o is None:
        o = torch.empty(H, T, dv, device=q.device, dtype=dt)
    _need(o, (H, T, dv), dt, "o")
    st = library().la_prefill_varlen(int(mode), dtype, N, H, T, dk, dv, _ptr(cu_seqlens), _ptr(q),
                                     _ptr(k), _ptr(v), _ptr(gate), _ptr(beta), _ptr(state),
                                     _ptr(z), _ptr(o), int(chunk),
                                     FLAG_INIT_STATE if init_state else 0,
                                     _stream_handle(q.device, stream))
    _check(st, "la_prefill_varlen")
    return o, state, (z if mode == MODE_ELU1_NORM else None)


def prefill_backward(q, k, v, dO, *, mode: int, gate=None, state0=None, dstate=None,
                     need_dgate: bool = True, need_dstate0: bool | None = None, stream=None):
    """Gradients of the prefill (``la_prefill_backward``, modes 1 and 4).

    q, k: [B,H,T,d_k]; v, dO: [B,H,T,d_v]; gate: [B,H,T] (mode 1) or [H] (mode 4);
    state0, dstate: [B,H,d_v,d_k] fp32 or None (zero).  Returns (dq, dk, dv, dgate, dstate0):
    dgate [B,H,T] fp32 for mode 1 with a gate (else None), dstate0 when ``need_dstate0``
    (default: when state0 is given).
    """
    B, H, T, dk_ = q.shape
    dv_ = v.shape[-1]
    dt = q.dtype
    dtype = _io_dtype(q)
    _need(q, (B, H, T, dk_), dt, "q")
    _need(k, (B, H, T, dk_), dt, "k")
    _need(v, (B, H, T, dv_), dt, "v")
    _need(dO, (B, H, T, dv_), dt, "dO")
    if gate is not None:
        _need(gate, _gate_shape(mode, (B, H, T), dk_, H), torch.float32, "gate")
    for name, t in (("state0", state0), ("dstate", dstate)):
        if t is not None:
            _need(t, (B, H, dv_, dk_), torch.float32, name)
    if need_dstate0 is None:
        need_dstate0 = state0 is not None
    dq = torch.empty_like(q)
    dk = torch.empty_like(k)
    dv = torch.empty_like(v)
    dgate = (torch.empty(B, H, T, device=q.device, dtype=torch.float32)
             if (need_dgate and mode == MODE_GATED and gate is not None) else None)
    dstate0 = (torch.empty(B, H, dv_, dk_, device=q.device, dtype=torch.float32)
               if need_dstate0 else None)
    nbytes = int(library().la_backward_workspace_size(int(mode), B, H, T, dk_, dv_))
    ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=q.device)
    if stream is not None:
        ws.record_stream(stream)   # freed on return: not reused before `stream`'s work is done
    st = library().la_prefill_backward(int(mode), dtype, B, H, T, dk_, dv_, _ptr(q), _ptr(k), _ptr(v),
                                       _ptr(gate), _ptr(state0), _ptr(dO), _ptr(dstate), _ptr(dq),
                                       _ptr(dk), _ptr(dv), _ptr(dgate), _ptr(dstate0), _ptr(ws),
                                       ws.numel(), _stream_handle(q.device, stream))
    _check(st, "la_prefill_backward")
    return dq, dk, dv, dgate, dstate0


def prefill_backward_delta(q, k, v, dO, *, mode: int, beta, gate=None, state0=None, dstate=None,
                           need_dgate: bool = True, need_dstate0: bool | None = None, stream=None):
    """Gradients of the delta-rule prefill (``la_prefill_backward_delta``, modes 2 and 3).

    q, k: [B,H,T,d_k]; v, dO: [B,H,T,d_v]; beta: [B,H,T] fp32; gate: [B,H,T] (mode 2) or
    [B,H,T,d_k] (mode 3) fp32, or None (a = 1); state0, dstate: [B,H,d_v,d_k] fp32 or None.
    Returns (dq, dk, dv, dgate, dbeta, dstate0): dgate shaped like gate (None without a
    gate), dbeta [B,H,T] fp32, dstate0 when ``need_dstate0`` (default: when state0 is given).
    """
    B, H, T, dk_ = q.shape
    dv_ = v.shape[-1]
    dt = q.dtype
    dtype = _io_dtype(q)
    _need(q, (B, H, T, dk_), dt, "q")
    _need(k, (B, H, T, dk_), dt, "k")
    _need(v, (B, H, T, dv_), dt, "v")
    _need(dO, (B, H, T, dv_), dt, "dO")
    _need(beta, (B, H, T), torch.float32, "beta")
    if gate is not None:
        _need(gate, _gate_shape(mode, (B, H, T), dk_, H), torch.float32, "gate")
    for name, t in (("state0", state0), ("dstate", dstate)):
        if t is not None:
            _need(t, (B, H, dv_, dk_), torch.float32, name)
    if need_dstate0 is None:
        need_dstate0 = state0 is not None
    dq = torch.empty_like(q)
    dk = torch.empty_like(k)
    dv = torch.empty_like(v)
    dgate = torch.empty_like(gate) if (need_dgate and gate is not None) else None
    dbeta = torch.empty_like(beta)
    dstate0 = (torch.empty(B, H, dv_, dk_, device=q.device, dtype=torch.float32)
               if need_dstate0 else None)
    nbytes = int(library().la_backward_workspace_size(int(mode), B, H, T, dk_, dv_))
    ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=q.device)
    if stream is not None:
        ws.record_stream(stream)   # freed on return: not reused before `stream`'s work is done
    st = library().la_prefill_backward_delta(
        int(mode), dtype, B, H, T, dk_, dv_, _ptr(q), _ptr(k), _ptr(v), _ptr(gate), _ptr(beta),
        _ptr(state0), _ptr(dO), _ptr(dstate), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dgate), _ptr(dbeta),
        _ptr(dstate0), _ptr(ws), ws.numel(), _stream_handle(q.device, stream))
    _check(st, "la_prefill_backward_delta")
    return dq, dk, dv, dgate, dbeta, dstate0


def decode_step(q, k, v, *, mode: int, state, gate=None, beta=None, z=None, o=None,
                stream=None):
    """One token for N sequences (``la_decode_step``), state updated in place.

    q, k: [N,H,d_k]; v: [N,H,d_v]; gate, beta: [N,H] fp32 (``MODE_KDA``: gate [N,H,d_k]);
    state: [N,H,d_v,d_k] fp32;
    z: [N,H,d_k] fp32 (mode 0).  Returns (o, state, z).  CPU inputs take the end-to-end
    path of ``prefill`` (copy in, run on the GPU, copy o, state and z back).
    """
    if q.device.type == "cpu":
        dev = torch.device("cuda", torch.cuda.current_device())
        move = (lambda t: None if t is None else t.to(dev, non_blocking=True))
        s_dev, z_dev = move(state), move(z)
        res = decode_step(move(q), move(k), move(v), mode=mode, state=s_dev, gate=move(gate),
                          beta=move(beta), z=z_dev, stream=stream)
        state.copy_(res[1].to("cpu"))
        if z is not None:
            z.copy_(res[2].to("cpu"))
        o_host = res[0].to("cpu")
        if o is not None:
            o.copy_(o_host)
            o_host = o
        return o_host, state, z
    N, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    dtype = _io_dtype(q)
    _need(q, (N, H, dk), dt, "q")
    _need(k, (N, H, dk), dt, "k")
    _need(v, (N, H, dv), dt, "v")
    _need(state, (N, H, dv, dk), torch.float32, "state")
    if gate is not None:
        _need(gate, _gate_shape(mode, (N, H), dk, H), torch.float32, "gate")
    if beta is not None:
        _need(beta, (N, H), torch.float32, "beta")
    if mode == MODE_ELU1_NORM:
        _need(z, (N, H, dk), torch.float32, "z")
    if o is None:
        o = torch.empty(N, H, dv, device=q.device, dtype=dt)
    _need(o, (N, H, dv), dt, "o")
    st = library().la_decode_step(int(mode), dtype, N, H, dk, dv, _ptr(q), _ptr(k), _ptr(v),
                                  _ptr(gate), _ptr(beta), _ptr(state), _ptr(z), _ptr(o),
                                  _stream_handle(q.device, stream))
    _check(st, "la_decode_step")
    return o, state, z


def _conv_flags(silu: bool, l2norm: bool) -> int:
    return (CONV_SILU if silu else 0) | (CONV_L2NORM if l2norm else 0)


def short_conv(x, w, *, heads: int, window=None, window_out=None, silu: bool = False,
               l2norm: bool = False, y=None, stream=None):
    """Short causal depthwise convolution over time (``la_short_conv``).

    x: [B, T, H*d] token-major (bf16 or fp32); w: [H*d, width] fp32 taps (tap width-1
    multiplies the current token); window: [B, width-1, H*d] in x's dtype, the inputs
    before x_0 (None: zeros).  ``silu`` applies u * sigmoid(u), ``l2norm`` normalises
    every head's d-row.  Returns (y [B, H, T, d], window_out [B, width-1, H*d]);
    ``window_out`` may be passed (``window`` itself updates the window in place).
    """
    B, T, C = x.shape
    width = w.shape[1]
    if C % heads:
        raise ValueError("x's last dimension must be heads * d")
    d = C // heads
    dt = x.dtype
    dtype = _io_dtype(x)
    _need(x, (B, T, C), dt, "x")
    _need(w, (C, width), torch.float32, "w")
    if window is not None:
        _need(window, (B, width - 1, C), dt, "window")
    if window_out is None:
        window_out = torch.empty(B, width - 1, C, device=x.device, dtype=dt)
    _need(window_out, (B, width - 1, C), dt, "window_out")
    if y is None:
        y = torch.empty(B, heads, T, d, device=x.device, dtype=dt)
    _need(y, (B, heads, T, d), dt, "y")
    st = library().la_short_conv(dtype, B, T, heads, d, width, _ptr(x), _ptr(w), _ptr(window),
                                 _ptr(window_out), _ptr(y), _conv_flags(silu, l2norm),
                                 _stream_handle(x.device, stream))
    _check(st, "la_short_conv")
    return y, window_out


def short_conv_varlen(x, w, cu_seqlens, *, heads: int, window=None, window_out=None,
                      silu: bool = False, l2norm: bool = False, y=None, stream=None):
    """Packed variable-length sequences (``la_short_conv_varlen``): x [T, H*d] holds N
    sequences back to back (cu_seqlens int32 [N+1] on the device), window / window_out
    [N, width-1, H*d].  Returns (y [H, T, d], window_out)."""
    T, C = x.shape
    width = w.shape[1]
    if C % heads:
        raise ValueError("x's last dimension must be heads * d")
    d = C // heads
    N = cu_seqlens.numel() - 1
    dt = x.dtype
    dtype = _io_dtype(x)
    _need(cu_seqlens, (N + 1,), torch.int32, "cu_seqlens")
    _need(x, (T, C), dt, "x")
    _need(w, (C, width), torch.float32, "w")
    if window is not None:
        _need(window, (N, width - 1, C), dt, "window")
    if window_out is None:
        window_out = torch.empty(N, width - 1, C, device=x.device, dtype=dt)
    _need(window_out, (N, width - 1, C), dt, "window_out")
    if y is None:
        y = torch.empty(heads, T, d, device=x.device, dtype=dt)
    _need(y, (heads, T, d), dt, "y")
    st = library().la_short_conv_varlen(dtype, N, T, heads, d, width, _ptr(cu_seqlens), _ptr(x),
                                        _ptr(w), _ptr(window), _ptr(window_out), _ptr(y),
                                        _conv_flags(silu, l2norm), _stream_handle(x.device, stream))
    _check(st, "la_short_conv_varlen")
    return y, window_out


def short_conv_step(x, w, window, *, heads: int, silu: bool = False, l2norm: bool = False,
                    y=None, stream=None):
    """One new token of N sequences (``la_short_conv_step``): x [N, H*d], window
    [N, width-1, H*d] updated in place.  Returns y [N, H, d]."""
    N, C = x.shape
    width = w.shape[1]
    if C % heads:
        raise ValueError("x's last dimension must be heads * d")
    d = C // heads
    dt = x.dtype
    dtype = _io_dtype(x)
    _need(x, (N, C), dt, "x")
    _need(w, (C, width), torch.float32, "w")
    if width > 1:
        _need(window, (N, width - 1, C), dt, "window")
    if y is None:
        y = torch.empty(N, heads, d, device=x.device, dtype=dt)
    _need(y, (N, heads, d), dt, "y")
    st = library().la_short_conv_step(dtype, N, heads, d, width, _ptr(x), _ptr(w),
                                      _ptr(window if width > 1 else None), _ptr(y),
                                      _conv_flags(silu, l2norm), _stream_handle(x.device, stream))
    _check(st, "la_short_conv_step")
    return y


def prefill_conv(xq, xk, xv, wq, wk, wv, *, heads: int, beta, gate=None, window=None,
                 window_out=None, qk_silu: bool = True, qk_l2norm: bool = True, v_silu: bool = True,
                 state=None, init_state: bool | None = None, y=None, o=None, stream=None):
    """A Gated DeltaNet layer's attention path from its projections (``la_prefill_conv``):
    the short convolution of xq, xk, xv fused into the gated-delta prefill's loads.

    xq, xk, xv: [B, T, H*128] bf16 token-major; wq, wk, wv: [H*128, width] fp32 taps;
    window: [3, B, width-1, H*128] bf16 (the q, k, v windows; None: zeros); gate, beta:
    [B, H, T] fp32; state: [B, H, 128, 128] fp32 (S_0 when ``init_state``, default: when
    given).  SiLU and the head-row L2 norm apply to q and k per ``qk_silu`` /
    ``qk_l2norm``, SiLU to v per ``v_silu``.  Returns (o [B, H, T, 128], state,
    y [3, B, H, T, 128] the convolved q, k, v, window_out [3, B, width-1, H*128]).
    """
    B, T, C = xq.shape
    width = wq.shape[1]
    if C % heads:
        raise ValueError("the projections' last dimension must be heads * d")
    d = C // heads
    dt = torch.bfloat16
    for name, t in (("xq", xq), ("xk", xk), ("xv", xv)):
        _need(t, (B, T, C), dt, name)
    for name, t in (("wq", wq), ("wk", wk), ("wv", wv)):
        _need(t, (C, width), torch.float32, name)
    _need(beta, (B, heads, T), torch.float32, "beta")
    if gate is not None:
        _need(gate, (B, heads, T), torch.float32, "gate")
    if window is not None:
        _need(window, (3, B, width - 1, C), dt, "window")
    if window_out is None:
        window_out = torch.empty(3, B, width - 1, C, device=xq.device, dtype=dt)
    _need(window_out, (3, B, width - 1, C), dt, "window_out")
    if init_state is None:
        init_state = state is not None
    if state is None:
        state = torch.empty(B, heads, d, d, device=xq.device, dtype=torch.float32)
    _need(state, (B, heads, d, d), torch.float32, "state")
    if y is None:
        y = torch.empty(3, B, heads, T, d, device=xq.device, dtype=dt)
    _need(y, (3, B, heads, T, d), dt, "y")
    if o is None:
        o = torch.empty(B, heads, T, d, device=xq.device, dtype=dt)
    _need(o, (B, heads, T, d), dt, "o")
    ws = _workspace(xq.device, int(library().la_prefill_conv_workspace_size(B, heads, T)), stream)
    ws_bytes = 0 if ws is None else ws.numel()
    st = library().la_prefill_conv(LA_BF16, B, heads, T, d, width, _ptr(xq), _ptr(xk), _ptr(xv),
                                   _ptr(wq), _ptr(wk), _ptr(wv), _ptr(window), _ptr(window_out),
                                   _conv_flags(qk_silu, qk_l2norm), _conv_flags(v_silu, False), _ptr(y),
                                   _ptr(gate), _ptr(beta), _ptr(state), _ptr(o),
                                   FLAG_INIT_STATE if init_state else 0, _ptr(ws), ws_bytes,
                                   _stream_handle(xq.device, stream))
    _check(st, "la_prefill_conv")
    return o, state, y, window_out


def selftest_wait_timeout(stream=None):
    """Enqueue the failure-path self-test (``la_selftest_wait_timeout``): the next
    ``check_status`` raises LaError with LA_ERR_TIMEOUT."""
    dev = torch.device("cuda", torch.cuda.current_device())
    _check(library().la_selftest_wait_timeout(_stream_handle(dev, stream)), "la_selftest_wait_timeout")


def check_status(stream=None):
    """Synchronise the stream and raise LaError if a kernel recorded a device failure."""
    dev = torch.device("cuda", torch.cuda.current_device())
    _check(library().la_check_status(_stream_handle(dev, stream)), "la_check_status")
