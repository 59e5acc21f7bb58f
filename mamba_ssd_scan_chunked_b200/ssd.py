"""Thin Python binding of libssd (include/ssd.h).

Argument marshalling only: every step of the SSD computation runs in the CUDA
kernels of ``libssd.so``.  PyTorch serves as the allocator of device memory and
the source of streams.  There is no fallback: if ``libssd.so`` is missing the
first call raises.

Raw names mirror the C ABI (``ssd_chunk_scan_fwd``, ``ssd_state_update``, ...)
and take integer device pointers; ``chunk_scan_fwd`` and ``state_update`` are
the tensor-level conveniences (shape checks, output and workspace allocation).
"""
from __future__ import annotations

import ctypes
import os
import threading

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libssd.so")

SSD_F32 = 0
SSD_BF16 = 1

STATUS = {0: "SSD_OK", 1: "SSD_ERR_INVALID_ARG", 2: "SSD_ERR_UNSUPPORTED", 3: "SSD_ERR_ALIGNMENT",
          4: "SSD_ERR_WORKSPACE", 5: "SSD_ERR_CUDA", 6: "SSD_ERR_DEVICE_TIMEOUT"}

# every symbol include/ssd.h declares
EXPORTS = ("ssd_version", "ssd_status_string", "ssd_chunk_scan_workspace_size", "ssd_chunk_scan_path",
           "ssd_chunk_scan_fwd", "ssd_chunk_scan_fwd_varlen", "ssd_chunk_scan_fwd_noalloc",
           "ssd_chunk_scan_bwd", "ssd_chunk_scan_bwd_workspace_size", "ssd_chunk_scan_bwd_launches",
           "ssd_chunk_scan_fwd_mamba3", "ssd_chunk_scan_mamba3_workspace_size", "ssd_chunk_scan_mamba3_launches",
           "ssd_state_update", "ssd_state_update_mimo", "ssd_state_update_mamba3",
           "ssd_replay_buffer_size",
           "ssd_replay_step", "ssd_get_device_error", "ssd_debug_inject")

# fault-injection bits of ssd_debug_inject
SSD_FAULT_DROP_RUN_PUBLISH = 0x1

# scratch size of ssd_chunk_scan_fwd_noalloc (SSD_NOALLOC_WORKSPACE_BYTES)
NOALLOC_WORKSPACE_BYTES = 32 << 20


class SsdError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)}")


class PrefillDesc(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64), ("nheads", ctypes.c_int64),
                ("headdim", ctypes.c_int64), ("dstate", ctypes.c_int64), ("ngroups", ctypes.c_int64),
                ("chunk", ctypes.c_int64), ("io_dtype", ctypes.c_int32), ("y_dtype", ctypes.c_int32),
                ("state_dtype", ctypes.c_int32)]


class DecodeDesc(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("nheads", ctypes.c_int64), ("headdim", ctypes.c_int64),
                ("dstate", ctypes.c_int64), ("ngroups", ctypes.c_int64), ("io_dtype", ctypes.c_int32),
                ("y_dtype", ctypes.c_int32), ("state_dtype", ctypes.c_int32)]


class MimoDesc(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("nheads", ctypes.c_int64), ("headdim", ctypes.c_int64),
                ("dstate", ctypes.c_int64), ("ngroups", ctypes.c_int64), ("rank", ctypes.c_int64),
                ("io_dtype", ctypes.c_int32), ("y_dtype", ctypes.c_int32), ("state_dtype", ctypes.c_int32)]


class ReplayDesc(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("nheads", ctypes.c_int64), ("headdim", ctypes.c_int64),
                ("dstate", ctypes.c_int64), ("ngroups", ctypes.c_int64), ("io_dtype", ctypes.c_int32),
                ("y_dtype", ctypes.c_int32), ("state_dtype", ctypes.c_int32), ("capacity", ctypes.c_int32)]


_lock = threading.Lock()
_lib = None
_VP = ctypes.c_void_p


def lib():
    """The loaded libssd.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                                   "`python -m mamba_ssd_scan_chunked_b200.build` (there is no fallback path)")
            L = ctypes.CDLL(LIB_PATH)
            L.ssd_version.restype = ctypes.c_int
            L.ssd_version.argtypes = []
            L.ssd_status_string.restype = ctypes.c_char_p
            L.ssd_status_string.argtypes = [ctypes.c_int]
            L.ssd_chunk_scan_workspace_size.restype = ctypes.c_int
            L.ssd_chunk_scan_workspace_size.argtypes = [ctypes.POINTER(PrefillDesc), ctypes.POINTER(ctypes.c_size_t)]
            L.ssd_chunk_scan_path.restype = ctypes.c_int
            L.ssd_chunk_scan_path.argtypes = [ctypes.POINTER(PrefillDesc), ctypes.POINTER(ctypes.c_int32)]
            L.ssd_chunk_scan_fwd.restype = ctypes.c_int
            L.ssd_chunk_scan_fwd.argtypes = [ctypes.POINTER(PrefillDesc)] + [_VP] * 10 + [_VP, ctypes.c_size_t, _VP]
            L.ssd_chunk_scan_fwd_varlen.restype = ctypes.c_int
            L.ssd_chunk_scan_fwd_varlen.argtypes = [ctypes.POINTER(PrefillDesc)] + [_VP] * 11 + [_VP, ctypes.c_size_t, _VP]
            L.ssd_chunk_scan_fwd_noalloc.restype = ctypes.c_int
            L.ssd_chunk_scan_fwd_noalloc.argtypes = [ctypes.POINTER(PrefillDesc)] + [_VP] * 11
            L.ssd_chunk_scan_bwd.restype = ctypes.c_int
            L.ssd_chunk_scan_bwd.argtypes = [ctypes.POINTER(PrefillDesc)] + [_VP] * 19 + [ctypes.c_size_t, _VP]
            L.ssd_chunk_scan_bwd_workspace_size.restype = ctypes.c_int
            L.ssd_chunk_scan_bwd_workspace_size.argtypes = [ctypes.POINTER(PrefillDesc),
                                                            ctypes.POINTER(ctypes.c_size_t)]
            L.ssd_chunk_scan_bwd_launches.restype = ctypes.c_int
            L.ssd_chunk_scan_bwd_launches.argtypes = [ctypes.POINTER(PrefillDesc), ctypes.c_int32,
                                                      ctypes.POINTER(ctypes.c_int32)]
            L.ssd_chunk_scan_fwd_mamba3.restype = ctypes.c_int
            L.ssd_chunk_scan_fwd_mamba3.argtypes = [ctypes.POINTER(PrefillDesc)] + [_VP] * 13 + [ctypes.c_size_t, _VP]
            L.ssd_chunk_scan_mamba3_workspace_size.restype = ctypes.c_int
            L.ssd_chunk_scan_mamba3_workspace_size.argtypes = [ctypes.POINTER(PrefillDesc),
                                                               ctypes.POINTER(ctypes.c_size_t)]
            L.ssd_chunk_scan_mamba3_launches.restype = ctypes.c_int
            L.ssd_chunk_scan_mamba3_launches.argtypes = [ctypes.POINTER(PrefillDesc)] + [ctypes.c_int32] * 3 + \
                [ctypes.POINTER(ctypes.c_int32)]
            L.ssd_state_update.restype = ctypes.c_int
            L.ssd_state_update.argtypes = [ctypes.POINTER(DecodeDesc)] + [_VP] * 10
            L.ssd_state_update_mimo.restype = ctypes.c_int
            L.ssd_state_update_mimo.argtypes = [ctypes.POINTER(MimoDesc)] + [_VP] * 10
            L.ssd_state_update_mamba3.restype = ctypes.c_int
            L.ssd_state_update_mamba3.argtypes = [ctypes.POINTER(DecodeDesc)] + [_VP] * 14
            L.ssd_replay_buffer_size.restype = ctypes.c_int
            L.ssd_replay_buffer_size.argtypes = [ctypes.POINTER(ReplayDesc), ctypes.POINTER(ctypes.c_size_t)]
            L.ssd_replay_step.restype = ctypes.c_int
            L.ssd_replay_step.argtypes = [ctypes.POINTER(ReplayDesc), _VP, _VP, ctypes.c_int32] + [_VP] * 9
            L.ssd_get_device_error.restype = ctypes.c_int
            L.ssd_get_device_error.argtypes = [_VP, ctypes.POINTER(ctypes.c_uint32)]
            L.ssd_debug_inject.restype = ctypes.c_int
            L.ssd_debug_inject.argtypes = [ctypes.c_uint32]
            _lib = L
    return _lib


# --------------------------------------------------------------------------
# raw C-ABI calls (integer device pointers; 0 = NULL)
# --------------------------------------------------------------------------
def ssd_version() -> int:
    return lib().ssd_version()


def ssd_status_string(status: int) -> str:
    return lib().ssd_status_string(status).decode()


def ssd_chunk_scan_workspace_size(desc: PrefillDesc) -> int:
    n = ctypes.c_size_t(0)
    st = lib().ssd_chunk_scan_workspace_size(ctypes.byref(desc), ctypes.byref(n))
    if st:
        raise SsdError(st, "ssd_chunk_scan_workspace_size")
    return n.value


def ssd_chunk_scan_path(desc: PrefillDesc) -> int:
    p = ctypes.c_int32(-1)
    st = lib().ssd_chunk_scan_path(ctypes.byref(desc), ctypes.byref(p))
    if st:
        raise SsdError(st, "ssd_chunk_scan_path")
    return p.value


def ssd_chunk_scan_fwd(desc, x, dt_raw, dt_bias, A, B, C, D, init_state, y, final_state,
                       workspace, workspace_bytes, stream) -> int:
    """Raw call; returns the status code (0 = enqueued)."""
    return lib().ssd_chunk_scan_fwd(ctypes.byref(desc), x or None, dt_raw or None, dt_bias or None, A or None,
                                     B or None, C or None, D or None, init_state or None, y or None,
                                     final_state or None, workspace or None, int(workspace_bytes), stream or None)


def ssd_chunk_scan_fwd_varlen(desc, x, dt_raw, dt_bias, A, B, C, D, init_state, pad_left, y, final_state,
                              workspace, workspace_bytes, stream) -> int:
    """Raw call of the left-padded variable-length variant; returns the status code."""
    return lib().ssd_chunk_scan_fwd_varlen(ctypes.byref(desc), x or None, dt_raw or None, dt_bias or None, A or None,
                                           B or None, C or None, D or None, init_state or None, pad_left or None,
                                           y or None, final_state or None, workspace or None, int(workspace_bytes),
                                           stream or None)


def ssd_chunk_scan_bwd(desc, x, dt_raw, dt_bias, A, B, C, D, init_state, dy, dfinal_state, dx, ddt_raw, ddt_bias, dA,
                       dB, dC, dD, dinit_state, workspace, workspace_bytes, stream) -> int:
    """Raw call of the backward pass; returns the status code (0 = enqueued)."""
    ptrs = (x, dt_raw, dt_bias, A, B, C, D, init_state, dy, dfinal_state, dx, ddt_raw, ddt_bias, dA, dB, dC, dD,
            dinit_state, workspace)
    return lib().ssd_chunk_scan_bwd(ctypes.byref(desc), *(p or None for p in ptrs), int(workspace_bytes),
                                     stream or None)


def ssd_chunk_scan_fwd_mamba3(desc, x, dt_raw, dt_bias, A, B, C, D, lam, theta, init_state, y, final_state,
                              workspace, workspace_bytes, stream) -> int:
    """Raw call of the Mamba-3 prefill; returns the status code (0 = enqueued)."""
    ptrs = (x, dt_raw, dt_bias, A, B, C, D, lam, theta, init_state, y, final_state, workspace)
    return lib().ssd_chunk_scan_fwd_mamba3(ctypes.byref(desc), *(p or None for p in ptrs), int(workspace_bytes),
                                            stream or None)


def ssd_chunk_scan_mamba3_workspace_size(desc: PrefillDesc) -> int:
    n = ctypes.c_size_t(0)
    st = lib().ssd_chunk_scan_mamba3_workspace_size(ctypes.byref(desc), ctypes.byref(n))
    if st:
        raise SsdError(st, "ssd_chunk_scan_mamba3_workspace_size")
    return int(n.value)


def ssd_chunk_scan_mamba3_launches(desc: PrefillDesc, has_lam: bool, has_theta: bool, has_final: bool) -> int:
    n = ctypes.c_int32(0)
    st = lib().ssd_chunk_scan_mamba3_launches(ctypes.byref(desc), int(bool(has_lam)), int(bool(has_theta)),
                                              int(bool(has_final)), ctypes.byref(n))
    if st:
        raise SsdError(st, "ssd_chunk_scan_mamba3_launches")
    return int(n.value)


def ssd_chunk_scan_bwd_workspace_size(desc: PrefillDesc) -> int:
    n = ctypes.c_size_t(0)
    st = lib().ssd_chunk_scan_bwd_workspace_size(ctypes.byref(desc), ctypes.byref(n))
    if st:
        raise SsdError(st, "ssd_chunk_scan_bwd_workspace_size")
    return int(n.value)


def ssd_chunk_scan_bwd_launches(desc: PrefillDesc, has_states: bool) -> int:
    n = ctypes.c_int32(0)
    st = lib().ssd_chunk_scan_bwd_launches(ctypes.byref(desc), int(bool(has_states)), ctypes.byref(n))
    if st:
        raise SsdError(st, "ssd_chunk_scan_bwd_launches")
    return int(n.value)


def ssd_chunk_scan_fwd_noalloc(desc, x, dt_raw, dt_bias, A, B, C, D, init_state, y, final_state, stream) -> int:
    """Raw call of the variant without a caller workspace; returns the status code."""
    return lib().ssd_chunk_scan_fwd_noalloc(ctypes.byref(desc), x or None, dt_raw or None, dt_bias or None, A or None,
                                            B or None, C or None, D or None, init_state or None, y or None,
                                            final_state or None, stream or None)


def ssd_state_update(desc, state, x, dt_raw, dt_bias, A, B, C, D, y, stream) -> int:
    """Raw call; returns the status code (0 = enqueued)."""
    return lib().ssd_state_update(ctypes.byref(desc), state or None, x or None, dt_raw or None, dt_bias or None,
                                  A or None, B or None, C or None, D or None, y or None, stream or None)


def ssd_state_update_mimo(desc, state, x, dt_raw, dt_bias, A, B, C, D, y, stream) -> int:
    """Raw call; returns the status code (0 = enqueued)."""
    return lib().ssd_state_update_mimo(ctypes.byref(desc), state or None, x or None, dt_raw or None, dt_bias or None,
                                       A or None, B or None, C or None, D or None, y or None, stream or None)


def ssd_state_update_mamba3(desc, state, x, x_prev, dt_raw, dt_bias, A, B, B_prev, C, D, lam, theta, y,
                            stream) -> int:
    """Raw call; returns the status code (0 = enqueued)."""
    return lib().ssd_state_update_mamba3(ctypes.byref(desc), state or None, x or None, x_prev or None, dt_raw or None,
                                         dt_bias or None, A or None, B or None, B_prev or None, C or None, D or None,
                                         lam or None, theta or None, y or None, stream or None)


def ssd_replay_buffer_size(desc: ReplayDesc) -> int:
    n = ctypes.c_size_t(0)
    st = lib().ssd_replay_buffer_size(ctypes.byref(desc), ctypes.byref(n))
    if st:
        raise SsdError(st, "ssd_replay_buffer_size")
    return n.value


def ssd_replay_step(desc, checkpoint, buffer, fill, x, dt_raw, dt_bias, A, B, C, D, y, stream) -> int:
    """Raw call; returns the status code (0 = enqueued)."""
    return lib().ssd_replay_step(ctypes.byref(desc), checkpoint or None, buffer or None, int(fill), x or None,
                                 dt_raw or None, dt_bias or None, A or None, B or None, C or None, D or None,
                                 y or None, stream or None)


def ssd_get_device_error(stream=None):
    """Synchronise ``stream`` and return (status, detail bits) of the device error word."""
    d = ctypes.c_uint32(0)
    st = lib().ssd_get_device_error(stream or None, ctypes.byref(d))
    return st, d.value


def ssd_debug_inject(faults: int) -> int:
    """Test hook: fault bits injected into every following launch (0 clears)."""
    return lib().ssd_debug_inject(int(faults))


# --------------------------------------------------------------------------
# tensor-level conveniences
# --------------------------------------------------------------------------
def _dtype_code(t) -> int:
    import torch
    if t == torch.float32:
        return SSD_F32
    if t == torch.bfloat16:
        return SSD_BF16
    raise TypeError(f"unsupported dtype {t}; libssd takes float32 or bfloat16")


def _torch_dtype(code: int):
    import torch
    return torch.bfloat16 if code == SSD_BF16 else torch.float32


def _ptr(t) -> int:
    return 0 if t is None else int(t.data_ptr())


def _stream(stream) -> int:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _expect(t, shape, name, dtype=None):
    """The C ABI takes bare pointers and sizes from the descriptor, so a tensor of
    another shape or dtype than the descriptor implies would be read or written
    out of bounds: refuse it here (None passes: optional arguments)."""
    if t is None:
        return
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name}: dtype {t.dtype}, expected {dtype}")


def prefill_desc(x, B, chunk, y_dtype=None, state_dtype=None) -> PrefillDesc:
    import torch
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    io = _dtype_code(x.dtype)
    return PrefillDesc(b, L, H, P, N, G, int(chunk), io,
                       _dtype_code(y_dtype) if y_dtype is not None else io,
                       _dtype_code(state_dtype) if state_dtype is not None else SSD_F32)


def workspace_bytes(x, B, chunk, y_dtype=None, state_dtype=None) -> int:
    return ssd_chunk_scan_workspace_size(prefill_desc(x, B, chunk, y_dtype, state_dtype))


def _check_prefill_args(desc, x, dt_raw, dt_bias, A, B, C, D, init_state):
    import torch
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    _expect(dt_raw, (b, L, H), "dt_raw", x.dtype)
    _expect(B, (b, L, G, N), "B", x.dtype)
    _expect(C, (b, L, G, N), "C", x.dtype)
    for name, t in (("dt_bias", dt_bias), ("A", A), ("D", D)):
        _expect(t, (H,), name, torch.float32)
    _expect(init_state, (b, H, N, P), "init_state", _torch_dtype(desc.state_dtype))


def chunk_scan_fwd(x, dt_raw, dt_bias, A, B, C, D, chunk, init_state=None, *, y=None, final_state=None,
                   y_dtype=None, state_dtype=None, want_final_state=True, workspace=None, pad_left=None, stream=None):
    """Chunked prefill scan.  Shapes: x [b,L,H,P], dt_raw [b,L,H], B/C [b,L,G,N], dt_bias/A/D [H] (fp32);
    ``pad_left`` (int32 [b], CUDA) marks left-padded variable-length sequences.

    Returns (y, final_state).  Outputs and workspace are allocated with torch
    when not given; ``state_dtype`` defaults to init_state's dtype, else fp32.
    """
    import torch
    if y_dtype is None and y is not None:
        y_dtype = y.dtype
    if state_dtype is None:
        state_dtype = (init_state.dtype if init_state is not None else
                       final_state.dtype if final_state is not None else torch.float32)
    desc = prefill_desc(x, B, chunk, y_dtype, state_dtype)
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    _check_prefill_args(desc, x, dt_raw, dt_bias, A, B, C, D, init_state)
    _expect(y, (b, L, H, P), "y", _torch_dtype(desc.y_dtype))
    _expect(final_state, (b, H, N, P), "final_state", _torch_dtype(desc.state_dtype))
    _expect(pad_left, (b,), "pad_left")
    for t in (x, dt_raw, B, C, dt_bias, A, D, init_state, y, final_state):
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("libssd takes contiguous CUDA tensors")
    if y is None:
        y = torch.empty((b, L, H, P), dtype=_torch_dtype(desc.y_dtype), device=x.device)
    if final_state is None and want_final_state:
        final_state = torch.empty((b, H, N, P), dtype=_torch_dtype(desc.state_dtype), device=x.device)
    need = ssd_chunk_scan_workspace_size(desc)
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=x.device)
    if pad_left is None:
        st = ssd_chunk_scan_fwd(desc, _ptr(x), _ptr(dt_raw), _ptr(dt_bias), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                                _ptr(init_state), _ptr(y), _ptr(final_state), _ptr(workspace), workspace.numel(),
                                _stream(stream))
    else:
        if pad_left.dtype != torch.int32 or not pad_left.is_cuda or not pad_left.is_contiguous():
            raise ValueError("pad_left must be a contiguous int32 CUDA tensor [batch]")
        st = ssd_chunk_scan_fwd_varlen(desc, _ptr(x), _ptr(dt_raw), _ptr(dt_bias), _ptr(A), _ptr(B), _ptr(C),
                                       _ptr(D), _ptr(init_state), _ptr(pad_left), _ptr(y), _ptr(final_state),
                                       _ptr(workspace), workspace.numel(), _stream(stream))
    if st:
        raise SsdError(st, "ssd_chunk_scan_fwd")
    return y, final_state


def chunk_scan_fwd_mamba3(x, dt_raw, dt_bias, A, B, C, D, chunk, lam=None, theta=None, init_state=None, *,
                          y_dtype=None, state_dtype=None, want_final_state=True, workspace=None, stream=None):
    """Mamba-3 prefill (trapezoidal input mix ``lam`` [b,L,H] fp32, rotation
    angles ``theta`` [b,L,G,N/2] fp32; either may be None).  Returns (y, final_state)."""
    import torch
    if state_dtype is None:
        state_dtype = init_state.dtype if init_state is not None else torch.float32
    desc = prefill_desc(x, B, chunk, y_dtype, state_dtype)
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    _check_prefill_args(desc, x, dt_raw, dt_bias, A, B, C, D, init_state)
    _expect(lam, (b, L, H), "lam")
    _expect(theta, (b, L, G, N // 2), "theta")
    for t in (x, dt_raw, B, C, dt_bias, A, D, lam, theta, init_state):
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("libssd takes contiguous CUDA tensors")
    for t in (lam, theta):
        if t is not None and t.dtype != torch.float32:
            raise ValueError("lam and theta are fp32")
    y = torch.empty((b, L, H, P), dtype=_torch_dtype(desc.y_dtype), device=x.device)
    final_state = (torch.empty((b, H, N, P), dtype=_torch_dtype(desc.state_dtype), device=x.device)
                   if want_final_state else None)
    need = ssd_chunk_scan_mamba3_workspace_size(desc)
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=x.device)
    st = ssd_chunk_scan_fwd_mamba3(desc, _ptr(x), _ptr(dt_raw), _ptr(dt_bias), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                                   _ptr(lam), _ptr(theta), _ptr(init_state), _ptr(y), _ptr(final_state),
                                   _ptr(workspace), workspace.numel(), _stream(stream))
    if st:
        raise SsdError(st, "ssd_chunk_scan_fwd_mamba3")
    return y, final_state


def chunk_scan_bwd(x, dt_raw, dt_bias, A, B, C, D, chunk, dy, init_state=None, dfinal_state=None, *,
                   grad_dtype=None, state_dtype=None, want_dinit=True, workspace=None, stream=None):
    """Backward pass of ``chunk_scan_fwd``: gradients of sum<dy, y> + <dfinal_state, final_state>.

    Returns a dict of CUDA tensors: dx, ddt_raw, dB, dC (``grad_dtype``, default
    x's dtype), dA, ddt_bias, dD (fp32 [H]) and dinit_state (state dtype, or
    None when ``want_dinit`` is false).
    """
    import torch
    if state_dtype is None:
        src = init_state if init_state is not None else dfinal_state
        state_dtype = src.dtype if src is not None else torch.float32
    desc = prefill_desc(x, B, chunk, grad_dtype, state_dtype)
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    _check_prefill_args(desc, x, dt_raw, dt_bias, A, B, C, D, init_state)
    _expect(dy, (b, L, H, P), "dy", x.dtype)
    _expect(dfinal_state, (b, H, N, P), "dfinal_state", _torch_dtype(desc.state_dtype))
    for t in (x, dt_raw, B, C, dt_bias, A, D, init_state, dy, dfinal_state):
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("libssd takes contiguous CUDA tensors")
    gd, dev = _torch_dtype(desc.y_dtype), x.device
    out = {"dx": torch.empty((b, L, H, P), dtype=gd, device=dev),
           "ddt_raw": torch.empty((b, L, H), dtype=gd, device=dev),
           "dB": torch.empty((b, L, G, N), dtype=gd, device=dev),
           "dC": torch.empty((b, L, G, N), dtype=gd, device=dev),
           "dA": torch.empty(H, dtype=torch.float32, device=dev),
           "ddt_bias": torch.empty(H, dtype=torch.float32, device=dev),
           "dD": torch.empty(H, dtype=torch.float32, device=dev),
           "dinit_state": (torch.empty((b, H, N, P), dtype=_torch_dtype(desc.state_dtype), device=dev)
                           if want_dinit else None)}
    need = ssd_chunk_scan_bwd_workspace_size(desc)
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    st = ssd_chunk_scan_bwd(desc, _ptr(x), _ptr(dt_raw), _ptr(dt_bias), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                            _ptr(init_state), _ptr(dy), _ptr(dfinal_state), _ptr(out["dx"]), _ptr(out["ddt_raw"]),
                            _ptr(out["ddt_bias"]), _ptr(out["dA"]), _ptr(out["dB"]), _ptr(out["dC"]),
                            _ptr(out["dD"]), _ptr(out["dinit_state"]), _ptr(workspace), workspace.numel(),
                            _stream(stream))
    if st:
        raise SsdError(st, "ssd_chunk_scan_bwd")
    return out


def _check_decode_args(state, x, dt_raw, dt_bias, A, B, C, D, y, y_dtype, bshape=None):
    import torch
    b, H = x.shape[0], x.shape[1]
    P = x.shape[-1]
    G, N = B.shape[1], B.shape[-1]
    _expect(state, (b, H, N, P), "state")
    _expect(dt_raw, (b, H), "dt_raw", x.dtype)
    _expect(B, bshape or (b, G, N), "B", x.dtype)
    _expect(C, bshape or (b, G, N), "C", x.dtype)
    for name, t in (("dt_bias", dt_bias), ("A", A), ("D", D)):
        _expect(t, (H,), name, torch.float32)
    _expect(y, tuple(x.shape), "y", y_dtype)


def state_update(state, x, dt_raw, dt_bias, A, B, C, D, *, y=None, y_dtype=None, stream=None):
    """Decode step in place on ``state`` [b,H,N,P].  x [b,H,P], dt_raw [b,H], B/C [b,G,N].  Returns y."""
    import torch
    b, H, P = x.shape
    G, N = B.shape[1], B.shape[2]
    if y_dtype is None and y is not None:
        y_dtype = y.dtype
    _check_decode_args(state, x, dt_raw, dt_bias, A, B, C, D, y, y_dtype)
    io = _dtype_code(x.dtype)
    desc = DecodeDesc(b, H, P, N, G, io, _dtype_code(y_dtype) if y_dtype is not None else io,
                      _dtype_code(state.dtype))
    for t in (state, x, dt_raw, B, C, dt_bias, A, D, y):
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("libssd takes contiguous CUDA tensors")
    if y is None:
        y = torch.empty((b, H, P), dtype=_torch_dtype(desc.y_dtype), device=x.device)
    st = ssd_state_update(desc, _ptr(state), _ptr(x), _ptr(dt_raw), _ptr(dt_bias), _ptr(A), _ptr(B), _ptr(C),
                          _ptr(D), _ptr(y), _stream(stream))
    if st:
        raise SsdError(st, "ssd_state_update")
    return y


def state_update_mamba3(state, x, dt_raw, dt_bias, A, B, C, D, *, x_prev=None, B_prev=None, lam=None, theta=None,
                        y=None, y_dtype=None, stream=None):
    """Mamba-3 decode step in place on ``state`` [b,H,N,P]: x, x_prev [b,H,P], dt_raw [b,H],
    B, B_prev, C [b,G,N], lam [b,H] (fp32), theta [b,G,N/2] (fp32).  x_prev and B_prev
    are the previous token's x and B (None before the first token).  Returns y."""
    import torch
    b, H, P = x.shape
    G, N = B.shape[1], B.shape[2]
    if y_dtype is None and y is not None:
        y_dtype = y.dtype
    _check_decode_args(state, x, dt_raw, dt_bias, A, B, C, D, y, y_dtype)
    _expect(x_prev, (b, H, P), "x_prev", x.dtype)
    _expect(B_prev, (b, G, N), "B_prev", x.dtype)
    _expect(lam, (b, H), "lam")
    _expect(theta, (b, G, N // 2), "theta")
    io = _dtype_code(x.dtype)
    desc = DecodeDesc(b, H, P, N, G, io, _dtype_code(y_dtype) if y_dtype is not None else io,
                      _dtype_code(state.dtype))
    for t in (state, x, x_prev, dt_raw, B, B_prev, C, dt_bias, A, D, lam, theta, y):
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("libssd takes contiguous CUDA tensors")
    if y is None:
        y = torch.empty((b, H, P), dtype=_torch_dtype(desc.y_dtype), device=x.device)
    st = ssd_state_update_mamba3(desc, _ptr(state), _ptr(x), _ptr(x_prev), _ptr(dt_raw), _ptr(dt_bias), _ptr(A),
                                 _ptr(B), _ptr(B_prev), _ptr(C), _ptr(D), _ptr(lam), _ptr(theta), _ptr(y),
                                 _stream(stream))
    if st:
        raise SsdError(st, "ssd_state_update_mamba3")
    return y


def replay_desc(checkpoint, x, B, capacity, y_dtype=None) -> ReplayDesc:
    b, H, P = x.shape
    G, N = B.shape[1], B.shape[2]
    io = _dtype_code(x.dtype)
    return ReplayDesc(b, H, P, N, G, io, _dtype_code(y_dtype) if y_dtype is not None else io,
                      _dtype_code(checkpoint.dtype), int(capacity))


def replay_buffer(checkpoint, x, B, capacity):
    """A device buffer of the size ssd_replay_step needs (uint8, 256-byte aligned by the allocator)."""
    import torch
    n = ssd_replay_buffer_size(replay_desc(checkpoint, x, B, capacity))
    return torch.empty(max(n, 1), dtype=torch.uint8, device=x.device)


def replay_step(checkpoint, buffer, fill, capacity, x, dt_raw, dt_bias, A, B, C, D, *, y=None, y_dtype=None,
                stream=None):
    """Replayed decode step: checkpoint [b,H,N,P] + buffer (``replay_buffer``) holding ``fill``
    tokens; x [b,H,P], dt_raw [b,H], B/C [b,G,N].  Returns (y, next fill)."""
    import torch
    if y_dtype is None and y is not None:
        y_dtype = y.dtype
    _check_decode_args(checkpoint, x, dt_raw, dt_bias, A, B, C, D, y, y_dtype)
    desc = replay_desc(checkpoint, x, B, capacity, y_dtype)
    if buffer is not None and buffer.numel() * buffer.element_size() < ssd_replay_buffer_size(desc):
        raise ValueError("buffer: smaller than ssd_replay_buffer_size")
    for t in (checkpoint, buffer, x, dt_raw, B, C, dt_bias, A, D, y):
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("libssd takes contiguous CUDA tensors")
    b, H, P = x.shape
    if y is None:
        y = torch.empty((b, H, P), dtype=_torch_dtype(desc.y_dtype), device=x.device)
    st = ssd_replay_step(desc, _ptr(checkpoint), _ptr(buffer), fill, _ptr(x), _ptr(dt_raw), _ptr(dt_bias), _ptr(A),
                         _ptr(B), _ptr(C), _ptr(D), _ptr(y), _stream(stream))
    if st:
        raise SsdError(st, "ssd_replay_step")
    return y, (fill + 1) % int(capacity)


def state_update_mimo(state, x, dt_raw, dt_bias, A, B, C, D, *, y=None, y_dtype=None, stream=None):
    """MIMO decode step in place on ``state`` [b,H,N,P].  x [b,H,R,P], dt_raw [b,H], B/C [b,G,R,N].  Returns y."""
    import torch
    b, H, R, P = x.shape
    G, N = B.shape[1], B.shape[3]
    if y_dtype is None and y is not None:
        y_dtype = y.dtype
    _check_decode_args(state, x, dt_raw, dt_bias, A, B, C, D, y, y_dtype, bshape=(b, G, R, N))
    io = _dtype_code(x.dtype)
    desc = MimoDesc(b, H, P, N, G, R, io, _dtype_code(y_dtype) if y_dtype is not None else io,
                    _dtype_code(state.dtype))
    for t in (state, x, dt_raw, B, C, dt_bias, A, D, y):
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("libssd takes contiguous CUDA tensors")
    if y is None:
        y = torch.empty((b, H, R, P), dtype=_torch_dtype(desc.y_dtype), device=x.device)
    st = ssd_state_update_mimo(desc, _ptr(state), _ptr(x), _ptr(dt_raw), _ptr(dt_bias), _ptr(A), _ptr(B), _ptr(C),
                               _ptr(D), _ptr(y), _stream(stream))
    if st:
        raise SsdError(st, "ssd_state_update_mimo")
    return y
