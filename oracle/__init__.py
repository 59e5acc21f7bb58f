"""Float64 CPU oracle of the Mamba-2 SSD layer core (test infrastructure).

Only the test-suite, ``__graft_entry__.smoke()`` and ``bench.py``'s
``cpu_baseline`` / ``--impl reference`` legs may import this package.  The
CUDA library never links, loads or calls it, and it shares no code with the
CUDA library.

The arithmetic lives in ``ssd_oracle.c`` (plain C, float64, OpenMP over the
independent (batch, head) recurrences); this module only compiles it with gcc
and marshals numpy arrays.  Every function cites the passage it follows in the
C file's header:

- ``recurrent``  -- the sequential recurrence (the definition): scalar-times-
  identity transition ("Mamba3", Telegram post; "Mamba-3 : SSM optimise
  inference", section "Du training-first a l'inference-first"), ZOH on the
  state and Euler on the input ("Mamba3", section "New discretisation scheme").
- ``quadratic``  -- the masked-attention contraction order of the same
  semiseparable matrix ("Mamba-2 vs Transformers / SSD", sections "How we
  compared" and "Mamba-2 and the SSD paper: what changed in practice").
- ``chunked``    -- the blocked two-pass contraction with per-chunk states
  recombined across chunks (same page, same section, and its table row
  "Mamba-2 SSD layer | Blocked two-pass contraction").
- ``backward``   -- reverse-mode gradients of the recurrence (the pages only
  say that end-to-end training also needs the backward pass: "Mamba-3 : SSM
  optimise inference", opening paragraph; the gradients follow from the
  forward definition).
- ``mamba3_recurrent`` -- the Mamba-3 recurrence: exponential-trapezoidal
  input and a rotational (complex) state ("Mamba3", sections "New
  discretisation scheme" and on complex-valued SSMs; "Mamba-3 : SSM optimise
  inference", "Etats complexes via RoPE").
- ``mamba3_decode_step`` -- one token of the Mamba-3 recurrence (the state
  plus the previous token's B and x, which the trapezoid's left end reads);
  ``mimo_recurrent`` -- a sequence of MIMO tokens.  Both are references for
  kernels not yet built, pinned like the rest.
- ``decode_step`` -- one token of the recurrent mode, in place on the state
  (same page, table "Evaluation criteria": O(1) recurrent step at inference).

Every entry point is pinned in ``tests/test_oracle_pins.py`` against closed
forms, textbook special cases and invariants (none of them re-types the C).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssd_oracle.c")
_LIB = os.path.join(_HERE, "libssd_oracle.so")
_lock = threading.Lock()
_lib = None

_D = ctypes.POINTER(ctypes.c_double)
_I64 = ctypes.c_int64


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (IEEE float64: no fast-math) and return the path."""
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-Wall", "-Werror",
           "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            sig6 = [_I64] * 6
            ptrs = [_D] * 10
            for name in ("oracle_ssd_recurrent", "oracle_ssd_quadratic"):
                fn = getattr(lib, name)
                fn.argtypes = sig6 + ptrs + [ctypes.c_int]
                fn.restype = ctypes.c_int
            lib.oracle_ssd_chunked.argtypes = sig6 + [_I64] + ptrs + [ctypes.c_int]
            lib.oracle_ssd_chunked.restype = ctypes.c_int
            lib.oracle_ssd_decode_step.argtypes = [_I64] * 5 + [_D] * 9 + [ctypes.c_int, ctypes.c_int]
            lib.oracle_ssd_decode_step.restype = ctypes.c_int
            lib.oracle_ssd_decode_step_mimo.argtypes = [_I64] * 6 + [_D] * 9 + [ctypes.c_int, ctypes.c_int]
            lib.oracle_ssd_decode_step_mimo.restype = ctypes.c_int
            lib.oracle_ssd_backward.argtypes = sig6 + [_D] * 18 + [ctypes.c_int]
            lib.oracle_ssd_backward.restype = ctypes.c_int
            lib.oracle_ssd_mamba3_recurrent.argtypes = sig6 + [_D] * 12 + [ctypes.c_int]
            lib.oracle_ssd_mamba3_recurrent.restype = ctypes.c_int
            lib.oracle_ssd_mamba3_decode_step.argtypes = [_I64] * 5 + [_D] * 13 + [ctypes.c_int]
            lib.oracle_ssd_mamba3_decode_step.restype = ctypes.c_int
            lib.oracle_ssd_mimo_recurrent.argtypes = sig6 + [_I64] + [_D] * 10 + [ctypes.c_int]
            lib.oracle_ssd_mimo_recurrent.restype = ctypes.c_int
            lib.oracle_round_bf16.argtypes = [ctypes.c_double]
            lib.oracle_round_bf16.restype = ctypes.c_double
            lib.oracle_round_bf16_array.argtypes = [_D, _D, _I64]
            lib.oracle_round_bf16_array.restype = None
            lib.oracle_softplus.argtypes = [ctypes.c_double]
            lib.oracle_softplus.restype = ctypes.c_double
            lib.oracle_num_threads.argtypes = []
            lib.oracle_num_threads.restype = ctypes.c_int
            _lib = lib
    return _lib


def _f64(a):
    if a is None:
        return None
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a):
    if a is None:
        return ctypes.cast(None, _D)
    return a.ctypes.data_as(_D)


def num_threads() -> int:
    """Threads the oracle's OpenMP loops use by default."""
    return int(_load().oracle_num_threads())


def softplus(z: float) -> float:
    return float(_load().oracle_softplus(float(z)))


def round_bf16(v) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 (ties to even), as float64."""
    a = np.ascontiguousarray(v, dtype=np.float64)
    out = np.empty_like(a)
    _load().oracle_round_bf16_array(_ptr(a), _ptr(out), a.size)
    return out


def _run_prefill(fn_name, x, dt_raw, dt_bias, A, B, C, D, init_state, extra=(), nthreads=0,
                 want_y=True):
    x, dt_raw, dt_bias, A, B, C, D, init_state = map(_f64, (x, dt_raw, dt_bias, A, B, C, D, init_state))
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    assert dt_raw.shape == (b, L, H) and B.shape == C.shape == (b, L, G, N)
    y = np.empty((b, L, H, P), dtype=np.float64) if want_y else None
    fs = np.empty((b, H, N, P), dtype=np.float64)
    fn = getattr(_load(), fn_name)
    rc = fn(b, L, H, P, N, G, *extra, _ptr(x), _ptr(dt_raw), _ptr(dt_bias), _ptr(A), _ptr(B), _ptr(C),
            _ptr(D), _ptr(init_state), _ptr(y), _ptr(fs), int(nthreads))
    if rc != 0:
        raise ValueError(f"{fn_name}: invalid arguments")
    return y, fs


def recurrent(x, dt_raw, dt_bias, A, B, C, D, init_state=None, nthreads=0, want_y=True):
    """Sequential recurrence.  x [b,L,H,P], dt_raw [b,L,H], B,C [b,L,G,N], dt_bias/A/D [H].

    Returns (y [b,L,H,P], final_state [b,H,N,P]) in float64.
    """
    return _run_prefill("oracle_ssd_recurrent", x, dt_raw, dt_bias, A, B, C, D, init_state,
                        nthreads=nthreads, want_y=want_y)


def quadratic(x, dt_raw, dt_bias, A, B, C, D, init_state=None, nthreads=0):
    """Masked-attention (quadratic) form of the same semiseparable matrix."""
    return _run_prefill("oracle_ssd_quadratic", x, dt_raw, dt_bias, A, B, C, D, init_state,
                        nthreads=nthreads)


def chunked(x, dt_raw, dt_bias, A, B, C, D, init_state=None, chunk=64, nthreads=0):
    """Blocked two-pass (chunked) form; the last chunk may be shorter."""
    return _run_prefill("oracle_ssd_chunked", x, dt_raw, dt_bias, A, B, C, D, init_state,
                        extra=(int(chunk),), nthreads=nthreads)


def decode_step(state, x, dt_raw, dt_bias, A, B, C, D, round_state_bf16=False, nthreads=0):
    """One recurrent step in place on ``state`` [b,H,N,P] (float64 array, modified).

    x [b,H,P], dt_raw [b,H], B,C [b,G,N].  Returns y [b,H,P].
    """
    if state.dtype != np.float64 or not state.flags.c_contiguous:
        raise TypeError("state must be a C-contiguous float64 array (updated in place)")
    x, dt_raw, dt_bias, A, B, C, D = map(_f64, (x, dt_raw, dt_bias, A, B, C, D))
    b, H, P = x.shape
    G, N = B.shape[1], B.shape[2]
    assert state.shape == (b, H, N, P) and dt_raw.shape == (b, H) and C.shape == B.shape
    y = np.empty((b, H, P), dtype=np.float64)
    rc = _load().oracle_ssd_decode_step(b, H, P, N, G, _ptr(state), _ptr(x), _ptr(dt_raw), _ptr(dt_bias),
                                        _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(y),
                                        int(bool(round_state_bf16)), int(nthreads))
    if rc != 0:
        raise ValueError("oracle_ssd_decode_step: invalid arguments")
    return y


def decode_step_mimo(state, x, dt_raw, dt_bias, A, B, C, D, round_state_bf16=False, nthreads=0):
    """One MIMO (rank-R) recurrent step in place on ``state`` [b,H,N,P] (float64, modified).

    x [b,H,R,P], dt_raw [b,H], B,C [b,G,R,N].  Returns y [b,H,R,P].
    """
    if state.dtype != np.float64 or not state.flags.c_contiguous:
        raise TypeError("state must be a C-contiguous float64 array (updated in place)")
    x, dt_raw, dt_bias, A, B, C, D = map(_f64, (x, dt_raw, dt_bias, A, B, C, D))
    b, H, R, P = x.shape
    G, N = B.shape[1], B.shape[3]
    assert state.shape == (b, H, N, P) and dt_raw.shape == (b, H) and B.shape == (b, G, R, N) and C.shape == B.shape
    y = np.empty((b, H, R, P), dtype=np.float64)
    rc = _load().oracle_ssd_decode_step_mimo(b, H, P, N, G, R, _ptr(state), _ptr(x), _ptr(dt_raw), _ptr(dt_bias),
                                             _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(y),
                                             int(bool(round_state_bf16)), int(nthreads))
    if rc != 0:
        raise ValueError("oracle_ssd_decode_step_mimo: invalid arguments")
    return y


def backward(x, dt_raw, dt_bias, A, B, C, D, init_state, dy, dfinal=None, nthreads=0):
    """Gradients of sum<dy, y> + <dfinal, final_state> through the recurrence.

    Shapes as in ``recurrent``; dy [b,L,H,P], dfinal [b,H,N,P] or None.
    Returns a dict of float64 arrays: dx, ddt_raw, ddt_bias, dA, dB, dC, dD,
    dinit_state (same shapes as the forward inputs).
    """
    x, dt_raw, dt_bias, A, B, C, D, init_state, dy, dfinal = map(
        _f64, (x, dt_raw, dt_bias, A, B, C, D, init_state, dy, dfinal))
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    assert dt_raw.shape == (b, L, H) and B.shape == C.shape == (b, L, G, N) and dy.shape == x.shape
    out = {"dx": np.empty_like(x), "ddt_raw": np.empty_like(dt_raw), "ddt_bias": np.empty(H),
           "dA": np.empty(H), "dB": np.empty_like(B), "dC": np.empty_like(C), "dD": np.empty(H),
           "dinit_state": np.empty((b, H, N, P))}
    rc = _load().oracle_ssd_backward(b, L, H, P, N, G, _ptr(x), _ptr(dt_raw), _ptr(dt_bias), _ptr(A), _ptr(B),
                                     _ptr(C), _ptr(D), _ptr(init_state), _ptr(dy), _ptr(dfinal),
                                     *(_ptr(out[k]) for k in ("dx", "ddt_raw", "ddt_bias", "dA", "dB", "dC",
                                                             "dD", "dinit_state")), int(nthreads))
    if rc != 0:
        raise ValueError("oracle_ssd_backward: invalid arguments")
    return out


def mamba3_recurrent(x, dt_raw, dt_bias, A, B, C, D, lam=None, theta=None, init_state=None, nthreads=0):
    """Mamba-3 sequential recurrence.  Shapes as ``recurrent``; lam [b,L,H] (the
    trapezoid's mix, None = 1), theta [b,L,G,N/2] (rotation angle per step and
    state pair, None = 0).  Returns (y, final_state) in float64."""
    x, dt_raw, dt_bias, A, B, C, D, lam, theta, init_state = map(
        _f64, (x, dt_raw, dt_bias, A, B, C, D, lam, theta, init_state))
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    assert dt_raw.shape == (b, L, H) and B.shape == C.shape == (b, L, G, N)
    assert lam is None or lam.shape == (b, L, H)
    assert theta is None or theta.shape == (b, L, G, N // 2)
    y = np.empty((b, L, H, P))
    fs = np.empty((b, H, N, P))
    rc = _load().oracle_ssd_mamba3_recurrent(b, L, H, P, N, G, _ptr(x), _ptr(dt_raw), _ptr(dt_bias), _ptr(A),
                                             _ptr(B), _ptr(C), _ptr(D), _ptr(lam), _ptr(theta), _ptr(init_state),
                                             _ptr(y), _ptr(fs), int(nthreads))
    if rc != 0:
        raise ValueError("oracle_ssd_mamba3_recurrent: invalid arguments")
    return y, fs


def mamba3_decode_step(state, B_prev, x_prev, x, dt_raw, dt_bias, A, B, C, D, lam=None, theta=None, nthreads=0):
    """One Mamba-3 token in place on ``state`` [b,H,N,P] and the previous-token
    buffers ``B_prev`` [b,G,N], ``x_prev`` [b,H,P] (float64, modified; zero
    before the first token).  x [b,H,P], dt_raw [b,H], B, C [b,G,N], lam [b,H],
    theta [b,G,N/2].  Returns y [b,H,P]."""
    for a in (state, B_prev, x_prev):
        if a.dtype != np.float64 or not a.flags.c_contiguous:
            raise TypeError("state and buffers must be C-contiguous float64 arrays (updated in place)")
    x, dt_raw, dt_bias, A, B, C, D, lam, theta = map(_f64, (x, dt_raw, dt_bias, A, B, C, D, lam, theta))
    b, H, P = x.shape
    G, N = B.shape[1], B.shape[2]
    assert state.shape == (b, H, N, P) and B_prev.shape == B.shape and x_prev.shape == x.shape
    y = np.empty((b, H, P))
    rc = _load().oracle_ssd_mamba3_decode_step(b, H, P, N, G, _ptr(state), _ptr(B_prev), _ptr(x_prev), _ptr(x),
                                               _ptr(dt_raw), _ptr(dt_bias), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                                               _ptr(lam), _ptr(theta), _ptr(y), int(nthreads))
    if rc != 0:
        raise ValueError("oracle_ssd_mamba3_decode_step: invalid arguments")
    return y


def mimo_recurrent(x, dt_raw, dt_bias, A, B, C, D, init_state=None, nthreads=0):
    """A sequence of MIMO tokens: x [b,L,H,R,P], dt_raw [b,L,H], B, C [b,L,G,R,N].
    Returns (y [b,L,H,R,P], final_state [b,H,N,P])."""
    x, dt_raw, dt_bias, A, B, C, D, init_state = map(_f64, (x, dt_raw, dt_bias, A, B, C, D, init_state))
    b, L, H, R, P = x.shape
    G, N = B.shape[2], B.shape[4]
    assert B.shape == C.shape == (b, L, G, R, N) and dt_raw.shape == (b, L, H)
    y = np.empty_like(x)
    fs = np.empty((b, H, N, P))
    rc = _load().oracle_ssd_mimo_recurrent(b, L, H, P, N, G, R, _ptr(x), _ptr(dt_raw), _ptr(dt_bias), _ptr(A),
                                           _ptr(B), _ptr(C), _ptr(D), _ptr(init_state), _ptr(y), _ptr(fs),
                                           int(nthreads))
    if rc != 0:
        raise ValueError("oracle_ssd_mimo_recurrent: invalid arguments")
    return y, fs
