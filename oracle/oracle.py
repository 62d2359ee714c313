"""fp64 CPU oracle for the key-gated GLA token mixer -- Python side.

TEST INFRASTRUCTURE ONLY: imported by the test suite, by the smoke check of
``__graft_entry__`` and by the CPU-baseline leg of ``bench.py``.  The product
library never imports, links or executes anything in this folder.

The arithmetic lives in ``gla_oracle.c`` (plain C, double precision); this
module compiles it with gcc, widens the caller's arrays to float64 and calls
it through ctypes.  Layout of every tensor: ``[B, N, heads, d]`` with the N
tokens in row-major spatial order of a ``grid_h x grid_w`` patch grid.
Directions: 0 = L->R, 1 = R->L, 2 = T->B, 3 = B->T.

Sources (by page and section; the equations are not legible on the pages):
  * ai.info summary of "GTR: Gated Token Recurrence for Efficient Dense
    Prediction", "Methodology in Plain English": key-only gated linear
    attention, one directional scan per block, spatial order restored,
    zero initial state for the inference operator.
  * GTR project page, "A Kernel That Makes Recurrence Fast": the chunkwise
    schedule (summaries, boundary scan, outputs) evaluates the exact
    recurrence.

Parity status: the serial recurrence and the chunked form are pinned by the
CPU tests against a brute-force quadratic form written independently in
numpy, against closed forms (zero gates = causal linear attention, a
constant gate = geometric decay weights, fully closed gates = memoryless
readout, a single token), against linearity, against chunk-size
independence and against the direction equivariances of the index map.
"""
from __future__ import annotations

import os
import subprocess
import ctypes
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gla_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "libgla_oracle.so")
_lib = None
_lock = threading.Lock()

DIRS = {"l2r": 0, "r2l": 1, "t2b": 2, "b2t": 3}


def build(force: bool = False) -> str:
    """Compile the C oracle into ``oracle/_build/libgla_oracle.so``."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O3", "-std=c11", "-fPIC", "-shared", "-pthread",
           "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.POINTER(ctypes.c_double)
            IP = ctypes.POINTER(ctypes.c_int)
            i = ctypes.c_int
            lib.gla_oracle_scan_index.restype = ctypes.c_int64
            lib.gla_oracle_scan_index.argtypes = [i, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64]
            lib.gla_oracle_serial.restype = i
            lib.gla_oracle_serial.argtypes = [P, P, P, P, i, i, i, i, i, i, i, P, i, P, IP, i, i]
            lib.gla_oracle_chunked.restype = i
            lib.gla_oracle_chunked.argtypes = [P, P, P, P, i, i, i, i, i, i, i, i, P, P, P, P, IP, i, i]
            lib.gla_oracle_serial_state.restype = i
            lib.gla_oracle_serial_state.argtypes = [P, P, P, P, i, i, i, i, i, i, i, P, P, P, IP, i, i]
            lib.gla_oracle_output_gate.restype = None
            lib.gla_oracle_output_gate.argtypes = [P, P, P, ctypes.c_double, ctypes.c_int64, i, P]
            lib.gla_oracle_sswiglu.restype = None
            lib.gla_oracle_sswiglu.argtypes = [P, P, P, P, i, i, i, i, P]
            _lib = lib
    return _lib


def _as_f64(x) -> np.ndarray:
    if hasattr(x, "detach"):  # torch tensor
        x = x.detach().cpu()
        if str(x.dtype) in ("torch.float16", "torch.bfloat16"):
            x = x.float()
        x = x.numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _slices_arg(slices):
    if slices is None:
        return None, None, 0
    arr = np.ascontiguousarray(np.asarray(slices, dtype=np.int32))
    return arr, arr.ctypes.data_as(ctypes.POINTER(ctypes.c_int)), int(arr.size)


def _dir(direction) -> int:
    return DIRS[direction] if isinstance(direction, str) else int(direction)


def default_threads() -> int:
    return max(1, os.cpu_count() or 1)


def scan_index(direction, t: int, grid_h: int, grid_w: int) -> int:
    """Row-major token index visited at scan position ``t``."""
    return int(_load().gla_oracle_scan_index(_dir(direction), int(t), int(grid_h), int(grid_w)))


def _shapes(q, v, grid_h, grid_w):
    B, N, heads, dk = q.shape
    dv = v.shape[3]
    if N != grid_h * grid_w:
        raise ValueError(f"N={N} != grid_h*grid_w={grid_h * grid_w}")
    return B, N, heads, dk, dv


def gla_serial(q, k, v, g, grid_h, grid_w, direction, *, chunk=0, return_states=False,
               slices=None, nthreads=None):
    """Serial recurrence S_t = diag(exp g_t) S_{t-1} + k_t^T v_t, o_t = q_t/sqrt(dk) S_t.

    Returns ``out`` (float64, same layout as v).  With ``return_states`` (needs
    ``chunk``) also returns the state after 0, chunk, 2*chunk, ..., N tokens,
    shape ``[B, heads, nc+1, dk, dv]``.  ``slices`` restricts the work to the
    listed ``b*heads + h`` slices (other outputs stay zero).
    """
    q, k, v, g = (_as_f64(x) for x in (q, k, v, g))
    B, N, heads, dk, dv = _shapes(q, v, grid_h, grid_w)
    out = np.zeros((B, N, heads, dv), dtype=np.float64)
    states = None
    if return_states:
        if chunk <= 0:
            raise ValueError("return_states needs chunk > 0")
        nc = (N + chunk - 1) // chunk
        states = np.zeros((B, heads, nc + 1, dk, dv), dtype=np.float64)
    keep, sp, ns = _slices_arg(slices)
    rc = _load().gla_oracle_serial(_ptr(q), _ptr(k), _ptr(v), _ptr(g), B, heads, grid_h, grid_w,
                                   dk, dv, _dir(direction), _ptr(out), int(chunk), _ptr(states),
                                   sp, ns, nthreads or default_threads())
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    return (out, states) if return_states else out


def gla_chunked(q, k, v, g, grid_h, grid_w, direction, chunk, *, slices=None, nthreads=None):
    """Chunkwise form: returns ``(out, dS, gamma, S_enter)``.

    ``dS[b,h,c]`` (dk x dv) is the decay-weighted summary of chunk c,
    ``gamma[b,h,c]`` (dk) its total decay, ``S_enter[b,h,c]`` the state that
    enters chunk c (zero for c = 0).
    """
    q, k, v, g = (_as_f64(x) for x in (q, k, v, g))
    B, N, heads, dk, dv = _shapes(q, v, grid_h, grid_w)
    nc = (N + chunk - 1) // chunk
    out = np.zeros((B, N, heads, dv), dtype=np.float64)
    dS = np.zeros((B, heads, nc, dk, dv), dtype=np.float64)
    gamma = np.zeros((B, heads, nc, dk), dtype=np.float64)
    S_enter = np.zeros((B, heads, nc, dk, dv), dtype=np.float64)
    keep, sp, ns = _slices_arg(slices)
    rc = _load().gla_oracle_chunked(_ptr(q), _ptr(k), _ptr(v), _ptr(g), B, heads, grid_h, grid_w,
                                    dk, dv, _dir(direction), int(chunk), _ptr(out), _ptr(dS),
                                    _ptr(gamma), _ptr(S_enter), sp, ns,
                                    nthreads or default_threads())
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    return out, dS, gamma, S_enter


def gla_serial_state(q, k, v, g, grid_h, grid_w, direction, S0=None, *, slices=None, nthreads=None):
    """Serial recurrence from the initial state ``S0`` (``[B, heads, dk, dv]``,
    None for zero); returns ``(out, SN)`` with ``SN`` the state after the last
    token, ``[B, heads, dk, dv]``."""
    q, k, v, g = (_as_f64(x) for x in (q, k, v, g))
    B, N, heads, dk, dv = _shapes(q, v, grid_h, grid_w)
    s0 = None
    if S0 is not None:
        s0 = _as_f64(S0)
        if s0.shape != (B, heads, dk, dv):
            raise ValueError(f"S0 shape {s0.shape} != {(B, heads, dk, dv)}")
    out = np.zeros((B, N, heads, dv), dtype=np.float64)
    SN = np.zeros((B, heads, dk, dv), dtype=np.float64)
    keep, sp, ns = _slices_arg(slices)
    rc = _load().gla_oracle_serial_state(_ptr(q), _ptr(k), _ptr(v), _ptr(g), B, heads, grid_h, grid_w,
                                         dk, dv, _dir(direction), _ptr(s0), _ptr(out), _ptr(SN), sp, ns,
                                         nthreads or default_threads())
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    return out, SN


def output_gate(o, r, w, eps=1e-5):
    """``o / sqrt(mean(o**2) + eps) * w * silu(r)`` over the last axis (d_v)."""
    o, r, w = _as_f64(o), _as_f64(r), _as_f64(w)
    if o.shape != r.shape or w.shape != (o.shape[-1],):
        raise ValueError("shapes: o and r alike, w of length d_v")
    dv = o.shape[-1]
    y = np.zeros(o.shape, dtype=np.float64)
    _load().gla_oracle_output_gate(_ptr(o), _ptr(r), _ptr(w), float(eps), int(o.size // dv), dv, _ptr(y))
    return y


def sswiglu(a, b, wc, bias, grid_h, grid_w):
    """Spatial SwiGLU gating: ``silu(a) * (3x3 depthwise conv of b + bias)``
    on the ``grid_h x grid_w`` patch grid, zero padding; ``a``, ``b``:
    ``[B, N, C]``, ``wc``: ``[C, 3, 3]``, ``bias``: ``[C]`` or None."""
    a, b, wc = _as_f64(a), _as_f64(b), _as_f64(wc)
    B, N, C = a.shape
    if N != grid_h * grid_w or b.shape != a.shape or wc.shape != (C, 3, 3):
        raise ValueError("shapes")
    bb = None if bias is None else _as_f64(bias)
    y = np.zeros(a.shape, dtype=np.float64)
    _load().gla_oracle_sswiglu(_ptr(a), _ptr(b), _ptr(wc), _ptr(bb), B, grid_h, grid_w, C, _ptr(y))
    return y
