"""ctypes binding of libgtr_gla.so (the C ABI in include/gtr_gla.h).

Argument marshalling only: every step of the GLA forward runs in the CUDA
library.  Functions named ``gtr_gla_*`` mirror the C entry points one to one
and accept torch tensors (their ``data_ptr()`` is passed) or raw integer
addresses; a ``stream`` argument may be a ``torch.cuda.Stream``, a raw
``cudaStream_t`` integer, or None for torch's current stream.  Each returns
the integer status; :func:`check` turns a non-zero status into
:class:`GtrError`.  :func:`forward` is the tensor-level convenience call.

The library must be built (``python -m recurrent_vision_backbone_key_b200.build``);
loading fails loudly otherwise -- there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgtr_gla.so")
CHECKED_LIB_PATH = os.path.join(_PKG, "libgtr_gla_checked.so")  # bounds-checked debug build

GTR_OK = 0
STATUS_NAMES = {
    0: "GTR_OK", 1: "GTR_ERR_INVALID_ARG", 2: "GTR_ERR_UNSUPPORTED_SHAPE",
    3: "GTR_ERR_MISALIGNED", 4: "GTR_ERR_ALIAS", 5: "GTR_ERR_CUDA", 6: "GTR_ERR_TIMEOUT",
    7: "GTR_ERR_OOM",
}
DIRECTIONS = {"l2r": 0, "r2l": 1, "t2b": 2, "b2t": 3}
SCHEDULES = {"auto": 0, "fused": 1, "three_phase": 2, "three_phase_simt": 3, "fused_tcgen05": 4,
             "walk_tcgen05": 5, "three_phase_mma": 6}

# Every symbol include/gtr_gla.h declares, with (restype, argtypes).
_P = ctypes.c_void_p
_I = ctypes.c_int
SIGNATURES = {
    "gtr_gla_forward": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _P, _P]),
    "gtr_gla_forward_ex": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _I, _P, _P]),
    "gtr_gla_forward_host": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _P, _P]),
    "gtr_gla_forward_noalloc": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _P, _P]),
    "gtr_gla_forward_bf16": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _P, _P]),
    "gtr_gla_forward_state": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _P, _P, _P]),
    "gtr_gla_forward_gated": (_I, [_P, _P, _P, _P, _P, _P, ctypes.c_float, _I, _I, _I, _I, _I, _I, _I, _I,
                                   _P, _P]),
    "gtr_sswiglu_forward": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _P, _P]),
    "gtr_gla_chunk_summary": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _P, _P, _P]),
    "gtr_gla_boundary_scan": (_I, [_P, _P, _I, _I, _I, _I, _I, _P, _P]),
    "gtr_gla_chunk_output": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _P, _P]),
    "gtr_gla_workspace_bytes": (ctypes.c_size_t, [_I, _I, _I, _I, _I, _I, _I]),
    "gtr_gla_workspace_bytes_ex": (ctypes.c_size_t, [_I, _I, _I, _I, _I, _I, _I, _I]),
    "gtr_gla_get_last_device_status": (_I, [_P]),
    "gtr_gla_debug_forward_fused": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _I, _I, _I,
                                         ctypes.c_longlong, _P, _P]),
    "gtr_gla_release_workspace": (_I, []),
    "gtr_gla_status_string": (ctypes.c_char_p, [_I]),
    "gtr_gla_last_error": (ctypes.c_char_p, []),
    "gtr_gla_launch_count": (ctypes.c_uint64, []),
    "gtr_gla_version": (_I, []),
    "gtr_gla_plan": (_I, [_I, _I, _I, _I, _I, _I, _I, _I, _I]),
    "gtr_gla_bounds_checked": (_I, []),
    "gtr_gla_debug_bounds_report": (_I, [ctypes.POINTER(ctypes.c_ulonglong), ctypes.POINTER(ctypes.c_int),
                                         ctypes.POINTER(ctypes.c_longlong), ctypes.POINTER(ctypes.c_longlong),
                                         _I]),
}

_lib = None


class GtrError(RuntimeError):
    def __init__(self, status: int, message: str):
        self.status = status
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")


def _open(path: str) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise RuntimeError(
            f"{path} is missing: build it with `python -m recurrent_vision_backbone_key_b200.build`"
            " (no CPU fallback exists)")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the CUDA library (once).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        _lib = _open(path)
    return _lib


_lib_checked = None


def load_checked(path: str = CHECKED_LIB_PATH) -> ctypes.CDLL:
    """Load the bounds-checked debug build (once), a separate library with the
    same C ABI.  Raises if it has not been built."""
    global _lib_checked
    if _lib_checked is None:
        _lib_checked = _open(path)
    return _lib_checked


def bounds_report(lib: ctypes.CDLL, clear: bool = True):
    """(count, site, index, limit) of the accesses a checked build skipped."""
    cnt, site = ctypes.c_ulonglong(0), ctypes.c_int(0)
    idx, lim = ctypes.c_longlong(0), ctypes.c_longlong(0)
    check(lib.gtr_gla_debug_bounds_report(ctypes.byref(cnt), ctypes.byref(site), ctypes.byref(idx),
                                          ctypes.byref(lim), int(clear)))
    return cnt.value, site.value, idx.value, lim.value


def _addr(x):
    if x is None:
        return None
    if isinstance(x, torch.Tensor):
        return x.data_ptr()
    return int(x)


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _dir(d):
    return DIRECTIONS[d] if isinstance(d, str) else int(d)


def last_error() -> str:
    return load().gtr_gla_last_error().decode()


def check(status: int) -> int:
    if status != GTR_OK:
        raise GtrError(status, last_error())
    return status


def gtr_gla_forward(q, k, v, g, B, heads, grid_h, grid_w, d_k, d_v, direction, chunk, out,
                    stream=None) -> int:
    return load().gtr_gla_forward(_addr(q), _addr(k), _addr(v), _addr(g), B, heads, grid_h, grid_w,
                                  d_k, d_v, _dir(direction), chunk, _addr(out), _stream(stream))


def gtr_gla_forward_ex(q, k, v, g, B, heads, grid_h, grid_w, d_k, d_v, direction, chunk, schedule,
                       out, stream=None) -> int:
    sched = SCHEDULES[schedule] if isinstance(schedule, str) else int(schedule)
    return load().gtr_gla_forward_ex(_addr(q), _addr(k), _addr(v), _addr(g), B, heads, grid_h,
                                     grid_w, d_k, d_v, _dir(direction), chunk, sched, _addr(out),
                                     _stream(stream))


def gtr_gla_forward_host(q, k, v, g, B, heads, grid_h, grid_w, d_k, d_v, direction, chunk, out,
                         stream=None) -> int:
    return load().gtr_gla_forward_host(_addr(q), _addr(k), _addr(v), _addr(g), B, heads, grid_h,
                                       grid_w, d_k, d_v, _dir(direction), chunk, _addr(out),
                                       _stream(stream))


def gtr_gla_forward_noalloc(q, k, v, g, B, heads, grid_h, grid_w, d_k, d_v, direction, chunk, out,
                            stream=None) -> int:
    return load().gtr_gla_forward_noalloc(_addr(q), _addr(k), _addr(v), _addr(g), B, heads, grid_h,
                                          grid_w, d_k, d_v, _dir(direction), chunk, _addr(out),
                                          _stream(stream))


def gtr_gla_forward_bf16(q, k, v, g, B, heads, grid_h, grid_w, d_k, d_v, direction, chunk, out,
                         stream=None) -> int:
    return load().gtr_gla_forward_bf16(_addr(q), _addr(k), _addr(v), _addr(g), B, heads, grid_h, grid_w,
                                       d_k, d_v, _dir(direction), chunk, _addr(out), _stream(stream))


def gtr_gla_forward_state(q, k, v, g, S0, B, heads, grid_h, grid_w, d_k, d_v, direction, chunk, out,
                          SN, stream=None) -> int:
    return load().gtr_gla_forward_state(_addr(q), _addr(k), _addr(v), _addr(g), _addr(S0), B, heads,
                                        grid_h, grid_w, d_k, d_v, _dir(direction), chunk, _addr(out),
                                        _addr(SN), _stream(stream))


def gtr_gla_forward_gated(q, k, v, g, gate, norm_weight, norm_eps, B, heads, grid_h, grid_w, d_k, d_v,
                          direction, chunk, out, stream=None) -> int:
    return load().gtr_gla_forward_gated(_addr(q), _addr(k), _addr(v), _addr(g), _addr(gate),
                                        _addr(norm_weight), float(norm_eps), B, heads, grid_h, grid_w,
                                        d_k, d_v, _dir(direction), chunk, _addr(out), _stream(stream))


def gtr_sswiglu_forward(a, v, w, bias, B, grid_h, grid_w, C, out, stream=None) -> int:
    return load().gtr_sswiglu_forward(_addr(a), _addr(v), _addr(w), _addr(bias), B, grid_h, grid_w, C,
                                      _addr(out), _stream(stream))


def gtr_gla_chunk_summary(k, v, g, B, heads, grid_h, grid_w, d_k, d_v, direction, chunk, dS, gamma,
                          stream=None) -> int:
    return load().gtr_gla_chunk_summary(_addr(k), _addr(v), _addr(g), B, heads, grid_h, grid_w,
                                        d_k, d_v, _dir(direction), chunk, _addr(dS), _addr(gamma),
                                        _stream(stream))


def gtr_gla_boundary_scan(dS, gamma, B, heads, n_chunks, d_k, d_v, S_enter, stream=None) -> int:
    return load().gtr_gla_boundary_scan(_addr(dS), _addr(gamma), B, heads, n_chunks, d_k, d_v,
                                        _addr(S_enter), _stream(stream))


def gtr_gla_chunk_output(q, k, v, g, S_enter, B, heads, grid_h, grid_w, d_k, d_v, direction, chunk,
                         out, stream=None) -> int:
    return load().gtr_gla_chunk_output(_addr(q), _addr(k), _addr(v), _addr(g), _addr(S_enter), B,
                                       heads, grid_h, grid_w, d_k, d_v, _dir(direction), chunk,
                                       _addr(out), _stream(stream))


def gtr_gla_workspace_bytes(B, heads, grid_h, grid_w, d_k, d_v, chunk) -> int:
    return int(load().gtr_gla_workspace_bytes(B, heads, grid_h, grid_w, d_k, d_v, chunk))


def gtr_gla_workspace_bytes_ex(B, heads, grid_h, grid_w, d_k, d_v, chunk, schedule) -> int:
    sched = SCHEDULES[schedule] if isinstance(schedule, str) else int(schedule)
    return int(load().gtr_gla_workspace_bytes_ex(B, heads, grid_h, grid_w, d_k, d_v, chunk, sched))


def gtr_gla_get_last_device_status(stream=None) -> int:
    return load().gtr_gla_get_last_device_status(_stream(stream))


def gtr_gla_debug_forward_fused(q, k, v, g, B, heads, grid_h, grid_w, d_k, d_v, direction, chunk,
                                schedule, hold_seq, hold_chunk, spin_limit, out, stream=None) -> int:
    sched = SCHEDULES[schedule] if isinstance(schedule, str) else int(schedule)
    return load().gtr_gla_debug_forward_fused(_addr(q), _addr(k), _addr(v), _addr(g), B, heads,
                                              grid_h, grid_w, d_k, d_v, _dir(direction), chunk,
                                              sched, hold_seq, hold_chunk, spin_limit, _addr(out),
                                              _stream(stream))


def gtr_gla_release_workspace() -> int:
    return load().gtr_gla_release_workspace()


def gtr_gla_status_string(status: int) -> str:
    return load().gtr_gla_status_string(status).decode()


def gtr_gla_launch_count() -> int:
    return int(load().gtr_gla_launch_count())


PLANS = {0: "three_phase", 1: "three_phase_simt", 2: "fused_mma", 3: "fused_mma_pair", 4: "fused_tcgen05",
         5: "walk_tcgen05", 6: "three_phase_mma"}


def gtr_gla_plan(B, heads, grid_h, grid_w, d_k, d_v, chunk, schedule, sm_count) -> int:
    sched = SCHEDULES[schedule] if isinstance(schedule, str) else int(schedule)
    return int(load().gtr_gla_plan(B, heads, grid_h, grid_w, d_k, d_v, chunk, sched, sm_count))


def gtr_gla_version() -> int:
    return int(load().gtr_gla_version())


def forward(q, k, v, g, grid_h, grid_w, direction=0, chunk=64, schedule=0, out=None, stream=None):
    """Tensor-level GLA forward: shapes taken from q [B,N,heads,d_k] and
    v [B,N,heads,d_v]; allocates ``out`` if not given; raises GtrError."""
    B, N, heads, d_k = q.shape
    d_v = v.shape[3]
    if out is None:
        out = torch.empty((B, N, heads, d_v), dtype=torch.float16, device=v.device)
    check(gtr_gla_forward_ex(q, k, v, g, B, heads, grid_h, grid_w, d_k, d_v, direction, chunk,
                             schedule, out, stream))
    return out
