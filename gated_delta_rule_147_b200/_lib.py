"""ctypes binding of libgdr.so (include/gdr.h). Argument marshalling only.

The library is built in-tree by gated_delta_rule_147_b200/build.py. Loading
fails loudly when it is missing and cannot be built: there is no other path.
"""
from __future__ import annotations

import ctypes
import os
import threading

from . import build as _build

GDR_OK, GDR_ERR_INVALID_ARG, GDR_ERR_UNSUPPORTED, GDR_ERR_MISALIGNED, GDR_ERR_LAUNCH, \
    GDR_ERR_NO_DEVICE = range(6)
GDR_DEVICE_TIMEOUT, GDR_DEVICE_DECAY_RANGE = 1, 2
GDR_BF16, GDR_FP32 = 0, 1
GATE_NONE, GATE_SCALAR, GATE_CHANNEL, GATE_TIED = 0, 1, 2, 3

EXPORTS = ("gdr_chunk_fwd", "gdr_chunk_fwd_grouped", "gdr_chunk_fwd_workspace_size",
           "gdr_chunk_fwd_static", "gdr_chunk_fwd_static_capacity", "gdr_chunk_bwd",
           "gdr_chunk_bwd_workspace_size", "gdr_chunk_bwd_grouped",
           "gdr_chunk_bwd_grouped_workspace_size", "gdr_decode_step",
           "gdr_decode_step_grouped", "gdr_selftest_bounded_wait", "gdr_status_string",
           "gdr_version")

_lock = threading.Lock()
_handle = None


class GdrError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} returned {status_string(status)} ({status})")


def library_path() -> str:
    return _build.LIB


def load(build_if_missing: bool = True) -> ctypes.CDLL:
    global _handle
    with _lock:
        if _handle is not None:
            return _handle
        path = _build.LIB
        if build_if_missing and _build._stale():
            _build.build()
        if not os.path.exists(path):
            raise OSError(f"CUDA library {path} is missing; run python -m gated_delta_rule_147_b200.build")
        lib = ctypes.CDLL(path)
        vp, ip = ctypes.c_void_p, ctypes.c_int
        sz = ctypes.c_size_t
        lib.gdr_chunk_fwd.argtypes = [vp] * 6 + [ip] * 3 + [vp, vp, vp, vp, sz] + [ip] * 7 + [vp, vp]
        lib.gdr_chunk_fwd.restype = ip
        lib.gdr_chunk_fwd_grouped.argtypes = [vp] * 6 + [ip] * 3 + [vp, vp, vp, vp, sz] + [ip] * 8 + [vp, vp]
        lib.gdr_chunk_fwd_grouped.restype = ip
        lib.gdr_decode_step_grouped.argtypes = [vp] * 6 + [ip] * 3 + [vp, vp] + [ip] * 6 + [vp, vp]
        lib.gdr_decode_step_grouped.restype = ip
        lib.gdr_chunk_fwd_workspace_size.argtypes = [ip] * 9
        lib.gdr_chunk_fwd_workspace_size.restype = sz
        lib.gdr_chunk_fwd_static.argtypes = [vp] * 6 + [ip] * 3 + [vp, vp, vp] + [ip] * 7 + [vp, vp]
        lib.gdr_chunk_fwd_static.restype = ip
        lib.gdr_chunk_fwd_static_capacity.argtypes = []
        lib.gdr_chunk_fwd_static_capacity.restype = sz
        lib.gdr_chunk_bwd.argtypes = [vp] * 6 + [ip] * 3 + [vp] * 11 + [sz] + [ip] * 7 + [vp, vp]
        lib.gdr_chunk_bwd.restype = ip
        lib.gdr_chunk_bwd_workspace_size.argtypes = [ip] * 5
        lib.gdr_chunk_bwd_workspace_size.restype = sz
        lib.gdr_chunk_bwd_grouped.argtypes = [vp] * 6 + [ip] * 3 + [vp] * 11 + [sz] + [ip] * 8 + [vp, vp]
        lib.gdr_chunk_bwd_grouped.restype = ip
        lib.gdr_chunk_bwd_grouped_workspace_size.argtypes = [ip] * 6
        lib.gdr_chunk_bwd_grouped_workspace_size.restype = sz
        lib.gdr_decode_step.argtypes = [vp] * 6 + [ip] * 3 + [vp, vp] + [ip] * 5 + [vp, vp]
        lib.gdr_decode_step.restype = ip
        lib.gdr_status_string.argtypes = [ip]
        lib.gdr_status_string.restype = ctypes.c_char_p
        lib.gdr_version.restype = ip
        lib.gdr_selftest_bounded_wait.argtypes = [vp, vp]
        lib.gdr_selftest_bounded_wait.restype = ip
        _handle = lib
        return lib


def status_string(s: int) -> str:
    return load().gdr_status_string(int(s)).decode()


def _p(x):
    """Device pointer of a tensor (or a raw int address); None -> NULL."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


def gdr_chunk_fwd(q, k, v, alpha, b, w, alpha_kind, b_kind, w_kind, S0, o, S_T, workspace,
                  workspace_bytes, B, T, H, d_k, d_v, chunk, dtype, d_status=None,
                  stream=None) -> None:
    """Same arguments as the C entry point; tensors are passed by device pointer."""
    st = load().gdr_chunk_fwd(_p(q), _p(k), _p(v), _p(alpha), _p(b), _p(w), alpha_kind, b_kind,
                              w_kind, _p(S0), _p(o), _p(S_T), _p(workspace), int(workspace_bytes),
                              B, T, H, d_k, d_v, chunk, dtype, _p(d_status), _stream(stream))
    if st != GDR_OK:
        raise GdrError("gdr_chunk_fwd", st)


def gdr_chunk_fwd_grouped(q, k, v, alpha, b, w, alpha_kind, b_kind, w_kind, S0, o, S_T, workspace,
                          workspace_bytes, B, T, H_qk, H, d_k, d_v, chunk, dtype, d_status=None,
                          stream=None) -> None:
    st = load().gdr_chunk_fwd_grouped(_p(q), _p(k), _p(v), _p(alpha), _p(b), _p(w), alpha_kind,
                                      b_kind, w_kind, _p(S0), _p(o), _p(S_T), _p(workspace),
                                      int(workspace_bytes), B, T, H_qk, H, d_k, d_v, chunk, dtype,
                                      _p(d_status), _stream(stream))
    if st != GDR_OK:
        raise GdrError("gdr_chunk_fwd_grouped", st)


def gdr_decode_step_grouped(q, k, v, alpha, b, w, alpha_kind, b_kind, w_kind, S, o, B, H_qk, H,
                            d_k, d_v, dtype, d_status=None, stream=None) -> None:
    st = load().gdr_decode_step_grouped(_p(q), _p(k), _p(v), _p(alpha), _p(b), _p(w), alpha_kind,
                                        b_kind, w_kind, _p(S), _p(o), B, H_qk, H, d_k, d_v, dtype,
                                        _p(d_status), _stream(stream))
    if st != GDR_OK:
        raise GdrError("gdr_decode_step_grouped", st)


def gdr_chunk_fwd_static(q, k, v, alpha, b, w, alpha_kind, b_kind, w_kind, S0, o, S_T, B, T, H,
                         d_k, d_v, chunk, dtype, d_status=None, stream=None) -> None:
    """gdr_chunk_fwd with the library's own scratch array (no workspace argument)."""
    st = load().gdr_chunk_fwd_static(_p(q), _p(k), _p(v), _p(alpha), _p(b), _p(w), alpha_kind,
                                     b_kind, w_kind, _p(S0), _p(o), _p(S_T), B, T, H, d_k, d_v,
                                     chunk, dtype, _p(d_status), _stream(stream))
    if st != GDR_OK:
        raise GdrError("gdr_chunk_fwd_static", st)


def gdr_chunk_fwd_static_capacity() -> int:
    return int(load().gdr_chunk_fwd_static_capacity())


def gdr_chunk_fwd_workspace_size(B, T, H, d_k, d_v, alpha_kind, b_kind, w_kind, dtype) -> int:
    return int(load().gdr_chunk_fwd_workspace_size(B, T, H, d_k, d_v, alpha_kind, b_kind, w_kind,
                                                   dtype))


def gdr_chunk_bwd(q, k, v, alpha, b, w, alpha_kind, b_kind, w_kind, S0, dO, dS_T, dq, dk, dv, dalpha,
                  db, dw, dS0, workspace, workspace_bytes, B, T, H, d_k, d_v, chunk, dtype,
                  d_status=None, stream=None) -> None:
    st = load().gdr_chunk_bwd(_p(q), _p(k), _p(v), _p(alpha), _p(b), _p(w), alpha_kind, b_kind,
                              w_kind, _p(S0), _p(dO), _p(dS_T), _p(dq), _p(dk), _p(dv), _p(dalpha),
                              _p(db), _p(dw), _p(dS0), _p(workspace), int(workspace_bytes), B, T, H,
                              d_k, d_v, chunk, dtype, _p(d_status), _stream(stream))
    if st != GDR_OK:
        raise GdrError("gdr_chunk_bwd", st)


def gdr_chunk_bwd_workspace_size(B, T, H, d_k, d_v) -> int:
    return int(load().gdr_chunk_bwd_workspace_size(B, T, H, d_k, d_v))


def gdr_chunk_bwd_grouped(q, k, v, alpha, b, w, alpha_kind, b_kind, w_kind, S0, dO, dS_T, dq, dk, dv,
                          dalpha, db, dw, dS0, workspace, workspace_bytes, B, T, H_qk, H, d_k, d_v,
                          chunk, dtype, d_status=None, stream=None) -> None:
    st = load().gdr_chunk_bwd_grouped(_p(q), _p(k), _p(v), _p(alpha), _p(b), _p(w), alpha_kind,
                                      b_kind, w_kind, _p(S0), _p(dO), _p(dS_T), _p(dq), _p(dk),
                                      _p(dv), _p(dalpha), _p(db), _p(dw), _p(dS0), _p(workspace),
                                      int(workspace_bytes), B, T, H_qk, H, d_k, d_v, chunk, dtype,
                                      _p(d_status), _stream(stream))
    if st != GDR_OK:
        raise GdrError("gdr_chunk_bwd_grouped", st)


def gdr_chunk_bwd_grouped_workspace_size(B, T, H_qk, H, d_k, d_v) -> int:
    return int(load().gdr_chunk_bwd_grouped_workspace_size(B, T, H_qk, H, d_k, d_v))


def gdr_decode_step(q, k, v, alpha, b, w, alpha_kind, b_kind, w_kind, S, o, B, H, d_k, d_v, dtype,
                    d_status=None, stream=None) -> None:
    st = load().gdr_decode_step(_p(q), _p(k), _p(v), _p(alpha), _p(b), _p(w), alpha_kind, b_kind,
                                w_kind, _p(S), _p(o), B, H, d_k, d_v, dtype, _p(d_status),
                                _stream(stream))
    if st != GDR_OK:
        raise GdrError("gdr_decode_step", st)


def gdr_selftest_bounded_wait(d_status, stream=None) -> None:
    st = load().gdr_selftest_bounded_wait(_p(d_status), _stream(stream))
    if st != GDR_OK:
        raise GdrError("gdr_selftest_bounded_wait", st)
