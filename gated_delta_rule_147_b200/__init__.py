"""B200-native gated delta-rule linear attention.

    S_t = (I - k_t^T (b_t . k_t)) Diag(alpha_t) S_{t-1} + (w_t . k_t)^T v_t,
    o_t = q_t S_t

Entry points (CUDA, sm_100a, through the C ABI in include/gdr.h):
  gdr_chunk_fwd / chunk_fwd     whole-sequence forward, chunkwise on tcgen05
  gdr_chunk_bwd / chunk_bwd     its backward pass (gradients of every input)
  gdr_decode_step / decode_step one token per head, state updated in place

torch is used for device memory and streams only; every step of the
recurrence runs in the library's kernels. Importing this package does not
load the library; the first call does (and fails loudly if it cannot).
"""
from __future__ import annotations

from ._lib import (GATE_CHANNEL, GATE_NONE, GATE_SCALAR, GATE_TIED, GDR_BF16, GDR_FP32,
                   GDR_DEVICE_DECAY_RANGE, GDR_DEVICE_TIMEOUT, GdrError, gdr_chunk_bwd,
                   gdr_chunk_bwd_grouped, gdr_chunk_bwd_grouped_workspace_size,
                   gdr_chunk_bwd_workspace_size, gdr_chunk_fwd, gdr_chunk_fwd_grouped, gdr_chunk_fwd_static, gdr_chunk_fwd_workspace_size,
                   gdr_decode_step, gdr_decode_step_grouped, load)

TIED = "tied"
_KIND = {"none": GATE_NONE, "scalar": GATE_SCALAR, "channel": GATE_CHANNEL, "tied": GATE_TIED}


def _dtype_code(t):
    import torch
    if t.dtype == torch.bfloat16:
        return GDR_BF16
    if t.dtype == torch.float32:
        return GDR_FP32
    raise TypeError(f"unsupported dtype {t.dtype}; use bfloat16 or float32")


def _check(*ts):
    for t in ts:
        if t is not None and not isinstance(t, str) and not t.is_contiguous():
            raise ValueError("tensors passed to the library must be contiguous")


def _check_types(ref, same=(), fp32=()):
    """The library reads raw device pointers with one element type: `ref` (q)
    and every (name, tensor) in `same` share q's dtype, every one in `fp32` is
    float32, and all live on one CUDA device. Raised before any call."""
    import torch
    _dtype_code(ref)
    tensors = [(n, t) for n, t in list(same) + list(fp32) if t is not None and not isinstance(t, str)]
    for name, t in same:
        if t is not None and not isinstance(t, str) and t.dtype != ref.dtype:
            raise TypeError(f"{name} has dtype {t.dtype}; expected {ref.dtype} like q")
    for name, t in fp32:
        if t is not None and t.dtype != torch.float32:
            raise TypeError(f"{name} has dtype {t.dtype}; the state is float32")
    if ref.device.type != "cuda":
        raise ValueError(f"q is on {ref.device}; the library takes CUDA tensors")
    for name, t in tensors:
        if t.device != ref.device:
            raise ValueError(f"{name} is on {t.device}; expected {ref.device} like q")


def _gate_kind(g, ndim_scalar: int):
    if g is None:
        return GATE_NONE
    if isinstance(g, str):
        if g != TIED:
            raise ValueError(g)
        return GATE_TIED
    return GATE_SCALAR if g.dim() == ndim_scalar else GATE_CHANNEL


def workspace_bytes(q, v, alpha=None, b=None, w=None) -> int:
    """Scratch bytes the two-pass chunk path wants for these inputs (0 when
    the shape / gate form has no two-pass path)."""
    B, T, _, dk = q.shape
    H = v.shape[2]
    return gdr_chunk_fwd_workspace_size(B, T, H, dk, v.shape[-1], _gate_kind(alpha, 3),
                                        _gate_kind(b, 3), _gate_kind(w, 3), _dtype_code(q))


def chunk_fwd(q, k, v, alpha=None, b=None, w=None, S0=None, *, out=None, final_state=True,
              S_T=None, chunk: int = 64, workspace="auto", d_status=None, stream=None):
    """Forward over [B,T,H,*] inputs. alpha/b/w: None, a [B,T,H] tensor
    (scalar gate), a [B,T,H,d_k] tensor (channel gate); w may be TIED (w := b).
    q and k may have fewer heads than v (grouped heads: H a multiple of
    H_qk, value head h reads q/k head h // (H // H_qk)).
    workspace: "auto" allocates the two-pass path's scratch with torch when
    the inputs have such a path; a uint8 device tensor supplies it; "static"
    uses the library's own scratch array (gdr_chunk_fwd_static); None runs
    the single-pass kernels. Returns (o, S_T) with S_T None when final_state
    is False."""
    import torch
    _check(q, k, v, alpha, b, w, S0, out, S_T)
    _check_types(q, [("k", k), ("v", v), ("alpha", alpha), ("b", b), ("w", w), ("out", out)],
                 [("S0", S0), ("S_T", S_T)])
    B, T, Hq, dk = q.shape
    H, dv = v.shape[2], v.shape[-1]
    o = out if out is not None else torch.empty((B, T, H, dv), dtype=v.dtype, device=v.device)
    if final_state and S_T is None:
        S_T = torch.empty((B, H, dk, dv), dtype=torch.float32, device=v.device)
    if isinstance(workspace, str) and workspace == "static":
        if Hq != H:
            raise ValueError("the static-scratch call takes ungrouped heads")
        gdr_chunk_fwd_static(q, k, v, alpha, b, None if isinstance(w, str) else w,
                             _gate_kind(alpha, 3), _gate_kind(b, 3), _gate_kind(w, 3), S0, o,
                             S_T if final_state else None, B, T, H, dk, dv, chunk, _dtype_code(q),
                             d_status, stream)
        return o, (S_T if final_state else None)
    if isinstance(workspace, str):
        if workspace != "auto":
            raise ValueError(workspace)
        nbytes = workspace_bytes(q, v, alpha, b, w)
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=v.device) if nbytes else None
    if workspace is not None and workspace.device != q.device:
        raise ValueError(f"workspace is on {workspace.device}; expected {q.device} like q")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    gdr_chunk_fwd_grouped(q, k, v, alpha, b, None if isinstance(w, str) else w,
                          _gate_kind(alpha, 3), _gate_kind(b, 3), _gate_kind(w, 3), S0, o,
                          S_T if final_state else None, workspace, ws_bytes, B, T, Hq, H, dk, dv,
                          chunk, _dtype_code(q), d_status, stream)
    return o, (S_T if final_state else None)


def chunk_bwd(q, k, v, alpha=None, b=None, w=None, S0=None, *, dO, dS_T=None, chunk: int = 64,
              workspace=None, need_dS0: bool = True, d_status=None, stream=None):
    """Backward of chunk_fwd for the same inputs: returns a dict with dq, dk,
    dv, dalpha, db, dw (None for an absent or tied gate) and dS0 (None when
    need_dS0 is False), all fp32. q and k may have fewer heads than v
    (grouped heads, as in chunk_fwd; dq and dk then sum over each group). dO has v's shape and dtype; dS_T is the
    gradient of the final state (None = 0). workspace: None allocates the
    chunk-checkpoint scratch with torch, or a uint8 device tensor of at least
    gdr_chunk_bwd_grouped_workspace_size bytes. d_status: optional int32
    device tensor the bounded waits of the tensor-core kernel OR their
    timeout flag into."""
    import torch
    _check(q, k, v, alpha, b, w, S0, dO, dS_T)
    _check_types(q, [("k", k), ("v", v), ("alpha", alpha), ("b", b), ("w", w), ("dO", dO)],
                 [("S0", S0), ("dS_T", dS_T)])
    B, T, Hq, dk = q.shape
    H, dv = v.shape[2], v.shape[-1]
    dev = v.device
    f32 = dict(dtype=torch.float32, device=dev)
    grads = {"dq": torch.empty((B, T, Hq, dk), **f32), "dk": torch.empty((B, T, Hq, dk), **f32),
             "dv": torch.empty((B, T, H, dv), **f32),
             "dS0": torch.empty((B, H, dk, dv), **f32) if need_dS0 else None}
    for name, g in (("dalpha", alpha), ("db", b), ("dw", w)):
        grads[name] = None if g is None or isinstance(g, str) else torch.empty(g.shape, **f32)
    if workspace is None:
        nbytes = gdr_chunk_bwd_grouped_workspace_size(B, T, Hq, H, dk, dv)
        workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=dev)
    if workspace.device != q.device:
        raise ValueError(f"workspace is on {workspace.device}; expected {q.device} like q")
    ws_bytes = workspace.numel() * workspace.element_size()
    gdr_chunk_bwd_grouped(q, k, v, alpha, b, None if isinstance(w, str) else w,
                          _gate_kind(alpha, 3), _gate_kind(b, 3), _gate_kind(w, 3), S0, dO, dS_T,
                          grads["dq"], grads["dk"], grads["dv"], grads["dalpha"], grads["db"],
                          grads["dw"], grads["dS0"], workspace, ws_bytes, B, T, Hq, H, dk, dv, chunk,
                          _dtype_code(q), d_status, stream)
    return grads


def decode_step(q, k, v, alpha, b, w, S, *, out=None, d_status=None, stream=None):
    """One token per head: q,k [B,H,d_k]; v [B,H,d_v]; gates [B,H] or
    [B,H,d_k] (w may be TIED); S [B,H,d_k,d_v] fp32 updated in place.
    Returns o [B,H,d_v]."""
    import torch
    _check(q, k, v, alpha, b, w, S, out)
    _check_types(q, [("k", k), ("v", v), ("alpha", alpha), ("b", b), ("w", w), ("out", out)],
                 [("S", S)])
    B, Hq, dk = q.shape
    H, dv = v.shape[1], v.shape[-1]
    o = out if out is not None else torch.empty((B, H, dv), dtype=v.dtype, device=v.device)
    gdr_decode_step_grouped(q, k, v, alpha, b, None if isinstance(w, str) else w,
                            _gate_kind(alpha, 2), _gate_kind(b, 2), _gate_kind(w, 2), S, o, B, Hq,
                            H, dk, dv, _dtype_code(q), d_status, stream)
    return o
