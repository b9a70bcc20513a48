"""CPU oracle for the gated delta-rule recurrence -- TEST INFRASTRUCTURE ONLY.

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may
import this package. It shares no code with the CUDA path
(gated_delta_rule_147_b200/); the only module both sides use is the seeded
input generator gated_delta_rule_147_b200.inputs, which holds none of the
recurrence's arithmetic.

Every route computes, per head, in fp64, on inputs already rounded to the
device dtype and then widened:

    S_t = (I - k_t^T (b_t . k_t)) Diag(alpha_t) S_{t-1} + (w_t . k_t)^T v_t
    o_t = q_t S_t

Routes (each follows a different passage, so they pin each other):
  recurrence            C token loop (gdr_oracle.c), the oracle proper.
  recurrence_bwd        its reverse-mode gradient (C, all states kept),
                        pinned by finite differences of `recurrence` and by
                        the linear-attention closed form.
  chunkwise_bwd         the same gradients per chunk as masked matrix
                        products (numpy, small cases), from the per-token
                        erase reads r_t and their gradients dr_t.
  recurrence_py         the same definition as a numpy token loop (small cases).
  unrolled_contributions  S_t = sum_i C_i^(t) with explicit d_k x d_k
                        transition matrices ("How Linear Attention Remembers",
                        Analytical Framework).
  masked_matrix         erase-free case b = 0 as a structured masked matrix
                        ("The Eraser Trilogy", "The Rosetta Stone").
  delta_three_line      tied gates b = w = beta written as read / delta /
                        write-back ("Recurrent Memory: Write, Erase, Decay,
                        Read", section 03) with decay (section 04).
  unified_decay_after_erase  the section-05 unified equation with decay applied
                        after the erase (the page's own order).

Parity: every route is pinned by the tests in tests/test_oracle_pins.py.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdr_oracle.c")
_SO = os.path.join(_HERE, "libgdr_oracle.so")
_lock = threading.Lock()
_lib_handle = None


def build(force: bool = False) -> str:
    """Compile the C oracle into oracle/libgdr_oracle.so (gcc, OpenMP)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", _SO, _SRC]
        subprocess.run(cmd, check=True)
    return _SO


def _lib():
    global _lib_handle
    with _lock:
        if _lib_handle is None:
            build()
            _lib_handle = load_library(_SO)
        return _lib_handle


def max_threads() -> int:
    return int(_lib().gdr_oracle_max_threads())


def f64(x):
    """Widen a torch tensor or numpy array (any float dtype) to contiguous fp64 numpy."""
    if x is None:
        return None
    if hasattr(x, "detach"):
        x = x.detach().to("cpu")
        import torch
        x = x.to(torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _resolve_gates(alpha, b, w, gates):
    """Returns (alpha, alpha_pc, b, b_pc, w, w_pc) with 'tied' resolved to w := b."""
    g = dict(gates or {})
    ka, kb, kw = g.get("alpha", "none"), g.get("b", "none"), g.get("w", "none")
    alpha = None if ka == "none" else f64(alpha)
    b = None if kb == "none" else f64(b)
    if kw == "tied":
        w, kw = b, kb
    else:
        w = None if kw == "none" else f64(w)
    return alpha, int(ka == "channel"), b, int(kb == "channel"), w, int(kw == "channel")


def load_library(path: str):
    """Load another build of gdr_oracle.c (tests compile deliberately broken
    copies to check that the pins catch each mistake)."""
    lib = ctypes.CDLL(path)
    dp = ctypes.POINTER(ctypes.c_double)
    lib.gdr_oracle_forward.argtypes = [ctypes.c_int] * 5 + [dp, dp, dp, dp, ctypes.c_int,
                                                            dp, ctypes.c_int, dp, ctypes.c_int,
                                                            dp, dp, dp, ctypes.c_int]
    lib.gdr_oracle_forward.restype = ctypes.c_int
    lib.gdr_oracle_backward.argtypes = [ctypes.c_int] * 5 + [dp, dp, dp, dp, ctypes.c_int,
                                                             dp, ctypes.c_int, dp, ctypes.c_int,
                                                             dp, dp, dp, dp, dp, dp, dp, dp, dp, dp,
                                                             ctypes.c_int]
    lib.gdr_oracle_backward.restype = ctypes.c_int
    lib.gdr_oracle_max_threads.restype = ctypes.c_int
    return lib


def recurrence(q, k, v, alpha=None, b=None, w=None, S0=None, gates=None, nthreads: int = 0,
               lib=None):
    """Token-by-token recurrence (the C oracle). Returns (o, S_T) in fp64.

    q,k [B,T,H,dk]; v [B,T,H,dv]; gates scalar [B,T,H] or channel [B,T,H,dk];
    S0 [B,H,dk,dv] or None. gates = {"alpha": kind, "b": kind, "w": kind},
    kinds "none" (alpha=1, b=0, w=1), "scalar", "channel", and for w "tied".
    """
    q, k, v = f64(q), f64(k), f64(v)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    a, apc, bb, bpc, ww, wpc = _resolve_gates(alpha, b, w, gates)
    S0 = f64(S0)
    o = np.zeros((B, T, H, dv), dtype=np.float64)
    S_T = np.zeros((B, H, dk, dv), dtype=np.float64)
    rc = (lib or _lib()).gdr_oracle_forward(B, T, H, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(a), apc,
                                   _ptr(bb), bpc, _ptr(ww), wpc, _ptr(S0), _ptr(o), _ptr(S_T),
                                   int(nthreads))
    if rc != 0:
        raise RuntimeError(f"gdr_oracle_forward returned {rc}")
    return o, S_T


def recurrence_bwd(q, k, v, alpha=None, b=None, w=None, S0=None, gates=None, dO=None, dS_T=None,
                   nthreads: int = 0, lib=None):
    """Gradients of L = sum(o * dO) + sum(S_T * dS_T) with respect to every
    input of `recurrence` (the C oracle's reverse-mode token loop), in fp64.

    Returns a dict: dq, dk [B,T,H,dk]; dv [B,T,H,dv]; dalpha, db, dw shaped like
    their gates (None for an absent gate; with w "tied", db holds the whole
    gradient of the shared beta and dw is None); dS0 [B,H,dk,dv] (the gradient
    with respect to the initial state, zero-state runs included).
    """
    q, k, v = f64(q), f64(k), f64(v)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    g = dict(gates or {})
    tied = g.get("w") == "tied"
    a, apc, bb, bpc, ww, wpc = _resolve_gates(alpha, b, w, gates)
    S0, dO, dS_T = f64(S0), f64(dO), f64(dS_T)
    gshape = lambda pc: (B, T, H, dk) if pc else (B, T, H)
    out = {"dq": np.zeros((B, T, H, dk)), "dk": np.zeros((B, T, H, dk)),
           "dv": np.zeros((B, T, H, dv)), "dS0": np.zeros((B, H, dk, dv))}
    da = None if a is None else np.zeros(gshape(apc))
    dbb = None if bb is None else np.zeros(gshape(bpc))
    dww = None if ww is None else np.zeros(gshape(wpc))
    rc = (lib or _lib()).gdr_oracle_backward(
        B, T, H, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(a), apc, _ptr(bb), bpc, _ptr(ww), wpc,
        _ptr(S0), _ptr(dO), _ptr(dS_T), _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]),
        _ptr(da), _ptr(dbb), _ptr(dww), _ptr(out["dS0"]), int(nthreads))
    if rc != 0:
        raise RuntimeError(f"gdr_oracle_backward returned {rc}")
    if tied:
        dbb, dww = dbb + dww, None
    out.update(dalpha=da, db=dbb, dw=dww)
    return out


def decode_step(q, k, v, alpha, b, w, S, gates=None, nthreads: int = 0):
    """One decode token per head: the recurrence with T = 1 and the state
    carried between calls. q,k [B,H,dk]; v [B,H,dv]; gates [B,H] or [B,H,dk];
    S [B,H,dk,dv]. Returns (o [B,H,dv], S_new)."""
    q, k, v = f64(q)[:, None], f64(k)[:, None], f64(v)[:, None]
    ex = lambda g: None if g is None else f64(g)[:, None]
    o, S_new = recurrence(q, k, v, ex(alpha), ex(b), ex(w), f64(S), gates, nthreads)
    return o[:, 0], S_new


# ---------------------------------------------------------------------------
# Independent routes used to pin the oracle (small inputs only).
# ---------------------------------------------------------------------------

def _full_gates(alpha, b, w, gates, B, T, H, dk):
    """Materialise all three gates as [B,T,H,dk] fp64 arrays (broadcasting only)."""
    a, apc, bb, bpc, ww, wpc = _resolve_gates(alpha, b, w, gates)

    def full(g, pc, dflt):
        if g is None:
            return np.full((B, T, H, dk), dflt)
        return np.broadcast_to(g if pc else g[..., None], (B, T, H, dk)).copy()
    return full(a, apc, 1.0), full(bb, bpc, 0.0), full(ww, wpc, 1.0)


def recurrence_py(q, k, v, alpha=None, b=None, w=None, S0=None, gates=None):
    """The definition again, as a numpy token loop (spec form:
    decay, then erase read with b.k, erase along k, write with key w.k)."""
    q, k, v = f64(q), f64(k), f64(v)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    A, Bg, W = _full_gates(alpha, b, w, gates, B, T, H, dk)
    S0 = f64(S0)
    o = np.zeros((B, T, H, dv))
    ST = np.zeros((B, H, dk, dv))
    for bi in range(B):
        for h in range(H):
            S = np.zeros((dk, dv)) if S0 is None else S0[bi, h].copy()
            for t in range(T):
                kt = k[bi, t, h]
                S = A[bi, t, h][:, None] * S
                r = (Bg[bi, t, h] * kt) @ S
                S = S - np.outer(kt, r) + np.outer(W[bi, t, h] * kt, v[bi, t, h])
                o[bi, t, h] = q[bi, t, h] @ S
            ST[bi, h] = S
    return o, ST


def unrolled_contributions(q, k, v, alpha=None, b=None, w=None, S0=None, gates=None):
    """State as a sum of per-position contributions ("How Linear Attention
    Remembers", Analytical Framework): S_t = T_t(S_{t-1}) + W_t with the
    linear map T_t(S) = M_t S, M_t = (I - k_t^T (b_t . k_t)) Diag(alpha_t)
    materialised as a d_k x d_k matrix, and the write W_t = (w_t . k_t)^T v_t.
    Then S_t = P_{t,0} S0 + sum_{i<=t} C_i^(t), C_i^(t) = P_{t,i} W_i with
    P_{t,i} = M_t M_{t-1} ... M_{i+1} (the product of transitions after i).
    o_t = q_t S_t. Cost O(T^2 d_k^2 (d_k + d_v)): tiny inputs only."""
    q, k, v = f64(q), f64(k), f64(v)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    A, Bg, Wg = _full_gates(alpha, b, w, gates, B, T, H, dk)
    S0 = f64(S0)
    I = np.eye(dk)
    o = np.zeros((B, T, H, dv))
    ST = np.zeros((B, H, dk, dv))
    for bi in range(B):
        for h in range(H):
            M = [(I - np.outer(k[bi, t, h], Bg[bi, t, h] * k[bi, t, h])) @ np.diag(A[bi, t, h])
                 for t in range(T)]
            Wr = [np.outer(Wg[bi, t, h] * k[bi, t, h], v[bi, t, h]) for t in range(T)]
            for t in range(T):
                S = np.zeros((dk, dv))
                for i in range(t + 1):
                    P = I.copy()
                    for j in range(i + 1, t + 1):
                        P = M[j] @ P
                    S += P @ Wr[i]
                if S0 is not None:
                    P = I.copy()
                    for j in range(0, t + 1):
                        P = M[j] @ P
                    S += P @ S0[bi, h]
                o[bi, t, h] = q[bi, t, h] @ S
                if t == T - 1:
                    ST[bi, h] = S
    return o, ST


def masked_matrix(q, k, v, alpha=None, w=None, gates=None):
    """Erase-free case (b = 0) read as a structured masked matrix ("The Eraser
    Trilogy", "The Rosetta Stone"): with gamma_t = prod_{j<=t} alpha_j (per
    channel), o_t = sum_{i<=t} [sum_c q_{t,c} (gamma_{t,c}/gamma_{i,c})
    w_{i,c} k_{i,c}] v_i. The decay ratio is formed as a product of alphas over
    (i, t], never as a quotient, so any alpha in (0, 1] works. S0 = 0."""
    q, k, v = f64(q), f64(k), f64(v)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    g = dict(gates or {})
    g["b"] = "none"
    A, _, W = _full_gates(alpha, None, w, g, B, T, H, dk)
    o = np.zeros((B, T, H, dv))
    for bi in range(B):
        for h in range(H):
            Mk = np.zeros((T, T))
            for t in range(T):
                ratio = np.ones(dk)
                for i in range(t, -1, -1):
                    Mk[t, i] = np.sum(q[bi, t, h] * ratio * W[bi, i, h] * k[bi, i, h])
                    ratio = ratio * A[bi, i, h]
            o[bi, :, h] = Mk @ v[bi, :, h]
    return o


def delta_three_line(q, k, v, alpha=None, beta=None, S0=None, alpha_kind="scalar"):
    """Tied gates b = w = beta (scalar per token-head) in the read / delta /
    write-back form ("Recurrent Memory: Write, Erase, Decay, Read", section 03)
    with the decay of section 04 applied to the carried state first:
        S'    = Diag(alpha_t) S_{t-1}
        v_old = k_t S'
        u_t   = beta_t (v_t - v_old)
        S_t   = S' + k_t^T u_t,     o_t = q_t S_t
    alpha [B,T,H] (scalar) or [B,T,H,dk] (channel), or None (alpha = 1)."""
    q, k, v = f64(q), f64(k), f64(v)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    beta = f64(beta)
    alpha = None if alpha is None else f64(alpha)
    S0 = f64(S0)
    o = np.zeros((B, T, H, dv))
    ST = np.zeros((B, H, dk, dv))
    for bi in range(B):
        for h in range(H):
            S = np.zeros((dk, dv)) if S0 is None else S0[bi, h].copy()
            for t in range(T):
                if alpha is not None:
                    a = alpha[bi, t, h]
                    S = (a[:, None] if alpha_kind == "channel" else a) * S
                v_old = k[bi, t, h] @ S
                u = beta[bi, t, h] * (v[bi, t, h] - v_old)
                S = S + np.outer(k[bi, t, h], u)
                o[bi, t, h] = q[bi, t, h] @ S
            ST[bi, h] = S
    return o, ST


def unified_decay_after_erase(q, k, v, alpha, beta, S0=None):
    """The unified equation in the order the section-05 equation of "Recurrent
    Memory: Write, Erase, Decay, Read" prints it: S_t = Diag(alpha_t)
    (I - beta_t k_t^T k_t) S_{t-1} + beta_t k_t^T v_t (decay after erase).
    alpha channel [B,T,H,dk]; beta scalar [B,T,H]."""
    q, k, v, alpha, beta = f64(q), f64(k), f64(v), f64(alpha), f64(beta)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    S0 = f64(S0)
    o = np.zeros((B, T, H, dv))
    I = np.eye(dk)
    for bi in range(B):
        for h in range(H):
            S = np.zeros((dk, dv)) if S0 is None else S0[bi, h].copy()
            for t in range(T):
                kt = k[bi, t, h]
                S = np.diag(alpha[bi, t, h]) @ (I - beta[bi, t, h] * np.outer(kt, kt)) @ S \
                    + beta[bi, t, h] * np.outer(kt, v[bi, t, h])
                o[bi, t, h] = q[bi, t, h] @ S
    return o


def chunkwise_bwd(q, k, v, alpha=None, b=None, w=None, S0=None, gates=None, dO=None, dS_T=None,
                  chunk: int = 8):
    """Gradients of L = sum(o * dO) + sum(S_T * dS_T), chunk by chunk.

    Two token scans give, per token, the erase read r_t = (b.k) Diag(alpha) S_{t-1}
    and its gradient dr_t = -k_t Ghat_t (Ghat_t = dL/dS_t after adding q_t^T dO_t),
    plus the state at every chunk start and the state gradient at every chunk
    end. With r and dr known, a chunk is a diagonal-decay (erase-free) system
    ("The Eraser Trilogy", "The Rosetta Stone": the masked-matrix form), so
    with gamma the running product of alpha inside the chunk (rows of Gam):
      dq  = Gam (dO S0^T) + Gam [(M o dO V^T)(U/Gam) - (M o dO R^T)(K/Gam)]
      de  = Gam (DR S0^T) + Gam [(M1 o DR V^T)(U/Gam) - (M1 o DR R^T)(K/Gam)]
      du  = [(M^T o V dO^T)(Q Gam) + (M1^T o V DR^T)(E Gam) + gamma_C (V Ge^T)] / Gam
      dkr = -[(M^T o R dO^T)(Q Gam) + (M1^T o R DR^T)(E Gam) + gamma_C (R Ge^T)] / Gam
    (M causal with the diagonal, M1 without; U = w.k, E = b.k, S0 / Ge the
    chunk's start state / end gradient), dk = dkr + b.de + w.du, db = k.de,
    dw = k.du, and the decay through the log of the running product: readers
    minus writers, q.dq + e.de - u.du - k.dkr, plus rowsum(Ge . S_end) on the
    chunk's last token, summed from each token to the chunk end, divided by
    alpha. Returns the dict of `recurrence_bwd` (per-channel gates only
    materialised: scalar and tied forms are summed / merged as there).

    Validity domain: alpha > 0 and short chunks (default 8 tokens). The route
    divides by running products of alpha inside a chunk (U/Gam, K/Gam, /Gam)
    and by alpha itself; it refuses (AssertionError) a chunk whose running
    product falls below 1e-200, where those quotients lose their precision.
    Outside that domain use `recurrence_bwd`, the reverse token loop."""
    q, k, v = f64(q), f64(k), f64(v)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    g = dict(gates or {})
    tied = g.get("w") == "tied"
    A, Bg, W = _full_gates(alpha, b, w, gates, B, T, H, dk)
    S0 = f64(S0)
    dO = f64(dO)
    dS_T = f64(dS_T)
    out = {n: np.zeros((B, T, H, dk)) for n in ("dq", "dk", "da", "db", "dw")}
    out["dv"] = np.zeros((B, T, H, dv))
    out["dS0"] = np.zeros((B, H, dk, dv))
    for bi in range(B):
        for h in range(H):
            qq, kk, vv, aa = q[bi, :, h], k[bi, :, h], v[bi, :, h], A[bi, :, h]
            e, u = Bg[bi, :, h] * kk, W[bi, :, h] * kk
            do = dO[bi, :, h]
            # forward scan: states and erase reads
            S = np.zeros((dk, dv)) if S0 is None else S0[bi, h].copy()
            states = [S.copy()]
            r = np.zeros((T, dv))
            for t in range(T):
                Sd = aa[t][:, None] * S
                r[t] = e[t] @ Sd
                S = Sd - np.outer(kk[t], r[t]) + np.outer(u[t], vv[t])
                states.append(S.copy())
            # backward scan: state-gradient at chunk ends, dr and dv per token
            G = np.zeros((dk, dv)) if dS_T is None else dS_T[bi, h].copy()
            g_end = {}
            dr = np.zeros((T, dv))
            for t in range(T - 1, -1, -1):
                if t == T - 1 or (t + 1) % chunk == 0:
                    g_end[t // chunk] = G.copy()
                G = G + np.outer(qq[t], do[t])
                dr[t] = -(kk[t] @ G)
                out["dv"][bi, t, h] = u[t] @ G
                G = aa[t][:, None] * (G + np.outer(e[t], dr[t]))
            out["dS0"][bi, h] = G
            for c in range((T + chunk - 1) // chunk):
                t0, t1 = c * chunk, min(T, c * chunk + chunk)
                n = t1 - t0
                sl = slice(t0, t1)
                Q, K, V, E, U, R, DR, DO = qq[sl], kk[sl], vv[sl], e[sl], u[sl], r[sl], dr[sl], do[sl]
                Gam = np.cumprod(aa[sl], axis=0)
                assert Gam.min() > 1e-200, "chunkwise_bwd: running decay product underflows; " \
                    "use a shorter chunk or recurrence_bwd"
                S_0, Ge, S_end = states[t0], g_end[c], states[t1]
                M = np.tril(np.ones((n, n)))
                M1 = np.tril(np.ones((n, n)), -1)
                DQ = Gam * (DO @ S_0.T) + Gam * ((M * (DO @ V.T)) @ (U / Gam) - (M * (DO @ R.T)) @ (K / Gam))
                DE = Gam * (DR @ S_0.T) + Gam * ((M1 * (DR @ V.T)) @ (U / Gam) - (M1 * (DR @ R.T)) @ (K / Gam))
                QG, EG = Q * Gam, E * Gam
                DU = ((M.T * (V @ DO.T)) @ QG + (M1.T * (V @ DR.T)) @ EG + (V @ Ge.T) * Gam[-1]) / Gam
                DKR = -((M.T * (R @ DO.T)) @ QG + (M1.T * (R @ DR.T)) @ EG + (R @ Ge.T) * Gam[-1]) / Gam
                dlam = Q * DQ + E * DE - U * DU - K * DKR
                dlam[-1] += np.sum(Ge * S_end, axis=1)
                dlam = np.cumsum(dlam[::-1], axis=0)[::-1]
                out["dq"][bi, sl, h] = DQ
                out["dk"][bi, sl, h] = DKR + Bg[bi, sl, h] * DE + W[bi, sl, h] * DU
                out["da"][bi, sl, h] = dlam / aa[sl]
                out["db"][bi, sl, h] = K * DE
                out["dw"][bi, sl, h] = K * DU

    def shape_like(kind, full):
        if kind in (None, "none", "tied"):
            return None
        return full if kind == "channel" else full.sum(axis=-1)
    ka, kb, kw = g.get("alpha", "none"), g.get("b", "none"), g.get("w", "none")
    db_full = out["db"] + (out["dw"] if tied else 0.0)
    return {"dq": out["dq"], "dk": out["dk"], "dv": out["dv"], "dS0": out["dS0"],
            "dalpha": shape_like(ka, out["da"]), "db": shape_like(kb, db_full),
            "dw": shape_like(kw, out["dw"])}
