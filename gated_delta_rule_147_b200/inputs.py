"""Seeded synthetic inputs for the gated delta-rule path.

This module is shared by the CUDA path's tests/bench and by the CPU oracle's
tests. It holds only the input recipes (random draws, L2 normalisation of q/k,
the gate activations that turn normal draws into gate values, and rounding to
the device dtype). It holds none of the recurrence's arithmetic.

Workloads (shapes and value distributions of the recurrence's standard forms;
"Recurrent Memory: Write, Erase, Decay, Read" section 05 for the gate
settings; "Erase-then-Delta Attention" abstract for the independent b/w gates;
"How Linear Attention Remembers", Table 1 for d_k = d_v = 128 heads):

  tiny   B=1,H=1,T=64,d=16 fp32; q,k L2-normalised; channel alpha;
         b,w ~ U(0,1)^d_k independent; S0 = 0; seed 0
  gdn    B=4,H=16,T=4096,d=128 bf16; k L2-normalised (q not); scalar alpha;
         b = w = beta scalar ~ sigmoid(N(0,1)); S0 = 0; seed 1
  kda    B=2,H=32,T=8192,d=128 bf16; q,k L2-normalised; channel alpha;
         beta scalar (tied); S0 ~ N(0, 0.02^2) fp32; seed 2
  gdn2   B=1,H=16,T=32768,d=128 bf16; q,k L2-normalised; channel alpha;
         b,w channel, independent, ~ sigmoid(N(0,1)); S0 = 0; seed 3
  decode B=256,H=32,d=128; fp32 state ~ N(0, 0.02^2); per step one bf16 token
         with gdn2 gates; 1000 steps; state from seed 4, step s from (4, s)
  gla    B=4,H=16,T=4096,d_k=128,d_v=256 bf16; q,k L2-normalised; channel
         alpha; no erase (b = 0), w = 1; S0 = 0; seed 5 (erase-free path)
  gdn_gqa B=2,H=32 value heads with 16 q/k heads (value head h reads q/k
         head h // 2),T=4096,d=128 bf16; gdn gates per value head; seed 6
  gdn256 B=2,H=16,T=4096,d_k=d_v=256 bf16 (the Gated DeltaNet head width of
         "How Linear Attention Remembers", Table 1); gdn gates and
         normalisation; S0 = 0; seed 7

Value recipes: q,k,v ~ N(0,1); alpha = exp(-softplus(x)), x ~ N(0,1);
sigmoid gates = 1/(1+exp(-x)), x ~ N(0,1). L2 normalisation is
x / max(||x||, 1e-6) in fp32, then rounding to the device dtype (bf16 is
round-to-nearest-even). Draw order: q, k, v, alpha, b, w, S0. Draws are fp32
from numpy's PCG64.
"""
from __future__ import annotations

from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, replace

import numpy as np
import torch

GATE_KINDS = ("none", "scalar", "channel")


@dataclass(frozen=True)
class ChunkWorkload:
    name: str
    B: int
    H: int
    T: int
    dk: int
    dv: int
    dtype: str          # "bf16" or "fp32": dtype of q, k, v, o and the gates
    alpha: str          # "none" | "scalar" | "channel"
    b: str              # "none" | "scalar" | "channel"
    w: str              # "none" | "scalar" | "channel" | "tied" (w := b)
    q_norm: bool
    k_norm: bool
    s0: bool            # random S0 ~ N(0, 0.02^2), else S0 = 0 (NULL)
    bw_dist: str        # "sigmoid" | "uniform"
    seed: int
    chunk: int = 64
    hq: int = 0         # q/k heads (grouped heads); 0 means H

    def with_(self, **kw) -> "ChunkWorkload":
        return replace(self, **kw)

    @property
    def Hq(self) -> int:
        return self.hq or self.H

    @property
    def tokens(self) -> int:
        return self.B * self.T * self.H


WORKLOADS = {
    "tiny": ChunkWorkload("tiny", 1, 1, 64, 16, 16, "fp32", "channel", "channel", "channel",
                          True, True, False, "uniform", 0),
    "gdn": ChunkWorkload("gdn", 4, 16, 4096, 128, 128, "bf16", "scalar", "scalar", "tied",
                         False, True, False, "sigmoid", 1),
    "kda": ChunkWorkload("kda", 2, 32, 8192, 128, 128, "bf16", "channel", "scalar", "tied",
                         True, True, True, "sigmoid", 2),
    "gdn2": ChunkWorkload("gdn2", 1, 16, 32768, 128, 128, "bf16", "channel", "channel", "channel",
                          True, True, False, "sigmoid", 3),
    # erase-free gated linear attention with the GLA head shape d_k=128, d_v=256
    # ("How Linear Attention Remembers", Table 1); q, k L2-normalised
    "gla": ChunkWorkload("gla", 4, 16, 4096, 128, 256, "bf16", "channel", "none", "none",
                         True, True, False, "sigmoid", 5),
    # Gated DeltaNet gates with grouped heads: 16 q/k heads serving 32 value heads
    # ("How Linear Attention Remembers", Table 1)
    "gdn_gqa": ChunkWorkload("gdn_gqa", 2, 32, 4096, 128, 128, "bf16", "scalar", "scalar", "tied",
                             False, True, False, "sigmoid", 6, hq=16),
    # Gated DeltaNet gates at the d_k = d_v = 256 head width ("How Linear
    # Attention Remembers", Table 1)
    "gdn256": ChunkWorkload("gdn256", 2, 16, 4096, 256, 256, "bf16", "scalar", "scalar", "tied",
                            False, True, False, "sigmoid", 7),
}


@dataclass(frozen=True)
class DecodeWorkload:
    name: str = "decode"
    B: int = 256
    H: int = 32
    dk: int = 128
    dv: int = 128
    steps: int = 1000
    seed: int = 4
    dtype: str = "bf16"


DECODE = DecodeWorkload()


def torch_dtype(name: str) -> torch.dtype:
    return {"bf16": torch.bfloat16, "fp32": torch.float32}[name]


def _l2norm(x: np.ndarray) -> np.ndarray:
    n = np.sqrt(np.sum(x.astype(np.float32) ** 2, axis=-1, keepdims=True, dtype=np.float32))
    return (x / np.maximum(n, np.float32(1e-6))).astype(np.float32)


def _softplus(x: np.ndarray) -> np.ndarray:
    return (np.maximum(x, 0) + np.log1p(np.exp(-np.abs(x)))).astype(np.float32)


def _sigmoid(x: np.ndarray) -> np.ndarray:
    return (1.0 / (1.0 + np.exp(-x))).astype(np.float32)


def _normal(rng: np.random.Generator, shape) -> np.ndarray:
    return rng.standard_normal(size=shape, dtype=np.float32)


def _gate(rng, kind: str, shape_scalar, shape_channel, recipe: str):
    if kind == "none" or kind == "tied":
        return None
    shape = shape_scalar if kind == "scalar" else shape_channel
    if recipe == "alpha":
        return np.exp(-_softplus(_normal(rng, shape))).astype(np.float32)
    if recipe == "sigmoid":
        return _sigmoid(_normal(rng, shape))
    if recipe == "uniform":
        return rng.random(size=shape, dtype=np.float32)
    raise ValueError(recipe)


def _to_dev_dtype(x, dtype: str):
    if x is None:
        return None
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch_dtype(dtype))


def make_chunk_inputs(wl: ChunkWorkload) -> dict:
    """Draw one workload's inputs; returns CPU torch tensors already in the
    device dtype (what the GPU consumes; the oracle widens these to fp64).

    Layout: q,k [B,T,Hq,dk] (Hq = H unless the heads are grouped); v
    [B,T,H,dv]; scalar gates [B,T,H]; channel gates [B,T,H,dk]; S0
    [B,H,dk,dv] fp32 or None.
    """
    rng = np.random.Generator(np.random.PCG64(wl.seed))
    B, T, H, dk, dv = wl.B, wl.T, wl.H, wl.dk, wl.dv
    q = _normal(rng, (B, T, wl.Hq, dk))
    k = _normal(rng, (B, T, wl.Hq, dk))
    v = _normal(rng, (B, T, H, dv))
    if wl.q_norm:
        q = _l2norm(q)
    if wl.k_norm:
        k = _l2norm(k)
    sc, ch = (B, T, H), (B, T, H, dk)
    alpha = _gate(rng, wl.alpha, sc, ch, "alpha")
    b = _gate(rng, wl.b, sc, ch, wl.bw_dist)
    w = _gate(rng, wl.w, sc, ch, wl.bw_dist)
    s0 = (0.02 * _normal(rng, (B, H, dk, dv))).astype(np.float32) if wl.s0 else None
    d = wl.dtype
    return {
        "q": _to_dev_dtype(q, d), "k": _to_dev_dtype(k, d), "v": _to_dev_dtype(v, d),
        "alpha": _to_dev_dtype(alpha, d), "b": _to_dev_dtype(b, d), "w": _to_dev_dtype(w, d),
        "S0": None if s0 is None else torch.from_numpy(s0),
        "gates": {"alpha": wl.alpha, "b": wl.b, "w": wl.w},
    }


def make_cotangents(wl: ChunkWorkload, with_dS_T: bool = True) -> dict:
    """Upstream gradients for a backward pass over `wl`, seed (wl.seed, 1):
    dO ~ N(0, 1) [B,T,H,dv] in the device dtype, then dS_T ~ N(0, 1)
    [B,H,dk,dv] fp32 (None when with_dS_T is False; still drawn, so dO does
    not depend on the flag)."""
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([wl.seed, 1])))
    dO = _normal(rng, (wl.B, wl.T, wl.H, wl.dv))
    dS_T = _normal(rng, (wl.B, wl.H, wl.dk, wl.dv))
    return {"dO": _to_dev_dtype(dO, wl.dtype),
            "dS_T": torch.from_numpy(dS_T) if with_dS_T else None}


def make_decode_state(dw: DecodeWorkload = DECODE) -> torch.Tensor:
    """Initial decode state S [B,H,dk,dv] fp32 ~ N(0, 0.02^2), seed (dw.seed)."""
    rng = np.random.Generator(np.random.PCG64(dw.seed))
    return torch.from_numpy((0.02 * _normal(rng, (dw.B, dw.H, dw.dk, dw.dv))).astype(np.float32))


def make_decode_step(dw: DecodeWorkload, step: int) -> dict:
    """One decode token per head for step `step`, seed (dw.seed, step).

    q,k,v [B,H,d] bf16 (q,k L2-normalised); alpha, b, w channel gates
    [B,H,dk] bf16 (alpha = exp(-softplus), b,w = sigmoid), drawn in that order.
    """
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([dw.seed, step])))
    B, H, dk, dv = dw.B, dw.H, dw.dk, dw.dv
    q = _l2norm(_normal(rng, (B, H, dk)))
    k = _l2norm(_normal(rng, (B, H, dk)))
    v = _normal(rng, (B, H, dv))
    alpha = np.exp(-_softplus(_normal(rng, (B, H, dk)))).astype(np.float32)
    b = _sigmoid(_normal(rng, (B, H, dk)))
    w = _sigmoid(_normal(rng, (B, H, dk)))
    d = dw.dtype
    return {"q": _to_dev_dtype(q, d), "k": _to_dev_dtype(k, d), "v": _to_dev_dtype(v, d),
            "alpha": _to_dev_dtype(alpha, d), "b": _to_dev_dtype(b, d), "w": _to_dev_dtype(w, d)}


def make_decode_steps(dw: DecodeWorkload, steps, threads: int = 8) -> list:
    """Draw several decode steps in parallel (numpy releases the GIL while drawing)."""
    steps = list(steps)
    with ThreadPoolExecutor(max_workers=max(1, threads)) as ex:
        return list(ex.map(lambda s: make_decode_step(dw, s), steps))
