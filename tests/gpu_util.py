"""Helpers shared by the GPU parity tests."""
import numpy as np
import torch

import oracle
from gated_delta_rule_147_b200 import TIED, chunk_fwd

TOL = {"bf16": 2e-2, "fp32": 1e-4}


def to_dev(x, dev):
    return None if x is None else x.to(dev).contiguous()


def run_chunk(inp, dev, S0="inp", final_state=True, d_status=None, workspace="auto"):
    """chunk_fwd on the device; workspace="auto" takes the two-pass path where
    the gate form has one, None forces the single-pass kernels."""
    g = inp["gates"]
    w = TIED if g["w"] == "tied" else to_dev(inp["w"], dev)
    s0 = inp["S0"] if isinstance(S0, str) else S0
    o, ST = chunk_fwd(to_dev(inp["q"], dev), to_dev(inp["k"], dev), to_dev(inp["v"], dev),
                      to_dev(inp["alpha"], dev), to_dev(inp["b"], dev), w, to_dev(s0, dev),
                      final_state=final_state, d_status=d_status, workspace=workspace)
    torch.cuda.synchronize()
    return o.float().cpu().numpy(), (None if ST is None else ST.cpu().numpy())


def run_oracle(inp, heads=None):
    """Oracle on all heads, or on a list of (b, h) pairs (returned stacked as
    [n, T, 1, dv] / [n, 1, dk, dv]). Grouped q/k heads are repeated per value
    head first (value head h reads q/k head h // group)."""
    g = inp["gates"]
    G = inp["v"].shape[2] // inp["q"].shape[2]
    if G > 1:
        inp = dict(inp, q=inp["q"].repeat_interleave(G, dim=2), k=inp["k"].repeat_interleave(G, dim=2))
    if heads is None:
        return oracle.recurrence(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["b"], inp["w"],
                                 inp["S0"], g)

    def pick(x, head_axis=2):
        if x is None:
            return None
        xs = [x[bi][:, hi] if head_axis == 2 else x[bi][hi] for bi, hi in heads]
        return torch.stack(xs)[:, :, None] if head_axis == 2 else torch.stack(xs)[:, None]
    return oracle.recurrence(pick(inp["q"]), pick(inp["k"]), pick(inp["v"]), pick(inp["alpha"]),
                             pick(inp["b"]), pick(inp["w"]), pick(inp["S0"], 1), g)


def gather_heads(o, ST, heads):
    os_ = np.stack([o[bi][:, hi] for bi, hi in heads])[:, :, None]
    ss = np.stack([ST[bi][hi] for bi, hi in heads])[:, None]
    return os_, ss


def rel_err(x, ref):
    return float(np.abs(x - ref).max() / max(np.abs(ref).max(), 1e-30))


def assert_close(x, ref, tol, what):
    e = rel_err(x, ref)
    assert np.all(np.isfinite(x)), f"{what}: non-finite values"
    assert e <= tol, f"{what}: max-abs error {e:.3e} x max|ref| exceeds {tol:.1e}"
    return e
