"""Backward pass (gdr_chunk_bwd) against the oracle's reverse-mode token loop.

The CUDA-core path computes the gradients in fp32 for both input dtypes,
from the same device-dtype inputs the oracle widens to fp64, so its cases are
held to the fp32 bar: max-abs error <= 1e-4 x max|oracle| per gradient
tensor. The Gated DeltaNet form in bf16 with d_k = d_v = 128 (scalar decay,
tied scalar beta) runs on tensor cores throughout: the forward's state
checkpoints, the chunkwise state-gradient pass (dv, dr, dS0 and the gradient
at every chunk end) and the chunk-parallel gradients, all with bf16 operands
(states, reads and their gradients rounded to bf16, fp32 accumulation), so
every gradient of that form is held to the bf16 bar, 2e-2 x max|oracle|.
"""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_147_b200 import TIED, chunk_bwd
from gated_delta_rule_147_b200.inputs import WORKLOADS, make_chunk_inputs, make_cotangents
from gpu_util import assert_close, to_dev

pytestmark = pytest.mark.gpu
TOL = 1e-4
TOL_TC = 2e-2
NAMES = ("dq", "dk", "dv", "dalpha", "db", "dw", "dS0")


def tensor_core_form(wl):
    return (wl.dtype == "bf16" and wl.dk == 128 and wl.dv == 128 and wl.alpha == "scalar"
            and wl.b == "scalar" and wl.w == "tied")


def tol_of(wl, name):
    return TOL_TC if tensor_core_form(wl) else TOL


def run_bwd(inp, cot, dev, workspace=None):
    g = inp["gates"]
    w = TIED if g["w"] == "tied" else to_dev(inp["w"], dev)
    out = chunk_bwd(to_dev(inp["q"], dev), to_dev(inp["k"], dev), to_dev(inp["v"], dev),
                    to_dev(inp["alpha"], dev), to_dev(inp["b"], dev), w, to_dev(inp["S0"], dev),
                    dO=to_dev(cot["dO"], dev), dS_T=to_dev(cot["dS_T"], dev), workspace=workspace)
    torch.cuda.synchronize()
    return {k: (None if v is None else v.cpu().numpy()) for k, v in out.items()}


def run_oracle_bwd(inp, cot, heads=None):
    def pick(x, state=False):
        if x is None or heads is None:
            return x
        xs = [x[bi][hi] if state else x[bi][:, hi] for bi, hi in heads]
        return torch.stack(xs)[:, None] if state else torch.stack(xs)[:, :, None]
    return oracle.recurrence_bwd(pick(inp["q"]), pick(inp["k"]), pick(inp["v"]),
                                 pick(inp["alpha"]), pick(inp["b"]), pick(inp["w"]),
                                 pick(inp["S0"], True), inp["gates"], pick(cot["dO"]),
                                 pick(cot["dS_T"], True))


def check(got, ref, wl, what=""):
    for n in NAMES:
        if ref[n] is None:
            assert got[n] is None, n
            continue
        assert got[n].shape == ref[n].shape, n
        assert_close(got[n], ref[n], tol_of(wl, n), f"{what}{n}")


FORMS = {
    "gdn": dict(alpha="scalar", b="scalar", w="tied"),
    "kda": dict(alpha="channel", b="scalar", w="tied"),
    "gdn2": dict(alpha="channel", b="channel", w="channel"),
    "gla": dict(alpha="channel", b="none", w="none"),
    "deltanet": dict(alpha="none", b="scalar", w="tied"),
    "linear": dict(alpha="none", b="none", w="none"),
    "mixed": dict(alpha="scalar", b="channel", w="scalar"),
}


@pytest.mark.parametrize("form", sorted(FORMS))
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_gate_forms(cuda_device, form, dtype):
    wl = WORKLOADS["kda"].with_(B=1, H=2, T=150, dtype=dtype, s0=True, seed=300, **FORMS[form])
    inp = make_chunk_inputs(wl)
    cot = make_cotangents(wl)
    check(run_bwd(inp, cot, cuda_device), run_oracle_bwd(inp, cot), wl, f"{form}/{dtype} ")


@pytest.mark.parametrize("T", [1, 7, 8, 9, 63, 64, 65, 200])
def test_ragged_lengths(cuda_device, T):
    """Sequence ends inside a sub-chunk, on a sub-chunk or chunk boundary, and
    after several chunks."""
    wl = WORKLOADS["gdn2"].with_(B=2, H=1, T=T, s0=True, seed=310 + T)
    inp = make_chunk_inputs(wl)
    cot = make_cotangents(wl)
    check(run_bwd(inp, cot, cuda_device), run_oracle_bwd(inp, cot), wl, f"T={T} ")


@pytest.mark.parametrize("dk,dv", [(128, 64), (64, 128), (40, 48), (16, 16), (100, 112), (128, 8),
                                   (128, 256), (7, 24), (256, 256), (200, 64), (256, 8)])
def test_head_shapes(cuda_device, dk, dv):
    """1 to 32 threads per state row (d_v / 8), some of them idle, row
    blocks that run past d_k, and d_k above 128 (8 state rows per lane in the
    scans)."""
    wl = WORKLOADS["kda"].with_(B=1, H=3, T=90, dk=dk, dv=dv, dtype="fp32", s0=True, seed=dk + dv)
    inp = make_chunk_inputs(wl)
    cot = make_cotangents(wl)
    check(run_bwd(inp, cot, cuda_device), run_oracle_bwd(inp, cot), wl, f"{dk}x{dv} ")


def test_no_initial_state_no_final_gradient(cuda_device):
    wl = WORKLOADS["gdn"].with_(B=1, H=2, T=100, seed=320)
    inp = make_chunk_inputs(wl)
    cot = make_cotangents(wl, with_dS_T=False)
    check(run_bwd(inp, cot, cuda_device), run_oracle_bwd(inp, cot), wl)


def test_zero_length_copies_final_gradient(cuda_device):
    wl = WORKLOADS["kda"].with_(B=1, H=2, T=0, seed=321)
    inp = make_chunk_inputs(wl)
    cot = make_cotangents(wl)
    got = run_bwd(inp, cot, cuda_device)
    np.testing.assert_array_equal(got["dS0"], cot["dS_T"].numpy())


def test_deterministic_and_workspace_reused(cuda_device):
    """No atomics: two runs (the second reusing a dirty workspace) agree bit for bit."""
    wl = WORKLOADS["gdn2"].with_(B=1, H=2, T=130, s0=True, seed=322)
    inp = make_chunk_inputs(wl)
    cot = make_cotangents(wl)
    from gated_delta_rule_147_b200 import gdr_chunk_bwd_workspace_size
    ws = torch.full((gdr_chunk_bwd_workspace_size(1, 130, 2, 128, 128),), 255, dtype=torch.uint8,
                    device=cuda_device)
    a = run_bwd(inp, cot, cuda_device, workspace=ws)
    b = run_bwd(inp, cot, cuda_device, workspace=ws)
    for n in NAMES:
        if a[n] is not None:
            np.testing.assert_array_equal(a[n], b[n])


def test_full_size_sampled_heads(cuda_device):
    """The Gated DeltaNet workload (B=4, H=16, T=4096, d=128, bf16) in the
    launch configuration the bench times; two heads checked against the
    oracle over the whole sequence."""
    wl = WORKLOADS["gdn"]
    inp = make_chunk_inputs(wl)
    cot = make_cotangents(wl)
    got = run_bwd(inp, cot, cuda_device)
    heads = [(0, 0), (3, 15)]
    ref = run_oracle_bwd(inp, cot, heads)
    for n in NAMES:
        if ref[n] is None:
            continue
        if n == "dS0":
            g = np.stack([got[n][bi][hi] for bi, hi in heads])[:, None]
        else:
            g = np.stack([got[n][bi][:, hi] for bi, hi in heads])[:, :, None]
        assert_close(g, ref[n], tol_of(wl, n), n)


@pytest.mark.parametrize("form", ["gdn", "gdn2"])
def test_grouped_heads(cuda_device, form):
    """q/k heads shared by pairs of value heads: dq, dk of a q/k head are the
    sums over its value heads of the oracle's gradients with q, k repeated."""
    wl = WORKLOADS["kda"].with_(B=2, H=4, hq=2, T=150, s0=True, seed=330, **FORMS[form])
    inp = make_chunk_inputs(wl)
    cot = make_cotangents(wl)
    got = run_bwd(inp, cot, cuda_device)
    G = wl.H // wl.hq
    rep = dict(inp, q=inp["q"].repeat_interleave(G, dim=2), k=inp["k"].repeat_interleave(G, dim=2))
    ref = run_oracle_bwd(rep, cot)
    for n in ("dq", "dk"):
        B, T, H, dk = ref[n].shape
        ref[n] = ref[n].reshape(B, T, H // G, G, dk).sum(axis=3)
    check(got, ref, wl, f"grouped {form} ")


@pytest.mark.parametrize("T", [1, 63, 64, 65, 200, 1000])
def test_tensor_core_ragged_lengths(cuda_device, T):
    """The tensor-core chunk kernel: one partial chunk, exactly one chunk, a
    one-token tail, several chunks (the final-state term lands on the last
    token of the last chunk)."""
    wl = WORKLOADS["gdn"].with_(B=2, H=2, T=T, s0=True, seed=340 + T)
    assert tensor_core_form(wl)
    inp = make_chunk_inputs(wl)
    cot = make_cotangents(wl)
    check(run_bwd(inp, cot, cuda_device), run_oracle_bwd(inp, cot), wl, f"T={T} ")


@pytest.mark.parametrize("alpha", [1.0, 0.01, 1e-4])
def test_tensor_core_decay_extremes(cuda_device, alpha):
    """Constant decay at the ends of (0, 1]: no decay, and decays whose
    64-token products underflow fp32; every factor the kernel forms is a
    ratio <= 1, so none overflows."""
    wl = WORKLOADS["gdn"].with_(B=1, H=2, T=150, s0=True, seed=350)
    inp = make_chunk_inputs(wl)
    inp["alpha"] = torch.full_like(inp["alpha"], alpha)
    cot = make_cotangents(wl)
    check(run_bwd(inp, cot, cuda_device), run_oracle_bwd(inp, cot), wl, f"alpha={alpha} ")


def test_tensor_core_deterministic_and_status(cuda_device):
    """Two runs over a dirty workspace agree bit for bit, and no bounded wait
    of the tensor-core kernel times out."""
    wl = WORKLOADS["gdn"].with_(B=1, H=3, T=300, s0=True, seed=360)
    inp = make_chunk_inputs(wl)
    cot = make_cotangents(wl)
    from gated_delta_rule_147_b200 import gdr_chunk_bwd_workspace_size
    ws = torch.full((gdr_chunk_bwd_workspace_size(1, 300, 3, 128, 128),), 255, dtype=torch.uint8,
                    device=cuda_device)
    st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    dev = cuda_device
    outs = []
    for _ in range(2):
        out = chunk_bwd(to_dev(inp["q"], dev), to_dev(inp["k"], dev), to_dev(inp["v"], dev),
                        to_dev(inp["alpha"], dev), to_dev(inp["b"], dev), TIED,
                        to_dev(inp["S0"], dev), dO=to_dev(cot["dO"], dev),
                        dS_T=to_dev(cot["dS_T"], dev), workspace=ws, d_status=st)
        torch.cuda.synchronize()
        outs.append({k: (None if v is None else v.cpu().numpy()) for k, v in out.items()})
    assert int(st.item()) == 0
    for n in NAMES:
        if outs[0][n] is not None:
            np.testing.assert_array_equal(outs[0][n], outs[1][n])
    check(outs[0], run_oracle_bwd(inp, cot), wl)


@pytest.mark.parametrize("T", [1, 70])
def test_dk256_gated_deltanet_bf16(cuda_device, T):
    """The Gated DeltaNet head width d_k = d_v = 256 in bf16 (its forward runs
    on tensor cores; its backward on the fp32 CUDA-core path, held to the
    fp32 bar)."""
    wl = WORKLOADS["gdn256"].with_(B=1, H=2, T=T, s0=True, seed=1900 + T)
    inp = make_chunk_inputs(wl)
    cot = make_cotangents(wl)
    check(run_bwd(inp, cot, cuda_device), run_oracle_bwd(inp, cot), wl, f"T={T} ")
