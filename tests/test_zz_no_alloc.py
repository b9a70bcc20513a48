"""gdr_chunk_fwd_static: the two-pass path on the library's own scratch array.

Collected last (file name) so the array's first lookup happens after every
other test's calls. Compares against gdr_chunk_fwd with a caller workspace on
two calls in a row (the second reuses the array the first filled).
"""
import numpy as np
import pytest
import torch

from gated_delta_rule_147_b200 import _lib
from gated_delta_rule_147_b200.inputs import WORKLOADS, make_chunk_inputs
from gated_delta_rule_147_b200._lib import GATE_SCALAR, GATE_TIED, GDR_BF16

KIND = {"none": 0, "scalar": 1, "channel": 2, "tied": 3}


def test_oversize_is_rejected_before_any_device_work():
    cap = _lib.gdr_chunk_fwd_static_capacity()
    assert cap == 64 << 20
    B, T, H = 8, 8192, 32   # GDN form needs B*T*H*(128 + 128 + 64)*2 bytes > 64 MiB
    need = _lib.gdr_chunk_fwd_workspace_size(B, T, H, 128, 128, GATE_SCALAR, GATE_SCALAR, GATE_TIED,
                                             GDR_BF16)
    assert need > cap
    P = 1 << 20
    st = _lib.load().gdr_chunk_fwd_static(P, P, P, P, P, None, GATE_SCALAR, GATE_SCALAR, GATE_TIED,
                                          None, P, P, B, T, H, 128, 128, 64, GDR_BF16, None, None)
    assert st == _lib.GDR_ERR_UNSUPPORTED


def _run(inp, dev, static):
    g = inp["gates"]
    q, k, v = (inp[x].to(dev) for x in ("q", "k", "v"))
    a = None if inp["alpha"] is None else inp["alpha"].to(dev)
    b = None if inp["b"] is None else inp["b"].to(dev)
    w = None if (inp["w"] is None or g["w"] == "tied") else inp["w"].to(dev)
    S0 = None if inp["S0"] is None else inp["S0"].to(dev)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = torch.empty((B, T, H, dv), dtype=v.dtype, device=dev)
    ST = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)
    args = (q, k, v, a, b, w, KIND[g["alpha"]], KIND[g["b"]], KIND[g["w"]], S0, o, ST)
    if static:
        _lib.gdr_chunk_fwd_static(*args, B, T, H, dk, dv, 64, GDR_BF16)
    else:
        n = _lib.gdr_chunk_fwd_workspace_size(B, T, H, dk, dv, KIND[g["alpha"]], KIND[g["b"]],
                                              KIND[g["w"]], GDR_BF16)
        ws = torch.empty(max(n, 1), dtype=torch.uint8, device=dev)
        _lib.gdr_chunk_fwd(*args, ws, n, B, T, H, dk, dv, 64, GDR_BF16)
    torch.cuda.synchronize()
    return o.cpu(), ST.cpu()


@pytest.mark.gpu
@pytest.mark.parametrize("family", ["gdn", "kda", "gdn2"])
def test_static_scratch_matches_caller_workspace_twice(cuda_device, family):
    """Two different inputs in a row through the static array give exactly
    the results of the caller-workspace entry point (same kernels)."""
    for seed in (501, 502):
        wl = WORKLOADS[family].with_(B=2, H=4, T=777, s0=True, seed=seed)
        inp = make_chunk_inputs(wl)
        o_ref, S_ref = _run(inp, cuda_device, static=False)
        o_st, S_st = _run(inp, cuda_device, static=True)
        assert torch.equal(o_ref.view(torch.int16), o_st.view(torch.int16))
        assert torch.equal(S_ref, S_st)
        assert np.isfinite(o_st.float().numpy()).all()


@pytest.mark.gpu
def test_static_scratch_long_sequence_few_heads(cuda_device):
    """A shape whose caller-workspace call splits the general state pass into
    segments (few heads, long sequence) and still fits the static array: the
    static call keeps one stream and gives the same bits."""
    wl = WORKLOADS["gdn2"].with_(B=1, H=2, T=9000, s0=True, seed=503)
    need = _lib.gdr_chunk_fwd_workspace_size(1, 9000, 2, 128, 128, KIND["channel"], KIND["channel"],
                                             KIND["channel"], GDR_BF16)
    assert 0 < need <= _lib.gdr_chunk_fwd_static_capacity()
    inp = make_chunk_inputs(wl)
    for _ in range(2):
        o_ref, S_ref = _run(inp, cuda_device, static=False)
        o_st, S_st = _run(inp, cuda_device, static=True)
        assert torch.equal(o_ref.view(torch.int16), o_st.view(torch.int16))
        assert torch.equal(S_ref, S_st)
