"""GPU parity of gdr_decode_step against the fp64 oracle (state carried
between calls, updated in place on the device)."""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_147_b200 import TIED, decode_step
from gated_delta_rule_147_b200.inputs import DECODE, DecodeWorkload, make_decode_state, make_decode_step, make_decode_steps
from gpu_util import TOL, assert_close

pytestmark = pytest.mark.gpu

GEN = {"alpha": "channel", "b": "channel", "w": "channel"}


def rand_step(rng, B, H, dk, dv, kinds, dtype):
    def n(*s):
        return torch.from_numpy(rng.standard_normal(s).astype(np.float32))
    q, k = n(B, H, dk), n(B, H, dk)
    q, k = q / q.norm(dim=-1, keepdim=True), k / k.norm(dim=-1, keepdim=True)
    v = n(B, H, dv)
    g = {}
    for name in ("alpha", "b", "w"):
        kind = kinds[name]
        if kind in ("none", "tied"):
            g[name] = None
            continue
        x = n(B, H) if kind == "scalar" else n(B, H, dk)
        g[name] = torch.exp(-torch.nn.functional.softplus(x)) if name == "alpha" else torch.sigmoid(x)
    cast = lambda x: None if x is None else x.to(dtype)
    return {"q": cast(q), "k": cast(k), "v": cast(v), "alpha": cast(g["alpha"]), "b": cast(g["b"]),
            "w": cast(g["w"])}


@pytest.mark.parametrize("dtype,dk,dv", [(torch.bfloat16, 128, 128), (torch.float32, 128, 128),
                                         (torch.bfloat16, 64, 32), (torch.float32, 96, 256),
                                         (torch.float32, 200, 16),
                                         # d_k = d_v = 256: each head's columns in two blocks
                                         (torch.bfloat16, 256, 256), (torch.float32, 200, 256)])
@pytest.mark.parametrize("kinds", [GEN, {"alpha": "scalar", "b": "scalar", "w": "tied"},
                                   {"alpha": "none", "b": "none", "w": "none"}])
def test_decode_steps_small(cuda_device, dtype, dk, dv, kinds):
    rng = np.random.default_rng(dk * 1000 + dv)
    B, H, steps = 3, 5, 12
    S0 = torch.from_numpy((0.02 * rng.standard_normal((B, H, dk, dv))).astype(np.float32))
    S_dev = S0.to(cuda_device)
    S_ref = S0.double().numpy()
    tol = TOL["fp32" if dtype == torch.float32 else "bf16"]
    for _ in range(steps):
        st = rand_step(rng, B, H, dk, dv, kinds, dtype)
        d = {k_: (None if x is None else x.to(cuda_device)) for k_, x in st.items()}
        w = TIED if kinds["w"] == "tied" else d["w"]
        o = decode_step(d["q"], d["k"], d["v"], d["alpha"], d["b"], w, S_dev)
        o_ref, S_ref = oracle.decode_step(st["q"], st["k"], st["v"], st["alpha"], st["b"], st["w"],
                                          S_ref, kinds)
        torch.cuda.synchronize()
        assert_close(o.float().cpu().numpy(), o_ref, tol, "o")
    assert_close(S_dev.cpu().numpy(), S_ref, tol, "S")


def test_decode_full_size_sampled_heads(cuda_device):
    """256 x 32 heads, d = 128, 1000 steps, GDN-2 gates; the oracle follows
    two whole batch rows (64 heads) through every step."""
    dw = DECODE
    S = make_decode_state(dw)
    rows = [17, 200]
    S_ref = S[rows].double().numpy()
    S_dev = S.to(cuda_device)
    o_dev = torch.empty((dw.B, dw.H, dw.dv), dtype=torch.bfloat16, device=cuda_device)
    worst = 0.0
    o_err_max, o_ref_max = 0.0, 0.0
    for s0 in range(0, dw.steps, 50):
        batch = make_decode_steps(dw, range(s0, min(s0 + 50, dw.steps)))
        for st in batch:
            d = {k_: x.to(cuda_device, non_blocking=False) for k_, x in st.items()}
            decode_step(d["q"], d["k"], d["v"], d["alpha"], d["b"], d["w"], S_dev, out=o_dev)
            o_ref, S_ref = oracle.decode_step(*(st[x][rows] for x in ("q", "k", "v", "alpha", "b", "w")),
                                              S_ref, GEN)
            o_got = o_dev[rows].float().cpu().numpy()
            o_err_max = max(o_err_max, float(np.abs(o_got - o_ref).max()))
            o_ref_max = max(o_ref_max, float(np.abs(o_ref).max()))
    assert o_err_max <= TOL["bf16"] * o_ref_max, (o_err_max, o_ref_max)
    worst = assert_close(S_dev[rows].cpu().numpy(), S_ref, TOL["bf16"], "S after 1000 steps")
    assert np.all(np.isfinite(S_dev.cpu().numpy()))


@pytest.mark.parametrize("family", ["gdn", "kda", "gdn2", "gdn256"])
def test_prefill_then_decode_continues_the_sequence(cuda_device, family):
    """The chunk forward's final state is the decode step's state layout:
    prefill T tokens, then decode m more from S_T; the decode outputs equal
    the oracle's outputs for tokens T..T+m-1 of one T+m sequence."""
    from gated_delta_rule_147_b200 import chunk_fwd
    from gated_delta_rule_147_b200.inputs import WORKLOADS, make_chunk_inputs
    T, m = 130, 6
    wl = WORKLOADS[family].with_(B=2, H=2, T=T + m, s0=True, seed=31)
    inp = make_chunk_inputs(wl)
    g = inp["gates"]
    dev = cuda_device
    pre = lambda x: None if x is None else x[:, :T].contiguous().to(dev)
    w_arg = TIED if g["w"] == "tied" else pre(inp["w"])
    _, S = chunk_fwd(pre(inp["q"]), pre(inp["k"]), pre(inp["v"]), pre(inp["alpha"]), pre(inp["b"]),
                     w_arg, inp["S0"].to(dev))
    o_ref, _ = oracle.recurrence(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["b"], inp["w"],
                                 inp["S0"], g)
    for t in range(T, T + m):
        tok = lambda x: None if x is None else x[:, t].contiguous().to(dev)
        w_t = TIED if g["w"] == "tied" else tok(inp["w"])
        o = decode_step(tok(inp["q"]), tok(inp["k"]), tok(inp["v"]), tok(inp["alpha"]), tok(inp["b"]),
                        w_t, S)
        torch.cuda.synchronize()
        assert_close(o.float().cpu().numpy(), o_ref[:, t], TOL["bf16"], f"decode token {t}")


def test_grouped_decode_equals_expanded(cuda_device):
    """Grouped q/k heads (H_qk = 2 for H = 4): equal, bit for bit, to the
    ungrouped step with q, k repeated per value head."""
    from gated_delta_rule_147_b200 import decode_step
    dw = DecodeWorkload(B=3, H=4, steps=1, seed=31)
    dev = cuda_device
    S1 = make_decode_state(dw).to(dev)
    S2 = S1.clone()
    st = {k: v.to(dev) for k, v in make_decode_step(dw, 0).items()}
    qg, kg = st["q"][:, ::2].contiguous(), st["k"][:, ::2].contiguous()
    o1 = decode_step(qg.repeat_interleave(2, dim=1).contiguous(), kg.repeat_interleave(2, dim=1).contiguous(),
                     st["v"], st["alpha"], st["b"], st["w"], S1)
    o2 = decode_step(qg, kg, st["v"], st["alpha"], st["b"], st["w"], S2)
    torch.cuda.synchronize()
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    assert torch.equal(S1, S2)
