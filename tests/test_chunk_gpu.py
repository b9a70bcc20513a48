"""GPU parity of gdr_chunk_fwd against the fp64 oracle.

Tolerances (max-abs error relative to max|ref|, for o and for S_T): 2e-2 for
bf16 inputs with fp32 accumulation, 1e-4 for fp32 inputs.
"""
import numpy as np
import pytest
import torch

from gated_delta_rule_147_b200 import GDR_DEVICE_DECAY_RANGE, TIED, chunk_fwd
from gated_delta_rule_147_b200.inputs import WORKLOADS, make_chunk_inputs
from gpu_util import TOL, assert_close, gather_heads, run_chunk, run_oracle

pytestmark = pytest.mark.gpu

FAMILIES = ["gdn", "kda", "gdn2"]


def small(family, **kw):
    base = dict(B=2, H=3, T=200)
    base.update(kw)
    return WORKLOADS[family].with_(**base)


@pytest.mark.parametrize("family", FAMILIES)
@pytest.mark.parametrize("T", [1, 64, 65, 200])
def test_small_ragged(cuda_device, family, T):
    """Several chunks and a ragged tail, two 64-column slices of d_v."""
    wl = small(family, T=T, s0=True, seed=100 + T)
    inp = make_chunk_inputs(wl)
    o, ST = run_chunk(inp, cuda_device)
    o_ref, ST_ref = run_oracle(inp)
    assert_close(o, o_ref, TOL["bf16"], "o")
    assert_close(ST, ST_ref, TOL["bf16"], "S_T")


@pytest.mark.parametrize("family", FAMILIES)
def test_slow_decay_carries_state_across_chunks(cuda_device, family):
    """alpha close to 1: the state survives many chunks, so inter-chunk
    propagation (and its bf16 operand rounding) is exercised."""
    wl = small(family, T=640, H=2, s0=True, seed=7)
    inp = make_chunk_inputs(wl)
    inp["alpha"] = (inp["alpha"].float() ** 0.02).to(inp["alpha"].dtype)
    o, ST = run_chunk(inp, cuda_device)
    o_ref, ST_ref = run_oracle(inp)
    assert_close(o, o_ref, TOL["bf16"], "o")
    assert_close(ST, ST_ref, TOL["bf16"], "S_T")


@pytest.mark.parametrize("gates", [
    {"alpha": "none", "b": "none", "w": "none"},          # linear attention
    {"alpha": "scalar", "b": "none", "w": "channel"},     # gated linear attention (no erase)
    {"alpha": "none", "b": "scalar", "w": "tied"},        # DeltaNet
    {"alpha": "channel", "b": "channel", "w": "tied"},    # channel b with w := b
    {"alpha": "scalar", "b": "scalar", "w": "scalar"},    # untied scalar gates
])
def test_gate_forms(cuda_device, gates):
    wl = small("gdn2", T=150, alpha=gates["alpha"], b=gates["b"], w=gates["w"], s0=True, seed=3)
    inp = make_chunk_inputs(wl)
    o, ST = run_chunk(inp, cuda_device)
    o_ref, ST_ref = run_oracle(inp)
    assert_close(o, o_ref, TOL["bf16"], "o")
    assert_close(ST, ST_ref, TOL["bf16"], "S_T")


def test_tiny_fp32(cuda_device):
    """B=1,H=1,T=64,d=16 fp32, channel alpha, independent b,w ~ U(0,1)."""
    inp = make_chunk_inputs(WORKLOADS["tiny"])
    o, ST = run_chunk(inp, cuda_device)
    o_ref, ST_ref = run_oracle(inp)
    assert_close(o, o_ref, TOL["fp32"], "o")
    assert_close(ST, ST_ref, TOL["fp32"], "S_T")


@pytest.mark.parametrize("family", FAMILIES)
def test_fp32_path_d128(cuda_device, family):
    wl = small(family, T=97, dtype="fp32", s0=True, seed=5)
    inp = make_chunk_inputs(wl)
    o, ST = run_chunk(inp, cuda_device)
    o_ref, ST_ref = run_oracle(inp)
    assert_close(o, o_ref, TOL["fp32"], "o")
    assert_close(ST, ST_ref, TOL["fp32"], "S_T")


def test_bf16_other_shapes_use_exact_path(cuda_device):
    wl = small("kda", T=70, dk=64, dv=48, s0=True, seed=9)
    inp = make_chunk_inputs(wl)
    o, ST = run_chunk(inp, cuda_device)
    o_ref, ST_ref = run_oracle(inp)
    assert_close(o, o_ref, TOL["bf16"], "o")
    assert_close(ST, ST_ref, TOL["bf16"], "S_T")


def test_split_sequence_resumes(cuda_device):
    """Two calls with S0 := S_T of the first equal one call."""
    wl = small("gdn2", T=256, s0=True, seed=11)
    inp = make_chunk_inputs(wl)
    dev = cuda_device
    o_full, ST_full = run_chunk(inp, dev)
    first = {k: (v[:, :128] if hasattr(v, "dim") and k not in ("S0",) else v) for k, v in inp.items()}
    second = {k: (v[:, 128:] if hasattr(v, "dim") and k not in ("S0",) else v) for k, v in inp.items()}
    o1, S1 = run_chunk(first, dev)
    second["S0"] = torch.from_numpy(S1)
    o2, S2 = run_chunk(second, dev)
    assert_close(np.concatenate([o1, o2], axis=1), o_full, 1e-2, "o (split)")
    assert_close(S2, ST_full, 1e-2, "S_T (split)")


def test_zero_length_copies_initial_state(cuda_device):
    wl = small("kda", T=0, s0=True)
    inp = make_chunk_inputs(wl)
    o, ST = run_chunk(inp, cuda_device)
    assert o.shape == (2, 0, 3, 128)
    np.testing.assert_array_equal(ST, inp["S0"].numpy())


def test_final_state_in_place(cuda_device):
    """S_T may alias S0."""
    wl = small("kda", T=130, s0=True, seed=12)
    inp = make_chunk_inputs(wl)
    dev = cuda_device
    S = inp["S0"].to(dev).clone()
    q, k, v = (inp[x].to(dev) for x in ("q", "k", "v"))
    o, ST = chunk_fwd(q, k, v, inp["alpha"].to(dev), inp["b"].to(dev), "tied", S, S_T=S)
    torch.cuda.synchronize()
    o_ref, ST_ref = run_oracle(inp)
    assert_close(S.cpu().numpy(), ST_ref, TOL["bf16"], "S_T in place")


def test_decay_range_flag(cuda_device):
    """A channel-decay chunk whose decay span exceeds the two-factor range is
    applied token by token (the result still matches the oracle) and reported
    through d_status; in-range inputs leave the status zero."""
    wl = small("kda", T=64, H=1, B=1, seed=13)
    inp = make_chunk_inputs(wl)
    st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    run_chunk(inp, cuda_device, d_status=st)
    assert int(st.item()) == 0
    inp["alpha"] = torch.full_like(inp["alpha"], 0.01)   # 63 x 4.6 nats > 160
    o, ST = run_chunk(inp, cuda_device, d_status=st)
    assert int(st.item()) & GDR_DEVICE_DECAY_RANGE
    o_ref, ST_ref = run_oracle(inp)
    assert_close(o, o_ref, TOL["bf16"], "o (fallback chunk)")
    assert_close(ST, ST_ref, TOL["bf16"], "S_T (fallback chunk)")


@pytest.mark.parametrize("family", FAMILIES)
def test_full_size_sampled_heads(cuda_device, family):
    """The full workload in the launch configuration the benchmark times;
    the oracle checks a seeded sample of heads over the whole sequence."""
    wl = WORKLOADS[family]
    inp = make_chunk_inputs(wl)
    o, ST = run_chunk(inp, cuda_device)
    rng = np.random.default_rng(2024)
    nh = 3 if family == "gdn2" else 4
    heads = sorted({(int(rng.integers(wl.B)), int(rng.integers(wl.H))) for _ in range(nh)})
    o_ref, ST_ref = run_oracle(inp, heads)
    o_s, ST_s = gather_heads(o, ST, heads)
    assert_close(o_s, o_ref, TOL["bf16"], f"o {heads}")
    assert_close(ST_s, ST_ref, TOL["bf16"], f"S_T {heads}")
    assert np.all(np.isfinite(o))


@pytest.mark.parametrize("akind,wkind", [("channel", "none"), ("scalar", "scalar"), ("none", "channel"),
                                         ("channel", "channel"), ("none", "none")])
@pytest.mark.parametrize("dv,T", [(64, 130), (256, 64), (128, 1)])
def test_erase_free_path(cuda_device, akind, wkind, dv, T):
    """b = 0 (no erase) runs the erase-free kernel: linear attention, gated
    linear attention and Mamba-2 shapes, with or without a write gate."""
    wl = small("gdn2", T=T, dv=dv, alpha=akind, b="none", w=wkind, s0=True, seed=40 + dv + T)
    inp = make_chunk_inputs(wl)
    o, ST = run_chunk(inp, cuda_device)
    o_ref, ST_ref = run_oracle(inp)
    assert_close(o, o_ref, TOL["bf16"], "o")
    assert_close(ST, ST_ref, TOL["bf16"], "S_T")


def test_gla_full_size_sampled_heads(cuda_device):
    """The erase-free workload (GLA head shape d_v = 256) at full size."""
    wl = WORKLOADS["gla"]
    inp = make_chunk_inputs(wl)
    o, ST = run_chunk(inp, cuda_device)
    heads = [(0, 3), (2, 11), (3, 15)]
    o_ref, ST_ref = run_oracle(inp, heads)
    o_s, ST_s = gather_heads(o, ST, heads)
    assert_close(o_s, o_ref, TOL["bf16"], f"o {heads}")
    assert_close(ST_s, ST_ref, TOL["bf16"], f"S_T {heads}")


# ---- two-pass path (per-chunk factors in parallel, then the state pass) -----
# Every erase-gated bf16 form with d_k = 128, d_v <= 128 takes it by default;
# these also run the same inputs through the single-pass kernels.

@pytest.mark.parametrize("family", FAMILIES)
@pytest.mark.parametrize("T", [1, 63, 64, 65, 200, 1000])
@pytest.mark.parametrize("dv", [64, 128])
def test_two_pass_matches_oracle_and_single_pass(cuda_device, family, T, dv):
    """Gated DeltaNet form: its own pair of kernels; KDA and GDN-2 forms: the
    general pair (channel decay, independent b and w)."""
    wl = small(family, T=T, dv=dv, s0=True, seed=300 + T + dv)
    inp = make_chunk_inputs(wl)
    o2, S2 = run_chunk(inp, cuda_device)                      # two-pass
    o1, S1 = run_chunk(inp, cuda_device, workspace=None)      # single pass
    o_ref, ST_ref = run_oracle(inp)
    assert_close(o2, o_ref, TOL["bf16"], "o (two-pass)")
    assert_close(S2, ST_ref, TOL["bf16"], "S_T (two-pass)")
    assert_close(o1, o_ref, TOL["bf16"], "o (single pass)")
    assert_close(S1, ST_ref, TOL["bf16"], "S_T (single pass)")


def test_two_pass_workspace_is_used(cuda_device):
    """The two-pass path writes the per-token rows of -W, P and Aq into the
    caller's workspace: row t of -W is -(T Diag(beta g) K)_t, so a token whose
    beta is 0 gets a zero row in both -W and P; Aq is lower triangular."""
    wl = small("gdn", T=130, B=1, H=2, seed=17)
    inp = make_chunk_inputs(wl)
    inp["b"][0, 5, 1] = 0.0
    dev = cuda_device
    q, k, v, a, b = (inp[x].to(dev) for x in ("q", "k", "v", "alpha", "b"))
    from gated_delta_rule_147_b200 import workspace_bytes
    nbytes = workspace_bytes(q, v, a, b, TIED)
    assert nbytes == 1 * 130 * 2 * (128 + 128 + 64) * 2
    ws = torch.full((nbytes,), 0x7F, dtype=torch.uint8, device=dev)
    chunk_fwd(q, k, v, a, b, TIED, None, workspace=ws)
    torch.cuda.synchronize()
    half = 130 * 2 * 128
    wneg = ws[: half * 2].view(torch.bfloat16).view(1, 130, 2, 128).float().cpu()
    p = ws[half * 2: half * 4].view(torch.bfloat16).view(1, 130, 2, 128).float().cpu()
    aq = ws[half * 4:].view(torch.bfloat16).view(1, 130, 2, 64).float().cpu()
    assert torch.all(wneg[0, 5, 1] == 0) and torch.all(p[0, 5, 1] == 0)
    assert torch.isfinite(wneg).all() and torch.isfinite(p).all() and torch.isfinite(aq).all()
    assert wneg.abs().sum() > 0 and p.abs().sum() > 0
    for t in (0, 5, 63, 64, 100, 129):  # token t of a chunk: Aq row zero past its own position
        j = t % 64
        assert torch.all(aq[0, t, :, j + 1:] == 0) and torch.all(aq[0, t, :, j] != 0)


@pytest.mark.parametrize("family", FAMILIES)
def test_two_pass_full_size_matches_single_pass(cuda_device, family):
    """Full workloads: the two paths agree everywhere (both were checked
    against the oracle on sampled heads above)."""
    wl = WORKLOADS[family]
    inp = make_chunk_inputs(wl)
    o2, S2 = run_chunk(inp, cuda_device)
    o1, S1 = run_chunk(inp, cuda_device, workspace=None)
    assert_close(o2, o1, 2e-2, "o two-pass vs single pass")
    assert_close(S2, S1, 2e-2, "S_T two-pass vs single pass")


@pytest.mark.parametrize("family", ["kda", "gdn2"])
@pytest.mark.parametrize("T", [4200, 9000])
def test_two_pass_segmented_state_pass(cuda_device, family, T):
    """Few heads and a long sequence: the general form splits the state pass
    into segments (the first pass of later segments overlaps earlier state
    segments on a second stream, the state carried between them)."""
    wl = WORKLOADS[family].with_(B=1, H=2, T=T, s0=True, seed=900 + T)
    inp = make_chunk_inputs(wl)
    o2, S2 = run_chunk(inp, cuda_device)
    o1, S1 = run_chunk(inp, cuda_device, workspace=None)
    o_ref, ST_ref = run_oracle(inp)
    assert_close(o2, o_ref, TOL["bf16"], "o (segmented two-pass)")
    assert_close(S2, ST_ref, TOL["bf16"], "S_T (segmented two-pass)")
    assert_close(o2, o1, 2e-2, "o two-pass vs single pass")


# ---- grouped q/k heads ------------------------------------------------------

def _expand_heads(x, group):
    """q or k with H_qk heads -> H = H_qk * group heads (value head h reads h // group)."""
    return None if x is None else x.repeat_interleave(group, dim=2).contiguous()


@pytest.mark.parametrize("family,dv,workspace", [
    ("gdn", 128, "auto"), ("kda", 128, "auto"), ("gdn2", 64, "auto"),   # two-pass paths
    ("gdn", 128, None), ("kda", 64, None), ("gdn2", 128, None),         # single-pass kernels
    ("gla", 256, "auto"),                                               # erase-free kernel
])
def test_grouped_heads_equal_expanded_heads(cuda_device, family, dv, workspace):
    """16 q/k heads for 32 value heads in small: H_qk = 2, H = 4. The grouped
    call reads q/k head h // 2 and must equal, bit for bit, the ungrouped call
    with q, k repeated per value head (same kernels, same data); the result
    is also checked against the oracle."""
    wl = WORKLOADS[family].with_(B=2, H=4, T=150, dv=dv, s0=True, seed=77)
    inp = make_chunk_inputs(wl)
    dev = cuda_device
    qg = inp["q"][:, :, ::2].contiguous()     # H_qk = 2 q/k heads
    kg = inp["k"][:, :, ::2].contiguous()
    full = dict(inp, q=_expand_heads(qg, 2), k=_expand_heads(kg, 2))
    o_ref_dev, S_ref_dev = run_chunk(full, dev, workspace=workspace)
    w = TIED if inp["gates"]["w"] == "tied" else (None if inp["w"] is None else inp["w"].to(dev))
    a = None if inp["alpha"] is None else inp["alpha"].to(dev)
    b = None if inp["b"] is None else inp["b"].to(dev)
    s0 = None if inp["S0"] is None else inp["S0"].to(dev)
    o, ST = chunk_fwd(qg.to(dev), kg.to(dev), inp["v"].to(dev), a, b, w, s0, workspace=workspace)
    torch.cuda.synchronize()
    assert torch.equal(o.cpu().view(torch.int16), torch.from_numpy(o_ref_dev).to(o.dtype).view(torch.int16))
    assert np.array_equal(ST.cpu().numpy(), S_ref_dev)
    o_or, S_or = run_oracle(full)
    assert_close(o.float().cpu().numpy(), o_or, TOL["bf16"], "o (grouped)")
    assert_close(ST.cpu().numpy(), S_or, TOL["bf16"], "S_T (grouped)")


def test_grouped_heads_fp32_exact_path(cuda_device):
    wl = WORKLOADS["kda"].with_(B=1, H=4, T=70, dtype="fp32", s0=True, seed=78)
    inp = make_chunk_inputs(wl)
    dev = cuda_device
    qg, kg = inp["q"][:, :, ::2].contiguous(), inp["k"][:, :, ::2].contiguous()
    full = dict(inp, q=_expand_heads(qg, 2), k=_expand_heads(kg, 2))
    o_ref, S_ref = run_chunk(full, dev)
    o, ST = chunk_fwd(qg.to(dev), kg.to(dev), inp["v"].to(dev), inp["alpha"].to(dev),
                      inp["b"].to(dev), TIED, inp["S0"].to(dev))
    torch.cuda.synchronize()
    assert np.array_equal(o.cpu().numpy(), o_ref) and np.array_equal(ST.cpu().numpy(), S_ref)


@pytest.mark.parametrize("dtype,dv", [("bf16", 64), ("fp32", 128), ("bf16", 256)])
def test_dk256_exact_path(cuda_device, dtype, dv):
    """d_k = 256 heads (GDN-340M width) run on the exact token-by-token path."""
    wl = WORKLOADS["kda"].with_(B=1, H=2, T=70, dk=256, dv=dv, dtype=dtype, s0=True, seed=81)
    inp = make_chunk_inputs(wl)
    o, ST = run_chunk(inp, cuda_device)
    o_ref, ST_ref = run_oracle(inp)
    assert_close(o, o_ref, TOL[dtype], "o")
    assert_close(ST, ST_ref, TOL[dtype], "S_T")


def test_grouped_workload_full_size_sampled_heads(cuda_device):
    """The grouped-heads workload the benchmark times (32 value heads, 16 q/k
    heads, Gated DeltaNet gates) at full size, sampled heads against the oracle."""
    wl = WORKLOADS["gdn_gqa"]
    inp = make_chunk_inputs(wl)
    o, ST = run_chunk(inp, cuda_device)
    heads = [(0, 0), (0, 1), (1, 30)]
    o_ref, ST_ref = run_oracle(inp, heads)
    o_s, ST_s = gather_heads(o, ST, heads)
    assert_close(o_s, o_ref, TOL["bf16"], f"o {heads}")
    assert_close(ST_s, ST_ref, TOL["bf16"], f"S_T {heads}")


@pytest.mark.parametrize("H", [2, 40])
def test_erase_free_decay_range(cuda_device, H):
    """Erase-free chunks whose decay span is beyond the two-factor range are
    applied token by token, between ordinary chunks and twice in a row (the
    kernel builds the next chunk's operands while the current chunk's last
    product runs, and runs a flagged chunk after the previous state update).
    d_status carries the flag and the result matches the oracle. H = 40 takes
    the 128-column CTAs."""
    wl = small("gdn2", T=320, H=H, dv=128, alpha="channel", b="none", w="none", s0=True, seed=741)
    inp = make_chunk_inputs(wl)
    a = inp["alpha"].clone()
    for lo, hi in ((64, 128), (192, 256), (256, 320)):  # chunks 1, 3 and 4: 63 x 4.6 nats > 160
        a[:, lo:hi] = 0.01
    inp["alpha"] = a
    st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    o, ST = run_chunk(inp, cuda_device, d_status=st)
    assert int(st.item()) & GDR_DEVICE_DECAY_RANGE
    o_ref, ST_ref = run_oracle(inp)
    assert_close(o, o_ref, TOL["bf16"], "o")
    assert_close(ST, ST_ref, TOL["bf16"], "S_T")


@pytest.mark.parametrize("dv,akind,wkind", [(256, "channel", "none"), (128, "scalar", "channel")])
def test_erase_free_wide_ctas(cuda_device, dv, akind, wkind):
    """More 64-column tiles than SMs: the erase-free kernel carries 128 value
    columns per CTA (one wave of CTAs)."""
    wl = WORKLOADS["gla"].with_(B=2, H=40, T=200, dv=dv, alpha=akind, w=wkind, s0=True, seed=61)
    inp = make_chunk_inputs(wl)
    o, ST = run_chunk(inp, cuda_device)
    o_ref, ST_ref = run_oracle(inp)
    assert_close(o, o_ref, TOL["bf16"], "o")
    assert_close(ST, ST_ref, TOL["bf16"], "S_T")


# ---- d_k = 256 (Gated DeltaNet head width, "How Linear Attention Remembers", Table 1) ----

@pytest.mark.parametrize("dv,T", [(256, 200), (256, 64), (128, 65), (64, 1), (192, 130)])
def test_dk256_tensor_core_path(cuda_device, dv, T):
    """Gated DeltaNet gates at d_k = 256 run on the d_k = 256 two-pass
    kernels: several chunks, a ragged tail, every d_v tile count."""
    wl = WORKLOADS["gdn256"].with_(B=2, H=3, T=T, dv=dv, s0=True, seed=900 + T + dv)
    inp = make_chunk_inputs(wl)
    o, ST = run_chunk(inp, cuda_device)
    o_ref, ST_ref = run_oracle(inp)
    assert_close(o, o_ref, TOL["bf16"], "o")
    assert_close(ST, ST_ref, TOL["bf16"], "S_T")


def test_dk256_slow_decay_and_grouped_heads(cuda_device):
    """alpha close to 1 over ten chunks (the state crosses every chunk
    boundary), and value heads sharing q/k heads in pairs."""
    wl = WORKLOADS["gdn256"].with_(B=1, H=4, T=640, s0=True, seed=910)
    inp = make_chunk_inputs(wl)
    inp["alpha"] = (inp["alpha"].float() ** 0.02).to(inp["alpha"].dtype)
    qg, kg = inp["q"][:, :, ::2].contiguous(), inp["k"][:, :, ::2].contiguous()
    inp_g = dict(inp, q=qg, k=kg)
    o, ST = run_chunk(inp_g, cuda_device)
    o_ref, ST_ref = run_oracle(inp_g)
    assert_close(o, o_ref, TOL["bf16"], "o")
    assert_close(ST, ST_ref, TOL["bf16"], "S_T")


def test_dk256_workspace_is_used(cuda_device):
    """The d_k = 256 path writes -W, P, Aq and K~ = Diag(g_{n-1}/g) K into the
    caller's workspace: a token with beta = 0 gets zero rows of -W and P, Aq is
    lower triangular, and K~ of a chunk's last token equals its k."""
    T, H = 130, 2
    wl = WORKLOADS["gdn256"].with_(B=1, H=H, T=T, seed=917)
    inp = make_chunk_inputs(wl)
    inp["b"][0, 5, 1] = 0.0
    dev = cuda_device
    q, k, v, a, b = (inp[x].to(dev) for x in ("q", "k", "v", "alpha", "b"))
    from gated_delta_rule_147_b200 import workspace_bytes
    nbytes = workspace_bytes(q, v, a, b, TIED)
    assert nbytes == T * H * (256 + 256 + 64 + 256) * 2
    ws = torch.full((nbytes,), 0x7F, dtype=torch.uint8, device=dev)
    chunk_fwd(q, k, v, a, b, TIED, None, workspace=ws)
    torch.cuda.synchronize()
    n = T * H
    parts, off = {}, 0
    for name, d in (("wneg", 256), ("p", 256), ("aq", 64), ("kt", 256)):
        parts[name] = ws[off: off + n * d * 2].view(torch.bfloat16).view(1, T, H, d).float().cpu()
        off += n * d * 2
    assert all(torch.isfinite(x).all() for x in parts.values())
    assert torch.all(parts["wneg"][0, 5, 1] == 0) and torch.all(parts["p"][0, 5, 1] == 0)
    assert parts["wneg"].abs().sum() > 0 and parts["p"].abs().sum() > 0
    for t in (0, 5, 63, 64, 100, 129):
        j = t % 64
        assert torch.all(parts["aq"][0, t, :, j + 1:] == 0) and torch.all(parts["aq"][0, t, :, j] != 0)
    kk = inp["k"].float()
    for t in (63, 127, 129):  # the last token of each chunk: g_{n-1} / g = 1
        assert torch.equal(parts["kt"][0, t], kk[0, t])
    # an earlier token is scaled by a decay ratio in (0, 1]
    m = kk[0, 10].abs() > 1e-3
    r = parts["kt"][0, 10][m] / kk[0, 10][m]
    assert m.sum() > 100 and torch.all((r > 0) & (r <= 1.0 + 1e-2))


def test_dk256_full_size_sampled_heads(cuda_device):
    """The d_k = d_v = 256 workload in the launch configuration the benchmark
    times; the oracle checks sampled heads over the whole sequence."""
    wl = WORKLOADS["gdn256"]
    inp = make_chunk_inputs(wl)
    o, ST = run_chunk(inp, cuda_device)
    heads = [(0, 3), (1, 14)]
    o_ref, ST_ref = run_oracle(inp, heads)
    o_s, ST_s = gather_heads(o, ST, heads)
    assert_close(o_s, o_ref, TOL["bf16"], f"o {heads}")
    assert_close(ST_s, ST_ref, TOL["bf16"], f"S_T {heads}")
    assert np.all(np.isfinite(o))
