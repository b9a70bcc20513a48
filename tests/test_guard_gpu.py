"""Out-of-bounds write checks (in place of a memory checker): every output
buffer of every kernel path sits inside a larger allocation whose bands before
and after it hold a known byte pattern; after the call the bands must be
untouched. Covers ragged sequence lengths (the TMA boxes and plain stores of
the last chunk overhang the tensor), every value width and grouped heads.
"""
import pytest
import torch

from gated_delta_rule_147_b200 import TIED, chunk_bwd, chunk_fwd, decode_step, workspace_bytes
from gated_delta_rule_147_b200.inputs import WORKLOADS, make_chunk_inputs

pytestmark = pytest.mark.gpu

BAND = 4096          # bytes before and after each buffer (keeps 256-byte alignment)
PATTERN = 0xA5


class Guarded:
    """A tensor of `shape` inside a byte buffer with guard bands."""

    def __init__(self, shape, dtype, dev):
        n = 1
        for s in shape:
            n *= s
        self.nbytes = n * torch.tensor([], dtype=dtype).element_size()
        self.buf = torch.full((self.nbytes + 2 * BAND,), PATTERN, dtype=torch.uint8, device=dev)
        self.t = self.buf[BAND:BAND + self.nbytes].view(dtype).view(shape)

    def check(self, what):
        torch.cuda.synchronize()
        head = self.buf[:BAND].cpu()
        tail = self.buf[BAND + self.nbytes:].cpu()
        bad_h = int((head != PATTERN).sum())
        bad_t = int((tail != PATTERN).sum())
        assert bad_h == 0 and bad_t == 0, f"{what}: {bad_h} bytes written before, {bad_t} after the buffer"


def _dev(x, dev):
    return None if x is None else x.to(dev).contiguous()


def _fwd_guarded(inp, dev, workspace_mode, group=1):
    g = inp["gates"]
    q, k, v = (_dev(inp[x], dev) for x in ("q", "k", "v"))
    if group > 1:
        q, k = q[:, :, ::group].contiguous(), k[:, :, ::group].contiguous()
    a, b, s0 = _dev(inp["alpha"], dev), _dev(inp["b"], dev), _dev(inp["S0"], dev)
    w = TIED if g["w"] == "tied" else _dev(inp["w"], dev)
    B, T, H, dv = v.shape
    dk = q.shape[-1]
    o = Guarded((B, T, H, dv), v.dtype, dev)
    st = Guarded((B, H, dk, dv), torch.float32, dev)
    ws = None
    if workspace_mode == "auto":
        n = workspace_bytes(q, v, a, b, w)
        ws = Guarded((n,), torch.uint8, dev) if n else None
    chunk_fwd(q, k, v, a, b, w, s0, out=o.t, S_T=st.t, workspace=None if ws is None else ws.t)
    o.check("o")
    st.check("S_T")
    if ws is not None:
        ws.check("workspace")
    assert torch.isfinite(o.t.float()).all() and torch.isfinite(st.t).all()


@pytest.mark.parametrize("T", [1, 63, 65, 200])
@pytest.mark.parametrize("family,dv,workspace_mode", [
    ("gdn", 64, "auto"), ("gdn", 128, "auto"),       # two-pass, Gated DeltaNet kernels
    ("kda", 128, "auto"), ("gdn2", 64, "auto"),      # two-pass, general kernels
    ("gdn", 256, None), ("gdn2", 128, None),         # single-pass kernels
    ("gla", 256, "auto"), ("gla", 64, "auto"),       # erase-free kernel
    ("gdn256", 256, "auto"), ("gdn256", 64, "auto"), # two-pass, d_k = 256 kernels
])
def test_forward_writes_stay_in_bounds(cuda_device, family, dv, workspace_mode, T):
    wl = WORKLOADS[family].with_(B=2, H=3, T=T, dv=dv, s0=True, seed=1300 + T + dv)
    _fwd_guarded(make_chunk_inputs(wl), cuda_device, workspace_mode)


@pytest.mark.parametrize("family,workspace_mode", [("gdn", "auto"), ("kda", None), ("gla", "auto")])
def test_forward_grouped_heads_writes_stay_in_bounds(cuda_device, family, workspace_mode):
    wl = WORKLOADS[family].with_(B=2, H=4, T=65, s0=True, seed=1400)
    _fwd_guarded(make_chunk_inputs(wl), cuda_device, workspace_mode, group=2)


@pytest.mark.parametrize("dtype,dk,dv", [("fp32", 16, 16), ("bf16", 64, 48), ("bf16", 256, 64)])
def test_exact_path_writes_stay_in_bounds(cuda_device, dtype, dk, dv):
    wl = WORKLOADS["gdn2"].with_(B=2, H=3, T=65, dk=dk, dv=dv, dtype=dtype, s0=True, seed=1500)
    _fwd_guarded(make_chunk_inputs(wl), cuda_device, "auto")


@pytest.mark.parametrize("dk,dv", [(128, 64), (128, 128), (128, 256), (256, 256)])
def test_decode_writes_stay_in_bounds(cuda_device, dk, dv):
    dev = cuda_device
    wl = WORKLOADS["gdn2"].with_(B=3, H=5, T=1, dk=dk, dv=dv, s0=True, seed=1600)
    inp = make_chunk_inputs(wl)
    q, k, v, a, b, w = (inp[x][:, 0].to(dev).contiguous() for x in ("q", "k", "v", "alpha", "b", "w"))
    S = Guarded(tuple(inp["S0"].shape), torch.float32, dev)
    S.t.copy_(inp["S0"].to(dev))
    o = Guarded((3, 5, dv), torch.bfloat16, dev)
    decode_step(q, k, v, a, b, w, S.t, out=o.t)
    o.check("o")
    S.check("S")


@pytest.mark.parametrize("T", [1, 65])
def test_backward_writes_stay_in_bounds(cuda_device, T):
    dev = cuda_device
    wl = WORKLOADS["gdn2"].with_(B=2, H=3, T=T, dv=64, s0=True, seed=1700 + T)
    inp = make_chunk_inputs(wl)
    q, k, v, a, b, w, s0 = (_dev(inp[x], dev) for x in ("q", "k", "v", "alpha", "b", "w", "S0"))
    dO = torch.randn(v.shape, device=dev).to(v.dtype)
    from gated_delta_rule_147_b200 import gdr_chunk_bwd_grouped_workspace_size
    ws = Guarded((gdr_chunk_bwd_grouped_workspace_size(2, T, 3, 3, 128, 64),), torch.uint8, dev)
    g = chunk_bwd(q, k, v, a, b, w, s0, dO=dO, workspace=ws.t)
    ws.check("backward workspace")
    for name, t in g.items():
        assert t is None or torch.isfinite(t).all(), name
