"""Strong decay on the tensor-core paths: alpha anywhere in (0, 1] must give
the oracle's result (the chunk's decay ratios may span thousands of nats).

Tolerance as for every bf16 workload: max-abs error <= 2e-2 x max|ref|.
"""
import numpy as np
import pytest
import torch

from gated_delta_rule_147_b200.inputs import WORKLOADS, make_chunk_inputs
from gpu_util import TOL, assert_close, run_chunk, run_oracle

pytestmark = pytest.mark.gpu


def _with_alpha(inp, alpha_fn):
    a = inp["alpha"]
    inp["alpha"] = alpha_fn(a.float()).clamp(min=1e-30, max=1.0).to(a.dtype)
    return inp


ALPHAS = {
    "0.01": lambda a: torch.full_like(a, 0.01),
    "1e-4": lambda a: torch.full_like(a, 1e-4),
    # log-uniform in [1e-4, 1]: neighbouring tokens differ by orders of magnitude
    "mixed": lambda a: torch.exp(torch.empty_like(a).uniform_(np.log(1e-4), 0.0,
                                                              generator=torch.Generator().manual_seed(5))),
    # chunks that alternate between almost no decay and very strong decay
    "bursts": lambda a: torch.where((torch.arange(a.shape[1]) // 40 % 2 == 0).view(1, -1, *([1] * (a.dim() - 2))),
                                    torch.full_like(a, 0.999), torch.full_like(a, 1e-3)),
}


@pytest.mark.parametrize("workspace", ["auto", None], ids=["two_pass", "single_pass"])
@pytest.mark.parametrize("alpha", list(ALPHAS))
@pytest.mark.parametrize("family", ["gdn", "kda", "gdn2", "gla"])
def test_strong_decay(cuda_device, family, alpha, workspace):
    """gdn: scalar decay (ratios formed per element); kda, gdn2: channel decay
    (chunks outside the two-factor range are applied token by token); gla:
    the erase-free kernel with channel decay (its single-pass path only)."""
    wl = WORKLOADS[family].with_(B=2, H=3, T=200, s0=True, seed=2200)
    inp = _with_alpha(make_chunk_inputs(wl), ALPHAS[alpha])
    o, ST = run_chunk(inp, cuda_device, workspace=workspace)
    o_ref, ST_ref = run_oracle(inp)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(ST))
    assert_close(o, o_ref, TOL["bf16"], f"o (alpha {alpha})")
    assert_close(ST, ST_ref, TOL["bf16"], f"S_T (alpha {alpha})")


@pytest.mark.parametrize("alpha", ["mixed", "bursts", "1e-4"])
@pytest.mark.parametrize("family", ["kda", "gdn2"])
def test_strong_decay_segmented(cuda_device, family, alpha):
    """Few heads and a long sequence: the general form's state pass runs in
    segments; chunks whose decay span is outside the two-factor range run
    token by token in the middle of a segment's walk."""
    wl = WORKLOADS[family].with_(B=1, H=2, T=4200, s0=True, seed=2300)
    inp = _with_alpha(make_chunk_inputs(wl), ALPHAS[alpha])
    o, ST = run_chunk(inp, cuda_device)
    o_ref, ST_ref = run_oracle(inp)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(ST))
    assert_close(o, o_ref, TOL["bf16"], f"o (alpha {alpha})")
    assert_close(ST, ST_ref, TOL["bf16"], f"S_T (alpha {alpha})")
