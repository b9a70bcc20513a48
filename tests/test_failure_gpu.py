"""Failure handling on the GPU without a fault: a bounded wait that nothing
completes must give up, report GDR_DEVICE_TIMEOUT and leave the context
usable for the next call."""
import time

import numpy as np
import pytest
import torch

from gated_delta_rule_147_b200 import GDR_DEVICE_TIMEOUT
from gated_delta_rule_147_b200._lib import gdr_selftest_bounded_wait
from gated_delta_rule_147_b200.inputs import WORKLOADS, make_chunk_inputs
from gpu_util import TOL, assert_close, run_chunk, run_oracle

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives(cuda_device):
    st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    t = time.perf_counter()
    gdr_selftest_bounded_wait(st)
    torch.cuda.synchronize()
    dt = time.perf_counter() - t
    assert int(st.item()) & GDR_DEVICE_TIMEOUT
    assert dt < 30.0
    # the next call on the same context still computes the right answer
    wl = WORKLOADS["kda"].with_(B=1, H=2, T=100, s0=True, seed=21)
    inp = make_chunk_inputs(wl)
    st2 = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    o, ST = run_chunk(inp, cuda_device, d_status=st2)
    assert int(st2.item()) == 0
    o_ref, ST_ref = run_oracle(inp)
    assert_close(o, o_ref, TOL["bf16"], "o after timeout")


def test_selftest_rejects_null_status():
    from gated_delta_rule_147_b200._lib import GdrError
    with pytest.raises(GdrError):
        gdr_selftest_bounded_wait(None, stream=0)
