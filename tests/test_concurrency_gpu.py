"""Concurrent calls from several host threads on different streams.

The general-form state pass can split into segments that run the first pass
of later segments on the library's auxiliary stream; the auxiliary stream and
its events are shared by every call on the device. Two threads issuing such
calls at the same time must still each get their own correct result.
"""
import threading

import numpy as np
import pytest
import torch

from gated_delta_rule_147_b200 import chunk_fwd
from gated_delta_rule_147_b200.inputs import WORKLOADS, make_chunk_inputs
from gpu_util import TOL, assert_close, run_oracle

pytestmark = pytest.mark.gpu


def test_two_threads_segmented_general_calls(cuda_device):
    dev = cuda_device
    jobs = []
    for i, family in enumerate(("gdn2", "kda")):
        # 1 x 2 heads x 2 column tiles and 70 chunks: segmented state pass
        wl = WORKLOADS[family].with_(B=1, H=2, T=4480, s0=True, seed=2100 + i)
        inp = make_chunk_inputs(wl)
        d = {k: (v.to(dev) if hasattr(v, "to") else v) for k, v in inp.items()}
        w = "tied" if inp["gates"]["w"] == "tied" else d["w"]
        jobs.append((inp, d, w))
    results = [[] for _ in jobs]
    errors = []
    start = threading.Barrier(len(jobs))

    def worker(j):
        try:
            inp, d, w = jobs[j]
            stream = torch.cuda.Stream(device=dev)
            start.wait()
            with torch.cuda.stream(stream):
                for _ in range(6):
                    o, ST = chunk_fwd(d["q"], d["k"], d["v"], d["alpha"], d["b"], w, d["S0"],
                                      stream=stream)
                    results[j].append((o, ST))
            stream.synchronize()
        except Exception as e:  # reported on the main thread
            errors.append(e)

    threads = [threading.Thread(target=worker, args=(j,)) for j in range(len(jobs))]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    torch.cuda.synchronize()
    assert not errors, errors
    for j, (inp, _, _) in enumerate(jobs):
        o_ref, ST_ref = run_oracle(inp)
        first_o, first_S = results[j][0]
        for o, ST in results[j]:
            # every repetition equals the first bit for bit, and the first the oracle
            assert torch.equal(o.view(torch.int16), first_o.view(torch.int16))
            assert torch.equal(ST, first_S)
        assert_close(first_o.float().cpu().numpy(), o_ref, TOL["bf16"], f"o (thread {j})")
        assert_close(first_S.cpu().numpy(), ST_ref, TOL["bf16"], f"S_T (thread {j})")
        assert np.isfinite(first_o.float().cpu().numpy()).all()
