"""The multi-rank path on CPU: two gloo ranks (127.0.0.1).

Ranks shard independent sequences with no data-path collective; the only
cross-rank steps are the shard choice and the max-over-ranks timing. Here
each rank runs the oracle on its shard of a small batch, the results are
gathered on the host, and they must equal the one-process oracle on the
whole batch; the timing reduction must return the maximum.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from gated_delta_rule_147_b200.dist_util import max_over_ranks, shard_rows, shard_seed


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        from gated_delta_rule_147_b200.inputs import WORKLOADS, make_chunk_inputs
        wl = WORKLOADS["gdn2"].with_(B=5, H=2, T=70, s0=True, seed=21)
        inp = make_chunk_inputs(wl)          # the same global batch on every rank
        rows = shard_rows(wl.B, world, rank)
        sl = slice(rows.start, rows.stop)
        pick = {k: (v[sl] if hasattr(v, "dim") else v) for k, v in inp.items()}
        o, ST = oracle.recurrence(pick["q"], pick["k"], pick["v"], pick["alpha"], pick["b"],
                                  pick["w"], pick["S0"], inp["gates"], nthreads=1)
        np.save(os.path.join(out_dir, f"o{rank}.npy"), o)
        np.save(os.path.join(out_dir, f"s{rank}.npy"), ST)
        m = max_over_ranks(10.0 + rank)
        np.save(os.path.join(out_dir, f"max{rank}.npy"), np.array([m]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_shard_rows_partition():
    for n in (1, 5, 8, 13):
        for world in (1, 2, 3, 4):
            got = [i for r in range(world) for i in shard_rows(n, world, r)]
            assert got == list(range(n))


def test_shard_seeds_are_distinct_and_rank0_keeps_seed():
    assert shard_seed(1, 0) == 1
    assert len({shard_seed(1, r) for r in range(8)}) == 8


def test_two_gloo_ranks_shard_the_batch(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    import oracle
    from gated_delta_rule_147_b200.inputs import WORKLOADS, make_chunk_inputs
    wl = WORKLOADS["gdn2"].with_(B=5, H=2, T=70, s0=True, seed=21)
    inp = make_chunk_inputs(wl)
    o_ref, S_ref = oracle.recurrence(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["b"],
                                     inp["w"], inp["S0"], inp["gates"])
    o = np.concatenate([np.load(tmp_path / f"o{r}.npy") for r in range(world)])
    S = np.concatenate([np.load(tmp_path / f"s{r}.npy") for r in range(world)])
    np.testing.assert_array_equal(o, o_ref)
    np.testing.assert_array_equal(S, S_ref)
    for r in range(world):
        assert float(np.load(tmp_path / f"max{r}.npy")[0]) == 10.0 + world - 1
