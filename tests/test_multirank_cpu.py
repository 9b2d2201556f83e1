"""The N > 1 path of bench.py on CPU: two gloo ranks.

Each rank runs its own replica of the workload (weak scaling, inputs seeded by
rank) and the job's time is the max over ranks.  No GPU is involved.
"""
import os
import socket

import numpy as np
import pytest

torch = pytest.importorskip("torch")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    import torch.distributed as dist

    import bench
    from diffusion_transformer_attention_attn_b200 import inputs
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # per-rank timings; the slowest rank sets each entry
        vals = [10.0 + rank, 5.0 - rank, 7.5 * (rank + 1)]
        out = bench.max_over_ranks(vals, "cpu", world)
        case = bench.rank_case(inputs.AttnCase("small", 1, 2, 64, 64), rank)
        q, _, _ = inputs.attn_inputs(case)
        digest = int(np.asarray(q, dtype=np.uint64).sum())
        results[rank] = (out, case.seed, digest)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_distinct_replicas():
    import torch.multiprocessing as mp
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as mgr:
        results = mgr.dict()
        mp.spawn(_worker, args=(world, port, results), nprocs=world, join=True)
        res = dict(results)
    expect = [11.0, 5.0, 15.0]
    for r in range(world):
        assert res[r][0] == expect
        assert res[r][1] == r
    assert res[0][2] != res[1][2], "ranks must draw different inputs"
