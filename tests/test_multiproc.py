"""The N > 1 path on CPU: world_size-2 gloo ranks.

Tokens are independent, so each rank runs its own token batch with no
data-path collective (weak scaling). These tests check that premise with the
oracle (rank shards equal the single-process result) and the host logic
bench.py uses across ranks (max-over-ranks timing, whole-job rate).
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from grouped_top_routing_b200 import inputs as G
from oracle import moe_oracle as O

WORLD = 2


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        wl = G.tiny_workload(tokens=12 * world, num_experts=16, num_experts_per_tok=3, n_group=4, topk_group=2,
                             score_function="sigmoid", bias="normal", routed_scaling_factor=2.5)
        inp = G.make_inputs(wl, seed=0, device="cpu")  # identical replicas of the weights on every rank
        per = wl["tokens"] // world
        rows = np.arange(rank * per, (rank + 1) * per)
        y = torch.from_numpy(O.moe_block(inp, wl, tokens=rows)["y"])
        gathered = [torch.empty_like(y) for _ in range(world)]
        dist.all_gather(gathered, y)
        # timing reduction exactly as bench.py does it
        t = torch.tensor([1.0 + rank, 10.0 * (1 + rank)], dtype=torch.float64)
        bench.reduce_max_over_ranks(t, world)
        if rank == 0:
            torch.save({"shards": torch.cat(gathered), "t": t}, os.path.join(out_dir, "result.pt"))
    finally:
        dist.destroy_process_group()


def test_token_shards_over_gloo_ranks_match_single_process(tmp_path):
    port = _free_port()
    mp.start_processes(_worker, args=(WORLD, port, str(tmp_path)), nprocs=WORLD, join=True, start_method="spawn")
    res = torch.load(os.path.join(tmp_path, "result.pt"))
    wl = G.tiny_workload(tokens=12 * WORLD, num_experts=16, num_experts_per_tok=3, n_group=4, topk_group=2,
                         score_function="sigmoid", bias="normal", routed_scaling_factor=2.5)
    inp = G.make_inputs(wl, seed=0, device="cpu")
    full = O.moe_block(inp, wl)["y"]
    # same rows and arithmetic; BLAS blocking differs with the row count, so fp64 rounding-level agreement
    assert np.allclose(res["shards"].numpy(), full, rtol=1e-12, atol=1e-12)
    assert res["t"].tolist() == [float(WORLD), 10.0 * WORLD]


def test_whole_job_rate_and_seeds():
    # N ranks each finishing T tokens in the slowest rank's step time
    assert bench.whole_job_rate(512, 4, 1.0) == pytest.approx(512 * 4 * 1000.0)
    assert len({bench.rank_activation_seed(r) for r in range(8)}) == 8
    assert bench.reduce_max_over_ranks(torch.tensor([3.0]), 1).item() == 3.0
