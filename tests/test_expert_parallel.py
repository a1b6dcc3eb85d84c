"""Expert parallelism on CPU: the exchange logic of
grouped_top_routing_b200.expert_parallel over gloo ranks.

Each rank holds E/P experts and its own tokens; rows go to their experts'
owners and come back. The expert computation on the received rows is the
oracle here (injected by the test; on GPUs it is the library's kernels), so
these tests check the exchange: every rank's block output must equal the
single-process oracle on its tokens, with world sizes 2 and 4, skewed routing
(some ranks receive nothing from some others) and a rank with no tokens.
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from grouped_top_routing_b200 import expert_parallel as EP
from grouped_top_routing_b200 import inputs as G
from oracle import moe_oracle as O


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_placement_and_counts():
    p = EP.ExpertPlacement(16, 4)
    assert p.per_rank == 4 and p.owner(0) == 0 and p.owner(15) == 3 and p.local_range(2) == (8, 12)
    with pytest.raises(ValueError):
        EP.ExpertPlacement(10, 4)
    counts = torch.tensor([1, 0, 2, 3, 0, 0, 5, 1, 2, 2, 0, 1, 0, 0, 0, 4])
    assert EP.send_counts(counts, p).tolist() == [6, 6, 5, 4]
    recv = torch.tensor([[2, 0, 1], [0, 0, 0], [1, 3, 0]])  # from 3 sources, 3 local experts
    assert EP.received_local_experts(recv).tolist() == [0, 0, 2, 0, 1, 1, 1]


def test_host_lists():
    # the host form of the device lists (moe_ep_send / recv / scatter_back)
    p = EP.ExpertPlacement(4, 2)
    offsets = torch.tensor([0, 2, 2, 5, 6], dtype=torch.int32)
    tok_of = torch.tensor([3, 0, 5, 1, 2, 4], dtype=torch.int32)
    topk_w = torch.tensor([0.5, 0.25, 0.125, 1.0, 2.0, 4.0])
    L = EP.host_lists(2)
    counts, row_w = L.send(offsets, tok_of, topk_w, p)
    assert counts.tolist() == [[2, 0], [3, 1]] and counts.dtype == torch.int64
    assert row_w.tolist() == [1.0, 0.5, 4.0, 0.25, 0.125, 2.0]
    y_perm = torch.arange(12, dtype=torch.float32).reshape(6, 2)
    y = L.scatter_back(y_perm, tok_of, 6)
    assert y[3].tolist() == [0.0, 1.0] and y[0].tolist() == [2.0, 3.0] and y[4].tolist() == [10.0, 11.0]


def _oracle_experts(inp, I, lo):
    """weight * expert(row) for the rank's experts lo + local id, from the oracle."""
    def run(rows, local_expert, weight):
        X = O.as_f64(rows)
        out = np.zeros_like(X)
        le = local_expert.numpy()
        wt = weight.numpy().astype(np.float64)
        for e in np.unique(le):
            sel = le == e
            Wg, Wu, Wd = O.expert_weights_f64(inp["w_gate_up"], inp["w_down"], lo + int(e), I)
            out[sel] = wt[sel, None] * O.swiglu_mlp(X[sel], Wg, Wu, Wd)
        return torch.from_numpy(out)
    return run


def _worker(rank, world, port, out_dir, case):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        wl = G.tiny_workload(**case["wl"])
        inp = G.make_inputs(wl, seed=case["seed"], device="cpu")  # every rank draws the same weights
        counts = case["tokens_per_rank"]
        lo_t = sum(counts[:rank])
        rows = np.arange(lo_t, lo_t + counts[rank])
        x = inp["x"][torch.from_numpy(rows)] if len(rows) else inp["x"][:0]
        T, E, k, I = len(rows), wl["num_experts"], wl["num_experts_per_tok"], wl["moe_intermediate_size"]
        # local routing and permutation (the oracle's, standing in for the kernels)
        L = O.router_logits(O.as_f64(x), inp["router_w"]) if T else np.zeros((0, E), np.float32)
        bias = None if inp["expert_bias"] is None else inp["expert_bias"].numpy()
        idx, w = O.route(L, bias, wl) if T else (np.zeros((0, k), np.int32), np.zeros((0, k), np.float32))
        offsets, _, tok_of = O.permutation(idx, E)
        x_perm = x[torch.from_numpy((tok_of // k).astype(np.int64))]
        placement = EP.ExpertPlacement(E, world)
        lo, _ = placement.local_range(rank)
        y_slots = EP.routed_rows_ep(x_perm, torch.from_numpy(offsets), torch.from_numpy(tok_of.astype(np.int64)),
                                    torch.from_numpy(w), placement, _oracle_experts(inp, I, lo), EP.host_lists(k))
        # combine: slot rows in slot order, then the shared MLP (held by every rank)
        y = y_slots.reshape(T, k, -1).sum(1).numpy() if T else np.zeros((0, wl["hidden_size"]))
        if wl["shared_width"] > 0:
            Wg, Wu, Wd = O.shared_weights_f64(inp["ws_gate_up"], inp["ws_down"])
            y = y + O.swiglu_mlp(O.as_f64(x), Wg, Wu, Wd)
        ref = O.moe_block(inp, wl, tokens=rows)["y"] if T else np.zeros((0, wl["hidden_size"]))
        torch.save({"y": torch.from_numpy(np.asarray(y)), "ref": torch.from_numpy(ref)},
                   os.path.join(out_dir, f"rank{rank}.pt"))
    finally:
        dist.destroy_process_group()


EP_CASES = {
    "p2": dict(world=2, seed=1, tokens_per_rank=[9, 13],
               wl=dict(tokens=22, num_experts=8, num_experts_per_tok=3, n_group=4, topk_group=2,
                       score_function="sigmoid", bias="normal", routed_scaling_factor=2.5)),
    "p4_skewed": dict(world=4, seed=2, tokens_per_rank=[5, 0, 11, 3],
                      wl=dict(tokens=19, num_experts=16, num_experts_per_tok=2, score_function="softmax",
                              bias="zipf", norm_topk_prob=True)),
}


@pytest.mark.parametrize("name", sorted(EP_CASES))
def test_expert_parallel_block_matches_single_process(tmp_path, name):
    case = EP_CASES[name]
    world = case["world"]
    port = _free_port()
    mp.start_processes(_worker, args=(world, port, str(tmp_path), case), nprocs=world, join=True,
                       start_method="spawn")
    for r in range(world):
        res = torch.load(os.path.join(tmp_path, f"rank{r}.pt"))
        y, ref = res["y"].numpy(), res["ref"].numpy()
        assert y.shape == ref.shape
        assert np.allclose(y, ref, rtol=1e-12, atol=1e-12), (r, np.abs(y - ref).max())
