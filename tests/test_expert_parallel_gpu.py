"""Expert parallelism with this library's kernels on one GPU: a one-rank NCCL
group runs the exchange and ``library_experts`` (permutation and expert
kernels on the received rows). The routed sum must match the oracle's."""
import datetime
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import support as S
from grouped_top_routing_b200 import build as B
from grouped_top_routing_b200 import expert_parallel as EP
from grouped_top_routing_b200 import inputs as G
from oracle import moe_oracle as O

pytestmark = pytest.mark.gpu


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


@pytest.mark.parametrize("T", [3, 40])
def test_expert_parallel_library_experts_one_rank(T):
    B.build()
    from grouped_top_routing_b200 import moe as M
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    try:
        wl = G.tiny_workload(tokens=T, hidden_size=256, num_experts=32, num_experts_per_tok=4, n_group=4, topk_group=2,
                             score_function="sigmoid", bias="normal", routed_scaling_factor=2.5,
                             moe_intermediate_size=128, shared_width=128)
        inp = G.make_inputs(wl, seed=6, device="cuda")
        E, k = wl["num_experts"], wl["num_experts_per_tok"]
        L = G.random_logits(T, E, S.logit_std(wl), seed=7).numpy()
        idx, w = M.moe_route(wl, torch.from_numpy(L).cuda(), inp["expert_bias"])
        ws = M.Workspace(wl, T)
        offsets, _, tok_of, x_perm = M.moe_permute(wl, idx, ws, x=inp["x"], want_x_perm=True)
        placement = EP.ExpertPlacement(E, 1)
        ews = EP.experts_workspace(wl, placement, T * k)   # allocated once, reused by every step
        experts = EP.library_experts(wl, placement, inp["w_gate_up"], inp["w_down"], ews)
        lists = EP.library_lists(wl)
        for _ in range(2):  # the same workspace twice
            y_slots = EP.routed_rows_ep(x_perm, offsets, tok_of, w, placement, experts, lists)
        ews.check()
        torch.cuda.synchronize()
        routed = y_slots.reshape(T, k, -1).sum(1).double().cpu().numpy()
        ref = O.moe_block(inp, dict(wl, num_shared_experts=0), logits=L)["y"]
        S.compare(routed, ref, f"expert-parallel routed sum T={T}")
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("P,n_local,T,k", [(1, 32, 40, 4), (4, 8, 300, 6), (8, 64, 1000, 8)])
def test_device_lists_match_host_lists(P, n_local, T, k):
    # moe_ep_send / moe_ep_recv / moe_ep_scatter_back against the host form,
    # bit for bit, on a real permutation (rows grouped by expert)
    B.build()
    from grouped_top_routing_b200 import moe as M
    E = P * n_local
    wl = G.tiny_workload(tokens=T, hidden_size=64, num_experts=E, num_experts_per_tok=k, moe_intermediate_size=32,
                         shared_width=0, num_shared_experts=0)
    rng = np.random.default_rng(P * 1000 + T)
    idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    topk_w = torch.from_numpy(rng.random((T, k)).astype(np.float32)).cuda()
    ws = M.Workspace(wl, T)
    offsets, _, tok_of, _ = M.moe_permute(wl, torch.from_numpy(idx).cuda(), ws)
    placement = EP.ExpertPlacement(E, P)
    dev, host = EP.library_lists(wl), EP.host_lists(k)
    c_d, w_d = dev.send(offsets, tok_of, topk_w, placement)
    c_h, w_h = host.send(offsets.cpu(), tok_of.cpu(), topk_w.cpu(), placement)
    assert torch.equal(c_d.cpu(), c_h) and torch.equal(w_d.cpu(), w_h)
    # receive side: skewed counts from P sources, zeros included
    recv_counts = torch.from_numpy(rng.integers(0, 5, size=(P, n_local)) * rng.integers(0, 2, size=(P, n_local)))
    R = int(recv_counts.sum())
    le_d = dev.recv(recv_counts.cuda(), R)
    assert torch.equal(le_d.cpu(), EP.received_local_experts(recv_counts))
    y_perm = torch.randn(T * k, 64, device="cuda")
    y_d = dev.scatter_back(y_perm, tok_of, T * k)
    y_h = host.scatter_back(y_perm.cpu(), tok_of.cpu(), T * k)
    torch.cuda.synchronize()
    assert torch.equal(y_d.cpu(), y_h)

