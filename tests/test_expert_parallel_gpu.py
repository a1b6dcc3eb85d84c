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
        experts = EP.library_experts(wl, placement, inp["w_gate_up"], inp["w_down"])
        y_slots = EP.routed_rows_ep(x_perm, offsets, tok_of, w, placement, experts)
        torch.cuda.synchronize()
        routed = y_slots.reshape(T, k, -1).sum(1).double().cpu().numpy()
        ref = O.moe_block(inp, dict(wl, num_shared_experts=0), logits=L)["y"]
        S.compare(routed, ref, f"expert-parallel routed sum T={T}")
    finally:
        dist.destroy_process_group()
