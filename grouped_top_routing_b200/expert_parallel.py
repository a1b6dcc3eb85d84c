"""Expert parallelism: P ranks, each holding E/P of the routed experts and its
own token batch.

The block's routed sum is over experts, and an expert's rows are independent of
every other expert's, so the experts can live on different GPUs. Each rank
routes and permutes its own tokens (the permuted rows are grouped by expert,
hence by owner rank), sends every row to the rank that owns its expert, runs
its own experts on the rows it received, and sends the weighted results back.
The shared MLP is never routed (mlxcel issue #838, section "Shared experts are
one wide MLP, not N separate experts"), so every rank holds it and applies it
to its own tokens. The combine then sums each token's slot rows in slot order,
exactly as on one GPU. (The issue's "Touchpoints & acceptance criteria" list a
distributed entry; this file is this library's reading of it.)

The exchanges are two all-to-alls with variable split sizes over
torch.distributed: NCCL over NVLink on GPUs, gloo on CPU. One step:

  1. counts: the per-expert row counts [P, E/P] (all-to-all of equal splits)
  2. dispatch: the permuted token rows (bf16) and their routing weights (fp32)
  3. local experts on the received rows, as a block of E/P experts with one
     slot per received row (so each result row is weight * expert(x_row))
  4. return: the fp32 result rows, back in the order they were sent
  5. the rows are placed at their slots and combined with the shared MLP.

The row lists the exchange needs (per-expert counts, the routing weight of
every sent row, the local expert of every received row, and the results'
scatter back to slot order) are built on the device by the library's
moe_ep_send / moe_ep_recv / moe_ep_scatter_back kernels (``library_lists``);
the step itself does no tensor indexing. The expert computation on the
received rows is ``library_experts`` (this library's permutation and expert
kernels, on one workspace the caller allocates once). Both are injectable so
that the exchange logic can be exercised without a GPU: ``host_lists`` builds
the same lists with host tensor indexing, for CPU tests only.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable

import torch
import torch.distributed as dist


@dataclass(frozen=True)
class ExpertPlacement:
    """Contiguous placement: rank r owns experts [r*E/P, (r+1)*E/P)."""

    num_experts: int
    world: int

    def __post_init__(self):
        if self.world < 1 or self.num_experts < 1:
            raise ValueError(f"need at least one rank and one expert (E={self.num_experts}, P={self.world})")
        if self.num_experts % self.world != 0:
            raise ValueError(f"num_experts = {self.num_experts} is not divisible by the {self.world} ranks")

    @property
    def per_rank(self) -> int:
        return self.num_experts // self.world

    def owner(self, e: int) -> int:
        return e // self.per_rank

    def local_range(self, rank: int) -> tuple[int, int]:
        return rank * self.per_rank, (rank + 1) * self.per_rank


class Lists:
    """The device-side row lists of one exchange step (moe_ep_* kernels)."""

    def __init__(self, cfg: dict):
        from grouped_top_routing_b200 import moe as M
        self.M = M
        self.cfg = cfg

    def send(self, offsets, tok_of, topk_w, placement: "ExpertPlacement"):
        """Counts [P, E/P] int64 by owner, and the routing weight of every
        permuted row."""
        T = tok_of.numel() // self.cfg["num_experts_per_tok"]
        counts, row_w = self.M.ep_send(self.cfg, T, offsets, tok_of, topk_w.reshape(-1))
        return counts.reshape(placement.world, placement.per_rank), row_w

    def recv(self, recv_counts, R_recv: int):
        return self.M.ep_recv(recv_counts, R_recv)

    def scatter_back(self, y_perm, tok_of, n_slots: int):
        return self.M.ep_scatter_back(y_perm, tok_of, n_slots)


def library_lists(cfg: dict) -> Lists:
    """The row lists on the device, through the library's kernels."""
    return Lists(cfg)


class HostLists:
    """The same lists with host tensor indexing: a test aid for the CPU ranks
    (gloo), where the library's kernels cannot run."""

    def __init__(self, num_experts_per_tok: int):
        self.k = num_experts_per_tok

    def send(self, offsets, tok_of, topk_w, placement: "ExpertPlacement"):
        counts = (offsets[1:] - offsets[:-1]).to(torch.int64).reshape(placement.world, placement.per_rank)
        row_w = topk_w.reshape(-1)[tok_of.to(torch.int64)]
        return counts.contiguous(), row_w

    def recv(self, recv_counts, R_recv: int):
        return received_local_experts(recv_counts)

    def scatter_back(self, y_perm, tok_of, n_slots: int):
        y_slots = torch.empty((n_slots, y_perm.shape[1]), dtype=y_perm.dtype, device=y_perm.device)
        y_slots[tok_of[: y_perm.shape[0]].to(torch.int64)] = y_perm
        return y_slots


def host_lists(num_experts_per_tok: int) -> HostLists:
    return HostLists(num_experts_per_tok)


def send_counts(expert_counts: torch.Tensor, placement: ExpertPlacement) -> torch.Tensor:
    """Rows this rank sends to each rank: its per-expert counts [E] summed over
    each owner's experts -> [P]."""
    return expert_counts.reshape(placement.world, placement.per_rank).sum(1)


def received_local_experts(recv_counts: torch.Tensor) -> torch.Tensor:
    """Local expert id of every received row, given the counts [P, E/P] each
    source sent per local expert; rows arrive source by source, each source's
    rows grouped by expert in ascending order (host form of moe_ep_recv)."""
    P, n_local = recv_counts.shape
    ids = torch.arange(n_local, dtype=torch.int32, device=recv_counts.device).repeat(P)
    return torch.repeat_interleave(ids, recv_counts.reshape(-1).to(torch.int64))


def _all_to_all(out: torch.Tensor, inp: torch.Tensor, out_splits, in_splits, group) -> None:
    dist.all_to_all_single(out, inp, output_split_sizes=out_splits, input_split_sizes=in_splits, group=group)


@dataclass
class Dispatched:
    """What a rank received for its local experts, and how to send results back."""

    x: torch.Tensor              # [R_recv, H] bf16 rows
    local_expert: torch.Tensor   # [R_recv] int32, expert id within this rank
    weight: torch.Tensor         # [R_recv] fp32 routing weight of each row
    recv_splits: list            # rows received from each rank
    send_splits: list            # rows sent to each rank


def dispatch(x_perm: torch.Tensor, counts: torch.Tensor, row_weight: torch.Tensor, lists, group=None) -> Dispatched:
    """Sends every permuted row (grouped by expert; counts [P, E/P] rows per
    expert, by owner) and its routing weight to the rank owning its expert."""
    recv_counts = torch.empty_like(counts)
    _all_to_all(recv_counts, counts, None, None, group)
    send = [int(v) for v in counts.sum(1).tolist()]   # split sizes: the one host read of a step
    recv = [int(v) for v in recv_counts.sum(1).tolist()]
    H = x_perm.shape[1]
    rx = torch.empty((sum(recv), H), dtype=x_perm.dtype, device=x_perm.device)
    _all_to_all(rx, x_perm[: sum(send)], recv, send, group)
    rw = torch.empty(sum(recv), dtype=row_weight.dtype, device=row_weight.device)
    _all_to_all(rw, row_weight[: sum(send)], recv, send, group)
    return Dispatched(rx, lists.recv(recv_counts, sum(recv)), rw, recv, send)


def give_back(y_recv: torch.Tensor, d: Dispatched, group=None) -> torch.Tensor:
    """Returns the result rows [R_recv, H] to their senders; each rank gets its
    rows back in the order it sent them ([R_sent, H])."""
    out = torch.empty((sum(d.send_splits), y_recv.shape[1]), dtype=y_recv.dtype, device=y_recv.device)
    _all_to_all(out, y_recv.contiguous(), d.send_splits, d.recv_splits, group)
    return out


# The expert computation on the received rows: (rows [R, H] bf16, local expert
# id [R] int32, weight [R] fp32) -> weight * expert(row) [R, H] fp32.
LocalExperts = Callable[[torch.Tensor, torch.Tensor, torch.Tensor], torch.Tensor]


def local_config(cfg: dict, placement: ExpertPlacement) -> dict:
    """The block the owner runs on received rows: its E/P experts, one slot
    per row, no groups and no shared MLP."""
    return dict(cfg, num_experts=placement.per_rank, num_experts_per_tok=1, n_group=1, topk_group=1,
                num_shared_experts=0, moe_shared_expert_intermediate_size=0, shared_width=0)


def experts_workspace(cfg: dict, placement: ExpertPlacement, max_rows: int, device="cuda"):
    """The one workspace library_experts reuses every step: sized for the most
    rows a rank can receive (its peers' T*k at most)."""
    from grouped_top_routing_b200 import moe as M
    return M.Workspace(local_config(cfg, placement), max_rows, device=device)


def library_experts(cfg: dict, placement: ExpertPlacement, w_gate_up: torch.Tensor, w_down: torch.Tensor,
                    ws) -> LocalExperts:
    """This library's permutation and expert kernels on the rank's own experts
    (w_gate_up [E/P, 2I, H], w_down [E/P, H, I] of the block config cfg), as a
    block of E/P experts with one slot per received row and no shared MLP, in
    the caller's workspace ws (experts_workspace, allocated once)."""
    from grouped_top_routing_b200 import moe as M

    if w_gate_up.shape[0] != placement.per_rank or w_down.shape[0] != placement.per_rank:
        raise ValueError(f"expected the rank's {placement.per_rank} experts, got {w_gate_up.shape[0]} / {w_down.shape[0]}")
    lcfg = local_config(cfg, placement)

    def run(rows: torch.Tensor, local_expert: torch.Tensor, weight: torch.Tensor) -> torch.Tensor:
        R = rows.shape[0]
        if R == 0:
            return torch.zeros((0, rows.shape[1]), dtype=torch.float32, device=rows.device)
        if R > ws.max_tokens:
            raise ValueError(f"{R} received rows, but the experts' workspace holds {ws.max_tokens}")
        offsets, _, tok_of, x_perm = M.moe_permute(lcfg, local_expert.reshape(R, 1), ws, x=rows, want_x_perm=True)
        y_slots, _ = M.moe_expert_ffn(lcfg, rows, offsets, tok_of, weight, w_gate_up, w_down, ws, x_perm=x_perm)
        return y_slots

    return run


def routed_rows_ep(x_perm: torch.Tensor, offsets: torch.Tensor, tok_of: torch.Tensor, topk_w: torch.Tensor,
                   placement: ExpertPlacement, experts: LocalExperts, lists, group=None) -> torch.Tensor:
    """Steps 1-5 for one rank: its permuted rows go to their experts' owners,
    the local experts run on what arrived, and the weighted result rows come
    back to their slots. lists: library_lists(cfg) on GPUs. Returns y_slots
    [T*k, H] fp32 (row of slot t*k + j), ready for the combine."""
    counts, weight = lists.send(offsets, tok_of, topk_w, placement)   # per owner; weight of each permuted row
    d = dispatch(x_perm, counts, weight, lists, group)
    y_recv = experts(d.x, d.local_expert, d.weight)
    y_perm = give_back(y_recv, d, group)
    return lists.scatter_back(y_perm, tok_of, tok_of.numel())         # permuted row r holds slot tok_of[r]
