"""Bounded device waits run out without harming the GPU.

Every wait in the library's kernels (mbarrier phases, counters, flags) gives up
after moe_options.wait_limit_ns, records MOE_ERR_TIMEOUT in the workspace error
word and lets the kernel return (mlxcel issue #838, section "Defensive
requirements": reject instead of terminating). These tests make one wait
unreachable on purpose with the test aid moe_options.test_withhold, under a
1 ms limit, and check that the call ends, that moe_check_device reports the
timeout, and that the next call on the same workspace is correct.
"""
import time

import numpy as np
import pytest
import torch

import support as S
from grouped_top_routing_b200 import build as B
from grouped_top_routing_b200 import inputs as G
from oracle import moe_oracle as O

pytestmark = pytest.mark.gpu
DEV = "cuda"
LIMIT_NS = 1_000_000  # 1 ms


@pytest.fixture(scope="module")
def M():
    B.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from grouped_top_routing_b200 import moe
    return moe


def _run(M, wl, inp, ws, opts, logits):
    return M.moe_forward(wl, inp["x"], inp["router_w"], inp["expert_bias"], inp["w_gate_up"], inp["w_down"],
                         inp["ws_gate_up"], inp["ws_down"], ws, logits_override=logits, opts=opts)


def _expect_timeout_then_recover(M, wl, inp, withhold, ffn_path):
    T = inp["tokens"]
    L = G.random_logits(T, wl["num_experts"], S.logit_std(wl), seed=9).numpy()
    Ld = torch.from_numpy(L).to(DEV)
    ws = M.Workspace(wl, T)
    t0 = time.perf_counter()
    _run(M, wl, inp, ws, M.options(ffn_path=ffn_path, wait_limit_ns=LIMIT_NS, withhold=withhold), Ld)
    with pytest.raises(M.MoeError) as ei:
        ws.check()
    elapsed = time.perf_counter() - t0
    assert ei.value.status == 6, ei.value   # MOE_ERR_TIMEOUT
    assert elapsed < 5.0, f"the call took {elapsed:.2f} s to give up"
    print(f"withhold={withhold}: timed out and returned in {elapsed * 1e3:.1f} ms ({ei.value})")
    # the error word was cleared; the same workspace gives the right answer
    y = _run(M, wl, inp, ws, M.options(ffn_path=ffn_path), Ld)
    ws.check()
    ref = O.moe_block(inp, wl, logits=L)["y"]
    S.compare(O.as_f64(y), ref, f"after the timeout ({withhold})")


def test_expert_kernel_wait_runs_out(M):
    # The tensor-core expert kernel's MMA lane withholds its first
    # accumulator hand-over: the epilogue's wait on it runs out, the CTA's
    # roles wind down (copies and MMAs drained, TMEM freed) and the kernel
    # returns. Token-major tiles, ragged widths.
    wl = G.tiny_workload(tokens=600, hidden_size=200, num_experts=6, num_experts_per_tok=2,
                         moe_intermediate_size=136, shared_width=272, num_shared_experts=2, name="timeout-umma")
    inp = G.make_inputs(wl, seed=0, device=DEV)
    _expect_timeout_then_recover(M, wl, inp, "expert_accumulator", "tensor_cores")


def test_expert_kernel_wait_runs_out_skinny_tiles(M):
    # The same on weight-major (swap-AB) tiles: few tokens per expert.
    wl = G.tiny_workload(tokens=40, hidden_size=64, num_experts=8, num_experts_per_tok=6,
                         moe_intermediate_size=64, shared_width=64, name="timeout-umma-bn64")
    inp = G.make_inputs(wl, seed=1, device=DEV)
    _expect_timeout_then_recover(M, wl, inp, "expert_accumulator", "tensor_cores")


@pytest.mark.parametrize("T", [1, 2])
def test_fused_decode_wait_runs_out(M, T):
    # CTA 0 of the fused decode kernel never arrives at the grid barrier that
    # follows the router rows: every other CTA's wait there runs out after
    # 1 ms, and every producer's wait for the routing after another; all CTAs
    # leave with their copies drained. moe_check_device reports the timeout
    # and resets the barrier's arrival count with the header. Ling-3.0-flash
    # shapes, 64 experts.
    wl = G.workload("ling30_flash_decode_t8", num_experts=64, tokens=T)
    wl = dict(wl, name="timeout-decode")
    inp = G.make_inputs(wl, seed=2, device=DEV)
    n0 = M.launch_count()
    _expect_timeout_then_recover(M, wl, inp, "decode_routing", "auto")
    assert M.launch_count() - n0 == 2, "both calls ran as one fused launch each"
