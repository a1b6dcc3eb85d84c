"""moe_permute_static: the permutation for callers that cannot allocate.

Some callers may not call cudaMalloc at all: a host framework that owns every
device allocation, a plugin host that forbids allocation, or a latency-critical
loop where cudaMalloc's implicit device-wide synchronisation is unacceptable.
For them moe_permute_static keeps its scratch in one file-scope device array
(1 MiB) instead of a caller workspace. Its outputs must match moe_permute's bit
for bit, on consecutive calls that share (and must not be confused by) that
array. This file is named so pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

from grouped_top_routing_b200 import build as B
from grouped_top_routing_b200 import inputs as G
from oracle import moe_oracle as O


@pytest.fixture(scope="module")
def M():
    B.build()
    from grouped_top_routing_b200 import moe
    return moe


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _static_permute(M, wl, idx, x):
    c = M.config_from_workload(wl)
    T, k, E, H = idx.shape[0], c.num_experts_per_tok, c.num_experts, c.hidden_size
    dev = idx.device
    off = torch.full((E + 1,), -7, dtype=torch.int32, device=dev)
    row_of = torch.full((T, k), -7, dtype=torch.int32, device=dev)
    tok_of = torch.full((T * k,), -7, dtype=torch.int32, device=dev)
    x_perm = torch.zeros((T * k, H), dtype=torch.bfloat16, device=dev)
    st = M.lib.moe_permute_static(ctypes.byref(c), _p(idx), T, _p(x), _p(off), _p(row_of), _p(tok_of), _p(x_perm),
                                  ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, M.last_error()
    torch.cuda.synchronize()
    return off, row_of, tok_of, x_perm


@pytest.mark.gpu
def test_static_permute_matches_workspace_permute(M):
    # two calls in a row with different shapes: the second must not see the
    # first call's leftovers in the shared scratch array
    for T, E, k, seed in [(300, 256, 8, 1), (77, 64, 6, 2)]:
        wl = G.tiny_workload(tokens=T, num_experts=E, num_experts_per_tok=k, hidden_size=64,
                             score_function="sigmoid")
        L = G.random_logits(T, E, 1.0, seed=seed).numpy()
        idx_np, _ = O.route(L, None, wl)
        idx = torch.from_numpy(idx_np).cuda()
        x = G.make_inputs(wl, seed=seed, device="cpu", weights=False)["x"].cuda()
        ws = M.Workspace(wl, T)
        r_off, r_row, r_tok, r_xp = M.moe_permute(wl, idx, ws, x=x, want_x_perm=True)
        ws.check()
        off, row_of, tok_of, x_perm = _static_permute(M, wl, idx, x)
        assert torch.equal(off, r_off)
        assert torch.equal(row_of, r_row)
        assert torch.equal(tok_of, r_tok)
        assert torch.equal(x_perm.view(torch.int16), r_xp.view(torch.int16))
        assert int(off[-1]) == T * k  # no id was skipped
        # and both equal the oracle's permutation (its definition: sorted by
        # expert, then token)
        o_off, o_row, o_tok = O.permutation(idx_np, E)
        assert np.array_equal(off.cpu().numpy(), o_off)
        assert np.array_equal(row_of.cpu().numpy(), o_row)
        assert np.array_equal(tok_of.cpu().numpy(), o_tok)


@pytest.mark.gpu
def test_static_permute_signals_bad_ids(M):
    # With no workspace error word, invalid or repeated ids show as a short
    # total: expert_offsets[E] < T*k. The next call, with good ids, is whole.
    T, E, k = 200, 16, 2
    wl = G.tiny_workload(tokens=T, num_experts=E, num_experts_per_tok=k, hidden_size=64)
    idx = torch.zeros((T, k), dtype=torch.int32)
    idx[:, 0] = torch.arange(T) % E
    idx[:, 1] = (torch.arange(T) + 1) % E
    bad = idx.clone()
    bad[17, 1] = E          # out of range
    bad[30, 1] = bad[30, 0]  # repeated within a token
    x = G.make_inputs(wl, seed=3, device="cpu", weights=False)["x"].cuda()
    off, _, _, _ = _static_permute(M, wl, bad.cuda(), x)
    assert int(off[-1]) == T * k - 2
    off, row_of, tok_of, _ = _static_permute(M, wl, idx.cuda(), x)
    o_off, o_row, o_tok = O.permutation(idx.numpy(), E)
    assert np.array_equal(off.cpu().numpy(), o_off)
    assert np.array_equal(row_of.cpu().numpy(), o_row)
    assert np.array_equal(tok_of.cpu().numpy(), o_tok)


def test_static_permute_rejects_sizes_beyond_its_scratch(M):
    # host-side rejection: nothing is launched, so this runs without a GPU too
    wl = G.tiny_workload(tokens=1, num_experts=1024, num_experts_per_tok=8, hidden_size=64)
    c = M.config_from_workload(wl)
    fake = ctypes.c_void_p(1 << 20)
    st = M.lib.moe_permute_static(ctypes.byref(c), fake, 1 << 16, None, fake, fake, fake, None, None)
    assert st == 2
    msg = M.last_error()
    assert "static scratch" in msg and "1048576" in msg
