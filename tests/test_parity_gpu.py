"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Routing and permutation are compared bit for bit on identical inputs; the
expert FFN and the whole block within max-abs 2e-2 / rel-L2 5e-3 against the
fp64 oracle, near-tie tokens reported separately. Inputs are seeded and
synthetic (grouped_top_routing_b200.inputs); the oracle never sees a value the
CUDA path produced except where a test compares them.
"""
import math

import numpy as np
import pytest
import torch

import support as S
from grouped_top_routing_b200 import build as B
from grouped_top_routing_b200 import inputs as G
from oracle import moe_oracle as O

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def M():
    B.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from grouped_top_routing_b200 import moe
    return moe


_CACHE = {}


def _inputs(name, device=DEV, **over):
    """Full-size inputs of a workload family, generated once on the device."""
    key = (name, device, tuple(sorted(over.items())))
    if key not in _CACHE:
        _CACHE.clear()
        torch.cuda.empty_cache()
        wl = G.workload(name, **over)
        _CACHE[key] = (wl, G.make_inputs(wl, seed=0, device=device))
    return _CACHE[key]


def _np_bias(inp):
    b = inp["expert_bias"]
    return None if b is None else b.detach().cpu().numpy().astype(np.float32)


# ---------------------------------------------------------------------------
# routing workloads: (name, overrides)
# ---------------------------------------------------------------------------
ROUTE_CASES = [
    ("ling_lite_t64", {}),
    ("ling_lite_t64", dict(norm_topk_prob=True, routed_scaling_factor=2.5)),
    ("ling26_flash_t512", {}),
    ("ling30_flash_decode_t1", {}),
    ("ling30_flash_decode_t8", {}),
    ("ling30_flash_decode_t32", {}),
    ("ling30_flash_decode_t64", {}),
    ("ling30_flash_decode_t64", dict(norm_topk_prob=False, routed_scaling_factor=1.0)),
    ("ling26_flash_prefill_t8192", {}),
    ("ling26_flash_prefill_t32768", {}),
    ("ling30_flash_skew_t16384", {}),
    ("ling30_flash_skew_t16384", dict(norm_topk_prob=False, routed_scaling_factor=1.0)),
    # edge shapes: E not a multiple of 32, k == E, one expert per group, k = 1
    ("edge_e48_g4", dict(tokens=77, hidden_size=64, num_experts=48, num_experts_per_tok=5, n_group=4, topk_group=2,
                         score_function="softmax", bias="normal")),
    ("edge_k_eq_e", dict(tokens=33, hidden_size=64, num_experts=8, num_experts_per_tok=8, n_group=2, topk_group=2,
                         score_function="softmax", bias="none")),
    ("edge_group_of_one", dict(tokens=40, hidden_size=64, num_experts=16, num_experts_per_tok=2, n_group=16,
                               topk_group=4, score_function="sigmoid", bias="normal")),
    ("edge_k1", dict(tokens=50, hidden_size=64, num_experts=64, num_experts_per_tok=1, score_function="sigmoid",
                     bias="normal", norm_topk_prob=True, routed_scaling_factor=2.5)),
    ("edge_e1024", dict(tokens=20, hidden_size=64, num_experts=1024, num_experts_per_tok=16, n_group=32,
                        topk_group=8, score_function="sigmoid", bias="normal")),
]


def _route_wl(name, over):
    if name.startswith("edge_"):
        return G.tiny_workload(**over)
    return G.workload(name, **over)


@pytest.mark.parametrize("name,over", ROUTE_CASES, ids=[f"{n}-{i}" for i, (n, _) in enumerate(ROUTE_CASES)])
def test_route_bit_exact(M, name, over):
    wl = _route_wl(name, over)
    T, E, k = wl["tokens"], wl["num_experts"], wl["num_experts_per_tok"]
    inp = G.make_inputs(wl, seed=0, device="cpu", weights=False, tokens=1)
    bias = _np_bias(inp)
    L = G.random_logits(T, E, S.logit_std(wl), seed=1).numpy()
    ties = None
    if wl["bias"] == "zipf":
        toks, pairs = S.add_exact_ties(L, bias, k)
        S.check_ties_constructed(L, bias, wl, toks, pairs)
        ties = (toks, pairs)
    ref_idx, ref_w = O.route(L, bias, wl)
    Ld = torch.from_numpy(L).to(DEV)
    bd = None if bias is None else torch.from_numpy(bias).to(DEV)
    idx, w = M.moe_route(wl, Ld, bd)
    idx, w = idx.cpu().numpy(), w.cpu().numpy()
    bad = np.nonzero((idx != ref_idx).any(1))[0]
    assert bad.size == 0, f"{bad.size} tokens differ, first {bad[:5]}: gpu {idx[bad[:2]]} oracle {ref_idx[bad[:2]]}"
    assert np.array_equal(w.view(np.uint32), ref_w.view(np.uint32)), np.abs(w - ref_w).max()
    if ties is not None:
        toks, pairs = ties
        assert np.all(idx[toks, k - 1] == pairs), "exact ties must go to the lower expert id"
        print(f"{len(toks)} exact-tie tokens resolved to the lower id")
    near, _ = S.near_tie_tokens(L, bias, wl)
    print(f"{name}: {T} tokens bit-exact; {int(near.sum())} near-tie tokens (gap < 1e-6) included")


@pytest.mark.parametrize("name,T", [("ling_lite_t64", 64), ("ling26_flash_t512", 512), ("ling30_flash_decode_t1", 1),
                                    ("ling30_flash_decode_t8", 8), ("ling30_flash_decode_t32", 32),
                                    ("ling26_flash_t512", 77), ("ling30_flash_decode_t8", 16),
                                    ("ling30_flash_decode_t8", 17), ("ling26_flash_prefill_t8192", 8192),
                                    ("ling30_flash_skew_t16384", 3000)])
def test_router_logits(M, name, T):
    wl = G.workload(name)
    inp = G.make_inputs(wl, seed=0, device="cpu", weights=False, tokens=T)
    ref = O.router_logits(inp["x"], inp["router_w"]).astype(np.float64)
    ws = M.Workspace(wl, T)
    got = M.moe_router_logits(wl, inp["x"].to(DEV), inp["router_w"].to(DEV), ws).cpu().numpy().astype(np.float64)
    ws.check()
    err = np.abs(got - ref).max()
    print(f"{name} T={T}: max |logit - oracle| = {err:.3e}")
    # fp32 accumulation over H terms of size ~0.02: a few 1e-6 typical
    assert err < 5e-5


@pytest.mark.parametrize("T,E,k", [(1, 512, 8), (5, 64, 6), (128, 256, 8), (129, 256, 8), (300, 48, 5),
                                   (4096, 512, 8), (32768, 256, 8), (1000, 1024, 16)])
def test_permute_bit_exact(M, T, E, k):
    wl = G.tiny_workload(tokens=T, num_experts=E, num_experts_per_tok=k, hidden_size=64, score_function="sigmoid")
    L = G.random_logits(T, E, 1.0, seed=T).numpy()
    idx, _ = O.route(L, None, wl)
    off, row_of, tok_of = O.permutation(idx, E)
    x = G.make_inputs(wl, seed=0, device="cpu", weights=False)["x"]
    ws = M.Workspace(wl, T)
    d_off, d_row, d_tok, d_xp = M.moe_permute(wl, torch.from_numpy(idx).to(DEV), ws, x=x.to(DEV), want_x_perm=True)
    ws.check()
    assert np.array_equal(d_off.cpu().numpy(), off)
    assert np.array_equal(d_row.cpu().numpy(), row_of)
    assert np.array_equal(d_tok.cpu().numpy(), tok_of)
    xp = d_xp.cpu().view(torch.int16).numpy()
    assert np.array_equal(xp, x.view(torch.int16).numpy()[tok_of // k])


def test_permute_rejects_bad_ids_on_device(M):
    wl = G.tiny_workload(tokens=200, num_experts=16, num_experts_per_tok=2, hidden_size=64)
    idx = torch.zeros((200, 2), dtype=torch.int32)
    idx[:, 0] = torch.arange(200) % 16
    idx[:, 1] = (torch.arange(200) + 1) % 16
    idx[17, 1] = 16       # out of range
    idx[30, 1] = idx[30, 0]  # repeated within a token
    ws = M.Workspace(wl, 200)
    M.moe_permute(wl, idx.to(DEV), ws)
    with pytest.raises(M.MoeError) as ei:
        ws.check()
    assert ei.value.status == 5
    ws.check()  # the word was cleared; the workspace is usable again
    idx[17, 1] = 3
    idx[30, 1] = 4
    off, _, _, _ = M.moe_permute(wl, idx.to(DEV), ws)
    ws.check()
    assert int(off[-1]) == 400


def test_combine_definition(M):
    # y[t] = bf16(sum_j y_slots[t*k+j] + shared[t]), fp32 in slot order, one rounding
    T, k, H = 37, 6, 256
    g = torch.Generator().manual_seed(3)
    ys = torch.randn((T * k, H), generator=g)
    sh = torch.randn((T, H), generator=g)
    wl = G.tiny_workload(hidden_size=H, num_experts=8, num_experts_per_tok=k)
    f = ys.numpy().reshape(T, k, H)
    acc = np.zeros((T, H), np.float32)
    for j in range(k):
        acc = (acc + f[:, j]).astype(np.float32)
    ref0 = torch.from_numpy(acc.copy()).to(torch.bfloat16)
    acc = (acc + sh.numpy()).astype(np.float32)
    ref = torch.from_numpy(acc).to(torch.bfloat16)
    y = M.moe_combine(wl, ys.to(DEV), sh.to(DEV), T).cpu()
    assert torch.equal(y.view(torch.int16), ref.view(torch.int16))
    y0 = M.moe_combine(wl, ys.to(DEV), None, T).cpu()
    assert torch.equal(y0.view(torch.int16), ref0.view(torch.int16))


FFN_CASES = [
    ("ling_lite_t64", {}),
    ("ling30_flash_decode_t8", {}),
    ("tiny_no_shared", dict(tokens=40, hidden_size=256, num_experts=16, num_experts_per_tok=4,
                            moe_intermediate_size=128, num_shared_experts=0, shared_width=0)),
    ("tiny_ragged", dict(tokens=13, hidden_size=136, num_experts=12, num_experts_per_tok=3,
                         moe_intermediate_size=72, shared_width=144, num_shared_experts=2)),
    # tile shapes of the tensor-core path, picked from the mean rows per expert:
    # ~30 rows -> 64-token tiles; ~68 -> 128-token tiles; >= 96 -> token-major
    # 128 x 256 tiles (here with ragged widths, so the store fallbacks run)
    ("tiny_bn64", dict(tokens=40, hidden_size=64, num_experts=8, num_experts_per_tok=6,
                       moe_intermediate_size=64, shared_width=64)),
    ("tiny_bn128", dict(tokens=90, hidden_size=64, num_experts=8, num_experts_per_tok=6,
                        moe_intermediate_size=64, shared_width=64)),
    ("tiny_token_major", dict(tokens=600, hidden_size=200, num_experts=6, num_experts_per_tok=2,
                              moe_intermediate_size=136, shared_width=272, num_shared_experts=2)),
    # more permuted rows (2400) than the streaming kernels stage per block, so
    # they read each row's slot id from global memory
    ("tiny_many_slots", dict(tokens=300, hidden_size=64, num_experts=16, num_experts_per_tok=8,
                             moe_intermediate_size=64, shared_width=64)),
]


@pytest.fixture(params=["streaming", "tensor_cores", "tensor_cores_f16"])
def path(request, M):
    return request.param


def _path_opts(M, path, inp):
    """moe_options for an expert path, and the inputs the oracle must see: on
    the fp16 down path the down weights are the fp16 copies the kernels read
    (equal to the bf16 ones except below 2^-14 in magnitude)."""
    if path != "tensor_cores_f16":
        return M.options(ffn_path=path), inp
    wd = M.convert_bf16_to_f16(inp["w_down"])
    wsd = None if inp["ws_down"] is None else M.convert_bf16_to_f16(inp["ws_down"])
    return (M.options(ffn_path="tensor_cores", w_down_f16=wd, ws_down_f16=wsd),
            dict(inp, w_down=wd, ws_down=wsd))


@pytest.mark.parametrize("name,over", FFN_CASES, ids=[c[0] for c in FFN_CASES])
def test_expert_ffn(M, name, over, path):
    if name.startswith("tiny"):
        wl = G.tiny_workload(**over)
        inp = S.inputs_to(G.make_inputs(wl, seed=0, device="cpu"), DEV)
    else:
        wl, inp = _inputs(name)
    T, E, k, H = inp["tokens"], wl["num_experts"], wl["num_experts_per_tok"], wl["hidden_size"]
    L = G.random_logits(T, E, S.logit_std(wl), seed=5).numpy()
    idx, w = O.route(L, _np_bias(inp), wl)
    ws = M.Workspace(wl, T)
    d_idx = torch.from_numpy(idx).to(DEV)
    d_w = torch.from_numpy(w).to(DEV)
    off, _, tok_of, _ = M.moe_permute(wl, d_idx, ws)
    has_shared = inp["ws_gate_up"] is not None
    opts, inp_o = _path_opts(M, path, inp)
    y_slots, shared = M.moe_expert_ffn(wl, inp["x"], off, tok_of, d_w.reshape(-1), inp["w_gate_up"], inp["w_down"],
                                       ws, ws_gate_up=inp["ws_gate_up"], ws_down=inp["ws_down"], opts=opts)
    ws.check()
    inp = inp_o
    X = O.as_f64(inp["x"])
    I = wl["moe_intermediate_size"]
    ref = np.zeros((T * k, H))
    for e in np.unique(idx):
        t_sel, j_sel = np.nonzero(idx == e)
        Wg, Wu, Wd = O.expert_weights_f64(inp["w_gate_up"], inp["w_down"], int(e), I)
        ref[t_sel * k + j_sel] = w[t_sel, j_sel][:, None].astype(np.float64) * O.swiglu_mlp(X[t_sel], Wg, Wu, Wd)
    S.compare(O.as_f64(y_slots), ref, f"{name} [{path}] y_slots", bf16_out=False)
    if has_shared:
        Wg, Wu, Wd = O.shared_weights_f64(inp["ws_gate_up"], inp["ws_down"])
        S.compare(O.as_f64(shared), O.swiglu_mlp(X, Wg, Wu, Wd), f"{name} [{path}] shared", bf16_out=False)


@pytest.mark.parametrize("name", ["tiny_bn64", "tiny_token_major"])
def test_expert_ffn_reads_given_x_perm(M, name):
    # moe_expert_ffn with a caller's x_perm reads the permuted rows as tiles;
    # without it the gate/up pass gathers the rows from x (the case above):
    # both must give the same slot rows bit for bit.
    over = dict(FFN_CASES)[name]
    wl = G.tiny_workload(**over)
    inp = S.inputs_to(G.make_inputs(wl, seed=3, device="cpu"), DEV)
    T, E = inp["tokens"], wl["num_experts"]
    L = G.random_logits(T, E, S.logit_std(wl), seed=8).numpy()
    idx, w = O.route(L, _np_bias(inp), wl)
    ws = M.Workspace(wl, T)
    off, _, tok_of, x_perm = M.moe_permute(wl, torch.from_numpy(idx).to(DEV), ws, x=inp["x"], want_x_perm=True)
    d_w = torch.from_numpy(w).to(DEV).reshape(-1)
    args = (wl, inp["x"], off, tok_of, d_w, inp["w_gate_up"], inp["w_down"], ws)
    kw = dict(ws_gate_up=inp["ws_gate_up"], ws_down=inp["ws_down"], opts=M.options(ffn_path="tensor_cores"))
    a_slots, a_sh = M.moe_expert_ffn(*args, **kw)
    a_slots, a_sh = a_slots.clone(), a_sh.clone()
    b_slots, b_sh = M.moe_expert_ffn(*args, x_perm=x_perm, **kw)
    ws.check()
    assert torch.equal(a_slots, b_slots) and torch.equal(a_sh, b_sh)


# ---------------------------------------------------------------------------
# whole block
# ---------------------------------------------------------------------------

def _oracle_rows(M, inp, rows):
    """The token rows `rows` of the block's inputs (the oracle evaluates only those)."""
    sub = dict(inp)
    sub["x"] = inp["x"][torch.from_numpy(np.asarray(rows)).to(inp["x"].device)]
    sub["tokens"] = len(rows)
    return sub


def _forward_and_compare(M, wl, inp, tokens=None, logits=None, opts=None, constructed_ties=0, oracle_inp=None):
    """Run moe_forward on all tokens and compare the output of every token in
    `tokens` (default: all) with the oracle.

    Tokens whose GPU routing equals the oracle's are compared with the oracle
    block on its own routing; among them the near-ties (k-th/(k+1)-th biased
    score, or topk_group-th/next group score, within 1e-6) are reported on a
    line of their own, to the same bars. Tokens whose routing flipped (only
    possible when each side computes its own router logits, and only inside a
    1e-5 gap) are compared with the oracle block evaluated on the GPU's
    routing, again on a line of their own. The near-tie count is bounded.
    oracle_inp: the weights the oracle uses, when they differ from the bf16
    ones passed to moe_forward (the fp16 down-weight copies)."""
    T = inp["tokens"]
    ws = M.Workspace(wl, T)
    Ld = None if logits is None else torch.from_numpy(logits).to(DEV)
    y, idx, w = M.moe_forward(wl, inp["x"], inp["router_w"], inp["expert_bias"], inp["w_gate_up"], inp["w_down"],
                              inp["ws_gate_up"], inp["ws_down"], ws, logits_override=Ld, return_routing=True,
                              opts=opts)
    ws.check()
    rows = np.arange(T) if tokens is None else np.asarray(tokens)
    bias = _np_bias(inp)
    if logits is None:
        L = O.router_logits(inp["x"][torch.from_numpy(rows).to(DEV)], inp["router_w"])
    else:
        L = logits[rows]
    ref_idx, ref_w = O.route(L, bias, wl)
    g_idx = idx.cpu().numpy()[rows]
    g_w = w.cpu().numpy()[rows]
    near, gap = S.near_tie_tokens(L, bias, wl)
    differ = (np.sort(g_idx, 1) != np.sort(ref_idx, 1)).any(1)
    name = wl.get("name", "")
    if logits is not None:
        assert not differ.any(), "identical logits must give identical routing"
        assert np.array_equal(g_idx, ref_idx), "identical logits must give the same slot order"
        assert np.array_equal(g_w.view(np.uint32), ref_w.view(np.uint32)), "and bitwise-equal weights"
    # With the router projection on both sides, fp32 accumulation order can flip
    # only tokens whose selection gap is within the logits' rounding (<< 1e-5).
    assert np.all(gap[differ] < 1e-5), f"routing differs off the tie band: gaps {gap[differ]}"
    bound = S.near_tie_bound(len(rows), constructed_ties)
    assert near.sum() <= bound, f"{int(near.sum())} near-tie tokens, more than {bound}"
    y_rows = O.as_f64(y[torch.from_numpy(rows).to(DEV)])
    same = ~differ
    if same.any():
        ref = O.moe_block(_oracle_rows(M, oracle_inp or inp, rows[same]), wl, logits=L[same])["y"]
        got = y_rows[same]
        plain = ~near[same]
        if plain.any():
            S.compare(got[plain], ref[plain], f"{name} T={T} y ({int(plain.sum())} tokens)")
        if (~plain).any():
            S.compare(got[~plain], ref[~plain], f"{name} T={T} near-tie: {int((~plain).sum())} tokens")
    if differ.any():
        ref = O.moe_block(_oracle_rows(M, oracle_inp or inp, rows[differ]), wl, idx=g_idx[differ],
                          w=g_w[differ])["y"]
        S.compare(y_rows[differ], ref, f"{name} T={T} routing flipped inside 1e-5: {int(differ.sum())} tokens, "
                                       "oracle on the GPU's routing")
    print(f"{name}: near-tie {int(near.sum())} (bound {bound}), flipped {int(differ.sum())}, compared {len(rows)}")
    return y


FORWARD_CASES = [
    ("ling_lite_t64", {}),
    ("ling_lite_t64", dict(norm_topk_prob=True, routed_scaling_factor=2.5)),
    ("ling26_flash_t512", {}),
    ("ling30_flash_decode_t64", {}),
    ("ling30_flash_decode_t64", dict(norm_topk_prob=False, routed_scaling_factor=1.0)),
]


@pytest.mark.parametrize("name,over", FORWARD_CASES, ids=[f"{n}-{i}" for i, (n, _) in enumerate(FORWARD_CASES)])
def test_forward_matches_oracle(M, name, over, path):
    wl, inp = _inputs(name)
    wl = dict(wl, **over, name=f"{name}[{path}]")
    opts, inp_o = _path_opts(M, path, inp)
    _forward_and_compare(M, wl, inp, opts=opts, oracle_inp=inp_o)


@pytest.mark.parametrize("T", [1, 8, 32])
def test_forward_decode_batches(M, T):
    wl, inp = _inputs("ling30_flash_decode_t64")
    sub = dict(inp, x=inp["x"][:T].contiguous(), tokens=T)
    _forward_and_compare(M, dict(wl, name=f"decode_t{T}"), sub)


@pytest.mark.parametrize("name,path", [("ling26_flash_prefill_t8192", "auto"),
                                       ("ling26_flash_prefill_t32768", "auto"),
                                       ("ling26_flash_prefill_t8192", "tensor_cores_f16"),
                                       ("ling26_flash_prefill_t32768", "tensor_cores_f16")])
def test_forward_prefill_every_token(M, name, path):
    # Full size, every token compared: every (expert, token tile) of both
    # expert passes, ragged last tiles included, holds compared rows; on the
    # bf16 (two h planes) and the fp16 down path.
    wl, inp = _inputs(name)
    opts, inp_o = _path_opts(M, path, inp)
    _forward_and_compare(M, dict(wl, name=f"{name}[{path}]"), inp, opts=opts, oracle_inp=inp_o)


@pytest.mark.parametrize("over,path", [({}, "auto"), (dict(norm_topk_prob=False, routed_scaling_factor=1.0), "auto"),
                                       ({}, "tensor_cores_f16"),
                                       (dict(norm_topk_prob=False, routed_scaling_factor=1.0), "tensor_cores_f16")])
def test_forward_skew_ties_every_token(M, over, path):
    # Skewed routing with 1% exact ties (given logits): every token compared.
    wl, inp = _inputs("ling30_flash_skew_t16384")
    wl = dict(wl, **over)
    opts, inp_o = _path_opts(M, path, inp)
    T, E, k = inp["tokens"], wl["num_experts"], wl["num_experts_per_tok"]
    bias = _np_bias(inp)
    L = G.random_logits(T, E, S.logit_std(wl), seed=2).numpy()
    toks, pairs = S.add_exact_ties(L, bias, k)
    S.check_ties_constructed(L, bias, wl, toks, pairs)
    _forward_and_compare(M, dict(wl, name=f"skew[{path}]"), inp, logits=L, constructed_ties=len(toks), opts=opts,
                         oracle_inp=inp_o)


def test_forward_skew_router_projection(M):
    # Skewed routing end to end through the router projection (no given
    # logits): router logits -> route -> experts at 16384 tokens.
    wl, inp = _inputs("ling30_flash_skew_t16384")
    _forward_and_compare(M, dict(wl, name="skew-projection"), inp)


FUSED_CASES = [
    ("ling30_flash_decode_t64", {}, 1),
    ("ling30_flash_decode_t64", dict(norm_topk_prob=False, routed_scaling_factor=1.0), 2),
    ("ling30_flash_decode_t64", {}, 5),
    ("ling30_flash_decode_t64", {}, 8),
    ("ling26_flash_t512", {}, 2),
    ("ling26_flash_t512", {}, 8),
    ("ling_lite_t64", {}, 1),
    ("ling_lite_t64", dict(norm_topk_prob=True, routed_scaling_factor=2.5), 2),
    ("ling_lite_t64", {}, 8),
]


@pytest.mark.parametrize("case", FUSED_CASES, ids=[f"{c[0]}-T{c[2]}-{i}" for i, c in enumerate(FUSED_CASES)])
def test_fused_decode(M, case):
    # one launch for up to two tokens (larger batches run as separate kernels
    # and are checked the same way): routing bit-exact on given logits, output
    # against the oracle, and the same routing when it computes the logits
    name, over, T = case
    wl, inp = _inputs(name)
    wl = dict(wl, **over, name=f"fused-{name}")
    sub = dict(inp, x=inp["x"][7:7 + T].contiguous(), tokens=T)
    L = G.random_logits(T, wl["num_experts"], S.logit_std(wl), seed=11).numpy()
    n0 = M.launch_count()
    _forward_and_compare(M, wl, sub, logits=L)
    if T <= M.FUSED_DECODE_MAX_TOKENS:
        assert M.launch_count() - n0 == 1, "the fused decode is a single launch"
    _forward_and_compare(M, wl, sub)


@pytest.mark.parametrize("name,T", [("ling26_flash_t512", 2), ("ling30_flash_decode_t64", 1),
                                    ("ling30_flash_decode_t64", 2), ("ling30_flash_decode_t64", 8),
                                    ("ling_lite_t64", 3)])
def test_fused_decode_repeatable(M, name, T):
    # Every sum in the fused kernel has a fixed order, so repeated launches
    # must agree bit for bit. Its consumer warps, producer and counters run
    # unsynchronised across SMs; a missed wait shows up here as a changed bit
    # (timing varies: some launches follow an L2 flush, some do not).
    wl, inp = _inputs(name)
    x = inp["x"][3:3 + T].contiguous()
    ws = M.Workspace(wl, T)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=DEV)
    args = (wl, x, inp["router_w"], inp["expert_bias"], inp["w_gate_up"], inp["w_down"], inp["ws_gate_up"],
            inp["ws_down"], ws)
    first = M.moe_forward(*args).clone()
    for i in range(40):
        if i % 3 == 0:
            flush.zero_()
        y = M.moe_forward(*args)
        assert torch.equal(y.view(torch.int16), first.view(torch.int16)), f"launch {i} differs"
    ws.check()


# The fused kernel routes the tokens in every CTA with all its warps, the
# router kernel each token with one warp: both must take the same decisions
# bit for bit, ties included: logits on a 1/4 grid tie often, zipf biases have
# bitwise twins, E not a multiple of 32 leaves padding lanes, and the cases
# reach the kernel's limits (32 slots, 1024 experts, every expert selected,
# k = 1). Batches the fused kernel does not take (more than two tokens or 32
# slots) run as separate kernels and must agree all the same.
FUSED_ROUTE_CASES = [
    # experts, k, n_group, topk_group, score, bias, tokens, shared MLP
    (64, 6, 1, 1, "softmax", "none", 1, True),
    (64, 6, 1, 1, "softmax", "none", 2, True),
    (40, 5, 4, 2, "softmax", "normal", 2, True),
    (256, 8, 8, 4, "sigmoid", "zipf", 2, True),
    (256, 8, 8, 4, "sigmoid", "zipf", 8, True),
    (512, 8, 1, 1, "sigmoid", "zipf", 1, False),
    (512, 8, 1, 1, "sigmoid", "zipf", 8, True),
    (512, 32, 1, 1, "sigmoid", "normal", 2, True),
    (1024, 16, 32, 3, "sigmoid", "zipf", 2, True),
    (8, 8, 1, 1, "sigmoid", "none", 2, True),
    (96, 1, 3, 1, "sigmoid", "normal", 2, False),
    (48, 6, 4, 2, "softmax", "normal", 7, True),
]


@pytest.mark.parametrize("hidden", [256, 512])
@pytest.mark.parametrize("case", FUSED_ROUTE_CASES,
                         ids=[f"E{c[0]}-k{c[1]}-g{c[2]}_{c[3]}-{c[4]}-T{c[6]}" for c in FUSED_ROUTE_CASES])
def test_fused_routing_matches_router_kernel(M, case, hidden):
    E, k, ng, tg, score, bias, T, shared = case
    wl = G.tiny_workload(tokens=T, hidden_size=hidden, num_experts=E, num_experts_per_tok=k, n_group=ng,
                         topk_group=tg, score_function=score, bias=bias, routed_scaling_factor=2.5,
                         moe_intermediate_size=64 if hidden == 256 else 128,
                         num_shared_experts=1 if shared else 0,
                         shared_width=(64 if hidden == 256 else 128) if shared else 0,
                         name=f"fused-route-E{E}-H{hidden}")
    inp = G.make_inputs(wl, seed=5, device=DEV)
    b = _np_bias(inp)
    fused = E <= 1024 and T <= M.FUSED_DECODE_MAX_TOKENS and T * k <= 32
    rng = np.random.default_rng(1000 * E + 10 * k + T)
    for rep in range(3):
        L = (np.round(rng.normal(0.0, 1.5, (T, E)) * 4.0) / 4.0).astype(np.float32)
        x = inp["x"]
        if rep == 2 and T >= 2:  # all tokens pick the same experts: every expert serves T slots
            L[1:] = L[0]
            x = x[:1].expand(T, -1).contiguous()
        Ld = torch.from_numpy(L).to(DEV)
        ws = M.Workspace(wl, T)
        n0 = M.launch_count()
        y, idx, w = M.moe_forward(wl, x, inp["router_w"], inp["expert_bias"], inp["w_gate_up"], inp["w_down"],
                                  inp["ws_gate_up"], inp["ws_down"], ws, logits_override=Ld, return_routing=True)
        ws.check()
        assert (M.launch_count() - n0 == 1) == fused
        r_idx, r_w = M.moe_route(wl, Ld, inp["expert_bias"])
        assert torch.equal(idx, r_idx), (idx, r_idx)
        assert torch.equal(w.view(torch.int32), r_w.view(torch.int32))
        o_idx, o_w = O.route(L, b, wl)
        assert np.array_equal(idx.cpu().numpy(), o_idx)
        assert np.array_equal(w.cpu().numpy().view(np.uint32), o_w.view(np.uint32))
        ref = O.moe_block(dict(inp, x=x, tokens=T), wl, logits=L)["y"]
        S.compare(O.as_f64(y), ref, f"fused E={E} k={k} T={T} rep {rep}")


def test_forward_deterministic(M):
    wl, inp = _inputs("ling26_flash_t512")
    ws = M.Workspace(wl, inp["tokens"])
    args = (wl, inp["x"], inp["router_w"], inp["expert_bias"], inp["w_gate_up"], inp["w_down"], inp["ws_gate_up"],
            inp["ws_down"], ws)
    a = M.moe_forward(*args).clone()
    b = M.moe_forward(*args).clone()
    ws.check()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_forward_zero_tokens_and_launch_count(M):
    wl, inp = _inputs("ling26_flash_t512")
    ws = M.Workspace(wl, 1)
    n0 = M.launch_count()
    x0 = inp["x"][:0]
    y = M.moe_forward(wl, x0, inp["router_w"], inp["expert_bias"], inp["w_gate_up"], inp["w_down"],
                      inp["ws_gate_up"], inp["ws_down"], ws)
    assert y.shape == (0, wl["hidden_size"]) and M.launch_count() == n0
    x1 = inp["x"][:1].contiguous()
    M.moe_forward(wl, x1, inp["router_w"], inp["expert_bias"], inp["w_gate_up"], inp["w_down"], inp["ws_gate_up"],
                  inp["ws_down"], ws)
    ws.check()
    assert M.launch_count() > n0


# ---------------------------------------------------------------------------
# dense-prefix MLP (moe_dense_mlp): the Ling-2.6-flash layer-0 MLP (hidden
# 4096, intermediate 9216) on both expert paths, and small ragged shapes
# ---------------------------------------------------------------------------
DENSE_CASES = [
    # hidden, intermediate, tokens, expert path
    (4096, 9216, 1, "auto"),          # streaming (T <= 2)
    (4096, 9216, 2, "auto"),
    (4096, 9216, 5, "auto"),          # tensor cores, one partial token tile
    (4096, 9216, 130, "auto"),        # token-major tiles: one full, one ragged
    (4096, 9216, 9, "streaming"),
    (192, 200, 37, "streaming"),      # K and N not multiples of the tile sizes
    (192, 200, 37, "tensor_cores"),
    (64, 32, 1, "tensor_cores"),
]


@pytest.mark.parametrize("H,Id,T,path", DENSE_CASES, ids=[f"H{c[0]}-I{c[1]}-T{c[2]}-{c[3]}" for c in DENSE_CASES])
def test_dense_mlp(M, H, Id, T, path):
    inp = G.make_dense_inputs(H, Id, T, seed=21, device=DEV)
    ws = M.dense_mlp_workspace(H, Id, T)
    y = M.moe_dense_mlp(inp["x"], inp["w_gate_up"], inp["w_down"], ws, opts=M.options(ffn_path=path))
    ws.check()
    ref = O.dense_mlp(inp["x"], inp["w_gate_up"], inp["w_down"])
    S.compare(O.as_f64(y), ref, f"dense MLP H={H} Id={Id} T={T} {path}")


def test_dense_mlp_zero_tokens_launches_nothing(M):
    inp = G.make_dense_inputs(64, 32, 1, seed=2, device=DEV)
    ws = M.dense_mlp_workspace(64, 32, 1)
    n0 = M.launch_count()
    y = M.moe_dense_mlp(inp["x"][:0], inp["w_gate_up"], inp["w_down"], ws)
    assert y.shape == (0, 64) and M.launch_count() == n0


# ---------------------------------------------------------------------------
# 8-bit affine expert weights (moe_forward_q8), dequantised in the streaming
# kernels: routing bit-exact on given logits, output against the oracle on the
# dequantised weights
# ---------------------------------------------------------------------------
Q8_CASES = [
    # workload, tokens, group size, shared MLP 8-bit (else bf16, the XL recipe)
    ("ling30_flash_decode_t1", 1, 64, True),
    ("ling30_flash_decode_t8", 2, 64, False),
    ("ling30_flash_decode_t8", 8, 64, True),
    ("ling26_flash_t512", 17, 128, True),    # grouped routing; 17 tokens: several token passes
    ("ling_lite_t64", 5, 64, True),          # softmax, Is = 2I
    ("tiny_q8", 37, 32, True),
    # 2250 permuted rows, more than the streaming kernels stage per block; the
    # shared MLP in many 4-token blocks, 8-bit and bf16
    ("tiny_q8", 450, 32, True),
    ("tiny_q8", 450, 32, False),
]


@pytest.mark.parametrize("name,T,group,shared", Q8_CASES, ids=[f"{c[0]}-T{c[1]}-g{c[2]}-{'q8' if c[3] else 'bf16'}shared"
                                                               for c in Q8_CASES])
def test_forward_q8(M, name, T, group, shared):
    if name == "tiny_q8":
        wl = G.tiny_workload(tokens=T, hidden_size=64, num_experts=48, num_experts_per_tok=5, n_group=4, topk_group=2,
                             score_function="sigmoid", bias="normal", moe_intermediate_size=96, shared_width=96,
                             routed_scaling_factor=2.5, name="tiny_q8")
        inp = G.make_inputs(wl, seed=4, device=DEV)
    else:
        wl, inp = _inputs(name)
    q8 = G.make_q8_weights(wl, seed=3, device=DEV, group_size=group, shared=shared)
    x = inp["x"][:T].contiguous()
    L = G.random_logits(T, wl["num_experts"], S.logit_std(wl), seed=31).numpy()
    ws = M.Workspace(wl, T)
    y, idx, w = M.moe_forward_q8(wl, x, inp["router_w"], inp["expert_bias"], q8, ws,
                                 ws_gate_up=None if shared else inp["ws_gate_up"],
                                 ws_down=None if shared else inp["ws_down"],
                                 logits_override=torch.from_numpy(L).to(DEV), return_routing=True)
    ws.check()
    ref = O.moe_block_q8(dict(inp, x=x, tokens=T), wl, q8, logits=L)
    assert np.array_equal(idx.cpu().numpy(), ref["idx"])
    assert np.array_equal(w.cpu().numpy().view(np.uint32), np.asarray(ref["w"], np.float32).view(np.uint32))
    S.compare(O.as_f64(y), ref["y"], f"q8 {name} T={T} group {group}")
