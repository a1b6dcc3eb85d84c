"""Pins of the CPU oracle against facts the pages and mathematics fix.

None of these calls the CUDA library. Each ``check_*`` function raises
AssertionError on a violation and takes ``mutate`` so the mutation test at the
bottom can plant each known bug in the oracle and show some pin catches it
(the mutation-check method of mlxcel issue #838, section "Touchpoints &
acceptance criteria": revert one behaviour, see a paired failure).
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from grouped_top_routing_b200 import inputs as G

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _f32(v):
    if isinstance(v, str) and v.startswith("ln"):
        return np.float32(math.log(float(v[2:])))
    return np.float32(v)


def _ulp_close(a, b, ulps):
    a = np.asarray(a, np.float32)
    b = np.asarray(b, np.float64).astype(np.float32)
    sp = np.spacing(np.maximum(np.abs(a), np.abs(b)).astype(np.float32))
    return np.all(np.abs(a.astype(np.float64) - b.astype(np.float64)) <= ulps * sp.astype(np.float64) + 0.0)


# --------------------------------------------------------------------------
# Worked examples (hand-derived, tests/golden/router_worked_examples.json)
# --------------------------------------------------------------------------

def check_worked_examples(mutate=None):
    with open(os.path.join(GOLDEN, "router_worked_examples.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        cfg = c["config"]
        L = np.array([[_f32(v) for v in c["logits"]]], dtype=np.float32)
        b = None if c["bias"] is None else np.array(c["bias"], np.float32)
        s = O.scores(L, cfg["score_function"])
        idx, w = O.route(L, b, cfg, mutate=mutate)
        assert list(idx[0]) == c["expect_idx"], (c["name"], idx[0], c["expect_idx"])
        if "ulps" in c:
            assert _ulp_close(s[0], c["expect_scores"], max(c["ulps"], 1)), (c["name"], s[0])
            assert _ulp_close(w[0], c["expect_w"], c["ulps"]), (c["name"], w[0], c["expect_w"])
        else:
            assert np.allclose(s[0], c["expect_scores"], rtol=c["rtol"], atol=0), (c["name"], s[0])
            assert np.allclose(w[0], c["expect_w"], rtol=c["rtol"], atol=0), (c["name"], w[0])


def test_worked_examples():
    check_worked_examples()


def test_shared_width_golden():
    with open(os.path.join(GOLDEN, "ling_lite_shapes.json")) as f:
        g = json.load(f)
    Is = O.shared_width(g["moe_intermediate_size"], g["num_shared_experts"],
                        g["moe_shared_expert_intermediate_size"])
    assert [Is, g["hidden_size"]] == g["shared_gate_proj_shape"]
    assert [g["hidden_size"], Is] == g["shared_down_proj_shape"]
    assert [g["num_experts"], g["hidden_size"]] == g["router_weight_shape"]
    # the workload generator writes the same width out literally
    assert G.WORKLOADS["ling_lite_t64"]["shared_width"] == Is
    # an explicit per-expert shared width takes precedence over moe_intermediate_size
    assert O.shared_width(1408, 2, 512) == 1024


# --------------------------------------------------------------------------
# Score closed forms
# --------------------------------------------------------------------------

def check_score_closed_forms(mutate=None):
    # sigmoid(0) = 1/2 exactly; sigmoid(-x) = 1 - sigmoid(x); sigmoid(ln 3) = 3/4
    L = np.array([[0.0, 1.0, -1.0, math.log(3.0), 50.0, -50.0]], np.float32)
    s = O.scores(L, "sigmoid")[0]
    assert s[0] == np.float32(0.5)
    assert abs(float(s[1]) + float(s[2]) - 1.0) <= 2 * np.spacing(np.float32(1.0))
    assert _ulp_close(s[3], 0.75, 1)
    assert s[4] == np.float32(1.0) and 0.0 < s[5] < 1e-20
    # softmax of equal logits over E = 2^m experts is exactly 1/E
    for E in (4, 8, 64):
        u = O.scores(np.full((1, E), 0.37, np.float32), "softmax")[0]
        assert np.all(u == np.float32(1.0 / E))
    # shift invariance and normalisation
    rng = np.random.default_rng(1)
    Lr = rng.normal(0, 2, size=(50, 16)).astype(np.float32)
    a = O.scores(Lr, "softmax")
    b = O.scores((Lr.astype(np.float64) + 8.0).astype(np.float32), "softmax")
    assert np.allclose(a, b, rtol=1e-5, atol=1e-7)
    assert np.allclose(a.astype(np.float64).sum(1), 1.0, atol=16 * 6e-8)
    # monotone in the logit
    z = np.sort(rng.normal(0, 3, size=(1, 200)).astype(np.float32), axis=1)
    assert np.all(np.diff(O.scores(z, "sigmoid")[0]) >= 0)


def test_score_closed_forms():
    check_score_closed_forms()


def test_unknown_score_function_rejected():
    with pytest.raises(ValueError):
        O.scores(np.zeros((1, 4), np.float32), "softplus")


def test_scores_match_library_routines():
    # softmax against scipy's and sigmoid against scipy's expit, both in fp64,
    # then rounded to fp32: the oracle must agree to the last bit on these.
    from scipy.special import expit, softmax
    rng = np.random.default_rng(2)
    L = rng.normal(0, 1.3, size=(64, 64)).astype(np.float32)
    ref_s = softmax(L.astype(np.float64), axis=1).astype(np.float32)
    assert np.max(np.abs(O.scores(L, "softmax").astype(np.float64) - ref_s)) <= np.spacing(np.float32(1.0))
    ref_g = expit(L.astype(np.float64)).astype(np.float32)
    assert np.max(np.abs(O.scores(L, "sigmoid").astype(np.float64) - ref_g)) <= np.spacing(np.float32(1.0))


# --------------------------------------------------------------------------
# Selection: brute force on tiny inputs
# --------------------------------------------------------------------------

def _brute_select(s, bias, k, G_, g_):
    """Brute-force selection for one token: group score = best fp32 pair sum
    over all pairs in the group; kept groups = the unique g-subset whose every
    member beats every non-member under (score desc, id asc); selected experts
    likewise over all k-subsets of the allowed experts."""
    E = len(s)
    sel = s.astype(np.float32) if bias is None else (s + bias).astype(np.float32)

    def beats(ka, ia, kb, ib):  # a ranks above b
        return ka > kb or (ka == kb and ia < ib)

    allowed = list(range(E))
    if G_ > 1 and g_ < G_:
        gsz = E // G_
        gs = []
        for q in range(G_):
            mem = range(q * gsz, (q + 1) * gsz)
            if gsz == 1:
                gs.append(sel[q])
            else:
                gs.append(max(np.float32(sel[a] + sel[b]) for a in mem for b in mem if a != b))
        kept = None
        for S in itertools.combinations(range(G_), g_):
            rest = [q for q in range(G_) if q not in S]
            if all(beats(gs[a], a, gs[b], b) for a in S for b in rest):
                assert kept is None
                kept = S
        allowed = [e for e in range(E) if e // gsz in kept]
    best = None
    for S in itertools.combinations(allowed, k):
        rest = [e for e in allowed if e not in S]
        if all(beats(sel[a], a, sel[b], b) for a in S for b in rest):
            assert best is None
            best = S
    # slot order: (sel desc, id asc)
    return sorted(best, key=lambda e: (-float(sel[e]), e))


def check_selection_brute_force(mutate=None):
    rng = np.random.default_rng(3)
    for (E, G_, g_, k) in [(8, 1, 1, 3), (8, 4, 2, 3), (8, 2, 1, 2), (12, 3, 2, 4), (8, 8, 3, 2), (6, 2, 2, 2)]:
        for trial in range(40):
            # coarse grids make exact ties common
            L = (rng.integers(-3, 4, size=(1, E)) * 0.5).astype(np.float32)
            bias = None if trial % 3 == 0 else (rng.integers(-2, 3, size=E) * 0.125).astype(np.float32)
            s = O.scores(L, "sigmoid")
            idx = O.select_experts(s, bias, k, G_, g_, mutate=mutate)[0]
            exp = _brute_select(s[0], bias, k, G_, g_)
            assert list(idx) == exp, (E, G_, g_, k, L, bias, idx, exp)
            if G_ > 1:  # selected experts lie inside the kept groups
                gsz = E // G_
                sel = s[0] if bias is None else (s[0] + bias).astype(np.float32)
                gsc = O.group_scores(sel[None], G_)[0]
                kept = [q for q, _ in sorted(enumerate(gsc), key=lambda p: (-p[1], p[0]))[:g_]]
                assert all(int(e) // gsz in kept for e in idx)


def test_selection_brute_force():
    check_selection_brute_force()


def check_selected_inside_groups_negative_keys(mutate=None):
    # kept groups whose biased keys are all negative: masking must still keep the
    # selection inside them (invariant named for the grouped branch).
    s = np.full((1, 8), 0.01, np.float32)
    bias = np.array([-0.5, -0.5, -0.9, -0.9, -0.9, -0.9, -0.5, -0.5], np.float32)
    idx = O.select_experts(s, bias, 3, 4, 2, mutate=mutate)[0]
    assert set(idx.tolist()) <= {0, 1, 6, 7}, idx


def test_selected_inside_groups_negative_keys():
    check_selected_inside_groups_negative_keys()


def check_topk_is_argsort_of_logits(mutate=None):
    # n_group = 1, softmax, no bias: top-k of the scores is top-k of the logits
    # (softmax is monotone). Logits well separated so fp32 scores stay distinct.
    rng = np.random.default_rng(4)
    for _ in range(20):
        L = (rng.permutation(16).astype(np.float32) * 0.25)[None, :]
        idx, _ = O.route(L, None, dict(num_experts_per_tok=5, score_function="softmax",
                                       norm_topk_prob=False, routed_scaling_factor=1.0), mutate=mutate)
        assert list(idx[0]) == list(np.argsort(-L[0], kind="stable")[:5])


def test_topk_is_argsort_of_logits():
    check_topk_is_argsort_of_logits()


# --------------------------------------------------------------------------
# Weights
# --------------------------------------------------------------------------

def check_bias_selection_only(mutate=None):
    rng = np.random.default_rng(5)
    L = rng.normal(0, 1.3, size=(200, 32)).astype(np.float32)
    bias = rng.normal(0, 0.1, size=32).astype(np.float32)
    cfg = dict(num_experts_per_tok=4, score_function="sigmoid", norm_topk_prob=True, routed_scaling_factor=2.5)
    s = O.scores(L, "sigmoid")
    idx_b, w_b, sel_b = O.route(L, bias, cfg, mutate=mutate, return_keys=True)
    # weights for a forced index set are bitwise equal with and without the bias
    w_nob = O.route_weights(s, s, idx_b, True, 2.5, mutate=mutate)
    assert np.array_equal(w_b, w_nob)
    # and equal the unbiased scores renormalised
    raw = np.take_along_axis(s, idx_b.astype(np.int64), 1)
    assert np.allclose(w_b, raw / raw.sum(1, keepdims=True) * 2.5, rtol=2e-6)
    # the bias does change the selection somewhere
    idx_n, _ = O.route(L, None, cfg, mutate=mutate)
    assert (np.sort(idx_b, 1) != np.sort(idx_n, 1)).any()


def test_bias_selection_only():
    check_bias_selection_only()


def check_normalisation(mutate=None):
    rng = np.random.default_rng(6)
    L = rng.normal(0, 1.3, size=(300, 64)).astype(np.float32)
    for k in (2, 6, 8):
        idx, w = O.route(L, None, dict(num_experts_per_tok=k, score_function="sigmoid", norm_topk_prob=True,
                                       routed_scaling_factor=2.5), mutate=mutate)
        tot = w.astype(np.float64).sum(1)
        assert np.all(np.abs(tot - 2.5) <= 2.5 * (k + 2) * 6e-8), tot
    # k = 1: the raw score times the scale, not the scale
    idx, w = O.route(L, None, dict(num_experts_per_tok=1, score_function="sigmoid", norm_topk_prob=True,
                                   routed_scaling_factor=2.5), mutate=mutate)
    s = O.scores(L, "sigmoid")
    assert np.array_equal(w[:, 0], (np.take_along_axis(s, idx.astype(np.int64), 1)[:, 0] * np.float32(2.5)))


def test_normalisation():
    check_normalisation()


# --------------------------------------------------------------------------
# Whole block: special cases and sparse == dense
# --------------------------------------------------------------------------

def _tiny_inputs(seed=0, **over):
    wl = G.tiny_workload(**over)
    return wl, G.make_inputs(wl, seed=seed, device="cpu")


def check_topk_all_is_dense_softmax(mutate=None):
    # top_k = E, softmax, renormalised, no bias, scale 1: the block is the dense
    # softmax mixture sum_e softmax_e(L) F_e(x) + F_shared(x) (scipy's softmax).
    from scipy.special import softmax
    wl, inp = _tiny_inputs(seed=7, num_experts=8, num_experts_per_tok=8, tokens=12)
    L = O.router_logits(inp["x"], inp["router_w"])
    out = O.moe_block(inp, wl, logits=L, mutate=mutate)
    X = O.as_f64(inp["x"])
    P = softmax(L.astype(np.float64), axis=1)
    y = np.zeros_like(out["y"])
    I = wl["moe_intermediate_size"]
    for e in range(8):
        wgu = O.as_f64(inp["w_gate_up"][e])
        g, u = X @ wgu[:I].T, X @ wgu[I:].T
        y += P[:, e:e + 1] * ((torch.nn.functional.silu(torch.from_numpy(g)).numpy() * u) @ O.as_f64(inp["w_down"][e]).T)
    wsg = O.as_f64(inp["ws_gate_up"])
    Is = wsg.shape[0] // 2
    g, u = X @ wsg[:Is].T, X @ wsg[Is:].T
    y += (torch.nn.functional.silu(torch.from_numpy(g)).numpy() * u) @ O.as_f64(inp["ws_down"]).T
    assert np.allclose(out["y"], y, rtol=1e-5, atol=1e-6), np.abs(out["y"] - y).max()


def test_topk_all_is_dense_softmax():
    check_topk_all_is_dense_softmax()


def check_sparse_equals_dense(mutate=None):
    for over in (dict(), dict(score_function="sigmoid", bias="normal", n_group=4, topk_group=2, num_experts_per_tok=3,
                              routed_scaling_factor=2.5),
                 dict(num_experts=16, n_group=4, topk_group=3, num_experts_per_tok=4, score_function="sigmoid",
                      bias="normal", norm_topk_prob=False, routed_scaling_factor=1.7)):
        wl, inp = _tiny_inputs(seed=8, **over)
        a = O.moe_block(inp, wl, mutate=mutate)["y"]
        b = O.moe_block_dense(inp, wl, mutate=mutate)
        assert np.allclose(a, b, rtol=1e-12, atol=1e-12), np.abs(a - b).max()


def test_sparse_equals_dense():
    check_sparse_equals_dense()


def check_scale_zero_leaves_shared_only(mutate=None):
    # routed_scaling_factor = 0 zeroes every routed weight: the block reduces to
    # the shared MLP at weight 1.0 (torch's silu as the library routine).
    wl, inp = _tiny_inputs(seed=9, routed_scaling_factor=0.0)
    y = O.moe_block(inp, wl, mutate=mutate)["y"]
    X = O.as_f64(inp["x"])
    wsg = O.as_f64(inp["ws_gate_up"])
    Is = wsg.shape[0] // 2
    ref = (torch.nn.functional.silu(torch.from_numpy(X @ wsg[:Is].T)).numpy() * (X @ wsg[Is:].T)) @ O.as_f64(inp["ws_down"]).T
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12)


def test_scale_zero_leaves_shared_only():
    check_scale_zero_leaves_shared_only()


def test_dense_mlp_brute_force():
    # [DENSE]: y[t, n] = sum_i Wd[n, i] * silu(g_i) * u_i with g_i = Wg[i] . x_t and
    # u_i = Wu[i] . x_t, written out with Python floats and math.exp (no numpy
    # matmul), gate rows first in the stacked weight.
    H, Id, T = 8, 4, 3
    inp = G.make_dense_inputs(H, Id, T, seed=3)
    y = O.dense_mlp(inp["x"], inp["w_gate_up"], inp["w_down"])
    x, wgu, wd = O.as_f64(inp["x"]), O.as_f64(inp["w_gate_up"]), O.as_f64(inp["w_down"])
    assert y.shape == (T, H)
    for t in range(T):
        h = []
        for i in range(Id):
            g = sum(float(wgu[i, c]) * float(x[t, c]) for c in range(H))
            u = sum(float(wgu[Id + i, c]) * float(x[t, c]) for c in range(H))
            h.append(g / (1.0 + math.exp(-g)) * u)
        for n in range(H):
            ref = sum(float(wd[n, i]) * h[i] for i in range(Id))
            assert abs(y[t, n] - ref) <= 1e-12 * (1.0 + abs(ref)), (t, n, y[t, n], ref)


def test_dense_mlp_is_a_one_expert_softmax_block():
    # A softmax over a single expert scores exactly 1, so a block with one routed
    # expert, k = 1, scale 1 and no shared MLP computes that expert's MLP: the
    # dense MLP with the expert's weights.
    wl, inp = _tiny_inputs(seed=12, num_experts=1, num_experts_per_tok=1, score_function="softmax",
                           norm_topk_prob=False, routed_scaling_factor=1.0, num_shared_experts=0, shared_width=0)
    y = O.moe_block(inp, wl)["y"]
    ref = O.dense_mlp(inp["x"], inp["w_gate_up"][0], inp["w_down"][0])
    assert np.allclose(y, ref, rtol=1e-13, atol=1e-13), np.abs(y - ref).max()


def test_dequant_affine_brute_force():
    # [Q8]: w[r, c] = scale[r, c // g] * q[r, c] + bias[r, c // g], written out
    # element by element with Python floats.
    wl = G.tiny_workload(num_experts=2, num_experts_per_tok=1, hidden_size=64, moe_intermediate_size=32, shared_width=32)
    q8 = G.make_q8_weights(wl, seed=4, group_size=32)
    q, sc, bi = q8["down"]  # [E, H, I] = [2, 64, 32]: one group per row
    w = O.dequant_affine(q, sc, bi, 32)
    qn, sn, bn = q.numpy(), O.as_f64(sc), O.as_f64(bi)
    q, sc, bi = q8["gate_up"]  # [2, 64, 64]: two groups per row
    w2 = O.dequant_affine(q, sc, bi, 32)
    qn2, sn2, bn2 = q.numpy(), O.as_f64(sc), O.as_f64(bi)
    for e in range(2):
        for r in range(64):
            for c in range(32):
                assert w[e, r, c] == float(sn[e, r, 0]) * int(qn[e, r, c]) + float(bn[e, r, 0])
            for c in range(64):
                assert w2[e, r, c] == float(sn2[e, r, c // 32]) * int(qn2[e, r, c]) + float(bn2[e, r, c // 32])


def test_q8_block_with_integer_weights_is_the_bf16_block():
    # scale 1/64 and bias -2 dequantise to q/64 - 2, which bf16 holds exactly
    # (at most 8 significant bits): the 8-bit block must then equal the bf16
    # block on those values.
    wl, inp = _tiny_inputs(seed=13, num_experts=4, num_experts_per_tok=2, score_function="sigmoid", bias="normal",
                           routed_scaling_factor=2.5)
    g = 32
    q8 = G.make_q8_weights(wl, seed=13, group_size=g)
    for key in ("gate_up", "down", "shared_gate_up", "shared_down"):
        q, sc, bi = q8[key]
        q8[key] = (q, torch.full_like(sc, 1.0 / 64.0), torch.full_like(bi, -2.0))
    ints = {key: (q8[key][0].to(torch.float32) / 64.0 - 2.0).to(torch.bfloat16)
            for key in ("gate_up", "down", "shared_gate_up", "shared_down")}
    bf = dict(inp, w_gate_up=ints["gate_up"], w_down=ints["down"], ws_gate_up=ints["shared_gate_up"],
              ws_down=ints["shared_down"])
    a = O.moe_block_q8(inp, wl, q8)["y"]
    b = O.moe_block(bf, wl)["y"]
    assert np.array_equal(a, b)


def test_permutation_definition():
    rng = np.random.default_rng(10)
    T, E, k = 37, 12, 3
    idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    off, row_of, tok_of = O.permutation(idx, E)
    assert off[0] == 0 and off[-1] == T * k
    assert np.array_equal(np.diff(off), np.bincount(idx.reshape(-1), minlength=E))
    assert sorted(tok_of.tolist()) == list(range(T * k))
    for r in range(T * k):
        t, j = divmod(int(tok_of[r]), k)
        assert row_of[t, j] == r
        e = idx[t, j]
        assert off[e] <= r < off[e + 1]
    # within an expert, tokens ascend
    for e in range(E):
        toks = tok_of[off[e]:off[e + 1]] // k
        assert np.all(np.diff(toks) > 0)


@pytest.mark.parametrize("name", ["ling26_flash_t512"])
def test_zero_mask_reading_agrees_on_workload(name):
    # On the grouped workload the -inf mask and the pages' literal "zeroed"
    # mask select the same experts on every token.
    wl = G.workload(name)
    inp = G.make_inputs(wl, seed=0, device="cpu", weights=False)
    L = O.router_logits(inp["x"], inp["router_w"])
    s = O.scores(L, wl["score_function"])
    assert O.zero_mask_disagreements(s, inp["expert_bias"], wl) == 0


# --------------------------------------------------------------------------
# Router projection and the tie-band helpers
# --------------------------------------------------------------------------

def check_router_logits_exact(mutate=None):
    # logits[t, e] = sum_h x[t, h] * W[e, h], on non-square shapes (E != H)
    # whose inputs are small dyadic numbers: every product and partial sum is
    # exact in fp64, so the oracle must equal a plain Python double loop bit
    # for bit (mlxcel issue #838, section "Router: ...": gates = gate_proj(x)).
    rng = np.random.default_rng(7)
    for T, H, E in ((3, 5, 4), (2, 8, 3), (4, 6, 9)):
        x = (rng.integers(-8, 9, (T, H)) / 8.0).astype(np.float32)
        W = (rng.integers(-16, 17, (E, H)) / 16.0).astype(np.float32)
        got = O.router_logits(x, W, mutate=mutate)
        assert got.shape == (T, E) and got.dtype == np.float32
        for t in range(T):
            for e in range(E):
                acc = 0.0
                for h in range(H):
                    acc += float(x[t, h]) * float(W[e, h])
                assert got[t, e] == np.float32(acc), (T, H, E, t, e, got[t, e], acc)


def test_router_logits_exact():
    check_router_logits_exact()


def _f64(v):
    return np.float64(np.float32(v))


def check_selection_gaps(mutate=None):
    # Hand-worked gaps between the k-th and (k+1)-th biased keys.
    ninf = -np.inf
    sel = np.array([[0.9, 0.5, 0.5, 0.1],
                    [0.7, ninf, 0.3, ninf],
                    [0.2, 0.6, 0.4, 0.8]], dtype=np.float32)
    g1 = O.selection_gaps(sel, 1, mutate=mutate)
    assert g1[0] == _f64(0.9) - _f64(0.5) and g1[1] == _f64(0.7) - _f64(0.3)
    assert g1[2] == _f64(0.8) - _f64(0.6)
    g2 = O.selection_gaps(sel, 2, mutate=mutate)
    assert g2[0] == 0.0, g2          # an exact tie at the boundary: gap 0
    assert g2[1] == np.inf, g2        # the (k+1)-th is a masked expert
    assert g2[2] == _f64(0.6) - _f64(0.4)
    g3 = O.selection_gaps(sel, 3, mutate=mutate)
    assert g3[0] == _f64(0.5) - _f64(0.1) and g3[1] == np.inf
    assert np.all(O.selection_gaps(sel, 4, mutate=mutate) == np.inf)  # k == E: nothing left out


def test_selection_gaps():
    check_selection_gaps()


def check_group_gaps(mutate=None):
    # Four groups of two experts, top-2 groups kept. Group scores are top-1 +
    # top-2 of the BIASED keys, each an fp32 add; the gap is between the 2nd
    # and 3rd best group.
    s = np.array([[0.1, 0.2, 0.3, 0.4, 0.5, 0.6, 0.7, 0.8]], dtype=np.float32)
    b = np.array([0.5, 0.5, 0, 0, 0, 0, 0, 0], dtype=np.float32)
    sel = (s + b).astype(np.float32)
    gs = [np.float32(sel[0, 2 * q] + sel[0, 2 * q + 1]) for q in range(4)]  # 1.3, 0.7, 1.1, 1.5
    g = O.group_gaps(s, b, 4, 2, mutate=mutate)
    assert g[0] == np.float64(gs[0]) - np.float64(gs[2]), (g, gs)
    # without a bias the order changes: 1.5, 1.1, 0.7, 0.3
    g = O.group_gaps(s, None, 4, 2, mutate=mutate)
    assert g[0] == np.float64(np.float32(np.float32(0.5) + np.float32(0.6))) - \
        np.float64(np.float32(np.float32(0.3) + np.float32(0.4)))
    # two groups with bitwise-equal scores at the boundary: gap 0
    t = np.array([[0.2, 0.3, 0.3, 0.2, 0.9, 0.9, 0.0, 0.1]], dtype=np.float32)
    assert O.group_gaps(t, None, 4, 2, mutate=mutate)[0] == 0.0
    # every group kept, or no groups: no group boundary
    assert O.group_gaps(s, b, 4, 4, mutate=mutate)[0] == np.inf
    assert O.group_gaps(s, b, 1, 1, mutate=mutate)[0] == np.inf


def test_group_gaps():
    check_group_gaps()


# --------------------------------------------------------------------------
# Mutation checks: every planted bug must be caught by at least one pin.
# --------------------------------------------------------------------------

CHECKS = [check_worked_examples, check_score_closed_forms, check_selection_brute_force,
          check_selected_inside_groups_negative_keys, check_topk_is_argsort_of_logits,
          check_bias_selection_only, check_normalisation, check_topk_all_is_dense_softmax,
          check_sparse_equals_dense, check_scale_zero_leaves_shared_only, check_router_logits_exact,
          check_selection_gaps, check_group_gaps]


@pytest.mark.parametrize("mutation", O.MUTATIONS)
def test_mutation_is_caught(mutation):
    caught = []
    for chk in CHECKS:
        try:
            with np.errstate(all="ignore"):
                chk(mutate=mutation)
        except AssertionError:
            caught.append(chk.__name__)
    assert caught, f"mutation {mutation} passed every pin"
