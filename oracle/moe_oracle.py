"""CPU oracle for the Bailing/Ling grouped top-k MoE feed-forward block.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import, call or run
this module: only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` use it. It shares no code with the CUDA library.

It is the plain definition of what the block computes, written as slowly and
as literally as is practical. numpy supplies the library steps (exp, sort,
matmul); the block's own steps are in the order the pages give them.

Sources (page title, then section):

* [ROUTER] mlxcel issue #838 "add Ant Group Ling / Bailing MoE (bailing_moe)",
  section "Router: selection uses biased scores, weights come from unbiased
  scores".
* [SCALE]  same issue, section "moe_router_enable_routed_scaling is dead code
  upstream": the routed scaling factor multiplies the weights unconditionally.
* [SHARED] same issue, section "Shared experts are one wide MLP, not N separate
  experts".
* [ARCH]   same issue, section "Architecture notes" (groups kept, the rest
  masked before top-k; norm only when k > 1 with a 1e-20 epsilon).
* [DEFAULTS] same issue, section "Config fields the checkpoint does not
  contain" (score_function defaults to softmax; n_group defaults to 1).
* [LING26] model card "Ling-2.6-flash-JANGTQ", section "Architecture
  (bailing_hybrid)", paragraph "MoE routing": sigmoid, 8 groups, top-4
  groups, top-8 experts, e_score_correction_bias for selection only, "same
  math as DeepSeek-V3".
* [Q8]     model card "Ling-3.0-tiny-8bit-XL-mlx", section "XL Quantization
  Recipe" (routed experts 8-bit); model card "Ling-2.6-flash-JANGTQ",
  quantization summary (8-bit affine on the shared experts); mlxcel issue
  #838, section "Upstream sanitize" (quantized expert tensors carry weight,
  scales and biases; group size 64). The affine form: for each row and each
  group of g consecutive inputs, w = scale * q + bias.
* [DENSE]  mlxcel issue #838, section "Architecture notes": the first
  first_k_dense_replace layers use a plain MLP at intermediate_size instead
  of the MoE block; model card "Ling-2.6-flash-JANGTQ", section
  "Architecture (bailing_hybrid)", layer table: layer 0 is a dense MLP of
  intermediate size 9216.

Precision. The pages fix the router's precision: the score function runs in
float32 and the weights stay float32 through normalisation and scaling
([ROUTER]). Here each fp32 score is the fp32 rounding of the score computed in
fp64. Bias add, group scores, the normalisation sum and divide and the
scaling are single fp32 operations. Every routing decision is therefore taken
on fp32 values, as the pages state. The expert FFNs are not fixed by the pages
and run in fp64 on the exact upcast of the bf16 inputs.

Readings where the pages are silent (each one is listed in the design doc):

* group score = top-1 + top-2 of the biased scores inside the group (the
  DeepSeek-V3 rule [LING26]); a group of one expert scores that expert alone;
* the masked experts get -inf (the pages say "zeroed"; the two agree unless
  fewer than k experts of the kept groups have a positive biased score;
  ``zero_mask_disagreements`` counts such tokens);
* ties go to the lower expert id and the lower group id;
* the output slots are ordered by (biased score descending, expert id
  ascending);
* the normalisation sum runs in slot order;
* topk_group == n_group keeps every group.

Parity of this file with the pages' own (unpublished) code is pinned only by
the invariants, closed forms, brute force and mutation checks in
``tests/test_oracle_pins.py``. No worked numeric example exists on the pages.
"""
from __future__ import annotations

import numpy as np

SOFTMAX = "softmax"
SIGMOID = "sigmoid"
NORM_EPS = np.float32(1e-20)

# Deliberate bugs, switched on one at a time by the mutation tests to show that
# the pins catch each of them. None is ever active outside those tests.
MUTATIONS = (
    "bias_in_weights",      # weights gathered from the biased scores
    "norm_when_k1",         # renormalise even when k == 1
    "no_eps",               # drop the 1e-20 epsilon
    "zero_mask",            # mask dropped groups with 0 instead of -inf
    "skip_scale",           # routed scaling not applied
    "tie_high_id",          # ties go to the higher expert id
    "group_top1",           # group score from the top-1 only
    "shared_routed_weight",  # shared MLP weighted like a routed expert
    "bias_not_in_selection",  # bias ignored by the selection
    "logits_layout",        # router weight [E, H] read as if it were stored [H, E]
    "gap_next_pair",        # selection gap taken one rank too deep ((k+1)-th minus (k+2)-th)
    "group_gap_unbiased",   # group gaps ranked on the unbiased scores
)


# --------------------------------------------------------------------------
# bf16 helpers (storage only: the exact upcast of bf16 bit patterns)
# --------------------------------------------------------------------------

def bf16_bits_to_f32(u16: np.ndarray) -> np.ndarray:
    """Exact value of bf16 bit patterns as float32."""
    u = np.asarray(u16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32)


def as_f64(a) -> np.ndarray:
    """Accept torch tensors (any dtype incl. bfloat16) or numpy arrays; return fp64."""
    try:
        import torch
        if isinstance(a, torch.Tensor):
            a = a.detach().cpu()
            if a.dtype == torch.bfloat16:
                return bf16_bits_to_f32(a.view(torch.int16).numpy().view(np.uint16)).astype(np.float64)
            return a.numpy().astype(np.float64)
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(a, dtype=np.float64)


def as_f32(a) -> np.ndarray:
    try:
        import torch
        if isinstance(a, torch.Tensor):
            a = a.detach().cpu()
            if a.dtype == torch.bfloat16:
                return bf16_bits_to_f32(a.view(torch.int16).numpy().view(np.uint16))
            return a.numpy().astype(np.float32)
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(a, dtype=np.float32)


# --------------------------------------------------------------------------
# Config
# --------------------------------------------------------------------------

def shared_width(moe_intermediate_size: int, num_shared_experts: int,
                 moe_shared_expert_intermediate_size: int = 0) -> int:
    """Width of the single shared MLP [SHARED]: the per-expert shared width
    (moe_shared_expert_intermediate_size, or moe_intermediate_size when that
    is unset) times num_shared_experts."""
    per = moe_shared_expert_intermediate_size or moe_intermediate_size
    return per * num_shared_experts


# --------------------------------------------------------------------------
# Router
# --------------------------------------------------------------------------

def router_logits(x, router_w, mutate=None) -> np.ndarray:
    """gates = x . W_r^T for the router projection (mlp.gate, weight [E, H]),
    accumulated in fp64 and rounded once to the fp32 the router works in
    [ROUTER]: the gates are cast to float32 before the score function."""
    X = as_f64(x)
    W = as_f64(router_w)
    if mutate == "logits_layout":
        W = W.reshape(W.shape[1], W.shape[0]).T
    return (X @ W.T).astype(np.float32)


def scores(logits, score_function: str) -> np.ndarray:
    """Score function on fp32 gates [ROUTER], [DEFAULTS].

    softmax: exp(L_e - max L) / sum_j exp(L_j - max L) along the experts;
    sigmoid: 1 / (1 + exp(-L_e)). Evaluated in fp64, rounded once to fp32.
    An unknown score function is rejected, not defaulted [DEFAULTS]."""
    L = np.asarray(logits, dtype=np.float32).astype(np.float64)
    if score_function == SOFTMAX:
        m = L.max(axis=-1, keepdims=True)
        e = np.exp(L - m)
        return (e / e.sum(axis=-1, keepdims=True)).astype(np.float32)
    if score_function == SIGMOID:
        return (1.0 / (1.0 + np.exp(-L))).astype(np.float32)
    raise ValueError(f"unknown score_function {score_function!r}")


def _order_desc_id_asc(keys: np.ndarray, mutate=None) -> np.ndarray:
    """Row-wise order of the columns by (key descending, column id ascending)."""
    T, n = keys.shape
    ids = np.broadcast_to(np.arange(n), (T, n))
    if mutate == "tie_high_id":
        ids = -ids
    return np.lexsort((ids, -keys), axis=1)


def group_scores(sel: np.ndarray, n_group: int, mutate=None) -> np.ndarray:
    """Score of each contiguous group of E / n_group experts: the sum of the two
    largest biased scores in it (DeepSeek-V3 rule [LING26]; one expert alone
    when the group has one expert). fp32 add."""
    T, E = sel.shape
    gsz = E // n_group
    srt = np.sort(sel.reshape(T, n_group, gsz), axis=2)
    if gsz == 1 or mutate == "group_top1":
        return srt[:, :, -1].copy()
    return (srt[:, :, -1] + srt[:, :, -2]).astype(np.float32)


def select_experts(s: np.ndarray, expert_bias, num_experts_per_tok: int, n_group: int = 1,
                   topk_group: int = 1, mutate=None, return_keys=False):
    """Expert selection [ROUTER], [ARCH].

    1. sel = s + bias (fp32; the bias touches this copy only).
    2. If n_group > 1 and topk_group < n_group: rank the groups by group score
       (descending, lower group id first), keep topk_group of them, set sel of
       every expert outside them to -inf.
    3. The num_experts_per_tok largest sel, ordered by (sel desc, id asc).
    Returns idx [T, k] int32 (and the masked sel when asked)."""
    s = np.asarray(s, dtype=np.float32)
    T, E = s.shape
    k = num_experts_per_tok
    sel = s.copy()
    if expert_bias is not None and mutate != "bias_not_in_selection":
        sel = (sel + as_f32(expert_bias)[None, :]).astype(np.float32)
    if n_group > 1 and topk_group < n_group:
        gs = group_scores(sel, n_group, mutate)
        gorder = _order_desc_id_asc(gs, mutate)
        keep = np.zeros((T, n_group), dtype=bool)
        np.put_along_axis(keep, gorder[:, :topk_group], True, axis=1)
        keep_e = np.repeat(keep, E // n_group, axis=1)
        fill = np.float32(0.0) if mutate == "zero_mask" else np.float32(-np.inf)
        sel = np.where(keep_e, sel, fill).astype(np.float32)
    idx = _order_desc_id_asc(sel, mutate)[:, :k].astype(np.int32)
    if return_keys:
        return idx, sel
    return idx


def route_weights(s: np.ndarray, sel: np.ndarray, idx: np.ndarray, norm_topk_prob: bool,
                  routed_scaling_factor: float, mutate=None) -> np.ndarray:
    """Routing weights [ROUTER], [SCALE], [ARCH].

    w_j = s[idx_j] (the UNBIASED score); if norm_topk_prob and k > 1:
    w_j = w_j / (((w_0 + w_1) + ...) + 1e-20), the sum in slot order; then
    w_j = w_j * routed_scaling_factor, always. All fp32."""
    src = sel if mutate == "bias_in_weights" else s
    w = np.take_along_axis(np.asarray(src, dtype=np.float32), idx.astype(np.int64), axis=1).copy()
    k = idx.shape[1]
    if norm_topk_prob and (k > 1 or mutate == "norm_when_k1"):
        den = w[:, 0].copy()
        for j in range(1, k):
            den = (den + w[:, j]).astype(np.float32)
        if mutate != "no_eps":
            den = (den + NORM_EPS).astype(np.float32)
        with np.errstate(invalid="ignore", divide="ignore"):
            w = (w / den[:, None]).astype(np.float32)
    if mutate != "skip_scale":
        w = (w * np.float32(routed_scaling_factor)).astype(np.float32)
    return w


def route(logits, expert_bias, cfg: dict, mutate=None, return_keys=False):
    """The whole router on fp32 gates: returns (idx [T,k] int32, w [T,k] fp32)."""
    s = scores(logits, cfg["score_function"])
    idx, sel = select_experts(s, expert_bias, cfg["num_experts_per_tok"], cfg.get("n_group", 1),
                              cfg.get("topk_group", 1), mutate=mutate, return_keys=True)
    w = route_weights(s, sel, idx, cfg["norm_topk_prob"], cfg["routed_scaling_factor"], mutate)
    if return_keys:
        return idx, w, sel
    return idx, w


def selection_gaps(sel: np.ndarray, k: int, mutate=None) -> np.ndarray:
    """Per token, sel[k-th] - sel[(k+1)-th] of the masked biased scores
    (inf when k == E, and when the (k+1)-th is a masked -inf). Tokens with a
    gap under 1e-6 are near-ties."""
    srt = -np.sort(-sel, axis=1)
    d = 1 if mutate == "gap_next_pair" else 0
    if k + d >= sel.shape[1]:
        return np.full(sel.shape[0], np.inf)
    a = srt[:, k - 1 + d].astype(np.float64)
    b = srt[:, k + d].astype(np.float64)
    with np.errstate(invalid="ignore"):
        g = a - b
    return np.where(np.isfinite(b), g, np.inf)


def group_gaps(s: np.ndarray, expert_bias, n_group: int, topk_group: int, mutate=None) -> np.ndarray:
    """Per token, the gap between the topk_group-th and next group score, the
    group scores taken on the biased selection copy as the selection does
    (inf when every group is kept)."""
    T, E = s.shape
    if n_group <= 1 or topk_group >= n_group:
        return np.full(T, np.inf)
    unbiased = expert_bias is None or mutate == "group_gap_unbiased"
    sel = s if unbiased else (s + as_f32(expert_bias)[None, :]).astype(np.float32)
    gs = group_scores(sel, n_group)
    srt = -np.sort(-gs, axis=1)
    return srt[:, topk_group - 1].astype(np.float64) - srt[:, topk_group].astype(np.float64)


def zero_mask_disagreements(s: np.ndarray, expert_bias, cfg: dict) -> int:
    """Number of tokens whose selection changes if dropped groups are masked with
    0 (the pages' word "zeroed") instead of -inf."""
    a = select_experts(s, expert_bias, cfg["num_experts_per_tok"], cfg.get("n_group", 1),
                       cfg.get("topk_group", 1))
    b = select_experts(s, expert_bias, cfg["num_experts_per_tok"], cfg.get("n_group", 1),
                       cfg.get("topk_group", 1), mutate="zero_mask")
    return int((np.sort(a, 1) != np.sort(b, 1)).any(axis=1).sum())


# --------------------------------------------------------------------------
# Experts
# --------------------------------------------------------------------------

def silu(z: np.ndarray) -> np.ndarray:
    """silu(z) = z * sigmoid(z) = z / (1 + exp(-z))."""
    return z / (1.0 + np.exp(-z))


def swiglu_mlp(X: np.ndarray, w_gate: np.ndarray, w_up: np.ndarray, w_down: np.ndarray) -> np.ndarray:
    """SwiGLU expert [ARCH]: down_proj(silu(gate_proj(x)) * up_proj(x)), with
    gate_proj/up_proj [I, H] and down_proj [H, I]; fp64 throughout."""
    g = X @ w_gate.T
    u = X @ w_up.T
    return (silu(g) * u) @ w_down.T


def dense_mlp(x, w_gate_up, w_down) -> np.ndarray:
    """The dense-prefix MLP [DENSE]: down_proj(silu(gate_proj(x)) * up_proj(x))
    with the gate/up weights stacked [2*Id, H] (gate rows first) and down_proj
    [H, Id]; fp64 on the exact upcast of the bf16 inputs."""
    wgu = as_f64(w_gate_up)
    Id = wgu.shape[0] // 2
    return swiglu_mlp(as_f64(x), wgu[:Id], wgu[Id:], as_f64(w_down))


def dequant_affine(q, scale, bias, group_size: int) -> np.ndarray:
    """8-bit affine weights [Q8]: w[..., c] = scale[..., c // g] * q[..., c] +
    bias[..., c // g] with q uint8 and scale, bias bf16; exact in fp64."""
    qf = as_f64(q)
    s = np.repeat(as_f64(scale), group_size, axis=-1)
    b = np.repeat(as_f64(bias), group_size, axis=-1)
    return s * qf + b


class _DequantStack:
    """Expert-indexed view of stacked 8-bit weights (q [E, R, K], scale and
    bias [E, R, K / g]) that dequantises one expert when indexed."""

    def __init__(self, mat, group_size: int):
        self.q, self.scale, self.bias = mat
        self.g = group_size

    def __getitem__(self, e):
        return dequant_affine(self.q[e], self.scale[e], self.bias[e], self.g)


def moe_block_q8(inp: dict, cfg: dict, q8: dict, logits=None, tokens=None) -> dict:
    """The MoE block with 8-bit affine expert weights [Q8]: every expert's
    weights dequantised, then the block exactly as ``moe_block``. ``q8`` holds
    group_size and (q, scale, bias) triples gate_up [E, 2I, H], down [E, H, I]
    and, when the shared MLP is 8-bit, shared_gate_up [2Is, H] and shared_down
    [H, Is]; otherwise the shared MLP is ``inp``'s bf16 one."""
    g = q8["group_size"]
    view = dict(inp)
    view["w_gate_up"] = _DequantStack(q8["gate_up"], g)
    view["w_down"] = _DequantStack(q8["down"], g)
    if q8.get("shared_gate_up") is not None:
        view["ws_gate_up"] = dequant_affine(*q8["shared_gate_up"], g)
        view["ws_down"] = dequant_affine(*q8["shared_down"], g)
    return moe_block(view, cfg, logits=logits, tokens=tokens)


def expert_weights_f64(w_gate_up, w_down, e: int, I: int):
    """fp64 gate, up and down matrices of routed expert e, from the stacked
    layout w_gate_up [E, 2I, H] (gate rows first) and w_down [E, H, I]."""
    wgu = as_f64(w_gate_up[e])
    return wgu[:I], wgu[I:], as_f64(w_down[e])


def shared_weights_f64(ws_gate_up, ws_down):
    Is = ws_gate_up.shape[0] // 2
    wgu = as_f64(ws_gate_up)
    return wgu[:Is], wgu[Is:], as_f64(ws_down)


def moe_block(inp: dict, cfg: dict, logits=None, idx=None, w=None, mutate=None,
              tokens=None) -> dict:
    """The MoE feed-forward block [ROUTER], [SHARED]:

        y(x) = sum_j w_j * F_{idx_j}(x) + F_shared(x)

    with the shared MLP at fixed weight 1.0, never routed. ``logits`` (fp32
    [T, E]) replaces the router projection when given; ``idx``/``w`` replace
    the router output when given. ``tokens`` restricts the evaluation to a
    subset of token rows (tokens are independent). Returns fp64 y and the
    routing used."""
    x = inp["x"]
    T_all = x.shape[0]
    rows = np.arange(T_all) if tokens is None else np.asarray(tokens)
    X = as_f64(x)[rows]
    I = cfg["moe_intermediate_size"]
    if idx is None:
        if logits is None:
            L = router_logits(as_f64(x)[rows], inp["router_w"])
        else:
            L = np.asarray(logits, dtype=np.float32)[rows] if logits.shape[0] == T_all else np.asarray(logits, np.float32)
        idx, w, sel = route(L, inp["expert_bias"], cfg, mutate=mutate, return_keys=True)
    else:
        L, sel = None, None
    y = np.zeros((len(rows), X.shape[1]), dtype=np.float64)
    for e in np.unique(idx):
        t_sel, j_sel = np.nonzero(idx == e)
        Wg, Wu, Wd = expert_weights_f64(inp["w_gate_up"], inp["w_down"], int(e), I)
        Ye = swiglu_mlp(X[t_sel], Wg, Wu, Wd)
        wt = np.asarray(w, dtype=np.float32)[t_sel, j_sel].astype(np.float64)
        # a token holds an expert in at most one slot, so the rows of t_sel are
        # distinct and a plain indexed add is the per-row sum
        assert np.unique(t_sel).size == t_sel.size, "a token selected one expert twice"
        y[t_sel] += wt[:, None] * Ye
    if cfg.get("num_shared_experts", 0) > 0 and inp.get("ws_gate_up") is not None:
        Wg, Wu, Wd = shared_weights_f64(inp["ws_gate_up"], inp["ws_down"])
        ys = swiglu_mlp(X, Wg, Wu, Wd)
        if mutate == "shared_routed_weight":
            ys = ys * np.float64(cfg["routed_scaling_factor"])
        y += ys
    return {"y": y, "idx": idx, "w": w, "logits": L, "sel": sel}


def moe_block_dense(inp: dict, cfg: dict, logits=None, mutate=None) -> np.ndarray:
    """Dense reference: every routed expert on every token, then the routing
    mask (weight w_j for the selected experts, 0 for all others), plus the
    shared MLP. Equal to ``moe_block`` by definition; for tiny inputs only."""
    x = inp["x"]
    X = as_f64(x)
    T, H = X.shape
    E, I = cfg["num_experts"], cfg["moe_intermediate_size"]
    L = router_logits(x, inp["router_w"]) if logits is None else np.asarray(logits, np.float32)
    idx, w = route(L, inp["expert_bias"], cfg, mutate=mutate)
    mix = np.zeros((T, E), dtype=np.float64)
    for t in range(T):
        for j in range(idx.shape[1]):
            mix[t, idx[t, j]] += float(w[t, j])
    y = np.zeros((T, H), dtype=np.float64)
    for e in range(E):
        Wg, Wu, Wd = expert_weights_f64(inp["w_gate_up"], inp["w_down"], e, I)
        y += mix[:, e:e + 1] * swiglu_mlp(X, Wg, Wu, Wd)
    if cfg.get("num_shared_experts", 0) > 0 and inp.get("ws_gate_up") is not None:
        Wg, Wu, Wd = shared_weights_f64(inp["ws_gate_up"], inp["ws_down"])
        ys = swiglu_mlp(X, Wg, Wu, Wd)
        if mutate == "shared_routed_weight":
            ys = ys * np.float64(cfg["routed_scaling_factor"])
        y += ys
    return y


def permutation(idx: np.ndarray, num_experts: int):
    """Token-to-expert permutation of the routed assignments: the (token, slot)
    pairs sorted by (expert, token). Returns expert_offsets [E+1] (exclusive
    prefix sum of the per-expert counts), row_of [T, k] (the permuted row of
    each assignment) and tok_of [T*k] (the flat slot t*k + j held by each
    permuted row). Every (token, slot) pair appears exactly once."""
    T, k = idx.shape
    counts = np.bincount(idx.reshape(-1), minlength=num_experts)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    order = sorted(range(T * k), key=lambda p: (int(idx.reshape(-1)[p]), p // k))
    tok_of = np.asarray(order, dtype=np.int32)
    row_of = np.empty(T * k, dtype=np.int32)
    row_of[tok_of] = np.arange(T * k, dtype=np.int32)
    return offsets, row_of.reshape(T, k), tok_of
