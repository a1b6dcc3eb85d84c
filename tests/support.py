"""Helpers shared by the GPU parity tests: input preparation, the exact-tie
construction of the skewed workload, and the comparison rules.

Tolerances (end-to-end, bf16 I/O with fp32 accumulation): max-abs <= 2e-2 and
relative L2 <= 5e-3 against the fp64 oracle; for bf16 outputs at |y| >= 8 the
max-abs bar grows with bf16's half-ulp (see abs_tolerance). Routing: indices bit-exact and
weights bitwise equal given identical fp32 logits. Tokens whose k-th and
(k+1)-th biased scores (or topk_group-th and next group scores) lie within
1e-6 are near-ties and are reported separately.
"""
from __future__ import annotations

import math

import numpy as np
import torch

from grouped_top_routing_b200 import inputs as G
from oracle import moe_oracle as O

MAX_ABS = 2e-2
REL_L2 = 5e-3
TIE_BAND = 1e-6


def logit_std(wl):
    """Std of x . W_r for x ~ N(0,1), W_r ~ N(0, 0.02)."""
    return 0.02 * math.sqrt(wl["hidden_size"])


def add_exact_ties(L: np.ndarray, bias: np.ndarray, k: int, every: int = 100):
    """Rewrite every `every`-th token's logits so that one twin pair (a, a+1)
    (bitwise-equal bias) gets bitwise-equal keys exactly at the k-th/(k+1)-th
    boundary: k-1 experts forced far above, all others far below. Returns the
    tie tokens and their pair id a (the lower id, which must win)."""
    T, E = L.shape
    b = bias.astype(np.float64)
    twins = [e for e in G.ZIPF_TWIN_EXPERTS if e + 1 < E]
    toks, pairs = [], []
    for n, t in enumerate(range(0, T, every)):
        a = twins[n % len(twins)]
        others = [e for e in range(E) if e not in (a, a + 1)]
        order = sorted(others, key=lambda e: -b[e])
        high, low = order[:k - 1], order[k - 1:]
        row = np.full(E, -30.0, np.float32)
        row[high] = 30.0
        lo_key = max(b[low].max(), b[a]) if len(low) else b[a]
        hi_key = min(1.0 + b[high].min(), b[a] + 1.0) if high else b[a] + 1.0
        p = 0.5 * (lo_key + hi_key) - b[a]
        p = min(max(p, 1e-3), 1 - 1e-3)
        row[a] = row[a + 1] = np.float32(math.log(p / (1.0 - p)))
        L[t] = row
        toks.append(t)
        pairs.append(a)
    return np.asarray(toks), np.asarray(pairs)


def check_ties_constructed(L, bias, wl, toks, pairs):
    """The construction must put the pair exactly on the boundary (oracle keys)."""
    idx, w, sel = O.route(L[toks], bias, wl, return_keys=True)
    k = wl["num_experts_per_tok"]
    for i, a in enumerate(pairs):
        assert sel[i, a] == sel[i, a + 1], "twin keys differ"
        assert idx[i, k - 1] == a and (a + 1) not in idx[i], (idx[i], a)
    return idx


def near_tie_bound(T: int, constructed: int = 0) -> int:
    """Most near-tie tokens a workload of T random tokens may hold: the gap
    between the k-th and (k+1)-th biased score falls under 1e-6 about once in
    a few thousand tokens on these workloads (counted on the oracle: 2 of 8192
    and 1 of 16384). ``constructed`` adds tokens built as exact ties."""
    return 4 + T // 1000 + constructed


def near_tie_tokens(L, bias, wl):
    s = O.scores(L, wl["score_function"])
    _, sel = O.select_experts(s, bias, wl["num_experts_per_tok"], wl.get("n_group", 1), wl.get("topk_group", 1),
                              return_keys=True)
    gap = O.selection_gaps(sel, wl["num_experts_per_tok"])
    ggap = O.group_gaps(s, bias, wl.get("n_group", 1), wl.get("topk_group", 1))
    return (gap < TIE_BAND) | (ggap < TIE_BAND), np.minimum(gap, ggap)


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return O.as_f64(t)


def bf16_half_ulp(v: np.ndarray) -> np.ndarray:
    """Half the spacing of bf16 numbers at |v| (8 significant bits): the
    largest error a correctly rounded bf16 output can have there."""
    a = np.maximum(np.abs(np.asarray(v, np.float64)), 2.0 ** -126)
    return np.exp2(np.floor(np.log2(a)) - 8.0)


def abs_tolerance(ref: np.ndarray, max_abs=MAX_ABS, bf16_out=True) -> np.ndarray:
    """Per-element max-abs bar. For bf16 outputs the 2e-2 bar leaves, below
    |y| = 8, at least 2e-2 - 2^-6 for the arithmetic once the output's own
    rounding (half an ulp, 2^-6 at 4 <= |y| < 8) is paid. From |y| = 8 on a
    bf16 number alone can be 2^-5 away from the exact value, more than the bar,
    so the bar grows with the half-ulp and keeps that same allowance for the
    arithmetic (reading of "max-abs 2e-2 for bf16 I/O"). fp32 outputs keep 2e-2."""
    if not bf16_out:
        return np.full(np.shape(ref), max_abs)
    return max_abs + np.maximum(0.0, bf16_half_ulp(ref) - 2.0 ** -6)


def compare(gpu: np.ndarray, ref: np.ndarray, what: str, max_abs=MAX_ABS, rel_l2=REL_L2, bf16_out=True):
    d = np.abs(gpu - ref)
    ma = float(np.max(d)) if d.size else 0.0
    tol = abs_tolerance(ref, max_abs, bf16_out)
    over = float(np.max(d - tol)) if d.size else -1.0
    wide = int(np.sum(tol > max_abs))
    den = float(np.linalg.norm(ref))
    rl = float(np.linalg.norm(gpu - ref) / den) if den > 0 else float(np.linalg.norm(gpu - ref))
    msg = (f"{what}: max-abs {ma:.3e} (bar {max_abs}; {wide} elements at |y| >= 8 have the bar raised by the bf16 "
           f"half-ulp), worst margin {-over:.3e}, rel-L2 {rl:.3e} (<= {rel_l2}), max|ref| {np.max(np.abs(ref)):.3f}")
    print(msg)
    assert over <= 0.0 and rl <= rel_l2, msg
    return ma, rl


def inputs_to(inp: dict, device) -> dict:
    return {k: (v.to(device) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
