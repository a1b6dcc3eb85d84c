"""Seeded synthetic inputs for the grouped top-k MoE block.

This module only draws random tensors and lays them out. It holds none of the
block's arithmetic (no scores, no routing, no expert math), so that the CUDA
path and the CPU oracle can both consume the same bits without sharing any
computation.

Workloads are shaped like the Bailing/Ling models on the pages:

* ``ling_lite_t64``: Ling-lite-1.5 shapes (mlxcel issue #838, section
  "Validation checkpoint"): hidden 2048, 64 routed experts of intermediate
  1408, top-6, softmax, 2 shared experts fused into one MLP of width 2816
  (section "Shared experts are one wide MLP, not N separate experts").
* ``ling26_flash_t512`` and the ``ling26_flash_prefill_*`` pair:
  Ling-2.6-flash shapes (model card "Ling-2.6-flash-JANGTQ", section
  "Architecture (bailing_hybrid)", paragraph "MoE routing"): 256 routed + 1
  shared experts, sigmoid scores, 8 groups, top-4 groups, top-8 experts,
  e_score_correction_bias.
* ``ling30_flash_decode_t*`` and ``ling30_flash_skew_t16384``: Ling-3.0-flash
  shapes (page "Ling-3.0-flash-GGUF": 512 experts, 8 used).

Random recipe (seed 0 unless stated): x ~ N(0,1) bf16; router weight
~ N(0, 0.02) fp32; expert weights ~ N(0, 1/sqrt(fan_in)) bf16 (fan_in is the
hidden size for gate/up rows and the intermediate size for down rows);
expert_bias ~ N(0, 0.1) fp32, or the Zipf-like recipe of the skewed workload.

Layout handed to both sides:

* ``x``           [T, H]      bf16 row-major
* ``router_w``    [E, H]      fp32
* ``expert_bias`` [E]         fp32, or None
* ``w_gate_up``   [E, 2I, H]  bf16; rows [0, I) are gate_proj, rows [I, 2I) up_proj
* ``w_down``      [E, H, I]   bf16
* ``ws_gate_up``  [2Is, H]    bf16 (shared MLP, same gate/up row split)
* ``ws_down``     [H, Is]     bf16

``Is`` (the shared MLP width) is written out literally per workload.
"""
from __future__ import annotations

import copy
import math

import torch

# Field names follow the Bailing config fields named in mlxcel issue #838,
# section "Config fields the checkpoint does not contain".
_LING_LITE = dict(
    hidden_size=2048, num_experts=64, num_experts_per_tok=6, n_group=1, topk_group=1,
    score_function="softmax", norm_topk_prob=False, routed_scaling_factor=1.0,
    moe_intermediate_size=1408, num_shared_experts=2, moe_shared_expert_intermediate_size=0,
    shared_width=2816, bias="none",
)
_LING26_FLASH = dict(
    hidden_size=4096, num_experts=256, num_experts_per_tok=8, n_group=8, topk_group=4,
    score_function="sigmoid", norm_topk_prob=True, routed_scaling_factor=2.5,
    moe_intermediate_size=1024, num_shared_experts=1, moe_shared_expert_intermediate_size=0,
    shared_width=1024, bias="normal",
)
_LING30_FLASH = dict(
    hidden_size=4096, num_experts=512, num_experts_per_tok=8, n_group=1, topk_group=1,
    score_function="sigmoid", norm_topk_prob=True, routed_scaling_factor=2.5,
    moe_intermediate_size=512, num_shared_experts=1, moe_shared_expert_intermediate_size=0,
    shared_width=512, bias="normal",
)


def _wl(base, tokens, **over):
    d = dict(base)
    d["tokens"] = tokens
    d.update(over)
    return d


WORKLOADS = {
    "ling_lite_t64": _wl(_LING_LITE, 64),
    "ling26_flash_t512": _wl(_LING26_FLASH, 512),
    "ling30_flash_decode_t1": _wl(_LING30_FLASH, 1),
    "ling30_flash_decode_t8": _wl(_LING30_FLASH, 8),
    "ling30_flash_decode_t32": _wl(_LING30_FLASH, 32),
    "ling30_flash_decode_t64": _wl(_LING30_FLASH, 64),
    "ling26_flash_prefill_t8192": _wl(_LING26_FLASH, 8192),
    "ling26_flash_prefill_t32768": _wl(_LING26_FLASH, 32768),
    # Skewed load: Zipf-like bias, 1% of tokens carry exact ties (built by the tests).
    "ling30_flash_skew_t16384": _wl(_LING30_FLASH, 16384, bias="zipf"),
}

# Experts whose bias is copied to the next expert in the Zipf recipe, giving
# 16 pairs (e, e+1) with bitwise-equal bias. Ties between such a pair are exact
# when both experts also receive equal logits.
ZIPF_TWIN_EXPERTS = tuple(range(0, 512, 32))
ZIPF_S = 1.2
ZIPF_AMPLITUDE = 2.0
ACT_SEED_OFFSET = 1_000_003


def workload(name: str, **over) -> dict:
    """A copy of a named workload, with fields overridden."""
    d = copy.deepcopy(WORKLOADS[name])
    d.update(over)
    return d


def tiny_workload(**over) -> dict:
    """A small workload for CPU tests; every field may be overridden."""
    d = dict(
        tokens=16, hidden_size=64, num_experts=8, num_experts_per_tok=2, n_group=1, topk_group=1,
        score_function="softmax", norm_topk_prob=True, routed_scaling_factor=1.0,
        moe_intermediate_size=32, num_shared_experts=1, moe_shared_expert_intermediate_size=0,
        shared_width=32, bias="none",
    )
    d.update(over)
    return d


def _normal(shape, std, gen, device, dtype):
    t = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


def zipf_bias(num_experts: int, gen: torch.Generator, device="cpu") -> torch.Tensor:
    """Zipf-like selection bias: b_e = A * r_e^(-s), r a seeded permutation of
    1..E, then b[e+1] = b[e] for the designated twin experts."""
    r = torch.randperm(num_experts, generator=gen, device=device).to(torch.float64) + 1.0
    b = ZIPF_AMPLITUDE * torch.pow(r, -ZIPF_S)
    for e in ZIPF_TWIN_EXPERTS:
        if e + 1 < num_experts:
            b[e + 1] = b[e]
    return b.to(torch.float32)


def make_inputs(wl: dict, seed: int = 0, device="cpu", tokens: int | None = None,
                weights: bool = True) -> dict:
    """Draw all tensors of one workload. Same seed and device give the same bits.

    Parameters come from a generator seeded with ``seed`` and activations from
    one seeded with ``seed + ACT_SEED_OFFSET``, so the weights do not depend on
    the token count.
    """
    device = torch.device(device)
    T = wl["tokens"] if tokens is None else tokens
    H, E, I, Is = wl["hidden_size"], wl["num_experts"], wl["moe_intermediate_size"], wl["shared_width"]
    gw = torch.Generator(device=device)
    gw.manual_seed(seed)
    gx = torch.Generator(device=device)
    gx.manual_seed(seed + ACT_SEED_OFFSET)
    out = {"tokens": T}
    out["router_w"] = _normal((E, H), 0.02, gw, device, torch.float32)
    if wl["bias"] == "normal":
        out["expert_bias"] = _normal((E,), 0.1, gw, device, torch.float32)
    elif wl["bias"] == "zipf":
        out["expert_bias"] = zipf_bias(E, gw, device)
    else:
        out["expert_bias"] = None
    if weights:
        # One expert at a time keeps the fp32 temporaries small at full size.
        wgu = torch.empty((E, 2 * I, H), dtype=torch.bfloat16, device=device)
        wd = torch.empty((E, H, I), dtype=torch.bfloat16, device=device)
        sg, sd = 1.0 / math.sqrt(H), 1.0 / math.sqrt(I)
        for e in range(E):
            wgu[e] = _normal((2 * I, H), sg, gw, device, torch.bfloat16)
            wd[e] = _normal((H, I), sd, gw, device, torch.bfloat16)
        out["w_gate_up"] = wgu
        out["w_down"] = wd
        if Is > 0:
            out["ws_gate_up"] = _normal((2 * Is, H), sg, gw, device, torch.bfloat16)
            out["ws_down"] = _normal((H, Is), 1.0 / math.sqrt(Is), gw, device, torch.bfloat16)
        else:
            out["ws_gate_up"] = None
            out["ws_down"] = None
    out["x"] = _normal((T, H), 1.0, gx, device, torch.bfloat16)
    return out


def _q8_matrix(shape, group_size, gen, device):
    """Codes, scales and biases of an 8-bit affine matrix [..., R, K] whose
    dequantised weights are about N(0, 1/sqrt(K)): codes 128 + 40 N(0, 1)
    clipped to [0, 255], scale (sigma / 40) * U(0.75, 1.25) per group, bias
    -128 * scale + N(0, sigma / 16) per group (scale and bias bf16)."""
    K = shape[-1]
    sigma = 1.0 / math.sqrt(K)
    gshape = tuple(shape[:-1]) + (K // group_size,)
    q = (torch.randn(shape, generator=gen, device=device) * 40.0 + 128.0).round_().clamp_(0, 255).to(torch.uint8)
    scale = (torch.rand(gshape, generator=gen, device=device) * 0.5 + 0.75) * (sigma / 40.0)
    bias = -128.0 * scale + torch.randn(gshape, generator=gen, device=device) * (sigma / 16.0)
    return q, scale.to(torch.bfloat16), bias.to(torch.bfloat16)


def make_q8_weights(wl: dict, seed: int = 0, device="cpu", group_size: int = 64, shared: bool = True) -> dict:
    """8-bit affine expert weights for a workload (drawn directly, seeded):
    gate_up [E, 2I, H], down [E, H, I] and, when ``shared``, the shared MLP's
    [2Is, H] and [H, Is]; each a (q, scale, bias) triple."""
    device = torch.device(device)
    H, E, I, Is = wl["hidden_size"], wl["num_experts"], wl["moe_intermediate_size"], wl["shared_width"]
    gen = torch.Generator(device=device)
    gen.manual_seed(seed + 77)
    parts = [_q8_matrix((1, 2 * I, H), group_size, gen, device) for _ in range(E)]
    gate_up = tuple(torch.cat([p[i] for p in parts]) for i in range(3))
    parts = [_q8_matrix((1, H, I), group_size, gen, device) for _ in range(E)]
    down = tuple(torch.cat([p[i] for p in parts]) for i in range(3))
    out = {"group_size": group_size, "gate_up": gate_up, "down": down, "shared_gate_up": None, "shared_down": None}
    if shared and Is > 0:
        out["shared_gate_up"] = _q8_matrix((2 * Is, H), group_size, gen, device)
        out["shared_down"] = _q8_matrix((H, Is), group_size, gen, device)
    return out


# Dense-prefix MLP of Ling-2.6-flash: hidden 4096, intermediate 9216 (model card
# "Ling-2.6-flash-JANGTQ", section "Architecture (bailing_hybrid)", layer table).
LING26_DENSE = dict(hidden_size=4096, intermediate_size=9216)


def make_dense_inputs(hidden_size: int, intermediate_size: int, tokens: int, seed: int = 0, device="cpu") -> dict:
    """Weights and token rows of a dense SwiGLU MLP: gate/up [2*Id, H] with std
    1/sqrt(H), down [H, Id] with std 1/sqrt(Id), x ~ N(0, 1); all bf16."""
    device = torch.device(device)
    H, Id = hidden_size, intermediate_size
    gw = torch.Generator(device=device)
    gw.manual_seed(seed)
    gx = torch.Generator(device=device)
    gx.manual_seed(seed + ACT_SEED_OFFSET)
    return {
        "tokens": tokens,
        "w_gate_up": _normal((2 * Id, H), 1.0 / math.sqrt(H), gw, device, torch.bfloat16),
        "w_down": _normal((H, Id), 1.0 / math.sqrt(Id), gw, device, torch.bfloat16),
        "x": _normal((tokens, H), 1.0, gx, device, torch.bfloat16),
    }


def random_logits(T: int, E: int, std: float, seed: int = 0, device="cpu") -> torch.Tensor:
    """fp32 logits [T, E] ~ N(0, std), for routing-only tests."""
    gen = torch.Generator(device=torch.device(device))
    gen.manual_seed(seed)
    return _normal((T, E), std, gen, device, torch.float32)
