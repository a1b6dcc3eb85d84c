"""The synthetic input recipe (grouped_top_routing_b200/inputs.py) against its
stated parameters: seeds give the same bits, the weights do not depend on the
token count, the distributions have the stated spreads, the Zipf bias follows
b_e = 2.0 * r_e^-1.2 over a permutation r of 1..E with bitwise-equal twin
pairs, and the 8-bit weights dequantise to about the bf16 recipe's spread.
Inputs only: none of the method's arithmetic is here.
"""
import math

import numpy as np
import torch

from grouped_top_routing_b200 import inputs as G


def _std(t):
    return float(t.float().std())


def test_same_seed_same_bits_and_weights_independent_of_tokens():
    wl = G.tiny_workload(tokens=16, hidden_size=64, num_experts=8, num_experts_per_tok=2,
                         moe_intermediate_size=32, shared_width=32, bias="normal")
    a = G.make_inputs(wl, seed=5)
    b = G.make_inputs(wl, seed=5)
    c = G.make_inputs(wl, seed=5, tokens=40)
    for key in ("router_w", "expert_bias", "w_gate_up", "w_down", "ws_gate_up", "ws_down", "x"):
        assert torch.equal(a[key], b[key]), key
    for key in ("router_w", "expert_bias", "w_gate_up", "w_down", "ws_gate_up", "ws_down"):
        assert torch.equal(a[key], c[key]), key
    assert torch.equal(a["x"], c["x"][:16])  # the activation stream starts the same
    d = G.make_inputs(wl, seed=6)
    assert not torch.equal(a["w_gate_up"], d["w_gate_up"])


def test_spreads():
    wl = G.tiny_workload(tokens=256, hidden_size=512, num_experts=16, num_experts_per_tok=2,
                         moe_intermediate_size=256, shared_width=512, bias="normal")
    inp = G.make_inputs(wl, seed=0)
    H, I, Is = 512, 256, 512
    checks = [("x", 1.0), ("router_w", 0.02), ("expert_bias", 0.1), ("w_gate_up", 1 / math.sqrt(H)),
              ("w_down", 1 / math.sqrt(I)), ("ws_gate_up", 1 / math.sqrt(H)), ("ws_down", 1 / math.sqrt(Is))]
    for key, std in checks:
        got = _std(inp[key])
        tol = 0.25 if key == "expert_bias" else 0.05  # 16 bias values vs many weights
        assert abs(got / std - 1.0) < tol, (key, got, std)
    assert inp["x"].dtype == torch.bfloat16 and inp["router_w"].dtype == torch.float32
    assert inp["w_gate_up"].dtype == torch.bfloat16 and inp["expert_bias"].dtype == torch.float32


def test_zipf_bias():
    gen = torch.Generator()
    gen.manual_seed(3)
    E = 512
    b = G.zipf_bias(E, gen).double().numpy()
    gen.manual_seed(3)
    r = torch.randperm(E, generator=gen).double().numpy() + 1.0
    expect = 2.0 * r ** -1.2
    twins = [e for e in range(0, E, 32)]
    for e in twins:
        expect[e + 1] = expect[e]
    assert np.allclose(b, expect.astype(np.float32), rtol=0, atol=0)
    for e in twins:
        assert b[e] == b[e + 1]
    # a few experts carry most of the bias mass
    s = np.sort(b)[::-1]
    assert s[: E // 10].sum() > 0.5 * s.sum()


def test_q8_recipe():
    wl = G.tiny_workload(tokens=4, hidden_size=256, num_experts=4, num_experts_per_tok=2,
                         moe_intermediate_size=128, shared_width=128)
    q8 = G.make_q8_weights(wl, seed=1, group_size=64, shared=True)
    q, scale, bias = q8["gate_up"]
    assert q.dtype == torch.uint8 and scale.dtype == torch.bfloat16 and bias.dtype == torch.bfloat16
    assert q.shape == (4, 2 * 128, 256) and scale.shape == (4, 2 * 128, 256 // 64)
    qf = q.double()
    assert abs(float(qf.mean()) - 128.0) < 1.0 and abs(float(qf.std()) - 40.0) < 1.5
    sigma = 1 / math.sqrt(256)
    s = scale.double()
    assert float(s.min()) >= 0.74 * sigma / 40 and float(s.max()) <= 1.26 * sigma / 40
    resid = bias.double() + 128.0 * s
    assert abs(float(resid.std()) / (sigma / 16) - 1.0) < 0.15
    # dequantised weights: about N(0, sigma^2), the bf16 recipe's spread
    w = s.repeat_interleave(64, dim=-1) * qf + bias.double().repeat_interleave(64, dim=-1)
    assert abs(float(w.std()) / sigma - 1.0) < 0.1 and abs(float(w.mean())) < 0.1 * sigma
    assert q8["shared_gate_up"][0].shape == (2 * 128, 256) and q8["shared_down"][0].shape == (256, 128)
