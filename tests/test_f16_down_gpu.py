"""The fp16 down path: its weight conversion and its range check.

moe_convert_bf16_to_f16 must round exactly as IEEE fp16 round-to-nearest-even
does (numpy's float32 -> float16 conversion is that rounding) and count the
values fp16 cannot hold. With moe_options.w_down_f16 the tensor-core path keeps
the SwiGLU product in fp16: a product beyond fp16's range must be reported as
MOE_ERR_RANGE, not passed on as an infinity. The path's numerics against the
oracle are in test_parity_gpu.py (the "tensor_cores_f16" cases).
"""
import numpy as np
import pytest
import torch

from grouped_top_routing_b200 import build as B
from grouped_top_routing_b200 import inputs as G

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def M():
    B.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from grouped_top_routing_b200 import moe
    return moe


def _bf16_bits(vals) -> np.ndarray:
    f = np.asarray(vals, np.float32)
    return torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("n", [0, 1, 7, 8, 9, 4099, 1 << 20])
def test_conversion_rounds_like_ieee_fp16(M, n):
    rng = np.random.default_rng(n)
    # normal weights, and every 16-bit pattern class: subnormal and zero
    # results, ties, the largest finite values, overflow, inf and NaN
    vals = (rng.standard_normal(n) * 0.03).astype(np.float32)
    special = np.array([0.0, -0.0, 2.0 ** -14, 2.0 ** -15, 2.0 ** -24, 2.0 ** -25, 2.0 ** -26, 3 * 2.0 ** -26,
                        65504.0, -65504.0, 65520.0, 1.0e5, np.inf, -np.inf, np.nan, 1.0 + 2.0 ** -11], np.float32)
    vals[: min(n, special.size)] = special[: min(n, special.size)]
    bits = _bf16_bits(vals)
    src = torch.from_numpy(bits.view(np.int16)).to(DEV).view(torch.bfloat16)
    dst = torch.empty(n, dtype=torch.float16, device=DEV)
    bad = torch.full((1,), 99, dtype=torch.int32, device=DEV)
    import ctypes
    st = M.lib.moe_convert_bf16_to_f16(ctypes.c_void_p(src.data_ptr()) if n else None,
                                       ctypes.c_void_p(dst.data_ptr()) if n else None, n,
                                       ctypes.c_void_p(bad.data_ptr()), None)
    assert st == 0, M.last_error()
    torch.cuda.synchronize()
    exact = (bits.astype(np.uint32) << 16).view(np.float32)  # the bf16 values
    want = exact.astype(np.float16)
    got = dst.cpu().numpy()
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint16), want[~nan].view(np.uint16))
    assert int(bad.item()) == int(np.sum(~np.isfinite(want)))


def test_binding_conversion_raises_on_overflow(M):
    w = torch.tensor([1.0, 7.0e4, -2.0], dtype=torch.bfloat16, device=DEV)
    with pytest.raises(M.MoeError) as ei:
        M.convert_bf16_to_f16(w)
    assert ei.value.status == 7 and "1 values" in str(ei.value)
    ok = M.convert_bf16_to_f16(torch.tensor([1.0, -2.5], dtype=torch.bfloat16, device=DEV))
    assert ok.dtype == torch.float16 and ok.tolist() == [1.0, -2.5]


@pytest.mark.parametrize("tokens", [40, 600])  # weight-major tiles, token-major tiles
def test_swiglu_beyond_fp16_is_reported(M, tokens):
    wl = G.tiny_workload(tokens=tokens, hidden_size=200, num_experts=6, num_experts_per_tok=2,
                         moe_intermediate_size=136, shared_width=272, num_shared_experts=2, name="f16-range")
    inp = G.make_inputs(wl, seed=4, device=DEV)
    x = inp["x"].clone()
    x[5] *= 400.0  # gate and up both ~400x: h ~ 1e5 for this token
    wd = M.convert_bf16_to_f16(inp["w_down"])
    wsd = M.convert_bf16_to_f16(inp["ws_down"])
    opts = M.options(ffn_path="tensor_cores", w_down_f16=wd, ws_down_f16=wsd)
    ws = M.Workspace(wl, tokens)
    M.moe_forward(wl, x, inp["router_w"], inp["expert_bias"], inp["w_gate_up"], inp["w_down"], inp["ws_gate_up"],
                  inp["ws_down"], ws, opts=opts)
    with pytest.raises(M.MoeError) as ei:
        ws.check()
    assert ei.value.status == 7, ei.value
    # the same input on the bf16 path is fine, and so is the fp16 path again
    # on ordinary input (the error word was cleared)
    M.moe_forward(wl, x, inp["router_w"], inp["expert_bias"], inp["w_gate_up"], inp["w_down"], inp["ws_gate_up"],
                  inp["ws_down"], ws, opts=M.options(ffn_path="tensor_cores"))
    ws.check()
    M.moe_forward(wl, inp["x"], inp["router_w"], inp["expert_bias"], inp["w_gate_up"], inp["w_down"],
                  inp["ws_gate_up"], inp["ws_down"], ws, opts=opts)
    ws.check()


@pytest.mark.parametrize("tokens,hidden", [(40, 200), (90, 64), (600, 200), (600, 136)])
def test_forward_f16_ragged_shapes(M, tokens, hidden):
    # The whole block on the fp16 down path, where the routed slot rows are
    # fp16 too: weight-major tiles (40, 90 tokens) and token-major tiles (600),
    # hidden sizes that leave a ragged last 64-column chunk, against the oracle
    # on the fp16 weights.
    import support as S
    from oracle import moe_oracle as O
    wl = G.tiny_workload(tokens=tokens, hidden_size=hidden, num_experts=6, num_experts_per_tok=2,
                         moe_intermediate_size=136, shared_width=272, num_shared_experts=2, name="f16-forward")
    inp = G.make_inputs(wl, seed=6, device=DEV)
    wd = M.convert_bf16_to_f16(inp["w_down"])
    wsd = M.convert_bf16_to_f16(inp["ws_down"])
    L = G.random_logits(tokens, wl["num_experts"], 1.0, seed=7).numpy()
    ws = M.Workspace(wl, tokens)
    y = M.moe_forward(wl, inp["x"], inp["router_w"], inp["expert_bias"], inp["w_gate_up"], inp["w_down"],
                      inp["ws_gate_up"], inp["ws_down"], ws, logits_override=torch.from_numpy(L).to(DEV),
                      opts=M.options(ffn_path="tensor_cores", w_down_f16=wd, ws_down_f16=wsd))
    ws.check()
    ref = O.moe_block(dict(inp, w_down=wd, ws_down=wsd), wl, logits=L)["y"]
    S.compare(O.as_f64(y), ref, f"f16 forward T={tokens} H={hidden}")
