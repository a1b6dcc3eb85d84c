"""Host logic of bench.py: the algorithmic bytes and flops behind the roofline
figures, and the whole-job rate, against sums written out by hand here.

The expert block's decode step reads the chosen experts' weights, the shared
MLP's, the fp32 router projection, x and y (page "Ling-3.0-flash-GGUF",
section "Measured performance": a decode step touches just the selected
experts); the prefill passes are two grouped contractions per routed and
shared row.
"""
import bench
from grouped_top_routing_b200 import inputs as G


def test_decode_step_bytes_one_token_512_experts():
    wl = G.workload("ling30_flash_decode_t1")
    a = bench.algorithmic(wl, 1, 8)
    # 8 routed experts + the shared MLP, each gate, up and down: 3 * 512 * 4096 bf16
    weights = 9 * 3 * 512 * 4096 * 2
    router = 512 * 4096 * 4
    x_and_y = 2 * 4096 * 2
    assert a["step_bytes"] == weights + router + x_and_y == 121_651_200


def test_decode_gate_up_bytes_count_h_and_token_rows():
    wl = G.workload("ling30_flash_decode_t8")
    T, U = 8, 50
    a = bench.algorithmic(wl, T, U, h_bytes=4, slot_bytes=4)
    k, H, I, Is = 8, 4096, 512, 512
    w = (U * 2 * I + 2 * Is) * H * 2
    rows_in = (T * k + T) * H * 2
    h_out = (T * k * I + T * Is) * 4
    assert a["gate_up_bytes"] == w + rows_in + h_out
    wd = (U * I + Is) * H * 2
    assert a["down_bytes"] == wd + h_out + T * k * H * 4 + T * H * 4


def test_eight_bit_weights_count_codes_scales_and_biases():
    wl = G.workload("ling30_flash_decode_t1")
    a16 = bench.algorithmic(wl, 1, 8)
    a8 = bench.algorithmic(wl, 1, 8, weight_bytes=1.0 + 4.0 / 64)
    w16 = 9 * 2 * 512 * 4096 * 2
    w8 = 9 * 2 * 512 * 4096 * (1 + 4 / 64)
    assert a16["gate_up_bytes"] - a8["gate_up_bytes"] == int(w16) - int(w8)


def test_prefill_flops():
    # every routed slot row and every token's shared row goes through
    # gate+up (2 * H * 2I flops) and down (2 * H * I); plus the router
    for T, tflops in [(8192, 1.8726), (32768, 7.4904)]:
        wl = G.workload(f"ling26_flash_prefill_t{T}")
        a = bench.algorithmic(wl, T, 256)
        H, E, k, I, Is = 4096, 256, 8, 1024, 1024
        rows = T * k * I + T * Is
        expect = 2 * H * 2 * rows + 2 * H * rows + 2 * T * H * E
        assert a["flops"] == expect
        assert abs(a["flops"] / 1e12 - tflops) < 1e-3


def test_whole_job_rate():
    # 4 ranks, 32768 tokens each, slowest rank 8 ms per step
    assert bench.whole_job_rate(32768, 4, 8.0) == 32768 * 4 / 0.008
