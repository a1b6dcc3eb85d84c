"""Benchmark of the grouped top-k MoE block on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

One step = the whole block (router logits, route, permute, expert FFNs with
the shared MLP, combine) through ``moe_forward`` on one batch of synthetic
tokens already resident in HBM. Weak scaling: every rank runs its own batch
against its own weight replica; no data-path collective. Rank 0 prints one
JSON line.

``--impl reference`` times the CPU oracle (the reference arm: a plain fp64
program, no GPU work) on bounded token samples of the same workload.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from grouped_top_routing_b200 import inputs as G  # noqa: E402

METRIC = "MoE-block tokens/s at 1 B200; HBM GB/s (decode) & TFLOPS (prefill) vs roofline"
UNIT = "tokens/s"
DEFAULT_WORKLOAD = "ling26_flash_prefill_t32768"
L2_FLUSH_BYTES = 256 << 20
L2_BYTES = 126 << 20  # B200 L2
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def _env_int(name, default):
    try:
        return int(os.environ.get(name, default))
    except ValueError:
        return default


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
            "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ---------------------------------------------------------------------------
# algorithmic work of one step (counted from the step's actual routing)
# ---------------------------------------------------------------------------

# DRAM traffic per launch of the roofline kernel (dram__bytes_read.sum +
# dram__bytes_write.sum, one ncu capture of this script's own default command
# for the workload), with a hash of the kernel's source files at capture time.
# The figure is reported only while those sources are unchanged and the run
# uses the captured configuration.
KERNEL_SOURCES = {
    "expert_gate_up": ["umma_ffn.cu", "ffn.cuh", "mbarrier.cuh", "common.cuh"],
    "expert_down": ["umma_ffn.cu", "ffn.cuh", "mbarrier.cuh", "common.cuh"],
    "decode_fused": ["decode_fused.cu", "decode_fused.cuh", "fused_common.cuh", "route_block.cuh", "route.cuh",
                     "mbarrier.cuh", "common.cuh"],
}
MEASURED_TRAFFIC = {  # profiles/dram_traffic_ling26_prefill_t32768.md (fp16 down path, the default)
    ("expert_gate_up", "ling26_flash_prefill_t32768"): (6817733632, "465f18060116542f"),
    ("expert_down", "ling26_flash_prefill_t32768"): (5130166528, "465f18060116542f"),
}


def kernel_source_hash(kernel: str) -> str:
    import hashlib
    csrc = os.path.join(os.path.dirname(os.path.abspath(__file__)), "grouped_top_routing_b200", "csrc")
    h = hashlib.sha256()
    for name in sorted(KERNEL_SOURCES[kernel]):
        h.update(name.encode())
        with open(os.path.join(csrc, name), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_traffic(kernel: str, workload: str, overrides, ffn_path: str, decode: str = "auto",
                     down_weights: str = "f16"):
    """Bytes per launch from the capture, or None when it no longer applies."""
    entry = MEASURED_TRAFFIC.get((kernel, workload))
    if entry is None or overrides or ffn_path != "auto" or decode != "auto" or down_weights != "f16":
        return None
    return entry[0] if kernel_source_hash(kernel) == entry[1] else None


def algorithmic(wl, T, n_unique, weight_bytes=2.0, h_bytes=4, slot_bytes=4):
    """Bytes each expert pass must move, and the block's flops, given the
    number of distinct routed experts the batch touched. Expert weights count
    weight_bytes per element (2 for bf16 or fp16; 1 + 4 / group for 8-bit
    affine codes with a bf16 scale and bias per group). Activations count at
    the width this design stores them: token rows bf16 (2 B), the SwiGLU
    product h_bytes (two bf16 planes or fp32: 4 B; one fp16 plane: 2 B),
    routed slot rows slot_bytes (fp32 4 B, fp16 2 B) and the shared MLP output
    fp32 (4 B)."""
    H, E, k, I, Is = (wl["hidden_size"], wl["num_experts"], wl["num_experts_per_tok"],
                      wl["moe_intermediate_size"], wl["shared_width"])
    R = T * k
    w_gate_up = int((n_unique * 2 * I + 2 * Is) * H * weight_bytes)
    w_down = int((n_unique * I + Is) * H * weight_bytes)
    h_elems = R * I + T * Is
    gate_up_bytes = w_gate_up + (R + T) * H * 2 + h_elems * h_bytes   # weights + token rows in + h out
    down_bytes = w_down + h_elems * h_bytes + R * H * slot_bytes + T * H * 4  # weights + h in + rows out
    step_bytes = (w_gate_up + w_down + E * H * 4 + 2 * T * H * 2)  # weights + router + x in + y out
    gate_up_flops = 2 * H * 2 * h_elems          # gate and up projections of every routed and shared row
    down_flops = 2 * H * h_elems
    flops = gate_up_flops + down_flops + 2 * T * H * E
    return dict(gate_up_bytes=gate_up_bytes, down_bytes=down_bytes, step_bytes=step_bytes, flops=flops,
                gate_up_flops=gate_up_flops, down_flops=down_flops)


# ---------------------------------------------------------------------------
# multi-rank bookkeeping (weak scaling: one token batch per rank, no
# data-path collective; tokens are independent)
# ---------------------------------------------------------------------------

def rank_activation_seed(rank: int) -> int:
    """Seed of rank r's token batch (rank 0 uses the workload's own x)."""
    return 1000 + rank


def reduce_max_over_ranks(t: torch.Tensor, world: int) -> torch.Tensor:
    """Element-wise max of a timing tensor over all ranks (in place)."""
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t


def whole_job_rate(units_per_rank: int, world: int, ms_per_step: float) -> float:
    """Units all ranks processed per second, given the slowest rank's step time."""
    return units_per_rank * world / (ms_per_step / 1e3)


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks", suffix=".csv")
        os.close(fd)
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        if self.proc is None or self.path is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        rows = []
        with open(self.path) as f:
            for line in f:
                p = [x.strip() for x in line.split(",")]
                if len(p) >= 9:
                    rows.append(p)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None

        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        mx = [num(r[2]) for r in rows if num(r[2]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------------------
# CPU oracle timing (reference arm and cpu_baseline)
# ---------------------------------------------------------------------------

def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def time_oracle(wl, inp, token_rows):
    """Seconds the oracle takes for the block on the given token rows."""
    from oracle import moe_oracle as O
    sub = dict(inp)
    sub["x"] = inp["x"][token_rows]
    t0 = time.perf_counter()
    O.moe_block(sub, wl)
    return time.perf_counter() - t0


def workload_from_args(args):
    wl = G.workload(args.workload)
    for kv in args.set:
        key, val = kv.split("=", 1)
        if key not in wl:
            raise SystemExit(f"unknown workload field {key}")
        wl[key] = type(wl[key])(val) if not isinstance(wl[key], bool) else val.lower() in ("1", "true")
    return wl


def run_reference(args):
    rank = _env_int("RANK", 0)
    if rank != 0:
        return 0
    wl = workload_from_args(args)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    inp = G.make_inputs(wl, seed=0, device=dev)  # generation is not timed; the oracle pulls rows to the host
    T = inp["tokens"]
    per_step = args.ref_sample
    rng = np.random.default_rng(0)
    for _ in range(args.warmup):
        time_oracle(wl, inp, torch.from_numpy(rng.choice(T, per_step, replace=False)).to(dev))
    secs = []
    for _ in range(args.steps):
        secs.append(time_oracle(wl, inp, torch.from_numpy(rng.choice(T, per_step, replace=False)).to(dev)))
    total = sum(secs)
    value = per_step * args.steps / total
    sample = f"{per_step} random tokens of the {T}-token batch per step, fp64 numpy oracle"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload, "tokens_per_step": per_step},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def run_ours(args):
    import torch.distributed as dist
    from grouped_top_routing_b200 import build as B
    B.build()
    from grouped_top_routing_b200 import moe as M

    world = _env_int("WORLD_SIZE", 1)
    rank = _env_int("RANK", 0)
    local = _env_int("LOCAL_RANK", 0)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    wl = workload_from_args(args)
    inp = G.make_inputs(wl, seed=0, device=dev)
    T = inp["tokens"]
    q8 = G.make_q8_weights(wl, seed=0, device=dev, group_size=args.q8) if args.q8 else None
    fused = args.decode == "auto" and T <= M.FUSED_DECODE_MAX_TOKENS and q8 is None
    # kernels timed live inside the steps (steps alternate between them when
    # there are two); the roofline line reports the one that takes longer
    if args.kernel != "auto":
        timed = [args.kernel]
    else:
        timed = ["decode_fused"] if fused else ["expert_gate_up", "expert_down"]
    if rank > 0:  # each rank its own batch (weak scaling), same weights
        g = torch.Generator(device=dev)
        g.manual_seed(rank_activation_seed(rank))
        inp["x"] = torch.randn(inp["x"].shape, generator=g, device=dev).to(torch.bfloat16)
    ws = M.Workspace(wl, T, device=dev)
    y = torch.empty_like(inp["x"])
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    base_opts = dict(ffn_path=args.ffn_path, decode=args.decode)
    # fp16 copies of the down weights, made once before anything is timed (a
    # load-time conversion, exact for |w| >= 2^-14): the tensor-core down pass
    # then multiplies fp16 operands, one MMA per k-step
    f16 = q8 is None and args.down_weights == "f16"
    if f16:
        base_opts["w_down_f16"] = M.convert_bf16_to_f16(inp["w_down"])
        base_opts["ws_down_f16"] = None if inp["ws_down"] is None else M.convert_bf16_to_f16(inp["ws_down"])

    def step(x=None, out=None, timer=None):
        out = y if out is None else out
        opts = M.options(timer=timer, **base_opts)
        if q8 is not None:
            return M.moe_forward_q8(wl, inp["x"] if x is None else x, inp["router_w"], inp["expert_bias"], q8, ws,
                                    y=out, opts=opts)
        return M.moe_forward(wl, inp["x"] if x is None else x, inp["router_w"], inp["expert_bias"],
                             inp["w_gate_up"], inp["w_down"], inp["ws_gate_up"], inp["ws_down"], ws, y=out,
                             opts=opts)

    warm = max(args.warmup, 3)
    for _ in range(warm):
        step()
    torch.cuda.synchronize(dev)
    ws.check()

    # routing of this batch: distinct experts touched (algorithmic bytes)
    _, idx, _ = M.moe_forward(wl, inp["x"], inp["router_w"], inp["expert_bias"], inp["w_gate_up"], inp["w_down"],
                              inp["ws_gate_up"], inp["ws_down"], ws, return_routing=True,
                              opts=M.options(**base_opts))
    n_unique = int(torch.unique(idx).numel())
    tc_path = not fused and (args.ffn_path == "tensor_cores" or (args.ffn_path == "auto" and T > M.STREAM_MAX_TOKENS))
    f16_tc = f16 and tc_path  # h as one fp16 plane, routed slot rows fp16
    work = algorithmic(wl, T, n_unique, 1.0 + 4.0 / args.q8 if q8 is not None else 2.0,
                       h_bytes=2 if f16_tc else 4, slot_bytes=2 if f16_tc else 4)

    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    for a, b in kev:  # torch creates the CUDA event on first record; the library needs the handles
        a.record(stream)
        b.record(stream)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    launches0 = M.launch_count()
    with ClockSampler(local) as clk:
        for i in range(K):
            flush.zero_()  # L2 flush, outside the timed events
            ev[i][0].record(stream)
            step(timer=(timed[i % len(timed)], kev[i][0], kev[i][1]))
            ev[i][1].record(stream)
        torch.cuda.synchronize(dev)
    launches = M.launch_count() - launches0
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    ws.check()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    kern_ms = {name: [kev[i][0].elapsed_time(kev[i][1]) for i in range(K) if timed[i % len(timed)] == name]
               for name in timed}
    kernel = max(timed, key=lambda n: statistics.mean(kern_ms[n]))  # the dominant one
    total_ms = sum(step_ms)

    # e2e: host pinned x in, host y out, through the same public call. When a
    # step's weights exceed 16x the L2, the steps cannot reuse each other's
    # weights from L2, and the loop runs as a serving loop would: step i+1's
    # input copy (host -> device) and step i-1's output copy (device -> host)
    # on their own streams while step i computes, double-buffered, all inside
    # one timed region. Otherwise each step is timed alone, with the L2 flush
    # outside its events and both copies inside. Either way every step's bytes
    # cross the link inside the timed region.
    pipelined = work["step_bytes"] >= 16 * L2_BYTES
    x_host = [inp["x"].cpu().pin_memory() for _ in range(2)]
    y_host = [torch.empty_like(x_host[0]).pin_memory() for _ in range(2)]
    x_dev = [torch.empty_like(inp["x"]) for _ in range(2)]
    y_dev = [torch.empty_like(inp["x"]) for _ in range(2)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    if pipelined:
        h2d, d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev = lambda: torch.cuda.Event()  # noqa: E731
        in_ready, computed, out_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
        e_start, e_stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e_start.record(stream)
        h2d.wait_stream(stream)
        d2h.wait_stream(stream)
        with torch.cuda.stream(h2d):
            x_dev[0].copy_(x_host[0], non_blocking=True)
            in_ready[0].record(h2d)
        for i in range(K):
            b = i % 2
            if i + 1 < K:  # next input, once the step that last read that buffer is done
                nb = (i + 1) % 2
                if i >= 1:
                    h2d.wait_event(computed[nb])
                with torch.cuda.stream(h2d):
                    x_dev[nb].copy_(x_host[nb], non_blocking=True)
                    in_ready[nb].record(h2d)
            stream.wait_event(in_ready[b])
            if i >= 2:
                stream.wait_event(out_done[b])  # y_dev[b] read out by its previous copy
            step(x_dev[b], y_dev[b])
            computed[b].record(stream)
            d2h.wait_event(computed[b])
            with torch.cuda.stream(d2h):
                y_host[b].copy_(y_dev[b], non_blocking=True)
                out_done[b].record(d2h)
        stream.wait_stream(d2h)
        e_stop.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = e_start.elapsed_time(e_stop)
    else:
        eev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
        for i in range(K):
            b = i % 2
            flush.zero_()
            eev[i][0].record(stream)
            x_dev[b].copy_(x_host[b], non_blocking=True)
            step(x_dev[b], y_dev[b])
            y_host[b].copy_(y_dev[b], non_blocking=True)
            eev[i][1].record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = sum(a.elapsed_time(b) for a, b in eev)
    assert torch.equal(y_host[(K - 1) % 2].view(torch.int16), y.cpu().view(torch.int16)), "e2e output differs"

    t = torch.tensor([total_ms, e2e_ms], dtype=torch.float64, device=dev)
    reduce_max_over_ranks(t, world)
    if world > 1:
        dist.barrier()
    total_ms, e2e_ms = float(t[0]), float(t[1])
    ms_per_step = total_ms / K
    value = whole_job_rate(T, world, ms_per_step)
    e2e_value = whole_job_rate(T, world, e2e_ms / K)

    pk = peaks()
    kms = statistics.mean(kern_ms[kernel])
    if kernel == "decode_fused":  # the whole block in one kernel
        kbytes, kflops = work["step_bytes"], work["flops"]
    else:
        kbytes = work["gate_up_bytes"] if kernel == "expert_gate_up" else work["down_bytes"]
        kflops = work["gate_up_flops"] if kernel == "expert_gate_up" else work["down_flops"]
    traffic = None if q8 is not None else measured_traffic(kernel, args.workload, args.set, args.ffn_path, args.decode,
                                                           args.down_weights)
    others = {n: statistics.mean(v) for n, v in kern_ms.items() if n != kernel}
    # the bound is the resource the kernel's arithmetic intensity saturates first
    ridge = pk["bf16_tflops"] * 1e12 / (pk["hbm_gbs"] * 1e9)
    if kflops / kbytes > ridge:
        # The kernel runs inside long back-to-back steps (power-capped), so the
        # denominator is the sustained bf16 figure; the burst fraction is kept
        # beside it.
        achieved = kflops / (kms / 1e3) / 1e12
        peak = pk["bf16_tflops_sustained"]
        roofline = {"bound": "tensor", "kernel": kernel, "achieved": achieved, "peak": peak,
                    "unit": "TFLOP/s", "frac": achieved / peak, "traffic": traffic,
                    "peak_source": pk["source"] + " (bf16 sustained)", "frac_of_burst": achieved / pk["bf16_tflops"],
                    "algorithmic_flops": kflops, "algorithmic_bytes": kbytes, "kernel_ms": kms,
                    "hbm_gbs": kbytes / (kms / 1e3) / 1e9, "other_kernels_ms": others}
    else:
        achieved = kbytes / (kms / 1e3) / 1e9
        roofline = {"bound": "hbm", "kernel": kernel, "achieved": achieved, "peak": pk["hbm_gbs"],
                    "unit": "GB/s", "frac": achieved / pk["hbm_gbs"], "traffic": traffic, "peak_source": pk["source"],
                    "algorithmic_bytes": kbytes, "algorithmic_flops": kflops, "kernel_ms": kms,
                    "tflops": kflops / (kms / 1e3) / 1e12, "other_kernels_ms": others}
    step_gbs = work["step_bytes"] / (ms_per_step / 1e3) / 1e9
    step_tflops = work["flops"] / (ms_per_step / 1e3) / 1e12

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rows = torch.arange(0, T, max(1, T // args.cpu_sample), device=dev)[:args.cpu_sample]
        secs = time_oracle(wl, inp, rows)
        cpu = {"value": len(rows) / secs, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
               "sample": f"{len(rows)} evenly spaced tokens of the {T}-token batch, fp64 numpy oracle, one pass",
               "seconds": secs}

    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return 0
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": warm,
        "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": args.workload, "overrides": args.set, "ffn_path": args.ffn_path,
                   "down_weights": None if q8 is not None else args.down_weights,
                   "decode": args.decode, "tokens": T, "hidden_size": wl["hidden_size"],
                   "num_experts": wl["num_experts"], "top_k": wl["num_experts_per_tok"],
                   "n_group": wl["n_group"], "topk_group": wl["topk_group"],
                   "moe_intermediate_size": wl["moe_intermediate_size"], "shared_width": wl["shared_width"],
                   "experts_touched": n_unique, "parallelism": f"replicas x{world} (token batches)",
                   "expert_weights": (f"8-bit affine, group {args.q8}" if q8 is not None else
                                      "bf16; down_proj also as an fp16 copy made once before timing (exact for "
                                      "|w| >= 2^-14), read by the tensor-core down pass" if f16 else "bf16"),
                   "l2": "256 MiB L2 flush between timed steps; expert weights >> 126 MB L2"},
        "step_hbm_gbs": step_gbs, "step_tflops": step_tflops,
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": int(x_host[0].numel() * 2),
                "d2h_bytes_per_step": int(y_host[0].numel() * 2),
                "schedule": ("pipelined: copies on their own streams overlap the neighbouring steps' compute; "
                             "weights > 16x L2, no flush") if pipelined else
                            "per step: copies and step inside the events, 256 MiB L2 flush outside"},
        "gpu_launches": int(launches),
        "clocks": clk.summary(),
    }
    print(json.dumps(line))
    return 0


def dense_algorithmic(H, Id, T):
    """Bytes of each pass and flops of the dense MLP: weights once, token rows
    bf16 in, the SwiGLU product at 4 B per element, fp32 rows out of the down
    pass."""
    gate_up_bytes = 2 * Id * H * 2 + T * H * 2 + T * Id * 4
    down_bytes = H * Id * 2 + T * Id * 4 + T * H * 4
    return dict(gate_up_bytes=gate_up_bytes, down_bytes=down_bytes, step_bytes=3 * H * Id * 2 + 2 * T * H * 2,
                gate_up_flops=2 * T * H * 2 * Id, flops=2 * T * H * 3 * Id)


def run_dense(args):
    """The dense-prefix MLP (moe_dense_mlp) on the Ling-2.6-flash layer-0 shape
    (hidden 4096, intermediate 9216), one GPU, T = args.dense tokens."""
    from grouped_top_routing_b200 import moe as M
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    H, Id, T = G.LING26_DENSE["hidden_size"], G.LING26_DENSE["intermediate_size"], args.dense
    inp = G.make_dense_inputs(H, Id, T, seed=0, device=dev)
    ws = M.dense_mlp_workspace(H, Id, T)
    y = torch.empty_like(inp["x"])
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(x=None, timer=None):
        return M.moe_dense_mlp(inp["x"] if x is None else x, inp["w_gate_up"], inp["w_down"], ws, y=y,
                               opts=M.options(timer=timer))

    warm = max(args.warmup, 3)
    for _ in range(warm):
        step()
    torch.cuda.synchronize(dev)
    ws.check()
    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    for a, b in kev:
        a.record(stream)
        b.record(stream)
    torch.cuda.synchronize(dev)
    launches0 = M.launch_count()
    with ClockSampler(0) as clk:
        for i in range(K):
            flush.zero_()  # L2 flush, outside the timed events
            ev[i][0].record(stream)
            step(timer=("expert_gate_up", kev[i][0], kev[i][1]))
            ev[i][1].record(stream)
        torch.cuda.synchronize(dev)
    launches = M.launch_count() - launches0
    ws.check()
    ms_per_step = sum(a.elapsed_time(b) for a, b in ev) / K
    kms = statistics.mean(a.elapsed_time(b) for a, b in kev)

    x_host = inp["x"].cpu().pin_memory()
    y_host = torch.empty_like(x_host).pin_memory()
    x_dev = torch.empty_like(inp["x"])
    eev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    for i in range(K):
        flush.zero_()
        eev[i][0].record(stream)
        x_dev.copy_(x_host, non_blocking=True)
        step(x_dev)
        y_host.copy_(y, non_blocking=True)
        eev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = sum(a.elapsed_time(b) for a, b in eev) / K

    work = dense_algorithmic(H, Id, T)
    pk = peaks()
    ridge = pk["bf16_tflops"] * 1e12 / (pk["hbm_gbs"] * 1e9)
    kb, kf = work["gate_up_bytes"], work["gate_up_flops"]
    if kf / kb > ridge:
        achieved = kf / (kms / 1e3) / 1e12
        roofline = {"bound": "tensor", "kernel": "expert_gate_up", "achieved": achieved, "peak": pk["bf16_tflops"],
                    "unit": "TFLOP/s", "frac": achieved / pk["bf16_tflops"], "traffic": None,
                    "peak_source": pk["source"] + " (bf16 burst)", "algorithmic_flops": kf, "algorithmic_bytes": kb,
                    "kernel_ms": kms}
    else:
        achieved = kb / (kms / 1e3) / 1e9
        roofline = {"bound": "hbm", "kernel": "expert_gate_up", "achieved": achieved, "peak": pk["hbm_gbs"],
                    "unit": "GB/s", "frac": achieved / pk["hbm_gbs"], "traffic": None, "peak_source": pk["source"],
                    "algorithmic_bytes": kb, "algorithmic_flops": kf, "kernel_ms": kms}
    cpu = None
    if not args.no_cpu_baseline:
        from oracle import moe_oracle as O
        n = min(T, 8)
        t0 = time.perf_counter()
        O.dense_mlp(inp["x"][:n], inp["w_gate_up"], inp["w_down"])
        secs = time.perf_counter() - t0
        cpu = {"value": n / secs, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
               "sample": f"first {n} tokens, fp64 numpy oracle, one pass", "seconds": secs}
    line = {
        "metric": "dense-prefix MLP tokens/s at 1 B200 (Ling-2.6-flash layer 0)", "value": T / (ms_per_step / 1e3),
        "unit": "tokens/s", "n_gpus": 1, "steps": K, "warmup": warm, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"ling26_flash_dense_mlp_t{T}", "hidden_size": H, "intermediate_size": Id,
                   "tokens": T, "l2": "256 MiB L2 flush between timed steps; weights 226 MB > 126 MB L2"},
        "step_hbm_gbs": work["step_bytes"] / (ms_per_step / 1e3) / 1e9,
        "roofline": roofline, "cpu_baseline": cpu,
        "e2e": {"value": T / (e2e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": int(x_host.numel() * 2),
                "d2h_bytes_per_step": int(y_host.numel() * 2)},
        "gpu_launches": int(launches), "clocks": clk.summary(),
    }
    print(json.dumps(line))
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(G.WORKLOADS))
    ap.add_argument("--kernel", default="auto", choices=["auto", "expert_gate_up", "expert_down", "decode_fused"],
                    help="kernel whose live timing gives the roofline (auto: the fused decode kernel when the "
                         "library runs the block as one launch, else whichever expert pass takes longer)")
    ap.add_argument("--cpu-sample", type=int, default=256)
    ap.add_argument("--ref-sample", type=int, default=8)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ffn-path", default="auto", choices=["auto", "streaming", "tensor_cores"],
                    help="expert-FFN kernels (default: the library's automatic choice)")
    ap.add_argument("--down-weights", default="f16", choices=["f16", "bf16"],
                    help="down_proj operands of the tensor-core pass: an fp16 copy made before timing, or the bf16 "
                         "weights (h then kept as two bf16 planes)")
    ap.add_argument("--decode", default="auto", choices=["auto", "unfused"],
                    help="a few tokens as one fused launch (auto, the library's choice) or as separate kernels")
    ap.add_argument("--set", action="append", default=[], metavar="FIELD=VALUE",
                    help="override a workload field (e.g. num_experts=64 for a small profiling case)")
    ap.add_argument("--q8", type=int, default=0, metavar="GROUP",
                    help="run the block with 8-bit affine expert weights of this group size (32, 64 or 128)")
    ap.add_argument("--dense", type=int, default=0, metavar="TOKENS",
                    help="time the dense-prefix MLP (Ling-2.6-flash layer 0) on TOKENS tokens instead of the block")
    args = ap.parse_args()
    if args.dense > 0:
        return run_dense(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
