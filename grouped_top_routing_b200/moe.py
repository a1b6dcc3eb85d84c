"""ctypes binding of libmoe.so (declared in include/moe.h).

Argument marshalling only: every step of the block runs in the library's CUDA
kernels. torch supplies device memory and the current stream. Importing this
module raises if libmoe.so is missing; there is no other implementation to
fall back to.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_PKG, "libmoe.so")

MOE_OK = 0
STATUS_NAMES = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED", 3: "MOE_ERR_WORKSPACE",
                4: "MOE_ERR_CUDA", 5: "MOE_ERR_DEVICE_CHECK", 6: "MOE_ERR_TIMEOUT", 7: "MOE_ERR_RANGE"}
SCORE = {"softmax": 0, "sigmoid": 1}
KERNELS = {"router_logits": 0, "route": 1, "permute": 2, "expert_gate_up": 3, "expert_down": 4, "combine": 5,
           "decode_fused": 6}

# Every entry point include/moe.h declares.
EXPORTS = ("moe_workspace_size", "moe_workspace_init", "moe_router_logits", "moe_route", "moe_permute",
           "moe_expert_ffn", "moe_combine", "moe_forward", "moe_check_device", "moe_launch_count", "moe_last_error",
           "moe_permute_static", "moe_dense_mlp_workspace_size", "moe_dense_mlp", "moe_forward_q8",
           "moe_convert_bf16_to_f16", "moe_ep_send", "moe_ep_recv", "moe_ep_scatter_back")
FFN_PATHS = {"auto": 0, "streaming": 1, "tensor_cores": 2}
FUSED_DECODE_MAX_TOKENS = 2  # moe_forward runs the whole block as one launch up to this batch (shapes permitting)
STREAM_MAX_TOKENS = 2  # ffn_path "auto": the streaming expert kernels up to this batch, the tensor cores above
DECODE = {"auto": 0, "unfused": 1}
WITHHOLD = {None: 0, "decode_routing": 1, "expert_accumulator": 2}


class MoeError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


class MoeConfig(ctypes.Structure):
    _fields_ = [
        ("hidden_size", ctypes.c_int32),
        ("num_experts", ctypes.c_int32),
        ("num_experts_per_tok", ctypes.c_int32),
        ("n_group", ctypes.c_int32),
        ("topk_group", ctypes.c_int32),
        ("score_function", ctypes.c_int32),
        ("norm_topk_prob", ctypes.c_int32),
        ("routed_scaling_factor", ctypes.c_float),
        ("moe_intermediate_size", ctypes.c_int32),
        ("num_shared_experts", ctypes.c_int32),
        ("moe_shared_expert_intermediate_size", ctypes.c_int32),
    ]


def config_from_workload(wl: dict) -> MoeConfig:
    sf = wl["score_function"]
    return MoeConfig(
        hidden_size=wl["hidden_size"], num_experts=wl["num_experts"],
        num_experts_per_tok=wl["num_experts_per_tok"], n_group=wl.get("n_group", 1),
        topk_group=wl.get("topk_group", 1), score_function=SCORE[sf] if isinstance(sf, str) else int(sf),
        norm_topk_prob=int(bool(wl["norm_topk_prob"])), routed_scaling_factor=float(wl["routed_scaling_factor"]),
        moe_intermediate_size=wl["moe_intermediate_size"], num_shared_experts=wl.get("num_shared_experts", 0),
        moe_shared_expert_intermediate_size=wl.get("moe_shared_expert_intermediate_size", 0),
    )


class Options(ctypes.Structure):
    """moe_options: per-call kernel choices, wait limit, timing hook and the
    optional fp16 copies of the down weights."""
    _fields_ = [
        ("ffn_path", ctypes.c_int32),
        ("decode_kernel", ctypes.c_int32),
        ("wait_limit_ns", ctypes.c_uint64),
        ("timer_kernel", ctypes.c_int32),
        ("timer_start", ctypes.c_void_p),
        ("timer_stop", ctypes.c_void_p),
        ("test_withhold", ctypes.c_int32),
        ("w_down_f16", ctypes.c_void_p),
        ("ws_down_f16", ctypes.c_void_p),
    ]


def options(ffn_path: str = "auto", decode: str = "auto", timer=None, wait_limit_ns: int = 0,
            withhold=None, w_down_f16=None, ws_down_f16=None) -> Options:
    """Build a moe_options: ffn_path in FFN_PATHS, decode in DECODE, timer =
    (kernel name, start event, stop event) or None, withhold in WITHHOLD (a
    test aid that makes one device wait run out), and w_down_f16 /
    ws_down_f16: fp16 copies of the down weights (convert_bf16_to_f16) for the
    tensor-core down pass. The struct keeps the tensors alive."""
    o = Options(FFN_PATHS[ffn_path], DECODE[decode], int(wait_limit_ns), -1, None, None, WITHHOLD[withhold],
                None, None)
    if timer is not None:
        name, ev0, ev1 = timer
        o.timer_kernel = KERNELS[name]
        o.timer_start = ev0.cuda_event
        o.timer_stop = ev1.cuda_event
    o.f16_tensors = (w_down_f16, ws_down_f16)
    if w_down_f16 is not None:
        o.w_down_f16 = w_down_f16.data_ptr()
    if ws_down_f16 is not None:
        o.ws_down_f16 = ws_down_f16.data_ptr()
    return o


def _check_down_f16(opts, dev, n_routed: int, n_shared: int):
    """Size, dtype and device of the fp16 down-weight copies an Options holds."""
    if opts is None:
        return
    wd, wsd = getattr(opts, "f16_tensors", (None, None))
    _require(wd, "w_down_f16", n_routed, torch.float16)
    _require(wsd, "ws_down_f16", n_shared, torch.float16)
    _on_device(dev, w_down_f16=wd, ws_down_f16=wsd)


def convert_bf16_to_f16(w, out=None, stream=None):
    """fp16 copy of bf16 weights (moe_convert_bf16_to_f16), checked: raises if
    a value is beyond fp16's range. Blocking (it reads the count)."""
    if not isinstance(w, torch.Tensor) or w.dtype != torch.bfloat16 or not w.is_cuda or not w.is_contiguous():
        raise ValueError("w: expected a contiguous CUDA bf16 tensor")
    if out is None:
        out = torch.empty(w.shape, dtype=torch.float16, device=w.device)
    _require(out, "out", w.numel(), torch.float16)
    _on_device(w.device, out=out)
    bad = torch.empty(1, dtype=torch.int32, device=w.device)
    _check(lib.moe_convert_bf16_to_f16(_p(w), _p(out), w.numel(), _p(bad), _stream(stream)))
    n_bad = int(bad.item())
    if n_bad:
        raise MoeError(7, f"{n_bad} values are beyond fp16's range")
    return out


def _opts(o):
    return None if o is None else ctypes.byref(o)


class Q8Matrix(ctypes.Structure):
    """moe_q8_matrix: codes [R, K] uint8, scale and bias [R, K / group_size] bf16."""
    _fields_ = [("q", ctypes.c_void_p), ("scale", ctypes.c_void_p), ("bias", ctypes.c_void_p)]


class Q8Weights(ctypes.Structure):
    """moe_q8_weights."""
    _fields_ = [("group_size", ctypes.c_int32), ("gate_up", Q8Matrix), ("down", Q8Matrix),
                ("shared_gate_up", Q8Matrix), ("shared_down", Q8Matrix)]


def q8_weights(q8: dict) -> Q8Weights:
    """ctypes view of a dict of (q, scale, bias) tensor triples (see inputs.make_q8_weights)."""
    def mat(t):
        if t is None:
            return Q8Matrix(None, None, None)
        return Q8Matrix(*(ctypes.c_void_p(x.data_ptr()) for x in t))
    return Q8Weights(int(q8["group_size"]), mat(q8["gate_up"]), mat(q8["down"]), mat(q8.get("shared_gate_up")),
                     mat(q8.get("shared_down")))


def _load():
    if not os.path.exists(library_path):
        raise ImportError(f"{library_path} is not built; run `python -m grouped_top_routing_b200.build`")
    L = ctypes.CDLL(library_path)
    vp, i64, sz, cfgp = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.POINTER(MoeConfig)
    op = ctypes.POINTER(Options)
    st = ctypes.c_int
    sig = {
        "moe_workspace_size": (sz, [cfgp, i64]),
        "moe_workspace_init": (st, [vp, sz, vp]),
        "moe_router_logits": (st, [cfgp, vp, i64, vp, vp, vp, sz, vp]),
        "moe_route": (st, [cfgp, vp, vp, i64, vp, vp, vp]),
        "moe_permute": (st, [cfgp, vp, i64, vp, vp, vp, vp, vp, vp, sz, vp]),
        "moe_expert_ffn": (st, [cfgp, i64, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp, op]),
        "moe_combine": (st, [cfgp, i64, vp, vp, vp, vp]),
        "moe_forward": (st, [cfgp, vp, i64, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp, op]),
        "moe_check_device": (st, [vp, sz, vp]),
        "moe_permute_static": (st, [cfgp, vp, i64, vp, vp, vp, vp, vp, vp]),
        "moe_dense_mlp_workspace_size": (sz, [ctypes.c_int32, ctypes.c_int32, i64]),
        "moe_dense_mlp": (st, [ctypes.c_int32, ctypes.c_int32, vp, i64, vp, vp, vp, vp, sz, vp, op]),
        "moe_forward_q8": (st, [cfgp, vp, i64, vp, vp, vp, ctypes.POINTER(Q8Weights), vp, vp, vp, vp, vp, vp, sz, vp,
                                op]),
        "moe_convert_bf16_to_f16": (st, [vp, vp, i64, vp, vp]),
        "moe_ep_send": (st, [cfgp, i64, vp, vp, vp, vp, vp, vp]),
        "moe_ep_recv": (st, [vp, ctypes.c_int32, ctypes.c_int32, i64, vp, vp]),
        "moe_ep_scatter_back": (st, [vp, vp, i64, i64, ctypes.c_int32, vp, vp]),
        "moe_launch_count": (ctypes.c_uint64, []),
        "moe_last_error": (ctypes.c_char_p, []),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    return L


lib = _load()


def last_error() -> str:
    return lib.moe_last_error().decode()


def _check(status: int):
    if status != MOE_OK:
        raise MoeError(status, last_error())


def _p(t):
    """Device (or host) address of a tensor, or None."""
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _cfg(cfg):
    return ctypes.byref(cfg if isinstance(cfg, MoeConfig) else config_from_workload(cfg))


def _as_cfg(cfg):
    return cfg if isinstance(cfg, MoeConfig) else config_from_workload(cfg)


def moe_workspace_size(cfg, max_tokens: int) -> int:
    n = lib.moe_workspace_size(_cfg(cfg), int(max_tokens))
    if n == 0:
        raise MoeError(1, last_error())
    return n


class Workspace:
    """A device workspace sized by moe_workspace_size (or, given nbytes, of that
    size), header zeroed."""

    def __init__(self, cfg, max_tokens: int, device="cuda", nbytes: int | None = None):
        self.nbytes = moe_workspace_size(cfg, max_tokens) if nbytes is None else int(nbytes)
        self.max_tokens = int(max_tokens)
        self.buf = torch.empty(self.nbytes + 256, dtype=torch.uint8, device=device)
        base = self.buf.data_ptr()
        self.ptr = (base + 255) & ~255
        _check(lib.moe_workspace_init(ctypes.c_void_p(self.ptr), self.nbytes, _stream()))

    @property
    def cptr(self):
        return ctypes.c_void_p(self.ptr)

    def check(self, stream=None):
        """Synchronise and raise if a device-side check or wait failed."""
        _check(lib.moe_check_device(self.cptr, self.nbytes, _stream(stream)))


def shared_width(c: MoeConfig) -> int:
    """Width of the shared MLP as the library derives it from the config."""
    if c.num_shared_experts <= 0:
        return 0
    per = c.moe_shared_expert_intermediate_size or c.moe_intermediate_size
    return per * c.num_shared_experts


def _require(t, name: str, numel: int, dtype):
    """The C ABI sees raw pointers only: a tensor smaller than the config says
    would be read or written past its end on the device. Check size, dtype and
    layout here, before any launch (the device is checked by _on_device once
    every size has passed)."""
    if t is None:
        return
    if not isinstance(t, torch.Tensor):
        raise ValueError(f"{name}: expected a torch tensor, got {type(t).__name__}")
    if t.numel() != numel or t.dtype != dtype or not t.is_contiguous():
        raise ValueError(f"{name}: expected {numel} contiguous {dtype} elements for this config, got "
                         f"{tuple(t.shape)} {t.dtype}{'' if t.is_contiguous() else ' (not contiguous)'}")


def _on_device(dev, **tensors):
    """A host tensor, or one on another GPU, would be dereferenced as a device
    address of the call's GPU: refuse it before any launch."""
    for name, t in tensors.items():
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError(f"{name}: expected a CUDA tensor, got one on {t.device}")
        if t.device != dev:
            raise ValueError(f"{name}: on {t.device}, but the call runs on {dev}")


def _rows(t, name: str):
    if not isinstance(t, torch.Tensor) or t.dim() < 1:
        raise ValueError(f"{name}: expected a tensor with a leading token dimension")
    return int(t.shape[0])


def _check_block_tensors(c: MoeConfig, T, x, router_w, expert_bias, logits_override, w_gate_up, w_down,
                         ws_gate_up, ws_down, y=None):
    E, H, I, Is = c.num_experts, c.hidden_size, c.moe_intermediate_size, shared_width(c)
    dev = x.device
    _require(x, "x", T * H, torch.bfloat16)
    _require(router_w, "router_w", E * H, torch.float32)
    _require(expert_bias, "expert_bias", E, torch.float32)
    _require(logits_override, "logits_override", T * E, torch.float32)
    _require(w_gate_up, "w_gate_up", E * 2 * I * H, torch.bfloat16)
    _require(w_down, "w_down", E * H * I, torch.bfloat16)
    _require(ws_gate_up, "ws_gate_up", 2 * Is * H, torch.bfloat16)
    _require(ws_down, "ws_down", H * Is, torch.bfloat16)
    _require(y, "y", T * H, torch.bfloat16)
    _on_device(x.device, x=x, router_w=router_w, expert_bias=expert_bias, logits_override=logits_override,
               w_gate_up=w_gate_up, w_down=w_down, ws_gate_up=ws_gate_up, ws_down=ws_down, y=y)


def _check_ws(ws, dev):
    if not isinstance(ws, Workspace):
        raise ValueError("ws: expected a Workspace")
    if ws.buf.device != dev:
        raise ValueError(f"workspace: on {ws.buf.device}, but the call runs on {dev}")


def moe_router_logits(cfg, x, router_w, ws: "Workspace", out=None, stream=None):
    c = _as_cfg(cfg)
    T = _rows(x, "x")
    dev = x.device
    _require(x, "x", T * c.hidden_size, torch.bfloat16)
    _require(router_w, "router_w", c.num_experts * c.hidden_size, torch.float32)
    _require(out, "logits", T * c.num_experts, torch.float32)
    _on_device(dev, x=x, router_w=router_w, logits=out)
    _check_ws(ws, dev)
    if out is None:
        out = torch.empty((T, c.num_experts), dtype=torch.float32, device=dev)
    _check(lib.moe_router_logits(ctypes.byref(c), _p(x), T, _p(router_w), _p(out), ws.cptr, ws.nbytes,
                                 _stream(stream)))
    return out


def moe_route(cfg, logits, expert_bias=None, topk_idx=None, topk_w=None, stream=None):
    c = _as_cfg(cfg)
    T = _rows(logits, "logits")
    k, E = c.num_experts_per_tok, c.num_experts
    dev = logits.device
    _require(logits, "logits", T * E, torch.float32)
    _require(expert_bias, "expert_bias", E, torch.float32)
    if topk_idx is None:
        topk_idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    if topk_w is None:
        topk_w = torch.empty((T, k), dtype=torch.float32, device=dev)
    _require(topk_idx, "topk_idx", T * k, torch.int32)
    _require(topk_w, "topk_w", T * k, torch.float32)
    _on_device(dev, logits=logits, expert_bias=expert_bias, topk_idx=topk_idx, topk_w=topk_w)
    _check(lib.moe_route(ctypes.byref(c), _p(logits), _p(expert_bias), T, _p(topk_idx), _p(topk_w), _stream(stream)))
    return topk_idx, topk_w


def moe_permute(cfg, topk_idx, ws: Workspace, x=None, want_x_perm=False, stream=None):
    c = _as_cfg(cfg)
    T = _rows(topk_idx, "topk_idx")
    k, E, H = c.num_experts_per_tok, c.num_experts, c.hidden_size
    dev = topk_idx.device
    _require(topk_idx, "topk_idx", T * k, torch.int32)
    _require(x, "x", T * H, torch.bfloat16)
    if want_x_perm and x is None:
        raise ValueError("x_perm needs x")
    _on_device(dev, topk_idx=topk_idx, x=x)
    _check_ws(ws, dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    row_of = torch.empty((T, k), dtype=torch.int32, device=dev)
    tok_of = torch.empty(T * k, dtype=torch.int32, device=dev)
    x_perm = torch.empty((T * k, H), dtype=torch.bfloat16, device=dev) if want_x_perm else None
    _check(lib.moe_permute(ctypes.byref(c), _p(topk_idx), T, _p(x), _p(offsets), _p(row_of), _p(tok_of), _p(x_perm),
                           ws.cptr, ws.nbytes, _stream(stream)))
    return offsets, row_of, tok_of, x_perm


def moe_expert_ffn(cfg, x, expert_offsets, tok_of, topk_w, w_gate_up, w_down, ws: Workspace, ws_gate_up=None,
                   ws_down=None, x_perm=None, y_slots=None, shared_out=None, stream=None, opts: Options | None = None):
    c = _as_cfg(cfg)
    T = _rows(x, "x")
    k, H, E, I, Is = c.num_experts_per_tok, c.hidden_size, c.num_experts, c.moe_intermediate_size, shared_width(c)
    dev = x.device
    _require(x, "x", T * H, torch.bfloat16)
    _require(x_perm, "x_perm", T * k * H, torch.bfloat16)
    _require(expert_offsets, "expert_offsets", E + 1, torch.int32)
    _require(tok_of, "tok_of", T * k, torch.int32)
    _require(topk_w, "topk_w", T * k, torch.float32)
    _require(w_gate_up, "w_gate_up", E * 2 * I * H, torch.bfloat16)
    _require(w_down, "w_down", E * H * I, torch.bfloat16)
    _require(ws_gate_up, "ws_gate_up", 2 * Is * H, torch.bfloat16)
    _require(ws_down, "ws_down", H * Is, torch.bfloat16)
    _require(y_slots, "y_slots", T * k * H, torch.float32)
    _require(shared_out, "shared_out", T * H, torch.float32)
    _on_device(dev, x=x, x_perm=x_perm, expert_offsets=expert_offsets, tok_of=tok_of, topk_w=topk_w,
               w_gate_up=w_gate_up, w_down=w_down, ws_gate_up=ws_gate_up, ws_down=ws_down, y_slots=y_slots,
               shared_out=shared_out)
    _check_down_f16(opts, dev, E * H * I, H * Is)
    _check_ws(ws, dev)
    if y_slots is None:
        y_slots = torch.empty((T * k, H), dtype=torch.float32, device=dev)
    if ws_gate_up is not None and shared_out is None:
        shared_out = torch.empty((T, H), dtype=torch.float32, device=dev)
    _check(lib.moe_expert_ffn(ctypes.byref(c), T, _p(x), _p(x_perm), _p(expert_offsets), _p(tok_of), _p(topk_w),
                              _p(w_gate_up), _p(w_down), _p(ws_gate_up), _p(ws_down), _p(y_slots), _p(shared_out),
                              ws.cptr, ws.nbytes, _stream(stream), _opts(opts)))
    return y_slots, shared_out


def moe_combine(cfg, y_slots, shared_out, T: int, y=None, stream=None):
    c = _as_cfg(cfg)
    k, H = c.num_experts_per_tok, c.hidden_size
    dev = y_slots.device
    _require(y_slots, "y_slots", T * k * H, torch.float32)
    _require(shared_out, "shared_out", T * H, torch.float32)
    if y is None:
        y = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    _require(y, "y", T * H, torch.bfloat16)
    _on_device(dev, y_slots=y_slots, shared_out=shared_out, y=y)
    _check(lib.moe_combine(ctypes.byref(c), T, _p(y_slots), _p(shared_out), _p(y), _stream(stream)))
    return y


def moe_forward(cfg, x, router_w, expert_bias, w_gate_up, w_down, ws_gate_up, ws_down, ws: Workspace,
                logits_override=None, y=None, return_routing=False, stream=None, opts: Options | None = None):
    c = _as_cfg(cfg)
    T = _rows(x, "x")
    k = c.num_experts_per_tok
    _check_block_tensors(c, T, x, router_w, expert_bias, logits_override, w_gate_up, w_down, ws_gate_up, ws_down, y)
    _check_down_f16(opts, x.device, c.num_experts * c.hidden_size * c.moe_intermediate_size,
                    c.hidden_size * shared_width(c))
    _check_ws(ws, x.device)
    if y is None:
        y = torch.empty_like(x)
    idx = w = None
    if return_routing:
        idx = torch.empty((T, k), dtype=torch.int32, device=x.device)
        w = torch.empty((T, k), dtype=torch.float32, device=x.device)
    _check(lib.moe_forward(ctypes.byref(c), _p(x), T, _p(router_w), _p(expert_bias), _p(logits_override),
                           _p(w_gate_up), _p(w_down), _p(ws_gate_up), _p(ws_down), _p(y), _p(idx), _p(w),
                           ws.cptr, ws.nbytes, _stream(stream), _opts(opts)))
    if return_routing:
        return y, idx, w
    return y


def launch_count() -> int:
    """Kernel launches this library made from the calling thread."""
    return int(lib.moe_launch_count())


def dense_mlp_workspace(hidden_size: int, intermediate_size: int, max_tokens: int, device="cuda") -> Workspace:
    """Workspace for moe_dense_mlp."""
    n = lib.moe_dense_mlp_workspace_size(int(hidden_size), int(intermediate_size), int(max_tokens))
    if n == 0:
        raise MoeError(1, last_error())
    return Workspace(None, max_tokens, device=device, nbytes=n)


def moe_dense_mlp(x, w_gate_up, w_down, ws: Workspace, y=None, stream=None, opts: Options | None = None):
    """Dense-prefix SwiGLU MLP: w_gate_up [2*Id, H] (gate rows first), w_down [H, Id]."""
    T = _rows(x, "x")
    if x.dim() != 2 or w_down.dim() != 2:
        raise ValueError("x [T, H] and w_down [H, Id] must be 2-D")
    H = int(x.shape[1])
    Id = int(w_down.shape[1])
    dev = x.device
    _require(x, "x", T * H, torch.bfloat16)
    _require(w_gate_up, "w_gate_up", 2 * Id * H, torch.bfloat16)
    _require(w_down, "w_down", H * Id, torch.bfloat16)
    _require(y, "y", T * H, torch.bfloat16)
    _on_device(dev, x=x, w_gate_up=w_gate_up, w_down=w_down, y=y)
    _check_down_f16(opts, dev, H * Id, 0)
    _check_ws(ws, dev)
    if y is None:
        y = torch.empty_like(x)
    _check(lib.moe_dense_mlp(int(H), int(Id), _p(x), T, _p(w_gate_up), _p(w_down), _p(y), ws.cptr, ws.nbytes,
                             _stream(stream), _opts(opts)))
    return y


def _check_q8(c: MoeConfig, q8: dict, dev):
    g = int(q8["group_size"])
    E, H, I, Is = c.num_experts, c.hidden_size, c.moe_intermediate_size, shared_width(c)
    if g <= 0 or H % g or I % g:
        raise ValueError(f"group_size {g} must divide hidden_size {H} and moe_intermediate_size {I}")

    def mat(t, name, R, K):
        if t is None:
            return
        q, sc, bi = t
        _require(q, f"{name}.q", R * K, torch.uint8)
        _require(sc, f"{name}.scale", R * (K // g), torch.bfloat16)
        _require(bi, f"{name}.bias", R * (K // g), torch.bfloat16)
    mat(q8["gate_up"], "gate_up", E * 2 * I, H)
    mat(q8["down"], "down", E * H, I)
    if q8.get("shared_gate_up") is not None:
        if Is % g:
            raise ValueError(f"group_size {g} must divide the shared MLP width {Is}")
        mat(q8["shared_gate_up"], "shared_gate_up", 2 * Is, H)
        mat(q8.get("shared_down"), "shared_down", H, Is)


def moe_forward_q8(cfg, x, router_w, expert_bias, q8: dict, ws: Workspace, ws_gate_up=None, ws_down=None,
                   logits_override=None, y=None, return_routing=False, stream=None, opts: Options | None = None):
    """The block with 8-bit affine expert weights (q8 as in inputs.make_q8_weights);
    the shared MLP is q8's when present, else the bf16 ws_gate_up / ws_down."""
    c = _as_cfg(cfg)
    T = _rows(x, "x")
    k, E, H = c.num_experts_per_tok, c.num_experts, c.hidden_size
    Is = shared_width(c)
    dev = x.device
    _require(x, "x", T * H, torch.bfloat16)
    _require(router_w, "router_w", E * H, torch.float32)
    _require(expert_bias, "expert_bias", E, torch.float32)
    _require(logits_override, "logits_override", T * E, torch.float32)
    _require(ws_gate_up, "ws_gate_up", 2 * Is * H, torch.bfloat16)
    _require(ws_down, "ws_down", H * Is, torch.bfloat16)
    _check_q8(c, q8, dev)
    _require(y, "y", T * H, torch.bfloat16)
    _on_device(dev, x=x, router_w=router_w, expert_bias=expert_bias, logits_override=logits_override,
               ws_gate_up=ws_gate_up, ws_down=ws_down, y=y)
    for key in ("gate_up", "down", "shared_gate_up", "shared_down"):
        if q8.get(key) is not None:
            q, sc, bi = q8[key]
            _on_device(dev, **{f"{key}.q": q, f"{key}.scale": sc, f"{key}.bias": bi})
    _check_ws(ws, dev)
    if y is None:
        y = torch.empty_like(x)
    idx = w = None
    if return_routing:
        idx = torch.empty((T, k), dtype=torch.int32, device=dev)
        w = torch.empty((T, k), dtype=torch.float32, device=dev)
    qw = q8_weights(q8)
    _check(lib.moe_forward_q8(ctypes.byref(c), _p(x), T, _p(router_w), _p(expert_bias), _p(logits_override),
                              ctypes.byref(qw), _p(ws_gate_up), _p(ws_down), _p(y), _p(idx), _p(w), ws.cptr,
                              ws.nbytes, _stream(stream), _opts(opts)))
    if return_routing:
        return y, idx, w
    return y


# ---------------------------------------------------------------------------
# expert parallelism: the row lists around the all-to-alls (moe_ep_*)
# ---------------------------------------------------------------------------

def ep_send(cfg, T: int, offsets, tok_of, topk_w, counts=None, row_w=None, stream=None):
    """Per-expert row counts (int64 [E]) and the routing weight of every
    permuted row (fp32 [T*k]; rows past offsets[E] are not written)."""
    c = _as_cfg(cfg)
    E, k = c.num_experts, c.num_experts_per_tok
    dev = offsets.device
    _require(offsets, "expert_offsets", E + 1, torch.int32)
    _require(tok_of, "tok_of", T * k, torch.int32)
    _require(topk_w, "topk_w", T * k, torch.float32)
    if counts is None:
        counts = torch.empty(E, dtype=torch.int64, device=dev)
    if row_w is None:
        row_w = torch.empty(T * k, dtype=torch.float32, device=dev)
    _require(counts, "counts", E, torch.int64)
    _require(row_w, "row_w", T * k, torch.float32)
    _on_device(dev, offsets=offsets, tok_of=tok_of, topk_w=topk_w, counts=counts, row_w=row_w)
    _check(lib.moe_ep_send(ctypes.byref(c), T, _p(offsets), _p(tok_of), _p(topk_w), _p(counts), _p(row_w),
                           _stream(stream)))
    return counts, row_w


def ep_recv(recv_counts, R_recv: int, out=None, stream=None):
    """Local expert id (int32 [R_recv]) of every received row, from the
    exchanged counts recv_counts [P, n_local] (int64)."""
    if not isinstance(recv_counts, torch.Tensor) or recv_counts.dim() != 2:
        raise ValueError("recv_counts: expected an int64 tensor [P, n_local]")
    P, n_local = (int(v) for v in recv_counts.shape)
    _require(recv_counts, "recv_counts", P * n_local, torch.int64)
    dev = recv_counts.device
    if out is None:
        out = torch.empty(R_recv, dtype=torch.int32, device=dev)
    _require(out, "local_expert", R_recv, torch.int32)
    _on_device(dev, recv_counts=recv_counts, local_expert=out)
    _check(lib.moe_ep_recv(_p(recv_counts), P, n_local, int(R_recv), _p(out), _stream(stream)))
    return out


def ep_scatter_back(y_perm, tok_of, n_slots: int, out=None, stream=None):
    """y_slots[tok_of[r]] = y_perm[r] for the rows of y_perm (fp32 [R, H])."""
    if not isinstance(y_perm, torch.Tensor) or y_perm.dim() != 2:
        raise ValueError("y_perm: expected an fp32 tensor [R, H]")
    R, H = (int(v) for v in y_perm.shape)
    _require(y_perm, "y_perm", R * H, torch.float32)
    if not isinstance(tok_of, torch.Tensor) or tok_of.dtype != torch.int32 or tok_of.numel() < R:
        raise ValueError(f"tok_of: expected at least {R} int32 entries")
    dev = y_perm.device
    if out is None:
        out = torch.empty((n_slots, H), dtype=torch.float32, device=dev)
    _require(out, "y_slots", n_slots * H, torch.float32)
    _on_device(dev, y_perm=y_perm, tok_of=tok_of, y_slots=out)
    _check(lib.moe_ep_scatter_back(_p(y_perm), _p(tok_of), R, int(n_slots), H, _p(out), _stream(stream)))
    return out

