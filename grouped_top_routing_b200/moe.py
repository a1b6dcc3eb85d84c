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
                4: "MOE_ERR_CUDA", 5: "MOE_ERR_DEVICE_CHECK", 6: "MOE_ERR_TIMEOUT"}
SCORE = {"softmax": 0, "sigmoid": 1}
KERNELS = {"router_logits": 0, "route": 1, "permute": 2, "expert_gate_up": 3, "expert_down": 4, "combine": 5,
           "decode_fused": 6}
FUSED_DECODE_MAX_TOKENS = 2  # moe_forward runs the whole block as one launch at or below this batch

# Every entry point include/moe.h declares.
EXPORTS = ("moe_workspace_size", "moe_workspace_init", "moe_router_logits", "moe_route", "moe_permute",
           "moe_expert_ffn", "moe_combine", "moe_forward", "moe_check_device", "moe_set_kernel_timer",
           "moe_set_ffn_path", "moe_set_decode_kernel", "moe_launch_count", "moe_last_error", "moe_permute_static",
           "moe_dense_mlp_workspace_size", "moe_dense_mlp", "moe_forward_q8")
FFN_PATHS = {"auto": 0, "streaming": 1, "tensor_cores": 2}


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
    st = ctypes.c_int
    sig = {
        "moe_workspace_size": (sz, [cfgp, i64]),
        "moe_workspace_init": (st, [vp, sz, vp]),
        "moe_router_logits": (st, [cfgp, vp, i64, vp, vp, vp, sz, vp]),
        "moe_route": (st, [cfgp, vp, vp, i64, vp, vp, vp]),
        "moe_permute": (st, [cfgp, vp, i64, vp, vp, vp, vp, vp, vp, sz, vp]),
        "moe_expert_ffn": (st, [cfgp, i64, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
        "moe_combine": (st, [cfgp, i64, vp, vp, vp, vp]),
        "moe_forward": (st, [cfgp, vp, i64, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
        "moe_check_device": (st, [vp, sz, vp]),
        "moe_set_kernel_timer": (st, [ctypes.c_int32, vp, vp]),
        "moe_set_ffn_path": (st, [ctypes.c_int32]),
        "moe_set_decode_kernel": (st, [ctypes.c_int32]),
        "moe_permute_static": (st, [cfgp, vp, i64, vp, vp, vp, vp, vp, vp]),
        "moe_dense_mlp_workspace_size": (sz, [ctypes.c_int32, ctypes.c_int32, i64]),
        "moe_dense_mlp": (st, [ctypes.c_int32, ctypes.c_int32, vp, i64, vp, vp, vp, vp, sz, vp]),
        "moe_forward_q8": (st, [cfgp, vp, i64, vp, vp, vp, ctypes.POINTER(Q8Weights), vp, vp, vp, vp, vp, vp, sz, vp]),
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


def moe_router_logits(cfg, x, router_w, ws: "Workspace", out=None, stream=None):
    c = _as_cfg(cfg)
    T = x.shape[0]
    if out is None:
        out = torch.empty((T, c.num_experts), dtype=torch.float32, device=x.device)
    _check(lib.moe_router_logits(ctypes.byref(c), _p(x), T, _p(router_w), _p(out), ws.cptr, ws.nbytes,
                                 _stream(stream)))
    return out


def moe_route(cfg, logits, expert_bias=None, topk_idx=None, topk_w=None, stream=None):
    c = _as_cfg(cfg)
    T = logits.shape[0]
    k = c.num_experts_per_tok
    if topk_idx is None:
        topk_idx = torch.empty((T, k), dtype=torch.int32, device=logits.device)
    if topk_w is None:
        topk_w = torch.empty((T, k), dtype=torch.float32, device=logits.device)
    _check(lib.moe_route(ctypes.byref(c), _p(logits), _p(expert_bias), T, _p(topk_idx), _p(topk_w), _stream(stream)))
    return topk_idx, topk_w


def moe_permute(cfg, topk_idx, ws: Workspace, x=None, want_x_perm=False, stream=None):
    c = _as_cfg(cfg)
    T = topk_idx.shape[0]
    k, E, H = c.num_experts_per_tok, c.num_experts, c.hidden_size
    dev = topk_idx.device
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    row_of = torch.empty((T, k), dtype=torch.int32, device=dev)
    tok_of = torch.empty(T * k, dtype=torch.int32, device=dev)
    x_perm = torch.empty((T * k, H), dtype=torch.bfloat16, device=dev) if want_x_perm else None
    _check(lib.moe_permute(ctypes.byref(c), _p(topk_idx), T, _p(x), _p(offsets), _p(row_of), _p(tok_of), _p(x_perm),
                           ws.cptr, ws.nbytes, _stream(stream)))
    return offsets, row_of, tok_of, x_perm


def moe_expert_ffn(cfg, x, expert_offsets, tok_of, topk_w, w_gate_up, w_down, ws: Workspace, ws_gate_up=None,
                   ws_down=None, x_perm=None, y_slots=None, shared_out=None, stream=None):
    c = _as_cfg(cfg)
    T = x.shape[0]
    k, H = c.num_experts_per_tok, c.hidden_size
    if y_slots is None:
        y_slots = torch.empty((T * k, H), dtype=torch.float32, device=x.device)
    if ws_gate_up is not None and shared_out is None:
        shared_out = torch.empty((T, H), dtype=torch.float32, device=x.device)
    _check(lib.moe_expert_ffn(ctypes.byref(c), T, _p(x), _p(x_perm), _p(expert_offsets), _p(tok_of), _p(topk_w),
                              _p(w_gate_up), _p(w_down), _p(ws_gate_up), _p(ws_down), _p(y_slots), _p(shared_out),
                              ws.cptr, ws.nbytes, _stream(stream)))
    return y_slots, shared_out


def moe_combine(cfg, y_slots, shared_out, T: int, y=None, stream=None):
    c = _as_cfg(cfg)
    if y is None:
        y = torch.empty((T, c.hidden_size), dtype=torch.bfloat16, device=y_slots.device)
    _check(lib.moe_combine(ctypes.byref(c), T, _p(y_slots), _p(shared_out), _p(y), _stream(stream)))
    return y


def shared_width(c: MoeConfig) -> int:
    """Width of the shared MLP as the library derives it from the config."""
    if c.num_shared_experts <= 0:
        return 0
    per = c.moe_shared_expert_intermediate_size or c.moe_intermediate_size
    return per * c.num_shared_experts


def _require(t, name: str, numel: int, dtype):
    """The C ABI sees raw pointers only: a tensor smaller than the config says
    would be read past its end on the device, so check sizes here."""
    if t is None:
        return
    if t.numel() != numel or t.dtype != dtype or not t.is_contiguous():
        raise ValueError(f"{name}: expected {numel} contiguous {dtype} elements for this config, got "
                         f"{tuple(t.shape)} {t.dtype}{'' if t.is_contiguous() else ' (not contiguous)'}")


def _check_block_tensors(c: MoeConfig, T, x, router_w, expert_bias, logits_override, w_gate_up, w_down,
                         ws_gate_up, ws_down):
    E, H, I, Is = c.num_experts, c.hidden_size, c.moe_intermediate_size, shared_width(c)
    _require(x, "x", T * H, torch.bfloat16)
    _require(router_w, "router_w", E * H, torch.float32)
    _require(expert_bias, "expert_bias", E, torch.float32)
    _require(logits_override, "logits_override", T * E, torch.float32)
    _require(w_gate_up, "w_gate_up", E * 2 * I * H, torch.bfloat16)
    _require(w_down, "w_down", E * H * I, torch.bfloat16)
    _require(ws_gate_up, "ws_gate_up", 2 * Is * H, torch.bfloat16)
    _require(ws_down, "ws_down", H * Is, torch.bfloat16)


def moe_forward(cfg, x, router_w, expert_bias, w_gate_up, w_down, ws_gate_up, ws_down, ws: Workspace,
                logits_override=None, y=None, return_routing=False, stream=None):
    c = _as_cfg(cfg)
    T = x.shape[0]
    k = c.num_experts_per_tok
    _check_block_tensors(c, T, x, router_w, expert_bias, logits_override, w_gate_up, w_down, ws_gate_up, ws_down)
    if y is None:
        y = torch.empty_like(x)
    idx = w = None
    if return_routing:
        idx = torch.empty((T, k), dtype=torch.int32, device=x.device)
        w = torch.empty((T, k), dtype=torch.float32, device=x.device)
    _check(lib.moe_forward(ctypes.byref(c), _p(x), T, _p(router_w), _p(expert_bias), _p(logits_override),
                           _p(w_gate_up), _p(w_down), _p(ws_gate_up), _p(ws_down), _p(y), _p(idx), _p(w),
                           ws.cptr, ws.nbytes, _stream(stream)))
    if return_routing:
        return y, idx, w
    return y


def set_ffn_path(path: str = "auto"):
    """Expert-FFN kernels for later calls: "auto", "streaming" or "tensor_cores"."""
    _check(lib.moe_set_ffn_path(FFN_PATHS[path]))


DECODE_KERNELS = {"auto": 0, "cuda_cores": 1, "tensor_cores": 2}


def set_decode_kernel(which: str = "auto"):
    """Fused decode kernel for later calls: "auto" (the CUDA-core kernel),
    "cuda_cores", or "tensor_cores" (where its shapes fit)."""
    _check(lib.moe_set_decode_kernel(DECODE_KERNELS[which]))


def set_kernel_timer(kernel: str, ev_start=None, ev_stop=None):
    a = ctypes.c_void_p(ev_start.cuda_event) if ev_start is not None else None
    b = ctypes.c_void_p(ev_stop.cuda_event) if ev_stop is not None else None
    _check(lib.moe_set_kernel_timer(KERNELS[kernel], a, b))


def launch_count() -> int:
    return int(lib.moe_launch_count())


def dense_mlp_workspace(hidden_size: int, intermediate_size: int, max_tokens: int, device="cuda") -> Workspace:
    """Workspace for moe_dense_mlp."""
    n = lib.moe_dense_mlp_workspace_size(int(hidden_size), int(intermediate_size), int(max_tokens))
    if n == 0:
        raise MoeError(1, last_error())
    return Workspace(None, max_tokens, device=device, nbytes=n)


def moe_dense_mlp(x, w_gate_up, w_down, ws: Workspace, y=None, stream=None):
    """Dense-prefix SwiGLU MLP: w_gate_up [2*Id, H] (gate rows first), w_down [H, Id]."""
    T, H = x.shape
    Id = w_down.shape[1]
    if y is None:
        y = torch.empty_like(x)
    _check(lib.moe_dense_mlp(int(H), int(Id), _p(x), T, _p(w_gate_up), _p(w_down), _p(y), ws.cptr, ws.nbytes,
                             _stream(stream)))
    return y


def moe_forward_q8(cfg, x, router_w, expert_bias, q8: dict, ws: Workspace, ws_gate_up=None, ws_down=None,
                   logits_override=None, y=None, return_routing=False, stream=None):
    """The block with 8-bit affine expert weights (q8 as in inputs.make_q8_weights);
    the shared MLP is q8's when present, else the bf16 ws_gate_up / ws_down."""
    c = _as_cfg(cfg)
    T = x.shape[0]
    k = c.num_experts_per_tok
    if y is None:
        y = torch.empty_like(x)
    idx = w = None
    if return_routing:
        idx = torch.empty((T, k), dtype=torch.int32, device=x.device)
        w = torch.empty((T, k), dtype=torch.float32, device=x.device)
    qw = q8_weights(q8)
    _check(lib.moe_forward_q8(ctypes.byref(c), _p(x), T, _p(router_w), _p(expert_bias), _p(logits_override),
                              ctypes.byref(qw), _p(ws_gate_up), _p(ws_down), _p(y), _p(idx), _p(w), ws.cptr,
                              ws.nbytes, _stream(stream)))
    if return_routing:
        return y, idx, w
    return y
