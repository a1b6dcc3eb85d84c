"""The C-ABI boundary on the host: the library loads, exports every symbol
include/moe.h declares, and rejects each invalid argument with a status
before any launch (mlxcel issue #838, section "Defensive requirements": one
rejection test per validation rule). No call here reaches the GPU."""
import ctypes
import os
import re

import pytest
import torch

from grouped_top_routing_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def M():
    B.build()
    from grouped_top_routing_b200 import moe
    return moe


def _declared():
    with open(os.path.join(ROOT, "include", "moe.h")) as f:
        src = f.read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_\w+)\s*\(", src)))


def test_header_declares_the_entry_points(M):
    names = _declared()
    assert set(names) == set(M.EXPORTS), names
    for n in ("moe_route", "moe_permute", "moe_expert_ffn", "moe_combine", "moe_forward"):
        assert n in names


def test_library_exports_every_declared_symbol(M):
    lib = ctypes.CDLL(M.library_path)
    for n in _declared():
        assert hasattr(lib, n), n


def _good(**over):
    c = dict(hidden_size=4096, num_experts=256, num_experts_per_tok=8, n_group=8, topk_group=4,
             score_function=1, norm_topk_prob=1, routed_scaling_factor=2.5, moe_intermediate_size=1024,
             num_shared_experts=1, moe_shared_expert_intermediate_size=0)
    c.update(over)
    return c


def _cfg(M, **over):
    return M.MoeConfig(**_good(**over))


BAD_CONFIGS = [
    ("hidden_size", dict(hidden_size=0), 1),
    ("hidden_size", dict(hidden_size=-8), 1),
    ("hidden_size", dict(hidden_size=1 << 20), 1),
    ("hidden_size", dict(hidden_size=4100), 2),          # not a multiple of 8
    ("num_experts", dict(num_experts=0), 1),
    ("num_experts", dict(num_experts=4096, n_group=1, topk_group=1), 1),
    ("num_experts_per_tok", dict(num_experts_per_tok=0), 1),
    ("num_experts_per_tok", dict(num_experts_per_tok=257), 1),  # k > E
    ("n_group", dict(n_group=0), 1),                     # zero checked before divisibility
    ("n_group", dict(n_group=64, topk_group=4), 1),
    ("divisible", dict(n_group=7, topk_group=4), 1),     # 256 % 7 != 0
    ("topk_group", dict(topk_group=0), 1),
    ("topk_group", dict(topk_group=9), 1),               # > n_group
    ("topk_group", dict(n_group=8, topk_group=1, num_experts_per_tok=64), 1),  # too few experts kept
    ("score_function", dict(score_function=2), 1),
    ("score_function", dict(score_function=-1), 1),
    ("norm_topk_prob", dict(norm_topk_prob=2), 1),
    ("routed_scaling_factor", dict(routed_scaling_factor=float("nan")), 1),
    ("routed_scaling_factor", dict(routed_scaling_factor=float("inf")), 1),
    ("moe_intermediate_size", dict(moe_intermediate_size=0), 1),
    ("moe_intermediate_size", dict(moe_intermediate_size=1030), 2),
    ("num_shared_experts", dict(num_shared_experts=-1), 1),
    ("num_shared_experts", dict(num_shared_experts=1000), 1),
    ("moe_shared_expert_intermediate_size", dict(moe_shared_expert_intermediate_size=-8), 1),
    ("moe_shared_expert_intermediate_size", dict(moe_shared_expert_intermediate_size=12), 2),
]


@pytest.mark.parametrize("field,over,status", BAD_CONFIGS, ids=[f"{b[0]}-{i}" for i, b in enumerate(BAD_CONFIGS)])
def test_invalid_config_rejected(M, field, over, status):
    c = _cfg(M, **over)
    fake = ctypes.c_void_p(1 << 20)
    for call in (
        lambda: M.lib.moe_route(ctypes.byref(c), fake, None, 4, fake, fake, None),
        lambda: M.lib.moe_forward(ctypes.byref(c), fake, 4, fake, None, None, fake, fake, fake, fake, fake, None,
                                  None, fake, 1 << 40, None, None),
        lambda: M.lib.moe_combine(ctypes.byref(c), 4, fake, None, fake, None),
    ):
        st = call()
        assert st == status, (field, st, M.last_error())
        msg = M.last_error()
        key = "num_experts" if field == "divisible" else field
        assert key in msg, msg
    assert M.lib.moe_workspace_size(ctypes.byref(c), 16) == 0


def test_null_config_rejected(M):
    assert M.lib.moe_route(None, None, None, 1, None, None, None) == 1
    assert "cfg" in M.last_error()


def test_valid_config_sizes(M):
    c = _cfg(M)
    n1 = M.lib.moe_workspace_size(ctypes.byref(c), 1)
    n2 = M.lib.moe_workspace_size(ctypes.byref(c), 512)
    assert 0 < n1 < n2 and n2 % 256 == 0
    # topk_group == n_group is valid: every group kept
    c2 = _cfg(M, topk_group=8)
    assert M.lib.moe_workspace_size(ctypes.byref(c2), 8) > 0


def test_token_count_rejected(M):
    c = _cfg(M)
    fake = ctypes.c_void_p(1 << 20)
    assert M.lib.moe_route(ctypes.byref(c), fake, None, -1, fake, fake, None) == 1
    assert "T" in M.last_error()
    assert M.lib.moe_route(ctypes.byref(c), fake, None, 1 << 40, fake, fake, None) == 1


def test_zero_tokens_is_a_no_op(M):
    c = _cfg(M)
    assert M.lib.moe_route(ctypes.byref(c), None, None, 0, None, None, None) == 0
    assert M.lib.moe_combine(ctypes.byref(c), 0, None, None, None, None) == 0


def test_null_and_misaligned_pointers_rejected(M):
    c = _cfg(M)
    fake = ctypes.c_void_p(1 << 20)
    odd = ctypes.c_void_p((1 << 20) + 2)
    assert M.lib.moe_route(ctypes.byref(c), None, None, 4, fake, fake, None) == 1
    assert "logits" in M.last_error()
    assert M.lib.moe_route(ctypes.byref(c), fake, None, 4, None, fake, None) == 1
    assert "topk_idx" in M.last_error()
    assert M.lib.moe_combine(ctypes.byref(c), 4, odd, None, fake, None) == 1
    assert "y_slots" in M.last_error() and "aligned" in M.last_error()
    ws_need = M.lib.moe_workspace_size(ctypes.byref(c), 4)
    # forward: router weight required unless logits are given
    st = M.lib.moe_forward(ctypes.byref(c), fake, 4, None, None, None, fake, fake, fake, fake, fake, None, None, fake,
                           ws_need, None, None)
    assert st == 1 and "router_w" in M.last_error()
    # shared weights required when the config has a shared MLP
    st = M.lib.moe_forward(ctypes.byref(c), fake, 4, fake, None, None, fake, fake, None, None, fake, None, None, fake,
                           ws_need, None, None)
    assert st == 1 and "ws_gate_up" in M.last_error()
    # and rejected when it has none
    c0 = _cfg(M, num_shared_experts=0)
    ws0 = M.lib.moe_workspace_size(ctypes.byref(c0), 4)
    st = M.lib.moe_forward(ctypes.byref(c0), fake, 4, fake, None, None, fake, fake, fake, fake, fake, None, None, fake,
                           ws0, None, None)
    assert st == 1 and "shared" in M.last_error()


def test_workspace_rejected(M):
    c = _cfg(M)
    fake = ctypes.c_void_p(1 << 20)
    need = M.lib.moe_workspace_size(ctypes.byref(c), 64)
    st = M.lib.moe_permute(ctypes.byref(c), fake, 64, None, fake, fake, fake, None, fake, need - 1, None)
    assert st == 3 and "workspace" in M.last_error()
    st = M.lib.moe_permute(ctypes.byref(c), fake, 64, None, fake, fake, fake, None, None, need, None)
    assert st == 3
    st = M.lib.moe_permute(ctypes.byref(c), fake, 64, None, fake, fake, fake, None, ctypes.c_void_p((1 << 20) + 16),
                           need, None)
    assert st == 3 and "aligned" in M.last_error()
    assert M.lib.moe_workspace_init(None, 0, None) == 3


OPTION_BAD = [
    # field, value, text in the message
    ("ffn_path", 3, "ffn_path"),
    ("ffn_path", -1, "ffn_path"),
    ("decode_kernel", 2, "decode_kernel"),
    ("timer_kernel", 99, "timer_kernel"),
    ("timer_kernel", -2, "timer_kernel"),
    ("timer_kernel", 0, "timer events"),   # a kernel id without its events
    ("test_withhold", 3, "test_withhold"),
    ("w_down_f16", (1 << 20) + 8, "w_down_f16"),      # misaligned
    ("ws_down_f16", 1 << 20, "ws_down_f16"),          # the shared copy without the routed one
]


@pytest.mark.parametrize("field,value,text", OPTION_BAD, ids=[f"{f}={v}" for f, v, _ in OPTION_BAD])
def test_options_rejected_before_launch(M, field, value, text):
    # Per-call options are validated before anything else; a bad one launches nothing.
    c = _cfg(M)
    fake = ctypes.c_void_p(1 << 20)
    o = M.options()
    setattr(o, field, value)
    n0 = M.lib.moe_launch_count()
    st = M.lib.moe_forward(ctypes.byref(c), fake, 4, fake, None, None, fake, fake, fake, fake, fake, None, None,
                           fake, 1 << 40, None, ctypes.byref(o))
    assert st == 1 and text in M.last_error(), (st, M.last_error())
    st = M.lib.moe_dense_mlp(4096, 9216, fake, 4, fake, fake, fake, fake, 1 << 40, None, ctypes.byref(o))
    assert st == 1 and text in M.last_error()
    assert M.lib.moe_launch_count() == n0


def test_fp16_down_options_need_the_shared_copy(M):
    # A block with a shared MLP needs both fp16 copies; without a shared MLP
    # (dense MLP) the routed copy alone is enough.
    c = _cfg(M)
    assert M.shared_width(c) > 0
    fake = ctypes.c_void_p(1 << 20)
    o = M.options()
    o.w_down_f16 = 1 << 20
    n0 = M.lib.moe_launch_count()
    st = M.lib.moe_forward(ctypes.byref(c), fake, 4, fake, None, None, fake, fake, fake, fake, fake, None, None,
                           fake, 1 << 40, None, ctypes.byref(o))
    assert st == 1 and "ws_down_f16 is NULL" in M.last_error(), M.last_error()
    st = M.lib.moe_expert_ffn(ctypes.byref(c), 4, fake, None, fake, fake, None, fake, fake, fake, fake, fake, fake,
                              fake, 1 << 40, None, ctypes.byref(o))
    assert st == 1 and "ws_down_f16 is NULL" in M.last_error(), M.last_error()
    assert M.lib.moe_launch_count() == n0
    w = _q8(M, shared=False)
    st = M.lib.moe_forward_q8(ctypes.byref(c), fake, 4, fake, None, None, ctypes.byref(w), fake, fake, fake, None,
                              None, fake, 1 << 40, None, ctypes.byref(o))
    assert st == 1 and "moe_forward_q8" in M.last_error(), M.last_error()


def test_convert_rejects_before_launch(M):
    fake = 1 << 20
    n0 = M.lib.moe_launch_count()
    cnt = ctypes.c_void_p(fake)
    assert M.lib.moe_convert_bf16_to_f16(ctypes.c_void_p(fake), ctypes.c_void_p(fake * 2), -1, cnt, None) == 1
    assert "negative" in M.last_error()
    # dst starts inside src's range
    assert M.lib.moe_convert_bf16_to_f16(ctypes.c_void_p(fake), ctypes.c_void_p(fake + 64), 1000, cnt, None) == 1
    assert "overlap" in M.last_error()
    assert M.lib.moe_convert_bf16_to_f16(ctypes.c_void_p(fake), ctypes.c_void_p(fake + 8 * 1024), 16, None, None) == 1
    assert "out_of_range" in M.last_error()
    assert M.lib.moe_convert_bf16_to_f16(ctypes.c_void_p(fake + 2), ctypes.c_void_p(fake * 2), 16, cnt, None) == 1
    assert "src" in M.last_error()
    assert M.lib.moe_launch_count() == n0


def test_options_defaults(M):
    o = M.options()
    assert (o.ffn_path, o.decode_kernel, o.wait_limit_ns, o.timer_kernel, o.test_withhold) == (0, 0, 0, -1, 0)
    o = M.options("tensor_cores", "unfused", wait_limit_ns=1000, withhold="expert_accumulator")
    assert (o.ffn_path, o.decode_kernel, o.wait_limit_ns, o.test_withhold) == (2, 1, 1000, 2)


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    # The binding has no fallback: a missing library is an import error.
    import importlib.util
    import shutil
    pkg = tmp_path / "pkgcopy"
    pkg.mkdir()
    shutil.copy(os.path.join(ROOT, "grouped_top_routing_b200", "moe.py"), pkg / "moe.py")
    spec = importlib.util.spec_from_file_location("moe_nolib", pkg / "moe.py")
    mod = importlib.util.module_from_spec(spec)
    with pytest.raises(ImportError):
        spec.loader.exec_module(mod)


DENSE_BAD = [
    # hidden, intermediate, tokens, ws given, status, field named in the message
    (0, 9216, 1, True, 1, "hidden_size"),
    (4100, 9216, 1, True, 2, "hidden_size"),
    (4096, 0, 1, True, 1, "intermediate_size"),
    (4096, 9217, 1, True, 2, "intermediate_size"),
    (4096, 1 << 20, 1, True, 1, "intermediate_size"),
    (4096, 9216, -1, True, 1, "T"),
    (4096, 9216, 4, False, 3, "workspace"),
]


@pytest.mark.parametrize("H,Id,T,with_ws,status,field", DENSE_BAD)
def test_dense_mlp_rejects_before_launch(M, H, Id, T, with_ws, status, field):
    # Host-side rejection: nothing is launched, so this runs without a GPU.
    fake = ctypes.c_void_p(1 << 20)
    ws = fake if with_ws else None
    n0 = M.lib.moe_launch_count()
    st = M.lib.moe_dense_mlp(H, Id, fake, T, fake, fake, fake, ws, 1 << 40, None, None)
    assert st == status, (st, M.last_error())
    assert field in M.last_error()
    assert M.lib.moe_launch_count() == n0


def test_dense_mlp_workspace_size(M):
    assert M.lib.moe_dense_mlp_workspace_size(4096, 9216, 64) > 64 * 4096 * 4  # at least the fp32 rows
    assert M.lib.moe_dense_mlp_workspace_size(4096, 9217, 64) == 0
    assert "intermediate_size" in M.last_error()


def _q8(M, group=64, shared=True, misalign=None):
    fake = 1 << 20
    def mat(name):
        if name.startswith("shared") and not shared:
            return M.Q8Matrix(None, None, None)
        p = [ctypes.c_void_p(fake), ctypes.c_void_p(fake), ctypes.c_void_p(fake)]
        if misalign == name:
            p[0] = ctypes.c_void_p(fake + 8)
        return M.Q8Matrix(*p)
    return M.Q8Weights(group, mat("gate_up"), mat("down"), mat("shared_gate_up"), mat("shared_down"))


Q8_BAD = [
    # description, weights factory args, bf16 shared given, status, text in the message
    ("group 48", dict(group=48), False, 2, "group_size"),
    ("group 256", dict(group=256), False, 2, "group_size"),
    ("unaligned codes", dict(misalign="down"), False, 1, "down.q"),
    ("shared twice", dict(), True, 1, "both"),
    ("shared missing", dict(shared=False), False, 1, "ws_gate_up"),
]


@pytest.mark.parametrize("what,wargs,bf16_shared,status,text", Q8_BAD, ids=[b[0] for b in Q8_BAD])
def test_forward_q8_rejects_before_launch(M, what, wargs, bf16_shared, status, text):
    c = _cfg(M)
    fake = ctypes.c_void_p(1 << 20)
    w = _q8(M, **wargs)
    n0 = M.lib.moe_launch_count()
    st = M.lib.moe_forward_q8(ctypes.byref(c), fake, 4, fake, None, None, ctypes.byref(w),
                              fake if bf16_shared else None, fake if bf16_shared else None, fake, None, None,
                              fake, 1 << 40, None, None)
    assert st == status, (st, M.last_error())
    assert text in M.last_error(), M.last_error()
    assert M.lib.moe_launch_count() == n0


def test_forward_q8_rejects_null_weights(M):
    c = _cfg(M)
    fake = ctypes.c_void_p(1 << 20)
    st = M.lib.moe_forward_q8(ctypes.byref(c), fake, 4, fake, None, None, None, None, None, fake, None, None,
                              fake, 1 << 40, None, None)
    assert st == 1 and "NULL" in M.last_error()


def test_binding_checks_tensor_sizes_against_the_config(M):
    # The C ABI sees raw pointers only; the binding refuses tensors whose size
    # disagrees with the config before anything reaches the device.
    from grouped_top_routing_b200 import inputs as G
    wl = G.tiny_workload(tokens=2, hidden_size=64, moe_intermediate_size=32, shared_width=32)
    inp = G.make_inputs(wl, seed=0, device="cpu")
    args = dict(x=inp["x"], router_w=inp["router_w"], expert_bias=inp["expert_bias"], w_gate_up=inp["w_gate_up"],
                w_down=inp["w_down"], ws_gate_up=inp["ws_gate_up"], ws_down=inp["ws_down"])
    args["expert_bias"] = torch.zeros(wl["num_experts"])
    for name in ("router_w", "w_gate_up", "w_down", "ws_gate_up", "ws_down", "expert_bias"):
        bad = dict(args, **{name: args[name].reshape(-1)[:-1]})
        with pytest.raises(ValueError, match=name):
            M.moe_forward(wl, ws=None, **bad)
    with pytest.raises(ValueError, match="y:"):  # a caller-supplied output is checked too
        M.moe_forward(wl, ws=None, y=torch.empty(3, 64, dtype=torch.bfloat16), **args)
    # a shared MLP wider than the config says (the width the library derives is
    # moe_intermediate_size x num_shared_experts)
    wide = G.make_inputs(dict(wl, shared_width=64), seed=0, device="cpu")
    with pytest.raises(ValueError, match="ws_gate_up"):
        M.moe_forward(wl, ws=None, **dict(args, ws_gate_up=wide["ws_gate_up"], ws_down=wide["ws_down"]))
    assert M.shared_width(M.config_from_workload(wl)) == 32
    assert M.shared_width(M.config_from_workload(dict(wl, num_shared_experts=2))) == 64
    assert M.shared_width(M.config_from_workload(dict(wl, num_shared_experts=0))) == 0


def test_binding_rejects_host_tensors(M):
    # Right sizes but host memory: the kernels would dereference a host address
    # as a device one, so the binding refuses before any launch.
    from grouped_top_routing_b200 import inputs as G
    wl = G.tiny_workload(tokens=2, hidden_size=64, moe_intermediate_size=32, shared_width=32)
    inp = G.make_inputs(wl, seed=0, device="cpu")
    n0 = M.launch_count()
    with pytest.raises(ValueError, match="CUDA"):
        M.moe_forward(wl, inp["x"], inp["router_w"], inp["expert_bias"], inp["w_gate_up"], inp["w_down"],
                      inp["ws_gate_up"], inp["ws_down"], ws=None)
    with pytest.raises(ValueError, match="CUDA"):
        M.moe_route(wl, torch.zeros(2, wl["num_experts"]))
    assert M.launch_count() == n0


def test_component_wrappers_check_sizes(M):
    # Every component wrapper checks what it hands the C ABI (size first, so
    # these run on the host without a device).
    from grouped_top_routing_b200 import inputs as G
    wl = G.tiny_workload(tokens=4, hidden_size=64, num_experts=8, num_experts_per_tok=2, moe_intermediate_size=32,
                         shared_width=32)
    T, E, k, H = 4, 8, 2, 64
    f32, i32, bf = torch.float32, torch.int32, torch.bfloat16
    with pytest.raises(ValueError, match="logits"):
        M.moe_route(wl, torch.zeros(T, E - 1))
    with pytest.raises(ValueError, match="expert_bias"):
        M.moe_route(wl, torch.zeros(T, E), torch.zeros(E + 1))
    with pytest.raises(ValueError, match="topk_idx"):
        M.moe_route(wl, torch.zeros(T, E), topk_idx=torch.zeros(T, k + 1, dtype=i32))
    with pytest.raises(ValueError, match="topk_idx"):
        M.moe_permute(wl, torch.zeros(T, k, dtype=torch.int64), ws=None)
    with pytest.raises(ValueError, match="x:"):
        M.moe_permute(wl, torch.zeros(T, k, dtype=i32), ws=None, x=torch.zeros(T, H - 8, dtype=bf))
    with pytest.raises(ValueError, match="router_w"):
        M.moe_router_logits(wl, torch.zeros(T, H, dtype=bf), torch.zeros(E, H - 8), ws=None)
    good = dict(x=torch.zeros(T, H, dtype=bf), expert_offsets=torch.zeros(E + 1, dtype=i32),
                tok_of=torch.zeros(T * k, dtype=i32), topk_w=torch.zeros(T * k),
                w_gate_up=torch.zeros(E * 64 * H, dtype=bf), w_down=torch.zeros(E * H * 32, dtype=bf))
    for name, bad in (("expert_offsets", torch.zeros(E, dtype=i32)), ("tok_of", torch.zeros(T * k - 1, dtype=i32)),
                      ("topk_w", torch.zeros(T * k, dtype=torch.float64)), ("w_down", torch.zeros(7, dtype=bf))):
        with pytest.raises(ValueError, match=name):
            M.moe_expert_ffn(wl, ws=None, **dict(good, **{name: bad}))
    with pytest.raises(ValueError, match="y_slots"):
        M.moe_expert_ffn(wl, ws=None, y_slots=torch.zeros(T * k, H + 1), **good)
    with pytest.raises(ValueError, match="y_slots"):
        M.moe_combine(wl, torch.zeros(T * k - 1, H), None, T)
    with pytest.raises(ValueError, match="shared_out"):
        M.moe_combine(wl, torch.zeros(T * k, H), torch.zeros(T, H - 1), T)
    q8 = G.make_q8_weights(wl, seed=0, device="cpu", group_size=32, shared=True)
    bad_q8 = dict(q8, down=(q8["down"][0][:-16], q8["down"][1], q8["down"][2]))
    with pytest.raises(ValueError, match="down.q"):
        M.moe_forward_q8(wl, torch.zeros(T, H, dtype=bf), torch.zeros(E, H), None, bad_q8, ws=None)
    with pytest.raises(ValueError, match="router_w"):
        M.moe_forward_q8(wl, torch.zeros(T, H, dtype=bf), torch.zeros(E, H + 8), None, q8, ws=None)


def test_expert_parallel_lists_reject_before_launch(M):
    fake = ctypes.c_void_p(1 << 20)
    n0 = M.lib.moe_launch_count()
    assert M.lib.moe_ep_recv(fake, 33, 32, 10, fake, None) == 1 and "1024" in M.last_error()
    assert M.lib.moe_ep_recv(fake, 0, 8, 10, fake, None) == 1
    assert M.lib.moe_ep_recv(fake, 2, 8, -1, fake, None) == 1 and "R_recv" in M.last_error()
    assert M.lib.moe_ep_recv(None, 2, 8, 10, fake, None) == 1 and "recv_counts" in M.last_error()
    assert M.lib.moe_ep_scatter_back(fake, fake, 4, 4, 6, fake, None) == 1 and "multiple of 4" in M.last_error()
    assert M.lib.moe_ep_scatter_back(ctypes.c_void_p((1 << 20) + 4), fake, 4, 4, 64, fake, None) == 1
    assert "y_perm" in M.last_error()
    c = _cfg(M, num_experts_per_tok=0)
    assert M.lib.moe_ep_send(ctypes.byref(c), 4, fake, fake, fake, fake, fake, None) == 1
    c = _cfg(M)
    assert M.lib.moe_ep_send(ctypes.byref(c), 4, fake, fake, fake, ctypes.c_void_p((1 << 20) + 4), fake, None) == 1
    assert "counts" in M.last_error()
    assert M.lib.moe_launch_count() == n0
