"""The binding refuses tensors the library would overrun or misread, on the CPU.

Every entry point reads or writes a fixed number of elements through each
pointer (T*d for x, E*f*d for W1, ...). A caller's tensor of the wrong dtype or
with too few elements must be stopped before its address reaches the GPU. The
checks run before the device check, so CPU tensors exercise them here; a
well-formed CPU argument list gets as far as the "must live on a CUDA device"
refusal.
"""
import pytest
import torch

from mixture_experts_ffn_sigmoid_b200 import binding as B
from mixture_experts_ffn_sigmoid_b200.inputs import MoEConfig

CFG = MoEConfig("checks", T=6, d=16, E=4, k=2, f=24, f_shared=8)
T, d, E, k, f, fs = CFG.T, CFG.d, CFG.E, CFG.k, CFG.f, CFG.f_shared
R = T * k
bf, f32, i32 = torch.bfloat16, torch.float32, torch.int32


def t(shape, dtype=bf):
    return torch.zeros(shape, dtype=dtype)


def ws():
    return torch.zeros(1024, dtype=torch.uint8)


def route_args():
    return dict(x=t((T, d)), w_router=t((E, d)), bias=t((E,), f32), topk_idx=t((T, k), i32),
                topk_gate=t((T, k), f32), expert_counts=t((E,), i32), expert_offsets=t((E + 1,), i32),
                workspace=ws())


def block_args():
    return dict(x=t((T, d)), w_router=t((E, d)), bias=t((E,), f32), w1=t((E, f, d)), w3=t((E, f, d)),
                w2=t((E, d, f)), ws1=t((fs, d)), ws3=t((fs, d)), ws2=t((d, fs)), y=t((T, d)), workspace=ws())


def grad_args():
    return dict(dy=t((T, d)), dx=t((T, d)), dw_router=t((E, d)), dw1=t((E, f, d)), dw3=t((E, f, d)),
                dw2=t((E, d, f)), dws1=t((fs, d)), dws3=t((fs, d)), dws2=t((d, fs)))


CALLS = {
    "moe_route": (B.moe_route, route_args),
    "moe_route_noalloc": (B.moe_route_noalloc,
                          lambda: {kk: v for kk, v in route_args().items() if kk != "workspace"}),
    "moe_permute": (B.moe_permute, lambda: dict(x=t((T, d)), topk_idx=t((T, k), i32),
                                                expert_offsets=t((E + 1,), i32), x_perm=t((R, d)),
                                                perm_src=t((R,), i32), inv_row=t((T, k), i32), workspace=ws())),
    "moe_expert_swiglu": (B.moe_expert_swiglu, lambda: dict(
        x_perm=t((R, d)), expert_offsets=t((E + 1,), i32), w1=t((E, f, d)), w3=t((E, f, d)), w2=t((E, d, f)),
        x_shared=t((T, d)), ws1=t((fs, d)), ws3=t((fs, d)), ws2=t((d, fs)), y_perm=t((R, d)),
        y_shared=t((T, d)), workspace=ws())),
    "moe_expert_gate_up": (B.moe_expert_gate_up, lambda: dict(
        x_perm=t((R, d)), expert_offsets=t((E + 1,), i32), w1=t((E, f, d)), w3=t((E, f, d)),
        x_shared=t((T, d)), ws1=t((fs, d)), ws3=t((fs, d)), h=t((R, f)), h_shared=t((T, fs)), workspace=ws())),
    "moe_expert_gate_up_gather": (B.moe_expert_gate_up_gather, lambda: dict(
        x=t((T, d)), perm_src=t((R,), i32), expert_offsets=t((E + 1,), i32), w1=t((E, f, d)),
        w3=t((E, f, d)), ws1=t((fs, d)), ws3=t((fs, d)), h=t((R, f)), h_shared=t((T, fs)), workspace=ws())),
    "moe_expert_down": (B.moe_expert_down, lambda: dict(
        h=t((R, f)), expert_offsets=t((E + 1,), i32), w2=t((E, d, f)), h_shared=t((T, fs)), ws2=t((d, fs)),
        y_perm=t((R, d)), y_shared=t((T, d)), workspace=ws())),
    "moe_combine": (B.moe_combine, lambda: dict(y_perm=t((R, d)), inv_row=t((T, k), i32),
                                                topk_gate=t((T, k), f32), y_shared=t((T, d)), y=t((T, d)))),
    "moe_forward": (B.moe_forward, block_args),
    "moe_forward_train": (B.moe_forward_train, block_args),
    "moe_backward": (B.moe_backward,
                     lambda: {**{kk: v for kk, v in block_args().items() if kk != "y"}, **grad_args()}),
    "moe_backward_saved": (B.moe_backward_saved,
                           lambda: {**{kk: v for kk, v in block_args().items() if kk not in ("y", "bias")},
                                    **grad_args()}),
    "moe_balance_update": (B.moe_balance_update, lambda: dict(expert_counts=t((E,), i32), bias=t((E,), f32),
                                                              gamma=0.1, entropy=t((1,), f32))),
}
GELU_CFG = CFG.with_(f_shared=0)
GELU_CALLS = {
    "moe_expert_gelu": (B.moe_expert_gelu, lambda: dict(
        x_perm=t((R, d)), expert_offsets=t((E + 1,), i32), w1=t((E, f, d)), b1=t((E, f), f32),
        w2=t((E, d, f)), b2=t((E, d), f32), y_perm=t((R, d)), workspace=ws())),
    "moe_forward_gelu": (B.moe_forward_gelu, lambda: dict(
        x=t((T, d)), w_router=t((E, d)), bias=t((E,), f32), w1=t((E, f, d)), b1=t((E, f), f32),
        w2=t((E, d, f)), b2=t((E, d), f32), y=t((T, d)), workspace=ws())),
}
ALL = [(n, CFG, fn, mk) for n, (fn, mk) in CALLS.items()] + \
      [(n, GELU_CFG, fn, mk) for n, (fn, mk) in GELU_CALLS.items()]


@pytest.mark.parametrize("name,cfg,fn,make", ALL, ids=[a[0] for a in ALL])
def test_well_formed_arguments_reach_the_device_check(name, cfg, fn, make):
    with pytest.raises(ValueError, match="CUDA device"):
        fn(cfg, **make())


@pytest.mark.parametrize("name,cfg,fn,make", ALL, ids=[a[0] for a in ALL])
def test_every_tensor_is_checked(name, cfg, fn, make):
    """One tensor at a time: one element short, then the wrong dtype."""
    names = [kk for kk, v in make().items() if isinstance(v, torch.Tensor) and kk != "workspace"]
    assert names
    for arg in names:
        args = make()
        good = args[arg]
        args[arg] = good.flatten()[:-1] if good.numel() > 0 else good
        if good.numel() > 0:
            with pytest.raises(ValueError, match=f"{arg}: .* elements"):
                fn(cfg, **args)
        args = make()
        wrong = torch.float16 if good.dtype != torch.float16 else torch.float32
        args[arg] = good.to(wrong)
        with pytest.raises(ValueError, match=f"{arg}: dtype"):
            fn(cfg, **args)


@pytest.mark.parametrize("name,cfg,fn,make", ALL, ids=[a[0] for a in ALL])
def test_workspace_must_be_bytes(name, cfg, fn, make):
    args = make()
    if "workspace" not in args:
        pytest.skip("no workspace argument")
    args["workspace"] = torch.zeros(256, dtype=torch.float32)
    with pytest.raises(ValueError, match="workspace: dtype"):
        fn(cfg, **args)


def test_shared_expert_tensors_required_only_with_a_shared_expert():
    args = block_args()
    args["ws2"] = None
    with pytest.raises(ValueError, match="ws2 is required"):
        B.moe_forward(CFG, **args)
    plain = CFG.with_(f_shared=0)
    args = block_args()
    args.update(ws1=None, ws3=None, ws2=None)
    with pytest.raises(ValueError, match="CUDA device"):
        B.moe_forward(plain, **args)


def test_optional_pointers_may_be_none():
    args = route_args()
    args["bias"] = None
    with pytest.raises(ValueError, match="CUDA device"):
        B.moe_route(CFG, **args)
    # permute without x_perm writes the maps only, and then needs no x
    with pytest.raises(ValueError, match="CUDA device"):
        B.moe_permute(CFG, None, t((T, k), i32), t((E + 1,), i32), None, t((R,), i32), t((T, k), i32), ws())
    with pytest.raises(ValueError, match="x is required"):
        B.moe_permute(CFG, None, t((T, k), i32), t((E + 1,), i32), t((R, d)), t((R,), i32), t((T, k), i32),
                      ws())


def test_config_with_T_override_sizes_the_checks():
    c = B.make_config(CFG, T=3)
    args = block_args()
    args["x"] = t((3, d))
    args["y"] = t((3, d))
    with pytest.raises(ValueError, match="CUDA device"):
        B.moe_forward(c, **args)
    args["x"] = t((2, d))
    with pytest.raises(ValueError, match="x: .* elements"):
        B.moe_forward(c, **args)


def test_token_arrays_may_be_none_when_there_are_no_tokens():
    c = B.make_config(CFG, T=0)
    args = {**{kk: v for kk, v in block_args().items() if kk != "y"}, **grad_args()}
    args.update(x=None, dy=None, dx=None)
    with pytest.raises(ValueError, match="CUDA device"):
        B.moe_backward(c, **args)
    args["w1"] = None            # weights are still read when T = 0 (zero gradients are written)
    with pytest.raises(ValueError, match="w1 is required"):
        B.moe_backward(c, **args)


def test_workspace_is_required():
    args = block_args()
    args["workspace"] = None
    with pytest.raises(ValueError, match="workspace is required"):
        B.moe_forward(CFG, **args)
