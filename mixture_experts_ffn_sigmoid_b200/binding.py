"""ctypes binding of ``libmoe_b200.so`` (declared in ``include/moe.h``).

Argument marshalling only: every function here checks that each torch
tensor has the dtype the entry point expects and at least as many elements as
the library will read or write through it (a short buffer would be an
out-of-bounds access on the GPU), that it is a contiguous CUDA tensor, passes
the device pointers and the current CUDA stream to the C entry point of the
same name, and raises ``MoEError`` on a non-OK status. All compute runs in the library's CUDA kernels; there is no other
path. If the library is missing or cannot be loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

from .inputs import MoEConfig

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe_b200.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_MISALIGNED = 2
MOE_ERR_UNSUPPORTED = 3
MOE_ERR_WORKSPACE_TOO_SMALL = 4
MOE_ERR_CUDA = 5
MOE_ERR_TIMEOUT = 6

MOE_DTYPE_F32 = 0
MOE_DTYPE_BF16 = 1

EXPORTED = ("moe_check_config", "moe_workspace_size", "moe_route", "moe_permute",
            "moe_expert_swiglu", "moe_expert_gate_up", "moe_expert_gate_up_gather", "moe_expert_down",
            "moe_combine", "moe_forward", "moe_get_device_error",
            "moe_selftest_wait_timeout", "moe_route_noalloc", "moe_route_noalloc_device_error",
            "moe_forward_gathers_rows", "moe_route_maps", "moe_route_maps_supported",
            "moe_balance_update",
            "moe_expert_gelu", "moe_forward_gelu", "moe_backward_workspace_size", "moe_backward",
            "moe_forward_train", "moe_backward_saved", "moe_status_string")


class MoEError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


class CConfig(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("d", ctypes.c_int32), ("E", ctypes.c_int32),
                ("k", ctypes.c_int32), ("f", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("gate_mode", ctypes.c_int32), ("n_groups", ctypes.c_int32),
                ("topk_groups", ctypes.c_int32), ("route_scale", ctypes.c_float),
                ("f_shared", ctypes.c_int32)]


_lib = None


def library_path() -> str:
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    """Load the CUDA library once; raise if it is not there."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"{_LIB_PATH} is missing: build it with "
                               "`python -m mixture_experts_ffn_sigmoid_b200.build`")
        L = ctypes.CDLL(_LIB_PATH)
        vp, sz, i32p, f32p = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_void_p
        cfgp = ctypes.POINTER(CConfig)
        sig = {
            "moe_check_config": (ctypes.c_int, [cfgp]),
            "moe_workspace_size": (sz, [cfgp]),
            "moe_route": (ctypes.c_int, [cfgp, vp, vp, f32p, i32p, f32p, i32p, i32p, vp, sz, vp]),
            "moe_permute": (ctypes.c_int, [cfgp, vp, i32p, i32p, vp, i32p, i32p, vp, sz, vp]),
            "moe_expert_swiglu": (ctypes.c_int, [cfgp, vp, i32p, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                                 vp, sz, vp]),
            "moe_expert_gate_up": (ctypes.c_int, [cfgp, vp, i32p, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
            "moe_expert_gate_up_gather": (ctypes.c_int, [cfgp, vp, i32p, i32p, vp, vp, vp, vp, vp, vp, vp,
                                                         sz, vp]),
            "moe_expert_down": (ctypes.c_int, [cfgp, vp, i32p, vp, vp, vp, vp, vp, vp, sz, vp]),
            "moe_combine": (ctypes.c_int, [cfgp, vp, i32p, f32p, vp, vp, vp]),
            "moe_forward": (ctypes.c_int, [cfgp, vp, vp, f32p, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
            "moe_get_device_error": (ctypes.c_int, [vp, vp]),
            "moe_selftest_wait_timeout": (ctypes.c_int, [vp, sz, ctypes.c_int64, vp]),
            "moe_route_noalloc": (ctypes.c_int, [cfgp, vp, vp, f32p, i32p, f32p, i32p, i32p, vp]),
            "moe_route_noalloc_device_error": (ctypes.c_int, [vp]),
            "moe_forward_gathers_rows": (ctypes.c_int, [cfgp, vp]),
            "moe_route_maps": (ctypes.c_int, [cfgp, vp, vp, f32p, i32p, f32p, i32p, i32p, i32p, i32p, vp, sz, vp]),
            "moe_route_maps_supported": (ctypes.c_int, [cfgp]),
            "moe_balance_update": (ctypes.c_int, [cfgp, i32p, f32p, ctypes.c_float, f32p, vp]),
            "moe_expert_gelu": (ctypes.c_int, [cfgp, vp, i32p, vp, f32p, vp, f32p, vp, vp, sz, vp]),
            "moe_forward_gelu": (ctypes.c_int, [cfgp, vp, vp, f32p, vp, f32p, vp, f32p, vp, vp, sz, vp]),
            "moe_backward_workspace_size": (sz, [cfgp]),
            "moe_forward_train": (ctypes.c_int, [cfgp, vp, vp, f32p, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
            "moe_backward_saved": (ctypes.c_int, [cfgp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                                  vp, vp, vp, vp, sz, vp]),
            "moe_backward": (ctypes.c_int, [cfgp, vp, vp, f32p, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                            vp, vp, vp, vp, sz, vp]),
            "moe_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().moe_status_string(int(status)).decode()


def make_config(cfg: MoEConfig, T: Optional[int] = None) -> CConfig:
    return CConfig(T=cfg.T if T is None else T, d=cfg.d, E=cfg.E, k=cfg.k, f=cfg.f,
                   dtype=MOE_DTYPE_F32 if cfg.dtype == "f32" else MOE_DTYPE_BF16,
                   gate_mode=cfg.gate_mode, n_groups=cfg.n_groups, topk_groups=cfg.topk_groups,
                   route_scale=cfg.route_scale, f_shared=cfg.f_shared)


def _cfg(c) -> CConfig:
    return c if isinstance(c, CConfig) else make_config(c)


_I32, _F32, _U8 = torch.int32, torch.float32, torch.uint8


def _dt(c: CConfig) -> torch.dtype:
    return torch.float32 if c.dtype == MOE_DTYPE_F32 else torch.bfloat16


def _need(t, name: str, numel: int, dtype: torch.dtype, required: bool = True):
    """Refuse a tensor the library would overrun or misread: wrong dtype, or
    fewer than ``numel`` elements. None passes where the C entry point takes
    NULL (``required=False``) and where it reads or writes nothing through the
    pointer (``numel == 0``, e.g. token arrays when T = 0)."""
    if t is None:
        if required and numel > 0:
            raise ValueError(f"{name} is required")
        return
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor, not {type(t).__name__}")
    if t.dtype != dtype:
        raise ValueError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if t.numel() < numel:
        raise ValueError(f"{name}: {t.numel()} elements, needs at least {numel}")


def _need_routing_io(c: CConfig, x, w_router, bias, topk_idx, topk_gate, expert_counts, expert_offsets):
    T, d, E, k, dt = c.T, c.d, c.E, c.k, _dt(c)
    _need(x, "x", T * d, dt)
    _need(w_router, "w_router", E * d, dt)
    _need(bias, "bias", E, _F32, required=False)
    _need(topk_idx, "topk_idx", T * k, _I32)
    _need(topk_gate, "topk_gate", T * k, _F32)
    _need(expert_counts, "expert_counts", E, _I32)
    _need(expert_offsets, "expert_offsets", E + 1, _I32)


def _need_weights(c: CConfig, w1, w3, w2, ws1, ws3, ws2, prefix: str = ""):
    d, E, f, fs, dt = c.d, c.E, c.f, c.f_shared, _dt(c)
    sh = fs > 0
    _need(w1, prefix + "w1", E * f * d, dt)
    _need(w3, prefix + "w3", E * f * d, dt)
    _need(w2, prefix + "w2", E * d * f, dt)
    _need(ws1, prefix + "ws1", fs * d, dt, required=sh)
    _need(ws3, prefix + "ws3", fs * d, dt, required=sh)
    _need(ws2, prefix + "ws2", d * fs, dt, required=sh)


def _need_ws(workspace):
    if workspace is None:
        raise ValueError("workspace is required")
    _need(workspace, "workspace", 0, _U8)


def _need_block(c: CConfig, x, w_router, bias, w1, w3, w2, ws1, ws3, ws2, y, workspace):
    """Inputs of the whole block (y checked unless None is passed for it)."""
    dt = _dt(c)
    _need(x, "x", c.T * c.d, dt)
    _need(w_router, "w_router", c.E * c.d, dt)
    _need(bias, "bias", c.E, _F32, required=False)
    _need_weights(c, w1, w3, w2, ws1, ws3, ws2)
    if y is not None:
        _need(y, "y", c.T * c.d, dt)
    _need_ws(workspace)


def _need_grads(c: CConfig, dy, dx, dw_router, dw1, dw3, dw2, dws1, dws3, dws2):
    dt = _dt(c)
    _need(dy, "dy", c.T * c.d, dt)
    _need(dx, "dx", c.T * c.d, dt)
    _need(dw_router, "dw_router", c.E * c.d, dt)
    _need_weights(c, dw1, dw3, dw2, dws1, dws3, dws2, prefix="d")


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(status: int, where: str):
    if status != MOE_OK:
        raise MoEError(status, where)


def check_config(cfg) -> int:
    return lib().moe_check_config(ctypes.byref(_cfg(cfg)))


def workspace_size(cfg) -> int:
    return lib().moe_workspace_size(ctypes.byref(_cfg(cfg)))


def alloc_workspace(cfg, device="cuda") -> torch.Tensor:
    n = workspace_size(cfg)
    if n == 0:
        raise MoEError(check_config(cfg) or MOE_ERR_INVALID_ARG, "moe_workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=device)


def moe_route(cfg, x, w_router, bias, topk_idx, topk_gate, expert_counts, expert_offsets,
              workspace, stream=None):
    c = _cfg(cfg)
    _need_routing_io(c, x, w_router, bias, topk_idx, topk_gate, expert_counts, expert_offsets)
    _need_ws(workspace)
    _check(lib().moe_route(ctypes.byref(c), _ptr(x), _ptr(w_router), _ptr(bias), _ptr(topk_idx),
                           _ptr(topk_gate), _ptr(expert_counts), _ptr(expert_offsets),
                           _ptr(workspace), workspace.numel(), _stream(stream)), "moe_route")


def moe_route_maps(cfg, x, w_router, bias, topk_idx, topk_gate, expert_counts, expert_offsets, perm_src,
                   inv_row, workspace, stream=None):
    """moe_route plus the maps-only permute in one launch (one-tile batches)."""
    c = _cfg(cfg)
    _need_routing_io(c, x, w_router, bias, topk_idx, topk_gate, expert_counts, expert_offsets)
    _need(perm_src, "perm_src", c.T * c.k, _I32)
    _need(inv_row, "inv_row", c.T * c.k, _I32)
    _need_ws(workspace)
    _check(lib().moe_route_maps(ctypes.byref(c), _ptr(x), _ptr(w_router), _ptr(bias), _ptr(topk_idx),
                                _ptr(topk_gate), _ptr(expert_counts), _ptr(expert_offsets), _ptr(perm_src),
                                _ptr(inv_row), _ptr(workspace), workspace.numel(), _stream(stream)),
           "moe_route_maps")


def moe_route_maps_supported(cfg) -> bool:
    """Whether moe_route_maps runs for cfg (else it returns MOE_ERR_UNSUPPORTED)."""
    r = lib().moe_route_maps_supported(ctypes.byref(_cfg(cfg)))
    if r < 0:
        raise MoEError(MOE_ERR_INVALID_ARG, "moe_route_maps_supported")
    return r == 1


def moe_permute(cfg, x, topk_idx, expert_offsets, x_perm, perm_src, inv_row, workspace, stream=None):
    c = _cfg(cfg)
    R, dt = c.T * c.k, _dt(c)
    _need(x, "x", c.T * c.d, dt, required=x_perm is not None)
    _need(topk_idx, "topk_idx", R, _I32)
    _need(expert_offsets, "expert_offsets", c.E + 1, _I32)
    _need(x_perm, "x_perm", R * c.d, dt, required=False)
    _need(perm_src, "perm_src", R, _I32)
    _need(inv_row, "inv_row", R, _I32)
    _need_ws(workspace)
    _check(lib().moe_permute(ctypes.byref(c), _ptr(x), _ptr(topk_idx), _ptr(expert_offsets),
                             _ptr(x_perm), _ptr(perm_src), _ptr(inv_row), _ptr(workspace),
                             workspace.numel(), _stream(stream)), "moe_permute")


def moe_expert_swiglu(cfg, x_perm, expert_offsets, w1, w3, w2, x_shared, ws1, ws3, ws2, y_perm,
                      y_shared, workspace, stream=None):
    c = _cfg(cfg)
    R, dt, sh = c.T * c.k, _dt(c), c.f_shared > 0
    _need(x_perm, "x_perm", R * c.d, dt)
    _need(expert_offsets, "expert_offsets", c.E + 1, _I32)
    _need_weights(c, w1, w3, w2, ws1, ws3, ws2)
    _need(x_shared, "x_shared", c.T * c.d, dt, required=sh)
    _need(y_perm, "y_perm", R * c.d, dt)
    _need(y_shared, "y_shared", c.T * c.d, dt, required=sh)
    _need_ws(workspace)
    _check(lib().moe_expert_swiglu(ctypes.byref(c), _ptr(x_perm), _ptr(expert_offsets), _ptr(w1),
                                   _ptr(w3), _ptr(w2), _ptr(x_shared), _ptr(ws1), _ptr(ws3),
                                   _ptr(ws2), _ptr(y_perm), _ptr(y_shared), _ptr(workspace),
                                   workspace.numel(), _stream(stream)), "moe_expert_swiglu")


def moe_expert_gate_up(cfg, x_perm, expert_offsets, w1, w3, x_shared, ws1, ws3, h, h_shared,
                       workspace, stream=None):
    c = _cfg(cfg)
    R, dt, sh, fs = c.T * c.k, _dt(c), c.f_shared > 0, c.f_shared
    _need(x_perm, "x_perm", R * c.d, dt)
    _need(expert_offsets, "expert_offsets", c.E + 1, _I32)
    _need(w1, "w1", c.E * c.f * c.d, dt)
    _need(w3, "w3", c.E * c.f * c.d, dt)
    _need(x_shared, "x_shared", c.T * c.d, dt, required=sh)
    _need(ws1, "ws1", fs * c.d, dt, required=sh)
    _need(ws3, "ws3", fs * c.d, dt, required=sh)
    _need(h, "h", R * c.f, dt)
    _need(h_shared, "h_shared", c.T * fs, dt, required=sh)
    _need_ws(workspace)
    _check(lib().moe_expert_gate_up(ctypes.byref(c), _ptr(x_perm), _ptr(expert_offsets), _ptr(w1),
                                    _ptr(w3), _ptr(x_shared), _ptr(ws1), _ptr(ws3), _ptr(h),
                                    _ptr(h_shared), _ptr(workspace), workspace.numel(),
                                    _stream(stream)), "moe_expert_gate_up")


def moe_expert_gate_up_gather(cfg, x, perm_src, expert_offsets, w1, w3, ws1, ws3, h, h_shared,
                              workspace, stream=None):
    c = _cfg(cfg)
    R, dt, sh, fs = c.T * c.k, _dt(c), c.f_shared > 0, c.f_shared
    _need(x, "x", c.T * c.d, dt)
    _need(perm_src, "perm_src", R, _I32)
    _need(expert_offsets, "expert_offsets", c.E + 1, _I32)
    _need(w1, "w1", c.E * c.f * c.d, dt)
    _need(w3, "w3", c.E * c.f * c.d, dt)
    _need(ws1, "ws1", fs * c.d, dt, required=sh)
    _need(ws3, "ws3", fs * c.d, dt, required=sh)
    _need(h, "h", R * c.f, dt)
    _need(h_shared, "h_shared", c.T * fs, dt, required=sh)
    _need_ws(workspace)
    _check(lib().moe_expert_gate_up_gather(ctypes.byref(c), _ptr(x), _ptr(perm_src), _ptr(expert_offsets),
                                           _ptr(w1), _ptr(w3), _ptr(ws1), _ptr(ws3), _ptr(h),
                                           _ptr(h_shared), _ptr(workspace), workspace.numel(),
                                           _stream(stream)), "moe_expert_gate_up_gather")


def moe_expert_down(cfg, h, expert_offsets, w2, h_shared, ws2, y_perm, y_shared, workspace,
                    stream=None):
    c = _cfg(cfg)
    R, dt, sh, fs = c.T * c.k, _dt(c), c.f_shared > 0, c.f_shared
    _need(h, "h", R * c.f, dt)
    _need(expert_offsets, "expert_offsets", c.E + 1, _I32)
    _need(w2, "w2", c.E * c.d * c.f, dt)
    _need(h_shared, "h_shared", c.T * fs, dt, required=sh)
    _need(ws2, "ws2", c.d * fs, dt, required=sh)
    _need(y_perm, "y_perm", R * c.d, dt)
    _need(y_shared, "y_shared", c.T * c.d, dt, required=sh)
    _need_ws(workspace)
    _check(lib().moe_expert_down(ctypes.byref(c), _ptr(h), _ptr(expert_offsets), _ptr(w2),
                                 _ptr(h_shared), _ptr(ws2), _ptr(y_perm), _ptr(y_shared),
                                 _ptr(workspace), workspace.numel(), _stream(stream)),
           "moe_expert_down")


def moe_combine(cfg, y_perm, inv_row, topk_gate, y_shared, y, stream=None):
    c = _cfg(cfg)
    R, dt = c.T * c.k, _dt(c)
    _need(y_perm, "y_perm", R * c.d, dt)
    _need(inv_row, "inv_row", R, _I32)
    _need(topk_gate, "topk_gate", R, _F32)
    _need(y_shared, "y_shared", c.T * c.d, dt, required=False)
    _need(y, "y", c.T * c.d, dt)
    _check(lib().moe_combine(ctypes.byref(c), _ptr(y_perm), _ptr(inv_row), _ptr(topk_gate),
                             _ptr(y_shared), _ptr(y), _stream(stream)), "moe_combine")


def moe_forward(cfg, x, w_router, bias, w1, w3, w2, ws1, ws3, ws2, y, workspace, stream=None):
    c = _cfg(cfg)
    _need_block(c, x, w_router, bias, w1, w3, w2, ws1, ws3, ws2, y, workspace)
    _check(lib().moe_forward(ctypes.byref(c), _ptr(x), _ptr(w_router), _ptr(bias), _ptr(w1),
                             _ptr(w3), _ptr(w2), _ptr(ws1), _ptr(ws3), _ptr(ws2), _ptr(y),
                             _ptr(workspace), workspace.numel(), _stream(stream)), "moe_forward")


def moe_expert_gelu(cfg, x_perm, expert_offsets, w1, b1, w2, b2, y_perm, workspace, stream=None):
    """Generic experts on packed rows: y = W2 GELU(W1 x + b1) + b2 per segment."""
    c = _cfg(cfg)
    R, dt = c.T * c.k, _dt(c)
    _need(x_perm, "x_perm", R * c.d, dt)
    _need(expert_offsets, "expert_offsets", c.E + 1, _I32)
    _need(w1, "w1", c.E * c.f * c.d, dt)
    _need(b1, "b1", c.E * c.f, _F32, required=False)
    _need(w2, "w2", c.E * c.d * c.f, dt)
    _need(b2, "b2", c.E * c.d, _F32, required=False)
    _need(y_perm, "y_perm", R * c.d, dt)
    _need_ws(workspace)
    _check(lib().moe_expert_gelu(ctypes.byref(c), _ptr(x_perm), _ptr(expert_offsets), _ptr(w1), _ptr(b1),
                                 _ptr(w2), _ptr(b2), _ptr(y_perm), _ptr(workspace), workspace.numel(),
                                 _stream(stream)), "moe_expert_gelu")


def moe_forward_gelu(cfg, x, w_router, bias, w1, b1, w2, b2, y, workspace, stream=None):
    """The block with generic GELU experts (no shared expert)."""
    c = _cfg(cfg)
    dt = _dt(c)
    _need(x, "x", c.T * c.d, dt)
    _need(w_router, "w_router", c.E * c.d, dt)
    _need(bias, "bias", c.E, _F32, required=False)
    _need(w1, "w1", c.E * c.f * c.d, dt)
    _need(b1, "b1", c.E * c.f, _F32, required=False)
    _need(w2, "w2", c.E * c.d * c.f, dt)
    _need(b2, "b2", c.E * c.d, _F32, required=False)
    _need(y, "y", c.T * c.d, dt)
    _need_ws(workspace)
    _check(lib().moe_forward_gelu(ctypes.byref(c), _ptr(x), _ptr(w_router), _ptr(bias), _ptr(w1),
                                  _ptr(b1), _ptr(w2), _ptr(b2), _ptr(y), _ptr(workspace),
                                  workspace.numel(), _stream(stream)), "moe_forward_gelu")


def backward_workspace_size(cfg) -> int:
    c = _cfg(cfg)
    return int(lib().moe_backward_workspace_size(ctypes.byref(c)))


def alloc_backward_workspace(cfg, device="cuda") -> torch.Tensor:
    n = backward_workspace_size(cfg)
    if n == 0:
        raise MoEError(MOE_ERR_INVALID_ARG, "moe_backward_workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=device)


def moe_backward(cfg, x, w_router, bias, w1, w3, w2, ws1, ws3, ws2, dy, dx, dw_router, dw1, dw3, dw2,
                 dws1, dws3, dws2, workspace, stream=None):
    """Gradients of the block with respect to x and every weight, given dy."""
    c = _cfg(cfg)
    _need_block(c, x, w_router, bias, w1, w3, w2, ws1, ws3, ws2, None, workspace)
    _need_grads(c, dy, dx, dw_router, dw1, dw3, dw2, dws1, dws3, dws2)
    _check(lib().moe_backward(ctypes.byref(c), _ptr(x), _ptr(w_router), _ptr(bias), _ptr(w1), _ptr(w3),
                              _ptr(w2), _ptr(ws1), _ptr(ws3), _ptr(ws2), _ptr(dy), _ptr(dx), _ptr(dw_router),
                              _ptr(dw1), _ptr(dw3), _ptr(dw2), _ptr(dws1), _ptr(dws3), _ptr(dws2),
                              _ptr(workspace), workspace.numel(), _stream(stream)), "moe_backward")


def moe_forward_train(cfg, x, w_router, bias, w1, w3, w2, ws1, ws3, ws2, y, workspace, stream=None):
    """moe_forward that keeps routing and pre-activations in a backward-size workspace."""
    c = _cfg(cfg)
    _need_block(c, x, w_router, bias, w1, w3, w2, ws1, ws3, ws2, y, workspace)
    _check(lib().moe_forward_train(ctypes.byref(c), _ptr(x), _ptr(w_router), _ptr(bias), _ptr(w1), _ptr(w3),
                                   _ptr(w2), _ptr(ws1), _ptr(ws3), _ptr(ws2), _ptr(y), _ptr(workspace),
                                   workspace.numel(), _stream(stream)), "moe_forward_train")


def moe_backward_saved(cfg, x, w_router, w1, w3, w2, ws1, ws3, ws2, dy, dx, dw_router, dw1, dw3, dw2,
                       dws1, dws3, dws2, workspace, stream=None):
    """moe_backward on the state moe_forward_train left in `workspace`."""
    c = _cfg(cfg)
    _need_block(c, x, w_router, None, w1, w3, w2, ws1, ws3, ws2, None, workspace)
    _need_grads(c, dy, dx, dw_router, dw1, dw3, dw2, dws1, dws3, dws2)
    _check(lib().moe_backward_saved(ctypes.byref(c), _ptr(x), _ptr(w_router), _ptr(w1), _ptr(w3), _ptr(w2),
                                    _ptr(ws1), _ptr(ws3), _ptr(ws2), _ptr(dy), _ptr(dx), _ptr(dw_router),
                                    _ptr(dw1), _ptr(dw3), _ptr(dw2), _ptr(dws1), _ptr(dws3), _ptr(dws2),
                                    _ptr(workspace), workspace.numel(), _stream(stream)), "moe_backward_saved")


def moe_route_noalloc(cfg, x, w_router, bias, topk_idx, topk_gate, expert_counts, expert_offsets,
                      stream=None):
    """moe_route with the router's scratch in the library's fixed device array."""
    c = _cfg(cfg)
    _need_routing_io(c, x, w_router, bias, topk_idx, topk_gate, expert_counts, expert_offsets)
    _check(lib().moe_route_noalloc(ctypes.byref(c), _ptr(x), _ptr(w_router), _ptr(bias),
                                   _ptr(topk_idx), _ptr(topk_gate), _ptr(expert_counts),
                                   _ptr(expert_offsets), _stream(stream)), "moe_route_noalloc")


def moe_route_noalloc_device_error(stream=None) -> int:
    """Status of moe_route_noalloc's bounded device waits on the current
    device (synchronises the stream, then reads and clears the fixed array's
    error word): MOE_OK or MOE_ERR_TIMEOUT."""
    return lib().moe_route_noalloc_device_error(_stream(stream))


def moe_forward_gathers_rows(cfg, x) -> bool:
    """Whether moe_forward's gate/up GEMM gathers the token rows of x itself
    (the permute then writes the maps only) rather than reading a packed copy."""
    r = lib().moe_forward_gathers_rows(ctypes.byref(_cfg(cfg)), _ptr(x))
    if r < 0:
        raise MoEError(MOE_ERR_INVALID_ARG, "moe_forward_gathers_rows")
    return r == 1


def moe_balance_update(cfg, expert_counts, bias, gamma: float, entropy=None, stream=None):
    """Aux-loss-free bias step in place on `bias` and/or the routing entropy."""
    c = _cfg(cfg)
    _need(expert_counts, "expert_counts", c.E, _I32)
    _need(bias, "bias", c.E, _F32, required=False)
    _need(entropy, "entropy", 1, _F32, required=False)
    _check(lib().moe_balance_update(ctypes.byref(c), _ptr(expert_counts), _ptr(bias), float(gamma),
                                    _ptr(entropy), _stream(stream)), "moe_balance_update")


def moe_get_device_error(workspace, stream=None) -> int:
    _need_ws(workspace)
    return lib().moe_get_device_error(_ptr(workspace), _stream(stream))


def moe_selftest_wait_timeout(workspace, timeout_ns: int, stream=None):
    _need_ws(workspace)
    _check(lib().moe_selftest_wait_timeout(_ptr(workspace), workspace.numel(), int(timeout_ns),
                                           _stream(stream)), "moe_selftest_wait_timeout")


class MoEBlock:
    """Convenience wrapper holding one block's weights and workspace on the GPU.

    ``forward(x)`` returns a new ``[T, d]`` tensor (shared + routed, no
    residual) computed by ``moe_forward``.
    """

    def __init__(self, cfg: MoEConfig, weights: dict, device="cuda"):
        self.cfg = cfg
        self.w = weights
        self.device = torch.device(device)
        self._ws = {}

    def workspace(self, T: int) -> torch.Tensor:
        if T not in self._ws:
            self._ws[T] = alloc_workspace(make_config(self.cfg, T), self.device)
        return self._ws[T]

    def forward(self, x: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        T = x.shape[0]
        if out is None:
            out = torch.empty_like(x)
        w = self.w
        moe_forward(make_config(self.cfg, T), x, w["w_router"], w.get("bias"), w["w1"], w["w3"], w["w2"],
                    w.get("ws1"), w.get("ws3"), w.get("ws2"), out, self.workspace(T), stream)
        return out
