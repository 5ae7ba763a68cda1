"""The C-ABI library without a GPU: it loads, exports every function that
include/moe.h declares, and rejects bad arguments on the host with the
documented status before touching any device."""
import ctypes
import os
import re

import pytest

from mixture_experts_ffn_sigmoid_b200 import binding as B
from mixture_experts_ffn_sigmoid_b200 import build as build_mod
from mixture_experts_ffn_sigmoid_b200.inputs import CONFIGS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built_library():
    build_mod.build()
    return B.lib()


def header_functions():
    text = open(os.path.join(ROOT, "include", "moe.h")).read()
    return re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", text)


def test_header_declares_the_boundary():
    names = set(header_functions())
    for required in ("moe_route", "moe_permute", "moe_expert_swiglu", "moe_combine", "moe_forward",
                     "moe_workspace_size", "moe_status_string", "moe_get_device_error"):
        assert required in names


def test_every_declared_symbol_is_exported(built_library):
    names = header_functions()
    assert names
    for n in names:
        assert hasattr(built_library, n), n
    assert set(names) == set(B.EXPORTED)


def test_library_has_no_torch_dependency():
    # The boundary is plain C: the shared object must not link libtorch or python.
    needed = open(B.library_path(), "rb").read()
    assert b"libtorch" not in needed and b"libc10" not in needed and b"libpython" not in needed


def test_status_strings():
    for s in range(7):
        assert B.status_string(s) and B.status_string(s) != "unknown status"
    assert B.status_string(99) == "unknown status"


def test_config_struct_layout():
    assert ctypes.sizeof(B.CConfig) == 11 * 4


@pytest.mark.parametrize("name", sorted(CONFIGS))
def test_workload_configs_valid(name):
    c = B.make_config(CONFIGS[name])
    assert B.check_config(c) == B.MOE_OK
    assert B.workspace_size(c) > 0


def _cfg(**kw):
    base = dict(T=64, d=128, E=8, k=2, f=256, dtype=B.MOE_DTYPE_BF16, gate_mode=0, n_groups=1,
                topk_groups=1, route_scale=1.0, f_shared=0)
    base.update(kw)
    return B.CConfig(**base)


@pytest.mark.parametrize("kw,status", [
    (dict(k=9), B.MOE_ERR_INVALID_ARG),                       # k > E
    (dict(k=0), B.MOE_ERR_INVALID_ARG),
    (dict(T=-1), B.MOE_ERR_INVALID_ARG),
    (dict(d=0), B.MOE_ERR_INVALID_ARG),
    (dict(dtype=7), B.MOE_ERR_INVALID_ARG),
    (dict(gate_mode=2), B.MOE_ERR_INVALID_ARG),
    (dict(route_scale=0.0), B.MOE_ERR_INVALID_ARG),
    (dict(route_scale=float("nan")), B.MOE_ERR_INVALID_ARG),
    (dict(n_groups=3), B.MOE_ERR_INVALID_ARG),               # E % n_groups != 0
    (dict(n_groups=8, topk_groups=1), B.MOE_ERR_INVALID_ARG),  # group size 1
    (dict(n_groups=4, topk_groups=5), B.MOE_ERR_INVALID_ARG),
    (dict(n_groups=4, topk_groups=0), B.MOE_ERR_INVALID_ARG),
    (dict(n_groups=4, topk_groups=1, k=3), B.MOE_ERR_INVALID_ARG),  # 1 group of 2 < k
    (dict(E=2048, k=2), B.MOE_ERR_UNSUPPORTED),
    (dict(E=64, k=33), B.MOE_ERR_UNSUPPORTED),
    (dict(d=100), B.MOE_ERR_MISALIGNED),                      # bf16 rows must be 16 B multiples
    (dict(f=260), B.MOE_ERR_MISALIGNED),
    (dict(f_shared=12), B.MOE_ERR_MISALIGNED),
    (dict(dtype=B.MOE_DTYPE_F32, d=100), B.MOE_OK),           # fp32: multiples of 4 suffice
    (dict(n_groups=4, topk_groups=2, k=3), B.MOE_OK),
    (dict(T=0), B.MOE_OK),
])
def test_check_config(kw, status):
    c = _cfg(**kw)
    assert B.lib().moe_check_config(ctypes.byref(c)) == status
    if status != B.MOE_OK:
        assert B.lib().moe_workspace_size(ctypes.byref(c)) == 0


def test_workspace_size_grows_with_tokens():
    a = B.lib().moe_workspace_size(ctypes.byref(_cfg(T=64)))
    b = B.lib().moe_workspace_size(ctypes.byref(_cfg(T=128)))
    c = B.lib().moe_workspace_size(ctypes.byref(_cfg(T=64, f_shared=64)))
    assert 0 < a < b and a < c
    assert a % 256 == 0


def test_host_side_rejections_before_any_launch():
    L = B.lib()
    cfg = _cfg()
    fake = ctypes.c_void_p(0x10000)        # never dereferenced: every case fails on the host
    odd = ctypes.c_void_p(0x10008)
    nbytes = L.moe_workspace_size(ctypes.byref(cfg))
    # NULL config
    assert L.moe_route(None, fake, fake, None, fake, fake, fake, fake, fake, nbytes, None) == B.MOE_ERR_INVALID_ARG
    # invalid config
    bad = _cfg(k=9)
    assert L.moe_forward(ctypes.byref(bad), fake, fake, None, fake, fake, fake, None, None, None, fake,
                         fake, nbytes, None) == B.MOE_ERR_INVALID_ARG
    # workspace too small
    assert L.moe_forward(ctypes.byref(cfg), fake, fake, None, fake, fake, fake, None, None, None, fake,
                         fake, nbytes - 1, None) == B.MOE_ERR_WORKSPACE_TOO_SMALL
    # misaligned workspace / activation
    assert L.moe_forward(ctypes.byref(cfg), fake, fake, None, fake, fake, fake, None, None, None, fake,
                         odd, nbytes, None) == B.MOE_ERR_MISALIGNED
    assert L.moe_forward(ctypes.byref(cfg), odd, fake, None, fake, fake, fake, None, None, None, fake,
                         fake, nbytes, None) == B.MOE_ERR_MISALIGNED
    # missing weights
    assert L.moe_forward(ctypes.byref(cfg), fake, fake, None, None, fake, fake, None, None, None, fake,
                         fake, nbytes, None) == B.MOE_ERR_INVALID_ARG
    # shared expert configured but its weights missing
    cs = _cfg(f_shared=64)
    ns = L.moe_workspace_size(ctypes.byref(cs))
    assert L.moe_forward(ctypes.byref(cs), fake, fake, None, fake, fake, fake, None, None, None, fake,
                         fake, ns, None) == B.MOE_ERR_INVALID_ARG
    # combine and permute argument checks
    assert L.moe_combine(ctypes.byref(cfg), None, fake, fake, None, fake, None) == B.MOE_ERR_INVALID_ARG
    assert L.moe_permute(ctypes.byref(cfg), fake, fake, fake, odd, fake, fake, fake, nbytes,
                         None) == B.MOE_ERR_MISALIGNED
    assert L.moe_expert_swiglu(ctypes.byref(cfg), fake, fake, fake, fake, fake, None, None, None, None,
                               None, None, fake, nbytes, None) == B.MOE_ERR_INVALID_ARG
    # balance update: nothing to do is an error; a negative step is rejected
    assert L.moe_balance_update(ctypes.byref(cfg), fake, None, ctypes.c_float(0.1), None, None) == B.MOE_ERR_INVALID_ARG
    assert L.moe_balance_update(ctypes.byref(cfg), fake, fake, ctypes.c_float(-0.1), None, None) == B.MOE_ERR_INVALID_ARG
    assert L.moe_balance_update(ctypes.byref(cfg), None, fake, ctypes.c_float(0.1), None, None) == B.MOE_ERR_INVALID_ARG
    # generic (GELU) experts: no shared-expert form
    assert L.moe_forward_gelu(ctypes.byref(cs), fake, fake, None, fake, None, fake, None, fake, fake, ns,
                              None) == B.MOE_ERR_UNSUPPORTED
    assert L.moe_expert_gelu(ctypes.byref(cs), fake, fake, fake, None, fake, None, fake, fake, ns,
                             None) == B.MOE_ERR_UNSUPPORTED
    assert L.moe_forward_gelu(ctypes.byref(cfg), fake, fake, None, None, None, fake, None, fake, fake,
                              nbytes, None) == B.MOE_ERR_INVALID_ARG
    assert L.moe_expert_gelu(ctypes.byref(cfg), fake, fake, fake, ctypes.c_void_p(0x10002), fake, None,
                             fake, fake, nbytes, None) == B.MOE_ERR_MISALIGNED
    # backward: its workspace is larger than the forward's
    nb = L.moe_backward_workspace_size(ctypes.byref(cfg))
    assert nb > nbytes
    args = [fake] * 18
    assert L.moe_backward(ctypes.byref(cfg), *args, fake, nb - 1, None) == B.MOE_ERR_WORKSPACE_TOO_SMALL
    assert L.moe_backward(ctypes.byref(bad), *args, fake, nb, None) == B.MOE_ERR_INVALID_ARG
    # the timeout self-test needs a workspace and a positive bound
    assert L.moe_selftest_wait_timeout(None, 256, 1000, None) == B.MOE_ERR_INVALID_ARG
    assert L.moe_selftest_wait_timeout(fake, 256, 0, None) == B.MOE_ERR_INVALID_ARG
    # T = 0 with empty buffers: only the forward path's validation runs, nothing is enqueued
    c0 = _cfg(T=0)
    n0 = L.moe_workspace_size(ctypes.byref(c0))
    assert L.moe_forward(ctypes.byref(c0), None, None, None, None, None, None, None, None, None, None,
                         fake, n0, None) == B.MOE_OK


def test_binding_requires_cuda_tensors():
    import torch
    x = torch.zeros(64, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        B._ptr(x)


def test_route_maps_support_and_host_rejections():
    L = B.lib()
    # one tile of the fused router: bf16, E <= 256, T <= 128
    assert L.moe_route_maps_supported(ctypes.byref(_cfg(T=128))) == 1
    assert L.moe_route_maps_supported(ctypes.byref(_cfg(T=129))) == 0
    assert L.moe_route_maps_supported(ctypes.byref(_cfg(T=64, dtype=B.MOE_DTYPE_F32))) == 0
    assert L.moe_route_maps_supported(ctypes.byref(_cfg(T=64, E=320))) == 0
    assert L.moe_route_maps_supported(ctypes.byref(_cfg(k=9))) == -1
    fake = ctypes.c_void_p(0x10000)        # never dereferenced: every case fails on the host
    for cfg in (_cfg(T=129), _cfg(T=64, dtype=B.MOE_DTYPE_F32)):
        nbytes = L.moe_workspace_size(ctypes.byref(cfg))
        assert L.moe_route_maps(ctypes.byref(cfg), fake, fake, None, fake, fake, fake, fake, fake, fake, fake,
                                nbytes, None) == B.MOE_ERR_UNSUPPORTED
    cfg = _cfg(T=64)
    nbytes = L.moe_workspace_size(ctypes.byref(cfg))
    assert L.moe_route_maps(ctypes.byref(cfg), fake, fake, None, fake, fake, fake, fake, None, fake, fake,
                            nbytes, None) == B.MOE_ERR_INVALID_ARG
