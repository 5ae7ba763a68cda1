"""moe_route_noalloc: the router for callers that cannot allocate device
memory keeps its scratch in the library's fixed device array. Called through
the C ABI, it must give the same routing as moe_route (which uses a caller
workspace), call after call, although every call reuses the same array.

This file is collected last on purpose: it also runs after every other GPU
test has loaded and used the library in the same process.
"""
import numpy as np
import pytest
import torch

from mixture_experts_ffn_sigmoid_b200 import binding as B
from mixture_experts_ffn_sigmoid_b200.inputs import GATE_SIGMOID, MoEConfig, make_inputs

import gpu_harness as H

pytestmark = pytest.mark.gpu


def _route_both(cfg, seed):
    inp = make_inputs(cfg, "cuda", seed=seed)
    ref = H.gpu_route(cfg, inp)                      # moe_route with a workspace
    T, E, k = cfg.T, cfg.E, cfg.k
    idx = torch.full((T, k), -7, dtype=torch.int32, device="cuda")
    gate = torch.full((T, k), float("nan"), dtype=torch.float32, device="cuda")
    counts = torch.full((E,), -7, dtype=torch.int32, device="cuda")
    offsets = torch.full((E + 1,), -7, dtype=torch.int32, device="cuda")
    B.moe_route_noalloc(cfg, inp["x"], inp["w_router"], inp["bias"], idx, gate, counts, offsets)
    # The fixed array's error word: no bounded device wait of the call ran out.
    assert B.moe_route_noalloc_device_error() == B.MOE_OK
    torch.cuda.synchronize()
    return ref, dict(idx=idx, gate=gate, counts=counts, offsets=offsets)


def test_route_noalloc_matches_route_on_consecutive_calls():
    # Two calls in a row with different inputs (and token counts): the second
    # must not see anything the first left in the shared array.
    cases = [
        (MoEConfig("noalloc_a", T=1000, d=512, E=256, k=8, f=64, gate_mode=GATE_SIGMOID, n_groups=8,
                   topk_groups=4, route_scale=2.5, bias="uniform"), 11),
        (MoEConfig("noalloc_b", T=700, d=512, E=256, k=8, f=64, gate_mode=GATE_SIGMOID, n_groups=8,
                   topk_groups=4, route_scale=2.5, bias="uniform"), 12),
    ]
    for cfg, seed in cases:
        ref, got = _route_both(cfg, seed)
        assert torch.equal(got["idx"], ref["idx"])
        assert torch.equal(got["counts"], ref["counts"])
        assert torch.equal(got["offsets"], ref["offsets"])
        err = (got["gate"] - ref["gate"]).abs().max().item()
        assert err <= H.gate_tol(cfg), err


def test_route_noalloc_rejects_oversized_problem():
    # 256 experts x 32768 tokens of fp32 logits alone is 32 MiB > 24 MiB.
    cfg = MoEConfig("too_big", T=32768, d=512, E=256, k=8, f=64)
    c = B.make_config(cfg)
    fake = B.ctypes.c_void_p(0x10000)
    st = B.lib().moe_route_noalloc(B.ctypes.byref(c), fake, fake, None, fake, fake, fake, fake, None)
    assert st == B.MOE_ERR_WORKSPACE_TOO_SMALL
