"""Aux-loss-free balancing on the GPU (moe_balance_update) against the oracle.

The update applies +-gamma in fp32 on the GPU and in fp64 in the oracle, so a
bias may differ by the rounding of one fp32 addition: |b - b_ref| <= 2^-23 *
(|b| + gamma) per step. The entropy is accumulated in fp64 and rounded to fp32
once: relative error <= 1e-6.
"""
import math

import numpy as np
import pytest
import torch

import oracle.moe_oracle as orc
from mixture_experts_ffn_sigmoid_b200 import binding as B
from mixture_experts_ffn_sigmoid_b200.inputs import GATE_SIGMOID, GATE_SOFTMAX, MoEConfig

import gpu_harness as H

pytestmark = pytest.mark.gpu


def _bias_tol(ref, gamma):
    return 2.0 ** -23 * (np.abs(ref) + gamma) + 1e-30


def _step(cfg, counts, bias, gamma):
    ent = torch.full((1,), float("nan"), device="cuda")
    b = bias.clone()
    B.moe_balance_update(cfg, counts, b, gamma, ent)
    torch.cuda.synchronize()
    return b, ent.item()


def test_single_step_matches_oracle():
    cfg = MoEConfig("balance", T=1000, d=256, E=64, k=6, f=64, gate_mode=GATE_SIGMOID, n_groups=8,
                    topk_groups=4, route_scale=2.5, bias="uniform")
    inp = H.gpu_inputs(cfg)
    got = H.gpu_route(cfg, inp)
    counts = got["counts"]
    c = counts.cpu().numpy()
    b, ent = _step(cfg, counts, inp["bias"], 0.15)
    ref_b = orc.update_bias(inp["bias"].cpu().numpy(), c, orc.balance_target(cfg.T, cfg.k, cfg.E), 0.15)
    assert np.all(np.abs(b.cpu().numpy() - ref_b) <= _bias_tol(ref_b, 0.15))
    ref_h = orc.routing_entropy(c)
    assert abs(ent - ref_h) <= 1e-6 * ref_h


def test_on_target_expert_keeps_bias_and_entropy_only_call():
    # 4 experts, T*k = 8: target 2. Counts 2, 4, 0, 2.
    cfg = MoEConfig("balance_small", T=4, d=64, E=4, k=2, f=64)
    counts = torch.tensor([2, 4, 0, 2], dtype=torch.int32, device="cuda")
    bias = torch.tensor([0.5, 0.5, 0.5, -1.0], device="cuda")
    b, ent = _step(cfg, counts, bias, 0.25)
    assert b.tolist() == [0.5, 0.25, 0.75, -1.0]
    assert abs(ent - orc.routing_entropy([2, 4, 0, 2])) <= 1e-6
    e2 = torch.zeros(1, device="cuda")
    B.moe_balance_update(cfg, counts, None, 0.0, e2)          # entropy only, bias untouched
    torch.cuda.synchronize()
    assert abs(e2.item() - ent) <= 1e-7
    uniform = torch.full((4,), 2, dtype=torch.int32, device="cuda")
    B.moe_balance_update(cfg, uniform, None, 0.0, e2)
    torch.cuda.synchronize()
    assert abs(e2.item() - math.log(4)) <= 1e-6


def test_balance_loop_raises_entropy_on_gpu():
    # The page's demo: gamma = 0.15, 10 iterations of route -> count -> update.
    # A skewed bias makes the first experts popular; the loop must even them out.
    cfg = MoEConfig("balance_loop", T=2048, d=256, E=32, k=4, f=64, gate_mode=GATE_SOFTMAX)
    inp = H.gpu_inputs(cfg)
    bias = torch.linspace(1.5, -1.5, cfg.E, device="cuda")
    inp["bias"] = bias
    ws = B.alloc_workspace(cfg)
    target = orc.balance_target(cfg.T, cfg.k, cfg.E)
    ents = []
    for it in range(10):
        got = H.gpu_route(cfg, inp, ws)
        c = got["counts"].cpu().numpy()
        before = inp["bias"].cpu().numpy()
        b, ent = _step(cfg, got["counts"], inp["bias"], 0.15)
        ref_b = orc.update_bias(before, c, target, 0.15)
        assert np.all(np.abs(b.cpu().numpy() - ref_b) <= _bias_tol(ref_b, 0.15)), it
        assert abs(ent - orc.routing_entropy(c)) <= 1e-6 * max(1.0, ent)
        ents.append(ent)
        inp["bias"] = b
    assert ents[-1] > ents[0] + 0.2, ents
    assert ents[-1] > 0.95 * math.log(cfg.E), ents
