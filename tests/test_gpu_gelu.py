"""Generic experts on the GPU (moe_expert_gelu, moe_forward_gelu) against the
oracle's GELU expert: E_i(u) = W2_i GELU(W1_i u + b1_i) + b2_i, gated sum
over the top-k ("Lesson 2 - From the Dense FFN to a Layer of Experts",
section 2).

Tolerances are those of the SwiGLU path (gpu_harness): relative L2 <= 1e-5
for fp32; for bf16 storage (h rounded once to bf16 after bias and GELU in
fp32) relative L2 <= 2e-2 and |error| <= 5e-2 * RMS + 1e-2 * |ref| elementwise.
"""
import numpy as np
import pytest
import torch

import oracle.moe_oracle as orc
from mixture_experts_ffn_sigmoid_b200 import binding as B
from mixture_experts_ffn_sigmoid_b200.inputs import GATE_SIGMOID, MoEConfig, make_expert_biases, \
    sample_token_ids

import gpu_harness as H

pytestmark = pytest.mark.gpu

CASES = {
    "tiny_fp32": MoEConfig("tiny_gelu", T=64, d=128, E=8, k=2, f=256, dtype="f32"),
    "ragged_fp32": MoEConfig("ragged_gelu_f32", T=77, d=200, E=12, k=3, f=72, dtype="f32",
                             gate_mode=GATE_SIGMOID, bias="uniform"),
    "ragged_bf16": MoEConfig("ragged_gelu", T=77, d=200, E=12, k=3, f=72, gate_mode=GATE_SIGMOID,
                             route_scale=1.0, bias="uniform"),
    "grouped_bf16": MoEConfig("grouped_gelu", T=300, d=256, E=32, k=4, f=384, gate_mode=GATE_SIGMOID,
                              n_groups=8, topk_groups=4, route_scale=2.5, bias="uniform"),
    "long_segments_bf16": MoEConfig("long_gelu", T=700, d=320, E=4, k=2, f=136),
}


@pytest.fixture(scope="module")
def cases():
    out = {}
    for name, cfg in CASES.items():
        inp = H.gpu_inputs(cfg)
        inp.update(make_expert_biases(cfg, "cuda"))
        out[name] = (cfg, inp)
    return out


def _packed(cfg, inp):
    got = H.gpu_route(cfg, inp)
    rows = cfg.T * cfg.k
    x_perm = torch.empty((rows, cfg.d), dtype=cfg.torch_dtype, device="cuda")
    perm_src = torch.empty((rows,), dtype=torch.int32, device="cuda")
    inv_row = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device="cuda")
    B.moe_permute(cfg, inp["x"], got["idx"], got["offsets"], x_perm, perm_src, inv_row, got["ws"])
    return got, x_perm


@pytest.mark.parametrize("name", sorted(CASES))
def test_expert_gelu_per_segment(cases, name):
    cfg, inp = cases[name]
    got, x_perm = _packed(cfg, inp)
    rows = cfg.T * cfg.k
    y_perm = torch.full((rows, cfg.d), float("nan"), dtype=cfg.torch_dtype, device="cuda")
    B.moe_expert_gelu(cfg, x_perm, got["offsets"], inp["w1"], inp["b1"], inp["w2"], inp["b2"], y_perm,
                      got["ws"])
    assert B.moe_get_device_error(got["ws"]) == B.MOE_OK
    offs = got["offsets"].cpu().numpy()
    xp = H.f64(x_perm)
    w1, w2, b1, b2 = H.f64(inp["w1"]), H.f64(inp["w2"]), H.f64(inp["b1"]), H.f64(inp["b2"])
    ref = np.zeros((rows, cfg.d))
    for e in range(cfg.E):
        a, b = offs[e], offs[e + 1]
        if b > a:
            ref[a:b] = orc.gelu_ffn(xp[a:b], w1[e], b1[e], w2[e], b2[e])
    H.compare_outputs(cfg, H.f64(y_perm), ref, "y_perm")


def _forward(cfg, inp, b1, b2):
    y = torch.full((cfg.T, cfg.d), float("nan"), dtype=cfg.torch_dtype, device="cuda")
    ws = B.alloc_workspace(cfg)
    B.moe_forward_gelu(cfg, inp["x"], inp["w_router"], inp["bias"], inp["w1"], b1, inp["w2"], b2, y, ws)
    assert B.moe_get_device_error(ws) == B.MOE_OK
    return y


@pytest.mark.parametrize("name", sorted(CASES))
def test_forward_gelu_matches_oracle(cases, name):
    cfg, inp = cases[name]
    y = _forward(cfg, inp, inp["b1"], inp["b2"])
    ref = H.oracle_route(cfg, inp)
    flags = orc.near_tie_tokens(ref, cfg.k, cfg.n_groups, cfg.topk_groups, H.NEAR_TIE_EPS)
    tokens = np.nonzero(~flags)[0]
    assert tokens.size >= cfg.T - max(1, cfg.T // 100)
    x = H.f64(inp["x"])[tokens]
    y_ref = orc.expert_outputs_gelu(x, ref["idx"][tokens], ref["gates"][tokens], H.f64(inp["w1"]),
                                    H.f64(inp["b1"]), H.f64(inp["w2"]), H.f64(inp["b2"]))
    H.compare_outputs(cfg, H.f64(y)[tokens], y_ref)
    assert torch.isfinite(y.float()).all().item()


def test_null_biases_equal_zero_biases(cases):
    cfg, inp = cases["grouped_bf16"]
    y_null = _forward(cfg, inp, None, None)
    y_zero = _forward(cfg, inp, torch.zeros_like(inp["b1"]), torch.zeros_like(inp["b2"]))
    assert torch.equal(y_null, y_zero)


def test_forward_gelu_is_deterministic(cases):
    cfg, inp = cases["grouped_bf16"]
    assert torch.equal(_forward(cfg, inp, inp["b1"], inp["b2"]), _forward(cfg, inp, inp["b1"], inp["b2"]))


def test_shared_expert_is_unsupported(cases):
    cfg, inp = cases["ragged_bf16"]
    c2 = cfg.with_(f_shared=64)
    y = torch.empty((cfg.T, cfg.d), dtype=cfg.torch_dtype, device="cuda")
    ws = B.alloc_workspace(c2)
    with pytest.raises(B.MoEError) as ei:
        B.moe_forward_gelu(c2, inp["x"], inp["w_router"], inp["bias"], inp["w1"], inp["b1"], inp["w2"],
                           inp["b2"], y, ws)
    assert ei.value.status == B.MOE_ERR_UNSUPPORTED


def test_forward_gelu_mixtral_shape_sampled():
    # Mixtral 8x7B FFN dimensions with GELU experts, checked on sampled tokens
    # (the oracle widens only the experts those tokens chose).
    cfg = MoEConfig("mixtral_gelu", T=4096, d=4096, E=8, k=2, f=14336)
    inp = H.gpu_inputs(cfg)
    inp.update(make_expert_biases(cfg, "cuda"))
    y = _forward(cfg, inp, inp["b1"], inp["b2"])
    ref = H.oracle_route(cfg, inp)
    flags = orc.near_tie_tokens(ref, cfg.k, cfg.n_groups, cfg.topk_groups, H.NEAR_TIE_EPS)
    tokens = sample_token_ids(cfg.T, 48).numpy()
    tokens = tokens[~flags[tokens]]
    x = H.f64(inp["x"][torch.as_tensor(tokens, device="cuda")])
    y_ref = orc.expert_outputs_gelu(x, ref["idx"][tokens], ref["gates"][tokens], H.LazyStack(inp["w1"]),
                                    H.f64(inp["b1"]), H.LazyStack(inp["w2"]), H.f64(inp["b2"]))
    H.compare_outputs(cfg, H.f64(y[torch.as_tensor(tokens, device="cuda")]), y_ref)
    assert torch.isfinite(y.float()).all().item()
