"""The workload table and the seeded input recipe, against numbers the pages print."""
import json
import math
import os

import pytest
import torch

from mixture_experts_ffn_sigmoid_b200.inputs import CONFIGS, GATE_SIGMOID, GATE_SOFTMAX, make_inputs

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_numbers.json")))


def test_deepseek_dims_match_pages():
    v = GOLD["deepseek_v3_dims"]["value"]
    for name in ("deepseek_v3", "deepseek_v3_skewed"):
        c = CONFIGS[name]
        assert (c.d, c.f, c.E, c.k, c.f_shared) == (v["hidden_size"], v["moe_intermediate_size"],
                                                    v["num_experts"], v["num_experts_per_tok"],
                                                    v["shared_experts"] * v["moe_intermediate_size"])
        r = GOLD["deepseek_v3_routing"]["value"]
        assert (c.n_groups, c.topk_groups, c.route_scale, c.gate_mode) == (
            r["n_groups"], r["topk_groups"], r["route_scale"], GATE_SIGMOID)


def test_deepseek_expert_params_within_total():
    # 58 MoE layers x 257 SwiGLU experts x 3 d f parameters: the bulk of 671B.
    c = CONFIGS["deepseek_v3"]
    v = GOLD["deepseek_v3_dims"]["value"]
    moe_layers = v["num_hidden_layers"] - v["first_k_dense_layers"]
    experts = 3 * c.d * c.f * (c.E + 1) * moe_layers
    total, active = GOLD["deepseek_v3_total_active_params_billion"]["value"]
    assert 0.95 * total * 1e9 < experts < total * 1e9
    # Activated expert params: (8 routed + 1 shared) per layer, well under 37B.
    act = 3 * c.d * c.f * (c.k + 1) * moe_layers
    assert act < active * 1e9
    assert abs(100 * active / total - GOLD["deepseek_v3_sparsity_percent"]["value"]) < 0.05


def test_mixtral_dims_match_pages():
    c = CONFIGS["mixtral_8x7b"]
    m = GOLD["mixtral_8x7b"]["value"]
    assert (c.E, c.k, c.gate_mode) == (m["experts"], m["top_k"], GATE_SOFTMAX)
    assert round(3 * c.d * c.f / 1e6) == GOLD["swiglu_ffn_params_4096x14336_million"]["value"]
    experts_32_layers = 3 * c.d * c.f * c.E * 32
    assert experts_32_layers < m["total_params_billion"] * 1e9 < 1.1 * experts_32_layers
    assert 3 * c.d * c.f * c.k * 32 < m["active_params_billion"] * 1e9


def test_expert_sets_per_token():
    c = CONFIGS["deepseek_v3"]
    n = math.comb(c.E, c.k)
    assert abs(n / GOLD["deepseek_v3_expert_sets_per_token"]["value"] - 1) < 0.05


@pytest.mark.parametrize("name", ["tiny_fp32", "decode_fine"])
def test_input_recipe_shapes_and_stats(name):
    c = CONFIGS[name]
    inp = make_inputs(c, "cpu", seed=0)
    assert inp["x"].shape == (c.T, c.d) and inp["x"].dtype == c.torch_dtype
    assert inp["w_router"].shape == (c.E, c.d)
    assert inp["w1"].shape == (c.E, c.f, c.d) and inp["w3"].shape == (c.E, c.f, c.d)
    assert inp["w2"].shape == (c.E, c.d, c.f)
    assert inp["bias"] is None and inp["ws1"] is None
    w1 = inp["w1"].float()
    assert abs(w1.std().item() * math.sqrt(c.d) - 1) < 0.05
    assert abs(inp["w2"].float().std().item() * math.sqrt(c.f) - 1) < 0.05
    again = make_inputs(c, "cpu", seed=0)
    assert torch.equal(again["w2"], inp["w2"]) and torch.equal(again["x"], inp["x"])
    other = make_inputs(c, "cpu", seed=1)
    assert not torch.equal(other["x"], inp["x"])


def test_skewed_bias_recipe():
    c = CONFIGS["deepseek_v3_skewed"].with_(T=8, d=64, f=64, f_shared=64)
    inp = make_inputs(c, "cpu")
    b = inp["bias"]
    assert b[0].item() == 4.0 and torch.all(b[1:8] == 2.0)
    assert torch.all(b[8:].abs() <= 0.05)
    assert inp["ws1"].shape == (64, 64) and inp["ws2"].shape == (64, 64)


def test_skewed_bias_sends_every_token_to_experts_0_to_7():
    # Sigmoid scores lie in (0, 1); +4 and +2 biases put experts 0..7 above
    # every other expert, and group 0's top-2 sum (> 6) keeps it. The oracle
    # must route every token to exactly {0..7}.
    import oracle.moe_oracle as orc
    c = CONFIGS["deepseek_v3_skewed"].with_(T=64, d=128, f=64, f_shared=64)
    inp = make_inputs(c, "cpu")
    r = orc.route(inp["x"].float().numpy(), inp["w_router"].float().numpy(), inp["bias"].numpy(),
                  c.k, c.gate_mode, c.n_groups, c.topk_groups, c.route_scale)
    assert (r["idx"] == list(range(8))).all()
