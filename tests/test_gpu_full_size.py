"""Parity at the workloads' full sizes, through moe_forward (the call the
bench times). Routing (indices, counts, offsets) is checked for every token;
outputs for every token where the fp64 oracle finishes in seconds (tiny,
decode) and on a seeded sample of 512 tokens otherwise: each token's output
depends only on its own row and the weights, so a sample checks those
tokens exactly."""
import numpy as np
import pytest
import torch

from mixture_experts_ffn_sigmoid_b200.inputs import CONFIGS

import gpu_harness as H

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

SAMPLE = {"tiny_fp32": None, "decode_fine": None, "mixtral_8x7b": 512, "deepseek_v3": 512,
          "deepseek_v3_skewed": 512}


@pytest.mark.parametrize("name", ["tiny_fp32", "decode_fine", "deepseek_v3", "mixtral_8x7b",
                                  "deepseek_v3_skewed"])
def test_full_size_forward(name):
    cfg = CONFIGS[name]
    inp = H.gpu_inputs(cfg)
    got = H.gpu_route(cfg, inp)
    ref = H.oracle_route(cfg, inp)
    rep = H.check_route(cfg, ref, got)
    assert rep["near_ties"] <= max(2, cfg.T // 200), rep["near_ties"]
    if name == "deepseek_v3_skewed":
        counts = got["counts"].cpu().numpy()
        assert np.all(counts[:8] == cfg.T) and counts[8:].sum() == 0
    del got
    y = H.gpu_forward(cfg, inp)
    out = H.check_forward(cfg, inp, y, n_sample=SAMPLE[name], lazy=cfg.E * cfg.f * cfg.d > 2 ** 27)
    print(f"{name}: {out}")
