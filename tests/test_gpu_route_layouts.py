"""Routing on every layout of the warp-per-token top-k, GPU against the oracle.

Up to 256 experts, each lane of the routing warp holds NPL consecutive experts
(NPL = 1, 2, 4 or 8). A group of experts is then a run of whole lanes when its
size is a multiple of NPL and the lane count is a power of two; any other
grouping takes the general per-group path. The cases cover lanes past the last
expert, one lane per group, a lane holding parts of two groups, a lane count
that is not a power of two, expert counts that are not a multiple of 32 (the
last lanes read their biases one by one), both gate modes, the fused bf16
router and the fp32 router kernel.

The tie cases use integer router logits, so equal scores are equal in every
precision. The pages' rule then fixes the winners exactly: groups ranked by
score with equal scores to the lower group index, experts by biased score with
equal scores to the lower id (DeepSeek-V3 note, "How it works", Routing; MoE
cheat sheet, "The router in code": a stable sort by score). Those cases compare
every token, with no near-tie exclusion.
"""
import numpy as np
import pytest
import torch

from mixture_experts_ffn_sigmoid_b200.inputs import GATE_SIGMOID, GATE_SOFTMAX, MoEConfig

import gpu_harness as H
from mixture_experts_ffn_sigmoid_b200 import binding as B

pytestmark = pytest.mark.gpu


def _cfg(name, E, k, n_groups=1, topk_groups=1, gate=GATE_SIGMOID, dtype="bf16", T=200, scale=2.5):
    return MoEConfig(name, T=T, d=128, E=E, k=k, f=64, dtype=dtype, gate_mode=gate, n_groups=n_groups,
                     topk_groups=topk_groups, route_scale=scale if gate == GATE_SIGMOID else 1.0, bias="uniform")


LAYOUTS = {
    # 8 experts a lane, groups of 32 = 4 lanes; 20 of the 32 lanes hold experts
    "e160_g5_bf16": _cfg("e160_g5", 160, 8, 5, 2),
    "e192_g6_bf16": _cfg("e192_g6", 192, 6, 6, 3, T=130),
    # groups of 8 = one lane each, 32 groups ranked by shuffles
    "e256_g32_bf16": _cfg("e256_g32", 256, 8, 32, 4, T=150),
    # groups of 3 with 4 experts a lane: a lane spans two groups
    "e72_g24_bf16": _cfg("e72_g24", 72, 6, 24, 4, T=100),
    # groups of 24 = 6 lanes: not a power of two
    "e96_g4_fp32": _cfg("e96_g4_f32", 96, 6, 4, 2, dtype="f32", T=100),
    # 200 experts: the last lane holds experts past E
    "e200_softmax_bf16": _cfg("e200_softmax", 200, 8, gate=GATE_SOFTMAX),
    "e200_g8_fp32": _cfg("e200_g8_f32", 200, 8, 8, 4, dtype="f32", T=90),
    # the DeepSeek-V3 grouping on the fp32 router kernel
    "e256_g8_fp32": _cfg("e256_g8_f32", 256, 8, 8, 4, dtype="f32", T=70),
    # 2 and 1 experts a lane
    "e48_g6_bf16": _cfg("e48_g6", 48, 4, 6, 2, T=120),
    "e20_softmax_fp32": _cfg("e20_softmax_f32", 20, 3, gate=GATE_SOFTMAX, dtype="f32", T=60),
}


@pytest.mark.parametrize("name", sorted(LAYOUTS))
def test_route_layout(name):
    cfg = LAYOUTS[name]
    inp = H.gpu_inputs(cfg, seed=3)
    H.check_route(cfg, H.oracle_route(cfg, inp), H.gpu_route(cfg, inp))


def _integer_logit_inputs(cfg, seed, nonzeros=3, zero_router=False):
    """x in {-1, 0, 1}; each router row has `nonzeros` entries of +-1, so every
    logit is an integer in [-nonzeros, nonzeros] and many tie exactly."""
    g = np.random.default_rng(seed)
    inp = H.gpu_inputs(cfg, seed=seed)
    dt = cfg.torch_dtype
    x = g.integers(-1, 2, size=(cfg.T, cfg.d)).astype(np.float32)
    w = np.zeros((cfg.E, cfg.d), dtype=np.float32)
    if not zero_router:
        for e in range(cfg.E):
            cols = g.choice(cfg.d, size=nonzeros, replace=False)
            w[e, cols] = g.choice([-1.0, 1.0], size=nonzeros)
    inp["x"] = torch.as_tensor(x, device="cuda").to(dt)
    inp["w_router"] = torch.as_tensor(w, device="cuda").to(dt)
    inp["bias"] = torch.zeros(cfg.E, dtype=torch.float32, device="cuda")
    return inp


TIES = {
    "ties_e256_g8_bf16": _cfg("ties_e256_g8", 256, 8, 8, 4, T=160),
    "ties_e256_g8_fp32": _cfg("ties_e256_g8_f32", 256, 8, 8, 4, dtype="f32", T=96),
    "ties_e200_softmax_bf16": _cfg("ties_e200", 200, 8, gate=GATE_SOFTMAX, T=130),
    "ties_e72_g24_bf16": _cfg("ties_e72_g24", 72, 6, 24, 4, T=100),
    "ties_e128_bf16": _cfg("ties_e128", 128, 8, T=64),
}


@pytest.mark.parametrize("name", sorted(TIES))
def test_exact_ties_follow_the_lower_index_rule(name):
    cfg = TIES[name]
    inp = _integer_logit_inputs(cfg, seed=11)
    ref = H.oracle_route(cfg, inp)
    got = H.gpu_route(cfg, inp)
    gi = got["idx"].cpu().numpy().astype(np.int64)
    # many tokens do tie at the k-th place: the case tests the rule
    flags = H.orc.near_tie_tokens(ref, cfg.k, cfg.n_groups, cfg.topk_groups, H.NEAR_TIE_EPS)
    assert flags.mean() > 0.5, "the inputs were meant to tie"
    bad = np.nonzero(np.any(gi != ref["idx"], axis=1))[0]
    assert bad.size == 0, f"{bad.size} tokens differ, e.g. {bad[:3]}: gpu {gi[bad[:3]]} ref {ref['idx'][bad[:3]]}"
    gg = got["gate"].cpu().numpy().astype(np.float64)
    assert np.abs(gg - ref["gates"]).max() <= H.gate_tol(cfg)
    c_ref, o_ref = H.orc.expert_counts_offsets(ref["idx"], cfg.E)
    assert np.array_equal(got["counts"].cpu().numpy(), c_ref)
    assert np.array_equal(got["offsets"].cpu().numpy(), o_ref)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_all_scores_equal_pick_the_lowest_groups_and_ids(dtype):
    # A zero router matrix and zero bias: every expert and every group ties,
    # so groups 0..3 are kept and experts 0..7 (all in group 0) win, each
    # with the gate route_scale / k.
    cfg = _cfg("all_equal", 256, 8, 8, 4, dtype=dtype, T=40)
    inp = _integer_logit_inputs(cfg, seed=5, zero_router=True)
    got = H.gpu_route(cfg, inp)
    gi = got["idx"].cpu().numpy()
    assert np.array_equal(gi, np.tile(np.arange(8), (cfg.T, 1)))
    gg = got["gate"].cpu().numpy().astype(np.float64)
    assert np.abs(gg - cfg.route_scale / cfg.k).max() <= H.gate_tol(cfg)
    ref = H.oracle_route(cfg, inp)
    assert np.array_equal(ref["idx"], gi)


# moe_route_maps: the fused router of a one-tile batch also writes the row
# maps; they must equal moe_route followed by the maps-only moe_permute.
MAPS = {
    "maps_t1": _cfg("maps_t1", 16, 4, T=1),
    "maps_t33_e256_g8": _cfg("maps_t33", 256, 8, 8, 4, T=33),
    "maps_t128_e128_softmax": _cfg("maps_t128", 128, 8, gate=GATE_SOFTMAX, T=128),
    "maps_t100_e72_g24": _cfg("maps_t100", 72, 6, 24, 4, T=100),
    "maps_t64_e8_k8": _cfg("maps_t64_k8", 8, 8, T=64),
}


@pytest.mark.parametrize("name", sorted(MAPS))
def test_route_maps_equal_route_then_permute(name):
    cfg = MAPS[name]
    inp = H.gpu_inputs(cfg, seed=7)
    assert B.moe_route_maps_supported(cfg)
    ref = H.gpu_route(cfg, inp)
    rows = cfg.T * cfg.k
    src_a = torch.full((rows,), -7, dtype=torch.int32, device="cuda")
    inv_a = torch.full((cfg.T, cfg.k), -7, dtype=torch.int32, device="cuda")
    B.moe_permute(cfg, None, ref["idx"], ref["offsets"], None, src_a, inv_a, ref["ws"])
    ws = B.alloc_workspace(cfg)
    idx = torch.full((cfg.T, cfg.k), -7, dtype=torch.int32, device="cuda")
    gate = torch.full((cfg.T, cfg.k), float("nan"), dtype=torch.float32, device="cuda")
    counts = torch.full((cfg.E,), -7, dtype=torch.int32, device="cuda")
    offsets = torch.full((cfg.E + 1,), -7, dtype=torch.int32, device="cuda")
    src_b = torch.full((rows,), -7, dtype=torch.int32, device="cuda")
    inv_b = torch.full((cfg.T, cfg.k), -7, dtype=torch.int32, device="cuda")
    B.moe_route_maps(cfg, inp["x"], inp["w_router"], inp["bias"], idx, gate, counts, offsets, src_b, inv_b, ws)
    torch.cuda.synchronize()
    assert torch.equal(idx, ref["idx"]) and torch.equal(gate, ref["gate"])
    assert torch.equal(counts, ref["counts"]) and torch.equal(offsets, ref["offsets"])
    assert torch.equal(src_b, src_a) and torch.equal(inv_b, inv_a)
    assert B.moe_get_device_error(ws) == B.MOE_OK
    H.check_route(cfg, H.oracle_route(cfg, inp), ref)


@pytest.mark.parametrize("cfg", [_cfg("maps_t129", 64, 4, T=129), _cfg("maps_f32", 64, 4, dtype="f32", T=64),
                                 _cfg("maps_e320", 320, 4, T=64)], ids=lambda c: c.name)
def test_route_maps_unsupported_writes_nothing(cfg):
    assert not B.moe_route_maps_supported(cfg)
    inp = H.gpu_inputs(cfg, seed=7)
    ws = B.alloc_workspace(cfg)
    rows = cfg.T * cfg.k
    idx = torch.full((cfg.T, cfg.k), -7, dtype=torch.int32, device="cuda")
    gate = torch.zeros((cfg.T, cfg.k), dtype=torch.float32, device="cuda")
    counts = torch.full((cfg.E,), -7, dtype=torch.int32, device="cuda")
    offsets = torch.full((cfg.E + 1,), -7, dtype=torch.int32, device="cuda")
    src = torch.full((rows,), -7, dtype=torch.int32, device="cuda")
    inv = torch.full((cfg.T, cfg.k), -7, dtype=torch.int32, device="cuda")
    with pytest.raises(B.MoEError) as e:
        B.moe_route_maps(cfg, inp["x"], inp["w_router"], inp["bias"], idx, gate, counts, offsets, src, inv, ws)
    assert e.value.status == B.MOE_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert int(idx.min()) == -7 and int(src.max()) == -7 and int(counts.max()) == -7
