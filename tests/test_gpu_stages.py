"""Per-stage parity on the GPU: route, permute, experts, combine, each called
through the C ABI and compared with the CPU oracle on the same inputs.

Shapes are small enough for the full oracle, yet span several tiles and a
ragged tail: T not a multiple of the 32-token chunk, expert segments longer
than one 256-token tile, hidden and inner widths that are not multiples of
the 64-wide K step or the 128-row weight tile.
"""
import numpy as np
import pytest
import torch

import oracle.moe_oracle as orc
from mixture_experts_ffn_sigmoid_b200 import binding as B
from mixture_experts_ffn_sigmoid_b200.inputs import CONFIGS, GATE_SIGMOID, GATE_SOFTMAX, MoEConfig

import gpu_harness as H

pytestmark = pytest.mark.gpu

STAGE_CASES = {
    "tiny_fp32": CONFIGS["tiny_fp32"],
    "ds_like_small_bf16": MoEConfig("ds_like_small", T=300, d=256, E=32, k=4, f=384, gate_mode=GATE_SIGMOID,
                                    n_groups=8, topk_groups=4, route_scale=2.5, f_shared=256, bias="uniform"),
    "long_segments_bf16": MoEConfig("long_segments", T=700, d=320, E=4, k=2, f=136),
    "ragged_dims_bf16": MoEConfig("ragged_dims", T=77, d=200, E=12, k=3, f=72, gate_mode=GATE_SIGMOID,
                                  route_scale=1.0, f_shared=40, bias="uniform"),
    "ragged_dims_fp32": MoEConfig("ragged_dims_f32", T=77, d=200, E=12, k=3, f=72, dtype="f32",
                                  gate_mode=GATE_SIGMOID, f_shared=40, bias="uniform"),
    # More than 256 experts: the router's second expert tile; ragged T and
    # segments of a handful of rows.
    "wide_experts_bf16": MoEConfig("wide_experts", T=150, d=192, E=320, k=6, f=64, gate_mode=GATE_SIGMOID,
                                   n_groups=8, topk_groups=4, route_scale=2.5, f_shared=64, bias="uniform"),
    # d a multiple of the down tile's rows (512 on CTA pairs, 256 on single
    # CTAs), so no weight tile is ragged; token tiles of up to 256 rows (one
    # 128-row copy per CTA of a pair) and of 64 rows (single CTAs).
    "fused_blocks_pair_bf16": MoEConfig("fused_blocks_pair", T=256, d=512, E=8, k=2, f=256,
                                        gate_mode=GATE_SIGMOID, route_scale=1.0, f_shared=128, bias="uniform"),
    "fused_blocks_single_bf16": MoEConfig("fused_blocks_single", T=40, d=256, E=16, k=2, f=128,
                                          gate_mode=GATE_SIGMOID, route_scale=1.0, f_shared=64, bias="uniform"),
    # k >= 4 and 64 chunks of 32 tokens: the permute copies whole rows with
    # bulk copies (the smaller cases take the vector path).
    "bulk_permute_bf16": MoEConfig("bulk_permute", T=2048, d=256, E=64, k=4, f=128, gate_mode=GATE_SIGMOID,
                                   n_groups=8, topk_groups=4, route_scale=2.5, f_shared=128, bias="uniform"),
    "bulk_permute_fp32": MoEConfig("bulk_permute_f32", T=2040, d=136, E=32, k=4, f=64, dtype="f32",
                                   gate_mode=GATE_SIGMOID, route_scale=1.0, bias="uniform"),
    # More chunks than SMs (150 > 148): each chunk's rows are split over
    # eight four-token blocks, and the last chunk holds two tokens.
    "bulk_permute_split_bf16": MoEConfig("bulk_permute_split", T=4770, d=128, E=64, k=4, f=64,
                                         gate_mode=GATE_SIGMOID, n_groups=8, topk_groups=4, route_scale=2.5,
                                         f_shared=64, bias="uniform"),
}


@pytest.fixture(scope="module")
def cases():
    out = {}
    for name, cfg in STAGE_CASES.items():
        out[name] = (cfg, H.gpu_inputs(cfg))
    return out


@pytest.mark.parametrize("name", sorted(STAGE_CASES))
def test_route(cases, name):
    cfg, inp = cases[name]
    got = H.gpu_route(cfg, inp)
    rep = H.check_route(cfg, H.oracle_route(cfg, inp), got)
    assert rep["near_ties"] <= max(1, cfg.T // 100)


@pytest.mark.parametrize("name", sorted(STAGE_CASES))
def test_permute(cases, name):
    cfg, inp = cases[name]
    got = H.gpu_route(cfg, inp)
    rows = cfg.T * cfg.k
    x_perm = torch.full((rows, cfg.d), float("nan"), dtype=cfg.torch_dtype, device="cuda")
    perm_src = torch.full((rows,), -7, dtype=torch.int32, device="cuda")
    inv_row = torch.full((cfg.T, cfg.k), -7, dtype=torch.int32, device="cuda")
    B.moe_permute(cfg, inp["x"], got["idx"], got["offsets"], x_perm, perm_src, inv_row, got["ws"])
    assert B.moe_get_device_error(got["ws"]) == B.MOE_OK
    gi = got["idx"].cpu().numpy()
    inv_ref, src_ref = orc.permutation_rows(gi, got["offsets"].cpu().numpy())
    assert np.array_equal(inv_row.cpu().numpy(), inv_ref)
    assert np.array_equal(perm_src.cpu().numpy(), src_ref)
    # Copies are exact: packed row r is x[perm_src[r]] byte for byte.
    assert torch.equal(x_perm, inp["x"][perm_src.long()])


def _packed(cfg, inp):
    got = H.gpu_route(cfg, inp)
    rows = cfg.T * cfg.k
    x_perm = torch.empty((rows, cfg.d), dtype=cfg.torch_dtype, device="cuda")
    perm_src = torch.empty((rows,), dtype=torch.int32, device="cuda")
    inv_row = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device="cuda")
    B.moe_permute(cfg, inp["x"], got["idx"], got["offsets"], x_perm, perm_src, inv_row, got["ws"])
    return got, x_perm, perm_src, inv_row


@pytest.mark.parametrize("name", sorted(STAGE_CASES))
def test_expert_swiglu(cases, name):
    cfg, inp = cases[name]
    got, x_perm, perm_src, inv_row = _packed(cfg, inp)
    rows = cfg.T * cfg.k
    y_perm = torch.full((rows, cfg.d), float("nan"), dtype=cfg.torch_dtype, device="cuda")
    y_sh = torch.full((cfg.T, cfg.d), float("nan"), dtype=cfg.torch_dtype, device="cuda") \
        if cfg.f_shared else None
    B.moe_expert_swiglu(cfg, x_perm, got["offsets"], inp["w1"], inp["w3"], inp["w2"],
                        inp["x"] if cfg.f_shared else None, inp["ws1"], inp["ws3"], inp["ws2"],
                        y_perm, y_sh, got["ws"])
    assert B.moe_get_device_error(got["ws"]) == B.MOE_OK
    # Reference: FFN of the expert that owns each packed row, on that row.
    offs = got["offsets"].cpu().numpy()
    xp = H.f64(x_perm)
    w1, w3, w2 = H.f64(inp["w1"]), H.f64(inp["w3"]), H.f64(inp["w2"])
    ref = np.zeros((rows, cfg.d))
    for e in range(cfg.E):
        a, b = offs[e], offs[e + 1]
        if b > a:
            ref[a:b] = orc.swiglu_ffn(xp[a:b], w1[e], w3[e], w2[e])
    H.compare_outputs(cfg, H.f64(y_perm), ref, "y_perm")
    if cfg.f_shared:
        ref_s = orc.swiglu_ffn(H.f64(inp["x"]), H.f64(inp["ws1"]), H.f64(inp["ws3"]), H.f64(inp["ws2"]))
        H.compare_outputs(cfg, H.f64(y_sh), ref_s, "y_shared")


@pytest.mark.parametrize("name", sorted(STAGE_CASES))
def test_combine(cases, name):
    cfg, inp = cases[name]
    got, x_perm, perm_src, inv_row = _packed(cfg, inp)
    rows = cfg.T * cfg.k
    g = torch.Generator(device="cuda")
    g.manual_seed(5)
    y_perm = torch.randn((rows, cfg.d), generator=g, device="cuda").to(cfg.torch_dtype)
    y_sh = torch.randn((cfg.T, cfg.d), generator=g, device="cuda").to(cfg.torch_dtype) if cfg.f_shared else None
    y = torch.full((cfg.T, cfg.d), float("nan"), dtype=cfg.torch_dtype, device="cuda")
    B.moe_combine(cfg, y_perm, inv_row, got["gate"], y_sh, y)
    torch.cuda.synchronize()
    yp, inv, gate = H.f64(y_perm), inv_row.cpu().numpy(), got["gate"].cpu().numpy().astype(np.float64)
    ref = np.zeros((cfg.T, cfg.d))
    for j in range(cfg.k):
        ref += gate[:, j:j + 1] * yp[inv[:, j]]
    if cfg.f_shared:
        ref += H.f64(y_sh)
    # Only the final rounding to the storage type separates the two.
    err = np.abs(H.f64(y) - ref)
    bound = (2.0 ** -8 if cfg.dtype == "bf16" else 2.0 ** -22) * np.abs(ref) + 1e-6
    assert np.all(err <= bound), float((err - bound).max())


@pytest.mark.parametrize("name", sorted(STAGE_CASES))
def test_forward_full_oracle(cases, name):
    cfg, inp = cases[name]
    y = H.gpu_forward(cfg, inp)
    rep = H.check_forward(cfg, inp, y)
    assert rep["compared"] >= cfg.T - max(1, cfg.T // 100)


# ds_like_small runs its expert GEMMs on CTA pairs (moe_forward reads a packed
# copy of the token rows); fused_blocks_single on single CTAs (moe_forward's
# gate/up GEMM gathers the rows from x, the permute writes the maps only).
@pytest.mark.parametrize("name", ["ds_like_small_bf16", "fused_blocks_single_bf16"])
def test_forward_equals_stage_chain(cases, name):
    # moe_forward and the four stage calls give the same bytes.
    cfg, inp = cases[name]
    y_fwd = H.gpu_forward(cfg, inp)
    got, x_perm, perm_src, inv_row = _packed(cfg, inp)
    rows = cfg.T * cfg.k
    y_perm = torch.empty((rows, cfg.d), dtype=cfg.torch_dtype, device="cuda")
    y_sh = torch.empty((cfg.T, cfg.d), dtype=cfg.torch_dtype, device="cuda")
    B.moe_expert_swiglu(cfg, x_perm, got["offsets"], inp["w1"], inp["w3"], inp["w2"], inp["x"],
                        inp["ws1"], inp["ws3"], inp["ws2"], y_perm, y_sh, got["ws"])
    y = torch.empty_like(y_fwd)
    B.moe_combine(cfg, y_perm, inv_row, got["gate"], y_sh, y)
    torch.cuda.synchronize()
    assert torch.equal(y, y_fwd)


@pytest.mark.parametrize("name", ["ds_like_small_bf16", "fused_blocks_single_bf16"])
def test_forward_is_deterministic(cases, name):
    cfg, inp = cases[name]
    a = H.gpu_forward(cfg, inp)
    b = H.gpu_forward(cfg, inp)
    assert torch.equal(a, b)


@pytest.mark.parametrize("name", sorted(STAGE_CASES))
def test_gate_up_gather_matches_packed(cases, name):
    # Reading token rows through perm_src (cp.async gather) gives bit-identical h
    # to reading the packed copy x_perm; maps-only permute writes the same maps.
    cfg, inp = cases[name]
    got, x_perm, perm_src, inv_row = _packed(cfg, inp)
    rows = cfg.T * cfg.k
    src2 = torch.full((rows,), -7, dtype=torch.int32, device="cuda")
    inv2 = torch.full((cfg.T, cfg.k), -7, dtype=torch.int32, device="cuda")
    B.moe_permute(cfg, None, got["idx"], got["offsets"], None, src2, inv2, got["ws"])
    torch.cuda.synchronize()
    assert torch.equal(src2, perm_src) and torch.equal(inv2, inv_row)
    sh = cfg.f_shared > 0
    h_a = torch.full((rows, cfg.f), float("nan"), dtype=cfg.torch_dtype, device="cuda")
    h_b = torch.full((rows, cfg.f), float("nan"), dtype=cfg.torch_dtype, device="cuda")
    hs_a = torch.full((cfg.T, cfg.f_shared), float("nan"), dtype=cfg.torch_dtype, device="cuda") if sh else None
    hs_b = torch.full((cfg.T, cfg.f_shared), float("nan"), dtype=cfg.torch_dtype, device="cuda") if sh else None
    B.moe_expert_gate_up(cfg, x_perm, got["offsets"], inp["w1"], inp["w3"], inp["x"] if sh else None,
                         inp["ws1"], inp["ws3"], h_a, hs_a, got["ws"])
    if cfg.dtype == "f32":
        with pytest.raises(B.MoEError) as ei:
            B.moe_expert_gate_up_gather(cfg, inp["x"], perm_src, got["offsets"], inp["w1"], inp["w3"],
                                        inp["ws1"], inp["ws3"], h_b, hs_b, got["ws"])
        assert ei.value.status == B.MOE_ERR_UNSUPPORTED
        return
    B.moe_expert_gate_up_gather(cfg, inp["x"], perm_src, got["offsets"], inp["w1"], inp["w3"],
                                inp["ws1"], inp["ws3"], h_b, hs_b, got["ws"])
    assert B.moe_get_device_error(got["ws"]) == B.MOE_OK
    assert torch.equal(h_a, h_b)
    if sh:
        assert torch.equal(hs_a, hs_b)


@pytest.mark.parametrize("name", sorted(STAGE_CASES))
def test_gate_up_hidden_matches_oracle(cases, name):
    # The SwiGLU inner activation h = SiLU(x W1^T) * (x W3^T) (Sparse MoE FFN
    # note, SwiGLU equation) from moe_expert_gate_up, and from
    # moe_expert_gate_up_gather (rows of x read through perm_src: the note's
    # "Packed forward (official)" gathers each expert's tokens), each compared
    # with the oracle per expert segment and element by element: relative L2
    # <= 2e-2 and |error| <= 5e-2 RMS + 1e-2 |ref| for bf16 (h is stored in
    # bf16 after an fp32 epilogue), relative L2 <= 1e-5 for fp32.
    cfg, inp = cases[name]
    got, x_perm, perm_src, inv_row = _packed(cfg, inp)
    rows = cfg.T * cfg.k
    sh = cfg.f_shared > 0
    offs = got["offsets"].cpu().numpy()
    x64 = H.f64(inp["x"])
    _, src = orc.permutation_rows(got["idx"].cpu().numpy(), offs)   # the oracle's packed-row sources
    w1, w3 = H.f64(inp["w1"]), H.f64(inp["w3"])
    variants = ["packed"] + (["gather"] if cfg.dtype == "bf16" else [])
    for v in variants:
        h = torch.full((rows, cfg.f), float("nan"), dtype=cfg.torch_dtype, device="cuda")
        h_s = torch.full((cfg.T, cfg.f_shared), float("nan"), dtype=cfg.torch_dtype, device="cuda") if sh else None
        if v == "packed":
            B.moe_expert_gate_up(cfg, x_perm, got["offsets"], inp["w1"], inp["w3"], inp["x"] if sh else None,
                                 inp["ws1"], inp["ws3"], h, h_s, got["ws"])
        else:
            B.moe_expert_gate_up_gather(cfg, inp["x"], perm_src, got["offsets"], inp["w1"], inp["w3"],
                                        inp["ws1"], inp["ws3"], h, h_s, got["ws"])
        assert B.moe_get_device_error(got["ws"]) == B.MOE_OK
        h64 = H.f64(h)
        for e in range(cfg.E):
            a, b = offs[e], offs[e + 1]
            if b > a:
                # The oracle reads the token rows from x itself, through its
                # own packing of the GPU's expert choice.
                ref = orc.swiglu_hidden(x64[src[a:b]], w1[e], w3[e])
                H.compare_outputs(cfg, h64[a:b], ref, f"{v} h of expert {e}")
        if sh:
            ref_s = orc.swiglu_hidden(x64, H.f64(inp["ws1"]), H.f64(inp["ws3"]))
            H.compare_outputs(cfg, H.f64(h_s), ref_s, f"{v} shared h")


@pytest.mark.parametrize("name", sorted(STAGE_CASES))
def test_gate_up_weight_storage_order(cases, name):
    # W1 and W3 are two caller buffers at any addresses. h must not depend on
    # their order in memory: the same weights stored W1-then-W3 and
    # W3-then-W1 in one allocation give bit-identical h, and that h matches
    # the oracle (SwiGLU equation of the Sparse MoE FFN note).
    cfg, inp = cases[name]
    got, x_perm, _, _ = _packed(cfg, inp)
    rows = cfg.T * cfg.k
    sh = cfg.f_shared > 0
    outs = []
    for order in ("w1_first", "w3_first"):
        pair = torch.empty((2,) + tuple(inp["w1"].shape), dtype=inp["w1"].dtype, device="cuda")
        pair_s = torch.empty((2,) + tuple(inp["ws1"].shape), dtype=inp["ws1"].dtype, device="cuda") if sh else None
        i1, i3 = (0, 1) if order == "w1_first" else (1, 0)
        pair[i1].copy_(inp["w1"])
        pair[i3].copy_(inp["w3"])
        if sh:
            pair_s[i1].copy_(inp["ws1"])
            pair_s[i3].copy_(inp["ws3"])
        assert (pair[i3].data_ptr() < pair[i1].data_ptr()) == (order == "w3_first")
        h = torch.full((rows, cfg.f), float("nan"), dtype=cfg.torch_dtype, device="cuda")
        h_s = torch.full((cfg.T, cfg.f_shared), float("nan"), dtype=cfg.torch_dtype, device="cuda") if sh else None
        B.moe_expert_gate_up(cfg, x_perm, got["offsets"], pair[i1], pair[i3], inp["x"] if sh else None,
                             pair_s[i1] if sh else None, pair_s[i3] if sh else None, h, h_s, got["ws"])
        assert B.moe_get_device_error(got["ws"]) == B.MOE_OK
        outs.append((h, h_s))
    assert torch.equal(outs[0][0], outs[1][0])
    if sh:
        assert torch.equal(outs[0][1], outs[1][1])
    offs = got["offsets"].cpu().numpy()
    _, src = orc.permutation_rows(got["idx"].cpu().numpy(), offs)
    x64, h64 = H.f64(inp["x"]), H.f64(outs[1][0])
    for e in range(cfg.E):
        a, b = offs[e], offs[e + 1]
        if b > a:
            ref = orc.swiglu_hidden(x64[src[a:b]], H.f64(inp["w1"])[e], H.f64(inp["w3"])[e])
            H.compare_outputs(cfg, h64[a:b], ref, f"w3-first h of expert {e}")
