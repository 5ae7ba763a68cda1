"""Edge and degenerate cases of the block on the GPU, each against the oracle:
one token, a token count that leaves a ragged 32-token chunk, k = E (every
expert fires, bias irrelevant), all tokens on one expert (all other experts
empty), a single expert (a dense SwiGLU), group limits that keep one group,
no tokens at all, a token whose scores are NaN or infinite, caller indices
and offsets out of range (skipped or clamped, and reported), and the
bounded-wait error path."""
import numpy as np
import pytest
import torch

import oracle.moe_oracle as orc
from mixture_experts_ffn_sigmoid_b200 import binding as B
from mixture_experts_ffn_sigmoid_b200.inputs import GATE_SIGMOID, GATE_SOFTMAX, MoEConfig

import gpu_harness as H

pytestmark = pytest.mark.gpu

EDGE = {
    "one_token": MoEConfig("one_token", T=1, d=256, E=16, k=4, f=256, gate_mode=GATE_SIGMOID,
                           route_scale=2.5, f_shared=128, bias="uniform"),
    "ragged_chunk": MoEConfig("ragged_chunk", T=33, d=128, E=8, k=2, f=128),
    "k_equals_E": MoEConfig("k_equals_E", T=40, d=128, E=4, k=4, f=64, gate_mode=GATE_SIGMOID,
                            route_scale=2.5, bias="uniform"),
    "single_expert": MoEConfig("single_expert", T=100, d=192, E=1, k=1, f=320),
    "one_group_kept": MoEConfig("one_group_kept", T=96, d=128, E=64, k=6, f=128, gate_mode=GATE_SIGMOID,
                                n_groups=8, topk_groups=1, route_scale=2.5, bias="uniform"),
    "k1_fp32": MoEConfig("k1_fp32", T=50, d=64, E=5, k=1, f=48, dtype="f32"),
    "many_experts": MoEConfig("many_experts", T=64, d=128, E=1024, k=32, f=64),
    # One full router tile of a DeepSeek-V3-style routing (grouped sigmoid,
    # shared expert) at decode size: moe_forward routes and writes the row
    # maps in one launch and its gate/up GEMM gathers the rows from x.
    "one_tile_grouped": MoEConfig("one_tile_grouped", T=128, d=512, E=256, k=8, f=256, gate_mode=GATE_SIGMOID,
                                  n_groups=8, topk_groups=4, route_scale=2.5, f_shared=256, bias="uniform"),
}


@pytest.mark.parametrize("name", sorted(EDGE))
def test_edge_forward(name):
    cfg = EDGE[name]
    inp = H.gpu_inputs(cfg)
    if name == "one_tile_grouped":
        assert B.moe_forward_gathers_rows(cfg, inp["x"]) and B.moe_route_maps_supported(cfg)
    got = H.gpu_route(cfg, inp)
    H.check_route(cfg, H.oracle_route(cfg, inp), got)
    y = H.gpu_forward(cfg, inp)
    H.check_forward(cfg, inp, y)


def test_all_tokens_on_one_expert():
    # A +10 bias on expert 3 with k = 1: expert 3 gets every token (a segment
    # spanning several 256-token tiles), the other experts are empty.
    cfg = MoEConfig("hot_expert", T=600, d=128, E=8, k=1, f=128, gate_mode=GATE_SIGMOID, route_scale=1.0,
                    bias="uniform")
    inp = H.gpu_inputs(cfg)
    inp["bias"] = torch.zeros(8, device="cuda")
    inp["bias"][3] = 10.0
    got = H.gpu_route(cfg, inp)
    counts = got["counts"].cpu().numpy()
    assert counts[3] == 600 and counts.sum() == 600
    H.check_route(cfg, H.oracle_route(cfg, inp), got)
    y = H.gpu_forward(cfg, inp)
    H.check_forward(cfg, inp, y)


def test_zero_tokens():
    cfg = MoEConfig("empty", T=0, d=128, E=8, k=2, f=128)
    c = B.make_config(cfg)
    ws = B.alloc_workspace(c)
    counts = torch.full((8,), 5, dtype=torch.int32, device="cuda")
    offsets = torch.full((9,), 5, dtype=torch.int32, device="cuda")
    empty = torch.empty((0, 128), dtype=torch.bfloat16, device="cuda")
    wr = torch.zeros((8, 128), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((0, 2), dtype=torch.int32, device="cuda")
    gate = torch.empty((0, 2), dtype=torch.float32, device="cuda")
    B.lib()
    st = B.lib().moe_route(B.ctypes.byref(c), None, B._ptr(wr), None, None, None, B._ptr(counts),
                           B._ptr(offsets), B._ptr(ws), ws.numel(), B._stream(None))
    assert st == B.MOE_OK
    torch.cuda.synchronize()
    assert counts.sum().item() == 0 and offsets.sum().item() == 0


def test_bounded_wait_reports_timeout_and_context_survives():
    cfg = MoEConfig("after_timeout", T=64, d=128, E=8, k=2, f=128)
    ws = B.alloc_workspace(cfg)
    B.moe_selftest_wait_timeout(ws, 50_000_000)          # 50 ms bound, nothing ever arrives
    assert B.moe_get_device_error(ws) == B.MOE_ERR_TIMEOUT
    assert B.moe_get_device_error(ws) == B.MOE_OK         # the word was cleared
    inp = H.gpu_inputs(cfg)
    y = H.gpu_forward(cfg, inp, ws)                       # the context is still usable
    H.check_forward(cfg, inp, y)


def test_bad_indices_are_skipped_not_dereferenced():
    # Out-of-range expert ids from a caller: the permute skips them and
    # reports row -1 instead of writing out of bounds.
    cfg = MoEConfig("bad_idx", T=32, d=128, E=8, k=2, f=128)
    inp = H.gpu_inputs(cfg)
    got = H.gpu_route(cfg, inp)
    idx = got["idx"].clone()
    idx[5, 1] = 99
    idx[7, 0] = -3
    rows = cfg.T * cfg.k
    x_perm = torch.zeros((rows, cfg.d), dtype=cfg.torch_dtype, device="cuda")
    perm_src = torch.full((rows,), -1, dtype=torch.int32, device="cuda")
    inv_row = torch.zeros((cfg.T, cfg.k), dtype=torch.int32, device="cuda")
    B.moe_permute(cfg, inp["x"], idx, got["offsets"], x_perm, perm_src, inv_row, got["ws"])
    assert B.moe_get_device_error(got["ws"]) == B.MOE_ERR_INVALID_ARG   # recorded, then cleared
    assert B.moe_get_device_error(got["ws"]) == B.MOE_OK
    inv = inv_row.cpu().numpy()
    assert inv[5, 1] == -1 and inv[7, 0] == -1
    assert inv.max() < rows


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_corrupt_offsets_are_clamped_and_reported(dtype):
    # expert_offsets from a caller that leave the packed rows (negative, past
    # T*k) or decrease: the expert GEMMs clamp them into [0, T*k], so no tile
    # reads or writes outside x_perm, h or y_perm, and the error word reports
    # the call; the context and the workspace keep working afterwards.
    cfg = MoEConfig(f"bad_offsets_{dtype}", T=200, d=128, E=8, k=2, f=128, dtype=dtype,
                    gate_mode=GATE_SIGMOID, route_scale=2.5, f_shared=64, bias="uniform")
    inp = H.gpu_inputs(cfg)
    got = H.gpu_route(cfg, inp)
    rows = cfg.T * cfg.k
    x_perm = torch.zeros((rows, cfg.d), dtype=cfg.torch_dtype, device="cuda")
    perm_src = torch.empty((rows,), dtype=torch.int32, device="cuda")
    inv_row = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device="cuda")
    B.moe_permute(cfg, inp["x"], got["idx"], got["offsets"], x_perm, perm_src, inv_row, got["ws"])
    assert B.moe_get_device_error(got["ws"]) == B.MOE_OK
    offs = got["offsets"].clone()
    offs[0] = -5
    offs[3] = offs[4] + 7
    offs[cfg.E] = rows + 1000
    y_perm = torch.zeros((rows, cfg.d), dtype=cfg.torch_dtype, device="cuda")
    y_sh = torch.zeros((cfg.T, cfg.d), dtype=cfg.torch_dtype, device="cuda")
    B.moe_expert_swiglu(cfg, x_perm, offs, inp["w1"], inp["w3"], inp["w2"], inp["x"], inp["ws1"], inp["ws3"],
                        inp["ws2"], y_perm, y_sh, got["ws"])
    assert B.moe_get_device_error(got["ws"]) == B.MOE_ERR_INVALID_ARG
    y = H.gpu_forward(cfg, inp, got["ws"])                # same workspace, valid routing: OK again
    H.check_forward(cfg, inp, y)


def test_combine_skips_rows_past_the_packed_rows():
    # moe_combine has no error word: a caller row past T*k is skipped like a
    # missing one (-1), never read.
    cfg = MoEConfig("bad_inv_row", T=64, d=128, E=8, k=2, f=128)
    inp = H.gpu_inputs(cfg)
    got = H.gpu_route(cfg, inp)
    rows = cfg.T * cfg.k
    g = torch.Generator(device="cuda")
    g.manual_seed(4)
    y_perm = torch.randn((rows, cfg.d), generator=g, device="cuda").to(cfg.torch_dtype)
    inv = torch.arange(rows, dtype=torch.int32, device="cuda").reshape(cfg.T, cfg.k)
    bad, skipped = inv.clone(), inv.clone()
    bad[3, 0], skipped[3, 0] = rows + 50, -1
    y_bad = torch.empty((cfg.T, cfg.d), dtype=cfg.torch_dtype, device="cuda")
    y_ref = torch.empty_like(y_bad)
    B.moe_combine(cfg, y_perm, bad, got["gate"], None, y_bad)
    B.moe_combine(cfg, y_perm, skipped, got["gate"], None, y_ref)
    torch.cuda.synchronize()
    assert torch.equal(y_bad, y_ref)


NAN_CASES = {
    "grouped_sigmoid": MoEConfig("nan_grouped", T=70, d=256, E=64, k=6, f=64, gate_mode=GATE_SIGMOID,
                                 n_groups=8, topk_groups=4, route_scale=2.5, bias="uniform"),
    "softmax": MoEConfig("nan_softmax", T=70, d=256, E=16, k=4, f=64),
}


@pytest.mark.parametrize("name", sorted(NAN_CASES))
@pytest.mark.parametrize("bad", ["nan", "inf"])
def test_non_finite_token_gets_valid_expert_ids(name, bad):
    # One token row of NaN (or +inf) scores: its winners must still be k
    # distinct in-range ids in ascending order (no index derived from a NaN
    # comparison may leave [0, E)), counts still add up to T*k, and every
    # other token is routed exactly as without the bad row.
    cfg = NAN_CASES[name]
    inp = H.gpu_inputs(cfg)
    clean = H.gpu_route(cfg, inp)
    inp["x"][5] = float(bad)
    got = H.gpu_route(cfg, inp)
    gi = got["idx"].cpu().numpy()
    assert gi.min() >= 0 and gi.max() < cfg.E
    assert np.all(np.diff(gi, axis=1) > 0)
    assert int(got["counts"].sum().item()) == cfg.T * cfg.k
    c, o = orc.expert_counts_offsets(gi, cfg.E)
    assert np.array_equal(got["counts"].cpu().numpy(), c)
    assert np.array_equal(got["offsets"].cpu().numpy(), o)
    others = np.arange(cfg.T) != 5
    assert np.array_equal(gi[others], clean["idx"].cpu().numpy()[others])
    keep = torch.as_tensor(others, device="cuda")
    assert torch.equal(got["gate"][keep], clean["gate"][keep])
    # The whole block: the bad row stays in its own outputs. Every other
    # token's output is finite and bitwise that of the clean input: the bad
    # token's expert choice moves other tokens to other packed rows, but each
    # output element depends only on its own token's row (no step mixes
    # neighbouring tokens' values, not even in rounding).
    y_bad = H.gpu_forward(cfg, inp)
    x_clean = inp["x"].clone()
    x_clean[5] = H.gpu_inputs(cfg)["x"][5]
    inp["x"] = x_clean
    y_clean = H.gpu_forward(cfg, inp)
    assert torch.isfinite(y_bad[keep].float()).all().item()
    assert torch.equal(y_bad[keep], y_clean[keep])
