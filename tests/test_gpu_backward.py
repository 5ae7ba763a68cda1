"""Backward pass on the GPU (moe_backward) against the oracle's chain rule.

The oracle's gradients are pinned to central differences of the forward and
to torch autograd (``oracle_pins``). The GPU recomputes the routing in fp32;
where that choice differs from the oracle's on a near-tie token, the oracle
is evaluated on the GPU's choice (the gradient is defined for a fixed
choice; the choice itself is checked by the routing tests).

Tolerances: fp32 storage, relative L2 <= 1e-5 per gradient tensor. bf16
storage: the pre-activations a, b, the scaled hidden g*h and [da | db] are
each rounded once to bf16 (relative 2^-9) before fp32-accumulated sums over
tokens, and each output is rounded once more. Weight gradients are
heavy-tailed (entries of 10 RMS occur), and the final rounding alone moves
such an entry by up to 2^-9 of itself, so the elementwise bound scales with
the entry as well as with the tensor: |err| <= 5e-2 * RMS + 1e-2 * |ref|,
with relative L2 <= 2e-2 as in the forward. ``test_bwd_rounding_emulation``
applies these exact rounding points on the CPU against the fp64 oracle:
correct bf16 arithmetic reaches ~0.09 RMS at the largest weight-gradient
entries, fails 5e-2 * RMS alone and needs a |ref| coefficient of up to
~7.6e-3 there, so 1e-2 is within 2x of what the rounding requires. A weight
gradient of an expert no token chose must be exactly 0.
"""
import numpy as np
import pytest
import torch

import oracle.moe_oracle as orc
from mixture_experts_ffn_sigmoid_b200 import binding as B
from mixture_experts_ffn_sigmoid_b200.inputs import GATE_SIGMOID, MoEConfig, make_inputs

import gpu_harness as H

pytestmark = pytest.mark.gpu

CASES = {
    "tiny_fp32": MoEConfig("tiny_bwd_f32", T=64, d=128, E=8, k=2, f=256, dtype="f32"),
    "ragged_fp32": MoEConfig("ragged_bwd_f32", T=77, d=200, E=12, k=3, f=72, dtype="f32",
                             gate_mode=GATE_SIGMOID, route_scale=2.5, f_shared=40, bias="uniform"),
    "ragged_bf16": MoEConfig("ragged_bwd", T=77, d=200, E=12, k=3, f=72, gate_mode=GATE_SIGMOID,
                             route_scale=1.0, f_shared=40, bias="uniform"),
    "grouped_bf16": MoEConfig("grouped_bwd", T=300, d=256, E=32, k=4, f=384, gate_mode=GATE_SIGMOID,
                              n_groups=8, topk_groups=4, route_scale=2.5, f_shared=256, bias="uniform"),
    "softmax_bf16": MoEConfig("softmax_bwd", T=200, d=192, E=16, k=2, f=136),
    # ~512 rows per expert: the weight gradients take two 128-row M blocks per tile.
    "long_segments_bf16": MoEConfig("long_bwd", T=1024, d=256, E=4, k=2, f=200, f_shared=64),
}


def _dy(cfg, seed=9):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    return torch.randn((cfg.T, cfg.d), generator=g, device="cuda").to(cfg.torch_dtype)


def gpu_backward(cfg, inp, dy):
    dt, dev = cfg.torch_dtype, "cuda"
    nan = float("nan")
    out = dict(dx=torch.full((cfg.T, cfg.d), nan, dtype=dt, device=dev),
               dw_router=torch.full((cfg.E, cfg.d), nan, dtype=dt, device=dev),
               dw1=torch.full((cfg.E, cfg.f, cfg.d), nan, dtype=dt, device=dev),
               dw3=torch.full((cfg.E, cfg.f, cfg.d), nan, dtype=dt, device=dev),
               dw2=torch.full((cfg.E, cfg.d, cfg.f), nan, dtype=dt, device=dev))
    sh = cfg.f_shared > 0
    out["dws1"] = torch.full((cfg.f_shared, cfg.d), nan, dtype=dt, device=dev) if sh else None
    out["dws3"] = torch.full((cfg.f_shared, cfg.d), nan, dtype=dt, device=dev) if sh else None
    out["dws2"] = torch.full((cfg.d, cfg.f_shared), nan, dtype=dt, device=dev) if sh else None
    ws = B.alloc_backward_workspace(cfg)
    B.moe_backward(cfg, inp["x"], inp["w_router"], inp["bias"], inp["w1"], inp["w3"], inp["w2"], inp["ws1"],
                   inp["ws3"], inp["ws2"], dy, out["dx"], out["dw_router"], out["dw1"], out["dw3"], out["dw2"],
                   out["dws1"], out["dws3"], out["dws2"], ws)
    assert B.moe_get_device_error(ws) == B.MOE_OK
    return out


def oracle_backward(cfg, inp, dy, idx=None):
    return orc.moe_backward(H.f64(inp["x"]), H.f64(inp["w_router"]), H.f64(inp["bias"]), H.f64(inp["w1"]),
                            H.f64(inp["w3"]), H.f64(inp["w2"]), cfg.k, cfg.gate_mode, H.f64(dy), cfg.n_groups,
                            cfg.topk_groups, cfg.route_scale, H.f64(inp["ws1"]), H.f64(inp["ws3"]),
                            H.f64(inp["ws2"]), idx=idx)


@pytest.fixture(scope="module")
def results():
    out = {}
    for name, cfg in CASES.items():
        inp = H.gpu_inputs(cfg)
        dy = _dy(cfg)
        got = gpu_backward(cfg, inp, dy)
        gr = H.gpu_route(cfg, inp)
        rep = H.check_route(cfg, H.oracle_route(cfg, inp), gr)
        ref = oracle_backward(cfg, inp, dy, idx=gr["idx"].cpu().numpy())
        out[name] = (cfg, inp, dy, got, ref, rep)
    return out


NAMES = ["dx", "dw_router", "dw1", "dw3", "dw2", "dws1", "dws3", "dws2"]


@pytest.mark.parametrize("name", sorted(CASES))
@pytest.mark.parametrize("grad", NAMES)
def test_gradient_matches_oracle(results, name, grad):
    cfg, inp, dy, got, ref, rep = results[name]
    if ref[grad] is None:
        assert got[grad] is None
        return
    compare_grad(cfg, H.f64(got[grad]), ref[grad], grad)


def compare_grad(cfg, y, y_ref, what):
    if cfg.dtype == "f32":
        return H.compare_outputs(cfg, y, y_ref, what)
    assert np.all(np.isfinite(y)), f"{what}: non-finite values (unwritten entries?)"
    diff = np.abs(y - y_ref)
    rel = float(np.linalg.norm(diff) / max(np.linalg.norm(y_ref), 1e-300))
    assert rel <= 2e-2, f"{what}: relative L2 error {rel:.3e} > 2e-2"
    rms = float(np.sqrt(np.mean(y_ref ** 2)))
    bound = 5e-2 * rms + 1e-2 * np.abs(y_ref)
    worst = float((diff - bound).max())
    assert worst <= 0.0, f"{what}: elementwise error exceeds 5e-2*RMS + 1e-2*|ref| by {worst:.3e}"
    return dict(rel_l2=rel)


@pytest.mark.parametrize("name", sorted(CASES))
def test_unchosen_experts_get_zero_weight_gradient(results, name):
    cfg, inp, dy, got, ref, rep = results[name]
    chosen = np.zeros(cfg.E, dtype=bool)
    chosen[np.unique(ref["idx"])] = True
    for g in ("dw1", "dw3", "dw2"):
        w = got[g].float()
        for e in np.nonzero(~chosen)[0]:
            assert torch.count_nonzero(w[int(e)]).item() == 0, (g, e)


def test_backward_is_deterministic():
    cfg = CASES["grouped_bf16"]
    inp = H.gpu_inputs(cfg)
    dy = _dy(cfg)
    a = gpu_backward(cfg, inp, dy)
    b = gpu_backward(cfg, inp, dy)
    for n in NAMES:
        if a[n] is not None:
            assert torch.equal(a[n], b[n]), n


def test_backward_empty_tokens():
    cfg = CASES["ragged_bf16"].with_(T=0)
    inp = make_inputs(CASES["ragged_bf16"], "cuda")
    dt = cfg.torch_dtype
    dw = dict(dw_router=torch.full((cfg.E, cfg.d), 1.0, dtype=dt, device="cuda"),
              dw1=torch.full((cfg.E, cfg.f, cfg.d), 1.0, dtype=dt, device="cuda"),
              dw3=torch.full((cfg.E, cfg.f, cfg.d), 1.0, dtype=dt, device="cuda"),
              dw2=torch.full((cfg.E, cfg.d, cfg.f), 1.0, dtype=dt, device="cuda"),
              dws1=torch.full((cfg.f_shared, cfg.d), 1.0, dtype=dt, device="cuda"),
              dws3=torch.full((cfg.f_shared, cfg.d), 1.0, dtype=dt, device="cuda"),
              dws2=torch.full((cfg.d, cfg.f_shared), 1.0, dtype=dt, device="cuda"))
    ws = B.alloc_backward_workspace(cfg)
    B.moe_backward(cfg, None, inp["w_router"], inp["bias"], inp["w1"], inp["w3"], inp["w2"], inp["ws1"],
                   inp["ws3"], inp["ws2"], None, None, dw["dw_router"], dw["dw1"], dw["dw3"], dw["dw2"],
                   dw["dws1"], dw["dws3"], dw["dws2"], ws)
    torch.cuda.synchronize()
    for n, t in dw.items():
        assert torch.count_nonzero(t).item() == 0, n


def test_backward_full_size_sampled():
    # The DeepSeek-V3 workload the bench times, checked on outputs the oracle
    # can compute one at a time:
    #  * dx of sampled tokens: dx_t depends only on token t, so the oracle's
    #    backward over those tokens (on the GPU's expert choice) gives it;
    #  * the full dW1, dW3, dW2 of two experts (most and least loaded): each
    #    depends only on the tokens that chose the expert, their gates and dy;
    #  * rows of the shared expert's dWs1, dWs3 and columns of dWs2 for
    #    sampled inner units: given dy, inner units are independent, so the
    #    gradient of the FFN restricted to those units equals them.
    # The router's weight gradient needs every token's expert outputs; the
    # small cases above check it.
    from mixture_experts_ffn_sigmoid_b200.inputs import CONFIGS, sample_token_ids
    cfg = CONFIGS["deepseek_v3"]
    inp = H.gpu_inputs(cfg)
    dy = _dy(cfg)
    got = gpu_backward(cfg, inp, dy)
    gr = H.gpu_route(cfg, inp)
    ref_route = H.oracle_route(cfg, inp)
    rep = H.check_route(cfg, ref_route, gr)
    gidx = gr["idx"].cpu().numpy().astype(np.int64)
    w1, w3, w2 = H.LazyStack(inp["w1"]), H.LazyStack(inp["w3"]), H.LazyStack(inp["w2"])
    x64, dy64 = H.f64(inp["x"]), H.f64(dy)
    wr, bias = H.f64(inp["w_router"]), H.f64(inp["bias"])
    # dx on sampled tokens
    toks = sample_token_ids(cfg.T, 6).numpy()
    ref = orc.moe_backward(x64[toks], wr, bias, w1, w3, w2, cfg.k, cfg.gate_mode, dy64[toks], cfg.n_groups,
                           cfg.topk_groups, cfg.route_scale, H.f64(inp["ws1"]), H.f64(inp["ws3"]),
                           H.f64(inp["ws2"]), idx=gidx[toks])
    compare_grad(cfg, H.f64(got["dx"])[toks], ref["dx"], "dx (sampled tokens)")
    # whole weight gradients of two experts
    counts = np.bincount(gidx.ravel(), minlength=cfg.E)
    gates = orc.gate_values(ref_route["logits"], ref_route["scores"], gidx, cfg.gate_mode, cfg.route_scale)
    for e in (int(np.argmax(counts)), int(np.argmin(np.where(counts > 0, counts, 1 << 30)))):
        tok, slot = np.nonzero(gidx == e)
        g = gates[tok, slot][:, None]
        _, d1, d3, d2 = orc.swiglu_ffn_backward(x64[tok], w1[e], w3[e], w2[e], g * dy64[tok])
        compare_grad(cfg, H.f64(got["dw1"][e]), d1, f"dw1[{e}]")
        compare_grad(cfg, H.f64(got["dw3"][e]), d3, f"dw3[{e}]")
        compare_grad(cfg, H.f64(got["dw2"][e]), d2, f"dw2[{e}]")
    # sampled inner units of the shared expert
    units = np.sort(np.random.default_rng(3).choice(cfg.f_shared, 16, replace=False))
    ws1, ws3, ws2 = H.f64(inp["ws1"]), H.f64(inp["ws3"]), H.f64(inp["ws2"])
    _, s1, s3, s2 = orc.swiglu_ffn_backward(x64, ws1[units], ws3[units], ws2[:, units], dy64)
    compare_grad(cfg, H.f64(got["dws1"])[units], s1, "dws1 (sampled rows)")
    compare_grad(cfg, H.f64(got["dws3"])[units], s3, "dws3 (sampled rows)")
    compare_grad(cfg, H.f64(got["dws2"])[:, units], s2, "dws2 (sampled columns)")
    for n in NAMES:
        assert torch.isfinite(got[n].float()).all().item(), n


@pytest.mark.parametrize("name", sorted(CASES))
def test_training_forward_then_saved_backward(results, name):
    # moe_forward_train gives moe_forward's bytes, and moe_backward_saved on
    # its workspace gives moe_backward's bytes (same kernels, same operands:
    # the pre-activations come from the gate/up epilogue instead of a
    # recomputing GEMM with the same accumulation order).
    cfg, inp, dy, got, ref, rep = results[name]
    ws = B.alloc_backward_workspace(cfg)
    y = torch.full((cfg.T, cfg.d), float("nan"), dtype=cfg.torch_dtype, device="cuda")
    B.moe_forward_train(cfg, inp["x"], inp["w_router"], inp["bias"], inp["w1"], inp["w3"], inp["w2"], inp["ws1"],
                        inp["ws3"], inp["ws2"], y, ws)
    assert torch.equal(y, H.gpu_forward(cfg, inp))
    dt = cfg.torch_dtype
    out = {n: (torch.full_like(got[n], float("nan")) if got[n] is not None else None) for n in NAMES}
    B.moe_backward_saved(cfg, inp["x"], inp["w_router"], inp["w1"], inp["w3"], inp["w2"], inp["ws1"], inp["ws3"],
                         inp["ws2"], dy, out["dx"], out["dw_router"], out["dw1"], out["dw3"], out["dw2"],
                         out["dws1"], out["dws3"], out["dws2"], ws)
    assert B.moe_get_device_error(ws) == B.MOE_OK
    for n in NAMES:
        if got[n] is not None:
            assert torch.equal(out[n], got[n]), n
