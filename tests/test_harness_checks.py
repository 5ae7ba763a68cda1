"""The GPU parity checks themselves, on the CPU: each must reject a planted
error in a stand-in "GPU" result and accept the oracle's own result.

The stand-ins are the oracle's routing and outputs (as CPU tensors, the form
the harness receives from the device) with one mistake planted: a token routed
to another expert, a gate off by more than the tolerance, counts or offsets off
by one, an output element far from the reference, a uniform relative error
above the bound, a NaN row. Near-tie tokens may be routed differently; they are
excluded and counted.
"""
import numpy as np
import pytest
import torch

import gpu_harness as H
import oracle.moe_oracle as orc
from mixture_experts_ffn_sigmoid_b200.inputs import GATE_SIGMOID, MoEConfig

CFG = MoEConfig("harness", T=40, d=16, E=8, k=2, f=12, gate_mode=GATE_SIGMOID, n_groups=4, topk_groups=2,
                route_scale=2.5, bias="uniform")


def _reference(seed=0):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((CFG.T, CFG.d))
    wr = rng.standard_normal((CFG.E, CFG.d)) / 4
    bias = rng.uniform(-0.05, 0.05, CFG.E)
    return orc.route(x, wr, bias, CFG.k, CFG.gate_mode, CFG.n_groups, CFG.topk_groups, CFG.route_scale)


def _as_gpu(ref):
    counts, offsets = orc.expert_counts_offsets(ref["idx"], CFG.E)
    return dict(idx=torch.as_tensor(ref["idx"], dtype=torch.int32),
                gate=torch.as_tensor(ref["gates"], dtype=torch.float32),
                counts=torch.as_tensor(counts, dtype=torch.int32),
                offsets=torch.as_tensor(offsets, dtype=torch.int32))


def test_route_check_accepts_the_oracle_itself():
    ref = _reference()
    rep = H.check_route(CFG, ref, _as_gpu(ref))
    assert rep["gate_err"] < 1e-6


def test_route_check_rejects_a_wrong_expert():
    ref = _reference()
    got = _as_gpu(ref)
    flags = orc.near_tie_tokens(ref, CFG.k, CFG.n_groups, CFG.topk_groups, H.NEAR_TIE_EPS)
    t = int(np.nonzero(~flags)[0][0])
    row = got["idx"][t].clone()
    spare = [e for e in range(CFG.E) if e not in row.tolist()][0]
    row[-1] = spare
    got["idx"][t] = torch.sort(row).values
    got["counts"], got["offsets"] = (torch.as_tensor(a, dtype=torch.int32)
                                     for a in orc.expert_counts_offsets(got["idx"].numpy(), CFG.E))
    with pytest.raises(AssertionError, match="routed differently"):
        H.check_route(CFG, ref, got)


def test_route_check_excludes_and_counts_near_ties():
    # Two experts tied exactly at the k-th place for token 0: the GPU may pick either.
    ref = _reference()
    biased = ref["biased"].copy()
    sel = ref["idx"][0]
    out = [e for e in range(CFG.E) if ref["eligible"][0, e] and e not in sel][0]
    biased[0, out] = biased[0, sel[-1]] if biased[0, sel[-1]] < biased[0, sel[0]] else biased[0, sel[0]]
    r2 = dict(ref, biased=biased)
    flags = orc.near_tie_tokens(r2, CFG.k, CFG.n_groups, CFG.topk_groups, H.NEAR_TIE_EPS)
    assert flags[0]
    got = _as_gpu(ref)
    alt = sorted([int(e) for e in sel if biased[0, e] != biased[0, out]] + [out])
    got["idx"][0] = torch.as_tensor(alt, dtype=torch.int32)
    got["counts"], got["offsets"] = (torch.as_tensor(a, dtype=torch.int32)
                                     for a in orc.expert_counts_offsets(got["idx"].numpy(), CFG.E))
    rep = H.check_route(CFG, r2, got)
    assert rep["near_ties"] >= 1


def test_route_check_rejects_gate_errors_above_the_tolerance():
    ref = _reference()
    got = _as_gpu(ref)
    got["gate"][3, 0] += 10 * H.gate_tol(CFG)
    with pytest.raises(AssertionError, match="gate error"):
        H.check_route(CFG, ref, got)


def test_route_check_rejects_wrong_counts_or_offsets():
    ref = _reference()
    got = _as_gpu(ref)
    got["counts"][2] += 1
    with pytest.raises(AssertionError):
        H.check_route(CFG, ref, got)
    got = _as_gpu(ref)
    got["offsets"][5] += 1
    with pytest.raises(AssertionError):
        H.check_route(CFG, ref, got)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_output_check_bounds(dtype):
    cfg = CFG.with_(dtype=dtype)
    rng = np.random.default_rng(5)
    y_ref = rng.standard_normal((64, 32))
    rms = float(np.sqrt(np.mean(y_ref ** 2)))
    rel_tol, max_tol = H.out_tol(cfg)
    H.compare_outputs(cfg, y_ref.copy(), y_ref)
    # a uniform relative error just inside / well outside the L2 bound
    H.compare_outputs(cfg, y_ref * (1 + 0.5 * rel_tol), y_ref)
    with pytest.raises(AssertionError, match="relative L2"):
        H.compare_outputs(cfg, y_ref * (1 + 3 * rel_tol), y_ref)
    if max_tol is not None:
        # one element far off, the L2 error still small: the elementwise bound
        # (max_tol * RMS + BF16_REL * |ref|) catches it
        y = y_ref.copy()
        y[7, 3] += 2 * (max_tol * rms + H.BF16_REL * abs(y_ref[7, 3]))
        assert np.linalg.norm(y - y_ref) / np.linalg.norm(y_ref) < rel_tol
        with pytest.raises(AssertionError, match="max abs"):
            H.compare_outputs(cfg, y, y_ref)
    y = y_ref.copy()
    y[1] = np.nan
    with pytest.raises(AssertionError):
        H.compare_outputs(cfg, y, y_ref)


def test_gradient_check_bounds():
    from test_gpu_backward import compare_grad
    cfg = CFG.with_(dtype="bf16")
    rng = np.random.default_rng(9)
    g_ref = rng.standard_t(3, size=(48, 40))          # heavy-tailed, like weight gradients
    rms = float(np.sqrt(np.mean(g_ref ** 2)))
    compare_grad(cfg, g_ref.copy(), g_ref, "g")
    # every element off by a quarter of its own bound, in a random direction:
    # inside the elementwise rule and the relative L2 bound
    bound = 5e-2 * rms + 1e-2 * np.abs(g_ref)
    within = g_ref + 0.25 * bound * np.sign(rng.standard_normal(g_ref.shape))
    compare_grad(cfg, within, g_ref, "g")
    # one element beyond its bound
    y = g_ref.copy()
    y[4, 4] += 2 * (5e-2 * rms + 1e-2 * abs(g_ref[4, 4]))
    with pytest.raises(AssertionError, match="elementwise"):
        compare_grad(cfg, y, g_ref, "g")
    # a uniform 3% error: above the relative L2 bound
    with pytest.raises(AssertionError, match="relative L2"):
        compare_grad(cfg, g_ref * 1.03, g_ref, "g")
    # fp32 gradients use the 1e-5 relative L2 bound
    with pytest.raises(AssertionError, match="relative L2"):
        compare_grad(cfg.with_(dtype="f32"), g_ref * (1 + 1e-4), g_ref, "g")
