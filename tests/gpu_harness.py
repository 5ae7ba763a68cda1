"""Helpers for the GPU parity tests: run the C-ABI entry points on seeded
inputs and compare with the CPU oracle on the same bytes.

Tolerances (written where they are applied):
* routing indices, counts, offsets, permutation rows: bit-exact, except
  tokens the oracle flags as near ties (k-th/(k+1)-th biased-score gap, or a
  group-boundary gap that changes the selection, below 1e-5), which are
  excluded and counted;
* gates: |g - g_ref| <= 2e-5 * max(1, route_scale) for bf16 inputs (fp32
  logits of bf16 products summed over d terms), 1e-6 for fp32 inputs;
* outputs: relative L2 error <= 1e-5 for fp32; for bf16 storage with fp32
  accumulation, relative L2 <= 2e-2 and max-abs <= 5e-2 * RMS(reference).
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle.moe_oracle as orc
from mixture_experts_ffn_sigmoid_b200 import binding as B
from mixture_experts_ffn_sigmoid_b200.inputs import MoEConfig, make_inputs, sample_token_ids

NEAR_TIE_EPS = 1e-5


def f64(t):
    return None if t is None else t.detach().to("cpu").to(torch.float64).numpy()


class LazyStack:
    """expert e's matrix, widened to fp64 on the host only when the oracle asks."""

    def __init__(self, t: torch.Tensor):
        self.t = t

    def __getitem__(self, e):
        return f64(self.t[int(e)])


def gate_tol(cfg: MoEConfig) -> float:
    return 1e-6 if cfg.dtype == "f32" else 2e-5 * max(1.0, cfg.route_scale)


def out_tol(cfg: MoEConfig):
    return (1e-5, None) if cfg.dtype == "f32" else (2e-2, 5e-2)


def gpu_inputs(cfg: MoEConfig, seed: int = 0) -> dict:
    return make_inputs(cfg, "cuda", seed=seed)


def oracle_route(cfg: MoEConfig, inp: dict) -> dict:
    return orc.route(f64(inp["x"]), f64(inp["w_router"]), f64(inp["bias"]), cfg.k, cfg.gate_mode,
                     cfg.n_groups, cfg.topk_groups, cfg.route_scale)


def gpu_route(cfg: MoEConfig, inp: dict, ws=None):
    dev = inp["x"].device
    T, E, k = cfg.T, cfg.E, cfg.k
    idx = torch.full((T, k), -7, dtype=torch.int32, device=dev)
    gate = torch.full((T, k), float("nan"), dtype=torch.float32, device=dev)
    counts = torch.full((E,), -7, dtype=torch.int32, device=dev)
    offsets = torch.full((E + 1,), -7, dtype=torch.int32, device=dev)
    ws = B.alloc_workspace(cfg) if ws is None else ws
    B.moe_route(cfg, inp["x"], inp["w_router"], inp["bias"], idx, gate, counts, offsets, ws)
    assert B.moe_get_device_error(ws) == B.MOE_OK
    return dict(idx=idx, gate=gate, counts=counts, offsets=offsets, ws=ws)


def check_route(cfg: MoEConfig, ref: dict, got: dict) -> dict:
    """Bit-exact routing except near ties; returns a small report."""
    flags = orc.near_tie_tokens(ref, cfg.k, cfg.n_groups, cfg.topk_groups, NEAR_TIE_EPS)
    gi = got["idx"].cpu().numpy().astype(np.int64)
    ok = ~flags
    bad = np.nonzero(np.any(gi[ok] != ref["idx"][ok], axis=1))[0]
    assert bad.size == 0, f"{bad.size} unflagged tokens routed differently, e.g. " \
                          f"{np.nonzero(ok)[0][bad[:3]]}: gpu {gi[ok][bad[:3]]} ref {ref['idx'][ok][bad[:3]]}"
    # Every token got k distinct experts in ascending order.
    assert np.all(np.diff(gi, axis=1) > 0) if cfg.k > 1 else True
    assert gi.min() >= 0 and gi.max() < cfg.E
    gg = got["gate"].cpu().numpy().astype(np.float64)
    err = np.abs(gg[ok] - ref["gates"][ok]).max() if ok.any() else 0.0
    assert err <= gate_tol(cfg), f"gate error {err}"
    # Counts and offsets: exactly those of the GPU's own selection ...
    c_gpu, o_gpu = orc.expert_counts_offsets(gi, cfg.E)
    assert np.array_equal(got["counts"].cpu().numpy(), c_gpu)
    assert np.array_equal(got["offsets"].cpu().numpy(), o_gpu)
    # ... and exactly the oracle's when no token is a near tie.
    if not flags.any():
        c_ref, o_ref = orc.expert_counts_offsets(ref["idx"], cfg.E)
        assert np.array_equal(c_gpu, c_ref) and np.array_equal(o_gpu, o_ref)
    return dict(near_ties=int(flags.sum()), gate_err=float(err), flags=flags)


# Relative part of the bf16 elementwise bound: 2.6x the 2^-8 worst case of one
# round-to-nearest into bf16 (the backward tests use the same form).
BF16_REL = 1e-2


def compare_outputs(cfg: MoEConfig, y: np.ndarray, y_ref: np.ndarray, what: str = "y") -> dict:
    rel_tol, max_tol = out_tol(cfg)
    diff = y.astype(np.float64) - y_ref
    ref_norm = np.linalg.norm(y_ref)
    rel = float(np.linalg.norm(diff) / max(ref_norm, 1e-300))
    rms = float(np.sqrt(np.mean(y_ref ** 2))) if y_ref.size else 0.0
    mx = float(np.abs(diff).max()) if diff.size else 0.0
    assert np.all(np.isfinite(y)), f"{what}: non-finite values (unwritten rows?)"
    assert rel <= rel_tol, f"{what}: relative L2 error {rel:.3e} > {rel_tol}"
    if max_tol is not None:
        # Elementwise: max_tol * RMS for the accumulated error, plus 1e-2 * |ref|
        # for the final rounding to bf16, which moves a stored value by up to
        # 2^-8 of its own magnitude (half an ulp at the bottom of its binade),
        # so large entries carry a proportionally larger error.
        bound = max_tol * rms + BF16_REL * np.abs(y_ref)
        worst = int(np.argmax(np.abs(diff) - bound)) if diff.size else 0
        assert np.all(np.abs(diff) <= bound), (
            f"{what}: max abs error {np.abs(diff).flat[worst]:.3e} at |ref| {np.abs(y_ref).flat[worst]:.3e} > "
            f"{max_tol} * rms {rms:.3e} + {BF16_REL} * |ref|")
    return dict(rel_l2=rel, max_abs=mx, rms=rms)


def weights_f64(inp: dict, lazy: bool):
    if lazy:
        return LazyStack(inp["w1"]), LazyStack(inp["w3"]), LazyStack(inp["w2"])
    return f64(inp["w1"]), f64(inp["w3"]), f64(inp["w2"])


def oracle_outputs(cfg: MoEConfig, inp: dict, ref: dict, tokens: np.ndarray, lazy: bool) -> np.ndarray:
    """The oracle's block output for the given token ids (its own routing)."""
    w1, w3, w2 = weights_f64(inp, lazy)
    x = f64(inp["x"][torch.as_tensor(tokens, device=inp["x"].device)])
    return orc.expert_outputs(x, ref["idx"][tokens], ref["gates"][tokens], w1, w3, w2,
                              f64(inp["ws1"]), f64(inp["ws3"]), f64(inp["ws2"]))


def gpu_forward(cfg: MoEConfig, inp: dict, ws=None):
    y = torch.full((cfg.T, cfg.d), float("nan"), dtype=cfg.torch_dtype, device=inp["x"].device)
    ws = B.alloc_workspace(cfg) if ws is None else ws
    B.moe_forward(cfg, inp["x"], inp["w_router"], inp["bias"], inp["w1"], inp["w3"], inp["w2"],
                  inp["ws1"], inp["ws3"], inp["ws2"], y, ws)
    assert B.moe_get_device_error(ws) == B.MOE_OK
    return y


def check_forward(cfg: MoEConfig, inp: dict, y: torch.Tensor, n_sample=None, lazy=False) -> dict:
    ref = oracle_route(cfg, inp)
    flags = orc.near_tie_tokens(ref, cfg.k, cfg.n_groups, cfg.topk_groups, NEAR_TIE_EPS)
    if n_sample is None or n_sample >= cfg.T:
        tokens = np.arange(cfg.T)
    else:
        tokens = sample_token_ids(cfg.T, n_sample).numpy()
    tokens = tokens[~flags[tokens]]
    y_ref = oracle_outputs(cfg, inp, ref, tokens, lazy)
    y_gpu = f64(y[torch.as_tensor(tokens, device=y.device)])
    rep = compare_outputs(cfg, y_gpu, y_ref)
    rep.update(near_ties=int(flags.sum()), compared=int(tokens.size))
    # Every row of y was written (NaN canary), not only the sampled ones.
    assert torch.isfinite(y.float()).all().item()
    return rep
