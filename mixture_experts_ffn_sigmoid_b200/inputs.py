"""Seeded synthetic inputs for the sparse MoE FFN block.

This module is shared by the CUDA path's tests/bench and by the CPU oracle's
tests. It holds the workload table and the random-number recipe only; it
contains none of the block's arithmetic (no routing, no FFN, no combine).

Workloads (shapes follow the pages' description of the block):

* ``tiny_fp32``          T=64, d=128, E=8, k=2, f=256, softmax, fp32 end to end.
* ``mixtral_8x7b``       T=4096, d=4096, E=8, k=2, f=14336, softmax, bf16
                         (Mixtral 8x7B FFN shape, "8 experts, top-2" in the
                         moe-hybrid-architectures cheat sheet, "Models side by side").
* ``deepseek_v3``        T=4096, d=7168, E=256 (+1 shared, f_shared=2048), k=8,
                         f=2048, sigmoid, 8 groups keep 4, route_scale 2.5, bias
                         U(-0.05, 0.05) (ds3-sparse-moe-ffn, "How it works",
                         eq. 12, SwiGLU shapes and "Routing").
* ``decode_fine``        T=32, d=2048, E=128, k=8, f=768, softmax (decode regime:
                         nearly every expert is touched, weights stream from HBM).
* ``deepseek_v3_skewed`` T=16384, DeepSeek-V3 dims, bias +4 on expert 0, +2 on
                         experts 1..7, the rest U(-0.05, 0.05): every token
                         lands on experts 0..7 (stress case for ragged tiles).

Recipe (seed 0 unless told otherwise). One ``torch.Generator`` on the target
device, seeded once, draws in this fixed order: x, w_router, bias, w1, w3, w2,
ws1, ws3, ws2. Expert weights are drawn one expert at a time (``w1[0]``,
``w1[1]``, ...) so that the fp32 staging buffer stays one expert large. Normal
draws are fp32 ``randn`` times the stated standard deviation, then cast to the
workload's dtype; the uniform bias is ``(rand*2-1)*0.05``. x ~ N(0, 1);
w_router, w1, w3, ws1, ws3 ~ N(0, 1/d); w2 ~ N(0, 1/f); ws2 ~ N(0, 1/f_shared).
Bias is fp32 (None for the workloads whose bias is 0). The values differ
between a CPU and a CUDA generator; a parity check always copies the bytes one
side produced to the other side.

Generic (GELU) experts add two fp32 bias stacks, drawn by ``make_expert_biases``
from a second generator seeded with seed + 1000 (so the draws above do not
move): b1 [E][f] then b2 [E][d], both N(0, 0.5^2). The weights of such an
expert are the w1 and w2 drawn above (w3 is unused).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

GATE_SOFTMAX = 0
GATE_SIGMOID = 1


@dataclasses.dataclass(frozen=True)
class MoEConfig:
    name: str
    T: int
    d: int
    E: int
    k: int
    f: int
    dtype: str = "bf16"            # "bf16" or "f32"
    gate_mode: int = GATE_SOFTMAX
    n_groups: int = 1
    topk_groups: int = 1
    route_scale: float = 1.0
    f_shared: int = 0
    bias: str = "zero"             # "zero", "uniform", "skewed"

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    def with_(self, **kw) -> "MoEConfig":
        return dataclasses.replace(self, **kw)

    # Work accounting used by the bench (not by either implementation).
    def active_flops(self) -> float:
        """Router GEMM + (k routed + shared) SwiGLU experts, 2 flops per MAC."""
        routed = self.k * 3 * self.d * self.f
        shared = 3 * self.d * self.f_shared
        return 2.0 * self.T * (self.E * self.d + routed + shared)


CONFIGS = {
    "tiny_fp32": MoEConfig("tiny_fp32", T=64, d=128, E=8, k=2, f=256, dtype="f32"),
    "mixtral_8x7b": MoEConfig("mixtral_8x7b", T=4096, d=4096, E=8, k=2, f=14336),
    "deepseek_v3": MoEConfig("deepseek_v3", T=4096, d=7168, E=256, k=8, f=2048,
                             gate_mode=GATE_SIGMOID, n_groups=8, topk_groups=4,
                             route_scale=2.5, f_shared=2048, bias="uniform"),
    "decode_fine": MoEConfig("decode_fine", T=32, d=2048, E=128, k=8, f=768),
    "deepseek_v3_skewed": MoEConfig("deepseek_v3_skewed", T=16384, d=7168, E=256, k=8,
                                    f=2048, gate_mode=GATE_SIGMOID, n_groups=8,
                                    topk_groups=4, route_scale=2.5, f_shared=2048,
                                    bias="skewed"),
}


def _normal(g: torch.Generator, shape, std: float, dtype, device) -> torch.Tensor:
    t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


def _expert_stack(g, E, rows, cols, std, dtype, device) -> torch.Tensor:
    out = torch.empty((E, rows, cols), dtype=dtype, device=device)
    for e in range(E):
        out[e].copy_(_normal(g, (rows, cols), std, dtype, device))
    return out


def make_inputs(cfg: MoEConfig, device="cpu", seed: int = 0,
                x_only: bool = False) -> dict:
    """Draw every input of one workload on ``device`` with the recipe above.

    Returns a dict with keys x, w_router, bias (fp32 or None), w1, w3, w2 and,
    when ``cfg.f_shared > 0``, ws1, ws3, ws2 (else None).
    """
    device = torch.device(device)
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    dt = cfg.torch_dtype
    out = {}
    out["x"] = _normal(g, (cfg.T, cfg.d), 1.0, dt, device)
    if x_only:
        return out
    out["w_router"] = _normal(g, (cfg.E, cfg.d), 1.0 / math.sqrt(cfg.d), dt, device)
    if cfg.bias == "zero":
        out["bias"] = None
    else:
        b = torch.rand((cfg.E,), generator=g, device=device, dtype=torch.float32)
        b = (b * 2.0 - 1.0) * 0.05
        if cfg.bias == "skewed":
            b[0] = 4.0
            b[1:8] = 2.0
        out["bias"] = b
    sd_in = 1.0 / math.sqrt(cfg.d)
    out["w1"] = _expert_stack(g, cfg.E, cfg.f, cfg.d, sd_in, dt, device)
    out["w3"] = _expert_stack(g, cfg.E, cfg.f, cfg.d, sd_in, dt, device)
    out["w2"] = _expert_stack(g, cfg.E, cfg.d, cfg.f, 1.0 / math.sqrt(cfg.f), dt, device)
    if cfg.f_shared > 0:
        fs = cfg.f_shared
        out["ws1"] = _normal(g, (fs, cfg.d), sd_in, dt, device)
        out["ws3"] = _normal(g, (fs, cfg.d), sd_in, dt, device)
        out["ws2"] = _normal(g, (cfg.d, fs), 1.0 / math.sqrt(fs), dt, device)
    else:
        out["ws1"] = out["ws3"] = out["ws2"] = None
    return out


def make_expert_biases(cfg: MoEConfig, device="cpu", seed: int = 0) -> dict:
    """b1 [E][f] and b2 [E][d], fp32, for generic experts (recipe above)."""
    device = torch.device(device)
    g = torch.Generator(device=device)
    g.manual_seed(seed + 1000)
    return {"b1": _normal(g, (cfg.E, cfg.f), 0.5, torch.float32, device),
            "b2": _normal(g, (cfg.E, cfg.d), 0.5, torch.float32, device)}


def sample_token_ids(T: int, n: int, seed: int = 1) -> torch.Tensor:
    """A seeded, sorted sample of ``n`` distinct token ids in [0, T)."""
    g = torch.Generator()
    g.manual_seed(seed)
    n = min(n, T)
    return torch.randperm(T, generator=g)[:n].sort().values
