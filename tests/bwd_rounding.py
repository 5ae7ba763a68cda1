"""The backward pass with the GPU's bf16 rounding points, in fp64 on the CPU.

Test infrastructure (used by ``test_bwd_rounding_emulation``): a model of
the arithmetic the CUDA backward does in bf16 storage, built from the
oracle's own functions and numpy, so that the elementwise tolerance of the
bf16 gradient checks can be derived from the rounding the kernels are meant
to do rather than chosen by eye. Everything is exact (fp64) except the
values the CUDA path stores in bf16, each rounded here once, at the same
point:

* the pre-activations a = W1 u and b = W3 u of every routed and shared row;
* the scaled hidden g*h and the SwiGLU input gradients da, db;
* the router-logit gradients, before they meet the router weight and x;
* every output gradient (dx, dW_router, dW1, dW3, dW2 and the shared ones).

fp32 accumulation (rounding 2^-24 per term) is modelled as exact; its effect
is far below the bf16 roundings (2^-9).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle.moe_oracle as orc


def bf16(a) -> np.ndarray:
    """Round to bfloat16 (nearest even) and widen back to fp64."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64))
    return t.to(torch.float32).to(torch.bfloat16).to(torch.float64).numpy()


def _swiglu_bwd_rounded(u, w1, w3, w2, dy_rows, g):
    """One expert's rows: returns (dx rows, dW1, dW3, dW2, dgate)."""
    a = bf16(u @ w1.T)
    b = bf16(u @ w3.T)
    dhp = dy_rows @ w2                          # dh' = W2^T dy, gate not applied
    sg = 1.0 / (1.0 + np.exp(-a))
    silu = a * sg
    h = silu * b
    dgate = (dhp * h).sum(axis=1)
    dh = g[:, None] * dhp
    hg = bf16(g[:, None] * h)
    da = bf16(dh * b * sg * (1.0 + a * (1.0 - sg)))
    db = bf16(dh * silu)
    du = da @ w1 + db @ w3
    return du, bf16(da.T @ u), bf16(db.T @ u), bf16(dy_rows.T @ hg), dgate


def moe_backward_bf16_rounding(x, w_router, bias, w1, w3, w2, k, gate_mode, dy, n_groups=1, topk_groups=1,
                               route_scale=1.0, ws1=None, ws3=None, ws2=None, idx=None) -> dict:
    """Gradients as ``orc.moe_backward`` computes them, with the CUDA path's
    bf16 storage roundings applied (inputs must already be bf16 values)."""
    x, dy = np.asarray(x, np.float64), np.asarray(dy, np.float64)
    r = orc.route(x, w_router, bias, k, gate_mode, n_groups, topk_groups, route_scale)
    if idx is not None:
        r["idx"] = np.asarray(idx, dtype=np.int64)
        r["gates"] = orc.gate_values(r["logits"], r["scores"], r["idx"], gate_mode, route_scale)
    idx, gates = r["idx"], r["gates"]
    dx = np.zeros_like(x)
    dgates = np.zeros_like(gates)
    dw1, dw3, dw2 = np.zeros(np.shape(w1)), np.zeros(np.shape(w3)), np.zeros(np.shape(w2))
    for e in np.unique(idx):
        e = int(e)
        tok, slot = np.nonzero(idx == e)
        du, dw1[e], dw3[e], dw2[e], dg = _swiglu_bwd_rounded(x[tok], w1[e], w3[e], w2[e], dy[tok],
                                                             gates[tok, slot])
        dgates[tok, slot] = dg
        np.add.at(dx, tok, du)
    dws1 = dws3 = dws2 = None
    if ws1 is not None:
        du, dws1, dws3, dws2, _ = _swiglu_bwd_rounded(x, ws1, ws3, ws2, dy, np.ones(x.shape[0]))
        dx += du
    dl = bf16(orc.gate_backward(r["logits"], r["scores"], idx, gates, dgates, gate_mode, route_scale))
    dx += dl @ np.asarray(w_router, np.float64)
    return dict(dx=bf16(dx), dw_router=bf16(dl.T @ x), dw1=dw1, dw3=dw3, dw2=dw2, dws1=dws1, dws3=dws3,
                dws2=dws2, idx=idx)
