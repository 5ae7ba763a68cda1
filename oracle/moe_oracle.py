"""CPU oracle for the sparse Mixture-of-Experts FFN forward pass.

TEST INFRASTRUCTURE ONLY. This module is the plain, slow, fp64 statement of
what the block computes. Only the test suite, ``__graft_entry__.smoke()`` and
the CPU-baseline / reference arm of ``bench.py`` may import it. The product
path (the CUDA library and its Python binding) never imports, calls or links
anything here, and this module imports nothing from the product package.

Sources (web pages, cited by title and section):

* [CS]  "Mixture of Experts and Hybrid Architectures" cheat sheet
        (aiengineeringfromscratch.com), sections "One MoE layer", "The router
        in code", "Troubleshooting", "Aux-loss-free balance loop".
* [KB]  "Mixture of experts and architecture families" knowledge-base page
        (cv-page-czj.pages.dev), section "The router and load balancing".
* [DS]  "Sparse MoE FFN" DeepSeek-V3 study note (ai-engineer-exhaustive),
        section "How it works": eq. 12 (residual form), the SwiGLU equation,
        the "Routing" paragraph and the "Packed forward (official)" paragraph.
* [L2]  "Lesson 2 - From the Dense FFN to a Layer of Experts" (fanfani.net),
        section 1 (dense FFN with phi), section 2 (expert definition and the
        boxed MoE equation) and section 4 (shared experts equation).

Everything is computed in float64 from the exact input values (bf16 inputs
are widened exactly by the caller). No intermediate is rounded. Library
primitives used as single steps: ``numpy`` matmul, ``exp``, stable
``argsort``, ``bincount``, ``cumsum``.

Readings taken where the pages are silent or ambiguous (each one is listed
again in the design notes):

* route_scale multiplies the renormalised gates in both gating modes; the
  softmax workloads use 1.0, so their gates sum to 1 as [CS] states.
* The group score is the sum of the two largest biased scores of the group
  (bias 0 when absent); groups are runs of E/n_groups consecutive experts.
* Every tie (experts or groups) goes to the lower index, as a stable sort on
  the negated score gives ([CS] "The router in code" sorts with a key).
* The k winners are reported in ascending expert id.
* In softmax mode the bias is added to the raw logit; the gates are the
  max-subtracted softmax of the selected raw logits ([CS]). [KB]'s
  softmax-over-all-then-renormalise form is the same number in exact
  arithmetic; ``moe_forward_dense_loop`` restates it and a test checks it.
* Sigmoid mode always renormalises over the winners ([DS] "Routing").
* W1 sits inside SiLU, W3 is the multiplier, W2 projects down ([DS] SwiGLU
  equation); SwiGLU experts carry no bias vectors. The generic experts of
  [L2] section 2 (``gelu_ffn``) carry b1 and b2 and use the exact erf GELU;
  their gate scales the whole expert output, b2 included.
* The block returns shared + routed, without the residual ([DS] eq. 12 and
  the note under it).
"""
from __future__ import annotations

import itertools
import math
from typing import Optional, Sequence

import numpy as np

GATE_SOFTMAX = 0
GATE_SIGMOID = 1

__all__ = [
    "GATE_SOFTMAX", "GATE_SIGMOID", "router_logits", "affinity", "biased_scores",
    "group_scores", "group_eligibility", "select_experts", "gate_values", "route",
    "silu", "swiglu_hidden", "swiglu_ffn", "expert_outputs", "moe_forward", "moe_forward_dense_loop",
    "expert_counts_offsets", "permutation_rows", "near_tie_tokens",
    "balance_target", "update_bias", "routing_entropy",
    "gelu", "gelu_ffn", "expert_outputs_gelu", "moe_forward_gelu",
    "silu_grad", "swiglu_ffn_backward", "gate_backward", "moe_backward",
]


def _f64(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64)


# ---------------------------------------------------------------------------
# Routing
# ---------------------------------------------------------------------------

def router_logits(x, w_router) -> np.ndarray:
    """Router linear layer: ``l[t, e] = u_t . e_e`` for every expert.

    [DS] "Routing": the affinity argument is u_t^T e_i. [CS] "The router in
    code": one dot product of the hidden state with each router row.
    x: (T, d); w_router: (E, d). Returns (T, E).
    """
    return _f64(x) @ _f64(w_router).T


def affinity(logits, gate_mode: int) -> np.ndarray:
    """Token-to-expert affinity.

    Sigmoid mode: s = 1 / (1 + exp(-l))  ([DS] "Routing").
    Softmax mode: the raw logit itself; the softmax is taken over the
    selected experts only, after selection ([CS] "The router in code").
    """
    logits = _f64(logits)
    if gate_mode == GATE_SIGMOID:
        with np.errstate(over="ignore"):
            return 1.0 / (1.0 + np.exp(-logits))
    if gate_mode == GATE_SOFTMAX:
        return logits.copy()
    raise ValueError(f"unknown gate mode {gate_mode}")


def biased_scores(scores, bias) -> np.ndarray:
    """Selection score ``s + b``: the bias moves selection only.

    [CS] "The router in code" (bias added before the sort, gates from the
    unbiased values) and "Troubleshooting" (gate with the raw scores);
    [DS] "Routing" (top-K on s + b_i).
    """
    scores = _f64(scores)
    if bias is None:
        return scores.copy()
    return scores + _f64(bias)[None, :]


def group_scores(biased, n_groups: int) -> np.ndarray:
    """Score of each expert group: the sum of its two largest biased scores.

    [DS] "Routing": 8 groups, keep 4, group score = sum of top-2.
    Group G holds experts [G*E/n_groups, (G+1)*E/n_groups). Returns (T, n_groups).
    """
    biased = _f64(biased)
    T, E = biased.shape
    size = E // n_groups
    per_group = biased.reshape(T, n_groups, size)
    two_largest = np.sort(per_group, axis=2)[:, :, -2:]
    return two_largest.sum(axis=2)


def _kept_groups(gscore, topk_groups: int) -> np.ndarray:
    """Indices of the best ``topk_groups`` groups per token, ties to lower index."""
    order = np.argsort(-gscore, axis=1, kind="stable")
    return order[:, :topk_groups]


def group_eligibility(biased, n_groups: int, topk_groups: int) -> np.ndarray:
    """Boolean (T, E) mask of experts that sit in a kept group.

    With ``n_groups <= 1`` every expert is eligible (plain top-k).
    """
    biased = _f64(biased)
    T, E = biased.shape
    if n_groups <= 1:
        return np.ones((T, E), dtype=bool)
    keep = np.zeros((T, n_groups), dtype=bool)
    kept = _kept_groups(group_scores(biased, n_groups), topk_groups)
    keep[np.arange(T)[:, None], kept] = True
    return np.repeat(keep, E // n_groups, axis=1)


def select_experts(biased, eligible, k: int) -> np.ndarray:
    """Top-k of the biased scores among eligible experts, ascending expert id.

    A stable sort of the negated scores puts equal scores in index order, so a
    tie goes to the lower expert index. Returns int64 (T, k).
    """
    masked = np.where(eligible, _f64(biased), -np.inf)
    winners = np.argsort(-masked, axis=1, kind="stable")[:, :k]
    return np.sort(winners, axis=1)


def gate_values(logits, scores, idx, gate_mode: int, route_scale: float) -> np.ndarray:
    """Gate weight of each selected expert, from the UNBIASED values.

    Softmax: exp(l_i - max) / sum over the k selected raw logits
    ([CS] "The router in code": softmax over the chosen original scores).
    Sigmoid: s_i / sum of the k selected s ([DS] "Routing": renormalised
    over the K_r winners). Both are then multiplied by ``route_scale``
    ([DS] "Routing": route_scale = 2.5). Returns (T, k).
    """
    rows = np.arange(idx.shape[0])[:, None]
    if gate_mode == GATE_SOFTMAX:
        chosen = _f64(logits)[rows, idx]
        top = chosen.max(axis=1, keepdims=True)
        ex = np.exp(chosen - top)
        g = ex / ex.sum(axis=1, keepdims=True)
    elif gate_mode == GATE_SIGMOID:
        chosen = _f64(scores)[rows, idx]
        g = chosen / chosen.sum(axis=1, keepdims=True)
    else:
        raise ValueError(f"unknown gate mode {gate_mode}")
    return g * float(route_scale)


def route(x, w_router, bias, k: int, gate_mode: int, n_groups: int = 1,
          topk_groups: int = 1, route_scale: float = 1.0) -> dict:
    """The whole gate: logits, affinity, biased group-limited top-k, gates.

    Returns a dict with ``idx`` (T, k) ascending expert ids, ``gates`` (T, k),
    and the intermediates ``logits``, ``scores``, ``biased``, ``eligible``.
    """
    logits = router_logits(x, w_router)
    scores = affinity(logits, gate_mode)
    biased = biased_scores(scores, bias)
    eligible = group_eligibility(biased, n_groups, topk_groups)
    idx = select_experts(biased, eligible, k)
    gates = gate_values(logits, scores, idx, gate_mode, route_scale)
    return dict(idx=idx, gates=gates, logits=logits, scores=scores,
                biased=biased, eligible=eligible)


# ---------------------------------------------------------------------------
# Experts
# ---------------------------------------------------------------------------

def silu(z) -> np.ndarray:
    """SiLU(z) = z * sigmoid(z)."""
    z = _f64(z)
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def swiglu_hidden(u, w1, w3) -> np.ndarray:
    """The SwiGLU inner activation SiLU(W1 u) * W3 u, row-wise over u.

    [DS] SwiGLU equation: W1, W3 in R^{f x d}. u: (n, d). Returns (n, f).
    """
    u = _f64(u)
    return silu(u @ _f64(w1).T) * (u @ _f64(w3).T)


def swiglu_ffn(u, w1, w3, w2) -> np.ndarray:
    """FFN(u) = W2 (SiLU(W1 u) * W3 u), row-wise over u.

    [DS] SwiGLU equation: W2 in R^{d x f}. u: (n, d). Returns (n, d).
    """
    return swiglu_hidden(u, w1, w3) @ _f64(w2).T


def expert_outputs(x, idx, gates, w1, w3, w2, ws1=None, ws3=None, ws2=None) -> np.ndarray:
    """Routed sum plus shared expert, per the packed forward.

    [DS] "Packed forward (official)": for each expert, gather the tokens that
    chose it, run the SwiGLU, scale by the matching gate and scatter-add into
    a zero buffer; then add the shared FFN over all tokens; no residual
    ([DS] eq. 12 and the note under it). [L2] section 4 gives the same sum:
    shared experts with unit weight plus gated routed experts.

    ``w1``/``w3``/``w2`` may be any object whose ``[e]`` gives expert e's
    matrix (an array stack, or a lazy loader for large workloads).
    """
    x = _f64(x)
    T = x.shape[0]
    idx = np.asarray(idx)
    gates = _f64(gates)
    y = np.zeros_like(x)
    for e in np.unique(idx):
        tok, slot = np.nonzero(idx == e)
        out = swiglu_ffn(x[tok], w1[e], w3[e], w2[e])
        np.add.at(y, tok, gates[tok, slot][:, None] * out)
    if ws1 is not None:
        y += swiglu_ffn(x, ws1, ws3, ws2)
    return y


def moe_forward(x, w_router, bias, w1, w3, w2, k: int, gate_mode: int,
                n_groups: int = 1, topk_groups: int = 1, route_scale: float = 1.0,
                ws1=None, ws3=None, ws2=None) -> np.ndarray:
    """MoE(u) = sum_shared FFN_s(u) + sum_{i in TopK} g_i FFN_i(u).

    [DS] eq. 12 without the u_t skip term; [L2] section 4 shared-expert form.
    """
    r = route(x, w_router, bias, k, gate_mode, n_groups, topk_groups, route_scale)
    return expert_outputs(x, r["idx"], r["gates"], w1, w3, w2, ws1, ws3, ws2)


def moe_forward_dense_loop(x, w_router, w1, w3, w2, k: int) -> np.ndarray:
    """The per-expert loop form with softmax over ALL experts, then renormalise.

    [KB] "The router and load balancing": probabilities from a softmax over
    all E logits, keep the k largest, divide by their sum, then visit each
    expert in turn and add its weighted output to the tokens that chose it.
    No bias, no groups, no shared expert (the page's form has none).
    """
    x = _f64(x)
    logits = router_logits(x, w_router)
    shifted = logits - logits.max(axis=1, keepdims=True)
    p = np.exp(shifted)
    p /= p.sum(axis=1, keepdims=True)
    T, E = p.shape
    chosen = np.argsort(-p, axis=1, kind="stable")[:, :k]
    weight = np.zeros((T, E))
    rows = np.arange(T)[:, None]
    weight[rows, chosen] = p[rows, chosen]
    weight /= weight.sum(axis=1, keepdims=True)
    out = np.zeros_like(x)
    for e in range(E):
        tok = np.nonzero(weight[:, e] > 0)[0]
        if tok.size == 0:
            continue
        out[tok] += weight[tok, e][:, None] * swiglu_ffn(x[tok], w1[e], w3[e], w2[e])
    return out


# ---------------------------------------------------------------------------
# Packing: counts, offsets, permutation
# ---------------------------------------------------------------------------

def expert_counts_offsets(idx, E: int):
    """counts[e] = #tokens that chose e; offsets = exclusive prefix sum (E+1).

    The packed forward gathers, per expert, the tokens whose indices equal it
    ([DS] "Packed forward"); laying those groups end to end in expert order
    gives these offsets.
    """
    counts = np.bincount(np.asarray(idx).ravel(), minlength=E).astype(np.int64)
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    return counts, offsets


def permutation_rows(idx, offsets):
    """Packed row of every (token, slot) pair, tokens in index order per expert.

    row(t, j) = offsets[e] + #{t' < t : e in sel(t')} with e = idx[t, j].
    Returns (inv_row (T, k), perm_src (T*k,)): ``perm_src[inv_row[t, j]] == t``.
    """
    idx = np.asarray(idx)
    T, k = idx.shape
    next_free = np.asarray(offsets[:-1], dtype=np.int64).copy()
    inv_row = np.empty((T, k), dtype=np.int64)
    perm_src = np.full(int(offsets[-1]), -1, dtype=np.int64)
    for t in range(T):
        for j in range(k):
            e = idx[t, j]
            inv_row[t, j] = next_free[e]
            perm_src[next_free[e]] = t
            next_free[e] += 1
    return inv_row, perm_src


# ---------------------------------------------------------------------------
# Near ties (which tokens a finite-precision router may legitimately route
# differently from this fp64 statement)
# ---------------------------------------------------------------------------

def near_tie_tokens(routed: dict, k: int, n_groups: int = 1, topk_groups: int = 1,
                    eps: float = 1e-5) -> np.ndarray:
    """Boolean (T,) flags for tokens whose selection rests on a gap below eps.

    A token is flagged when the k-th and (k+1)-th largest eligible biased
    scores differ by less than ``eps``, or, with group-limited routing, when
    the group ranking is ambiguous at its boundary and that can change the
    selected set: the near groups are the kept ones less than ``eps`` above
    the first dropped score and the dropped ones less than ``eps`` below the
    last kept score; every way of filling the kept places those near groups
    compete for is tried, and the token is flagged if any of them selects a
    different set of experts.
    """
    biased = routed["biased"]
    eligible = routed["eligible"]
    T, E = biased.shape
    flags = np.zeros(T, dtype=bool)
    masked = np.where(eligible, biased, -np.inf)
    srt = -np.sort(-masked, axis=1)
    n_elig = eligible.sum(axis=1)
    for t in range(T):
        if k < n_elig[t] and srt[t, k - 1] - srt[t, k] < eps:
            flags[t] = True
    if n_groups > 1 and topk_groups < n_groups:
        gscore = group_scores(biased, n_groups)
        order = np.argsort(-gscore, axis=1, kind="stable")
        size = E // n_groups
        for t in range(T):
            kept, dropped = list(order[t, :topk_groups]), list(order[t, topk_groups:])
            hi, lo = gscore[t, kept[-1]], gscore[t, dropped[0]]
            if hi - lo >= eps:
                continue
            near = [g for g in kept if gscore[t, g] - lo < eps] + \
                   [g for g in dropped if hi - gscore[t, g] < eps]
            sure = [g for g in kept if g not in near]
            for pick in itertools.combinations(near, topk_groups - len(sure)):
                alt = np.zeros(E, dtype=bool)
                for g in sure + list(pick):
                    alt[g * size:(g + 1) * size] = True
                alt_sel = select_experts(biased[t:t + 1], alt[None, :], k)[0]
                if not np.array_equal(alt_sel, routed["idx"][t]):
                    flags[t] = True
                    break
    return flags


# ---------------------------------------------------------------------------
# Aux-loss-free load balancing (the step that follows routing in training)
# ---------------------------------------------------------------------------

def balance_target(T: int, k: int, E: int) -> float:
    """Per-expert target usage: n_tokens * top_k / n_experts.

    [CS] "Aux-loss-free balance loop", step 1.
    """
    return T * k / E


def update_bias(bias, counts, target: float, gamma: float) -> np.ndarray:
    """One bias update: experts over target lose gamma, experts under gain it.

    [CS] "Aux-loss-free balance loop", step 5 (over target: bias -= gamma;
    under target: bias += gamma). An expert exactly on target keeps its bias
    (the page names only the two strict cases).
    """
    bias = _f64(bias).copy()
    counts = np.asarray(counts, dtype=np.float64)
    bias[counts > target] -= gamma
    bias[counts < target] += gamma
    return bias


def routing_entropy(counts) -> float:
    """Shannon entropy (nats) of the expert-usage distribution counts / sum.

    [CS] "Aux-loss-free balance loop", step 7: it rises toward ln(n_experts),
    the value for uniform usage. Experts with zero count contribute 0.
    """
    c = np.asarray(counts, dtype=np.float64)
    total = c.sum()
    if total <= 0:
        return 0.0
    p = c[c > 0] / total
    return float(-(p * np.log(p)).sum())


# ---------------------------------------------------------------------------
# Generic experts: bias vectors and a GELU nonlinearity
# ---------------------------------------------------------------------------

def gelu(z) -> np.ndarray:
    """GELU(z) = z * Phi(z), Phi the standard normal CDF = (1 + erf(z/sqrt 2))/2.

    [L2] section 1 names GELU as the FFN nonlinearity phi without fixing a
    form; this is the exact (erf) definition, not the tanh approximation.
    ``math.erf`` is the library primitive, applied element by element.
    """
    z = _f64(z)
    erf = np.vectorize(math.erf, otypes=[np.float64])
    return 0.5 * z * (1.0 + erf(z / math.sqrt(2.0)))


def gelu_ffn(u, w1, b1, w2, b2) -> np.ndarray:
    """E_i(u) = W2 phi(W1 u + b1) + b2 with phi = GELU, row-wise over u.

    [L2] section 2, the expert definition: W1 in R^{f x d}, b1 in R^f,
    W2 in R^{d x f}, b2 in R^d. u: (n, d). Returns (n, d).
    """
    u = _f64(u)
    return gelu(u @ _f64(w1).T + _f64(b1)) @ _f64(w2).T + _f64(b2)


def expert_outputs_gelu(x, idx, gates, w1, b1, w2, b2) -> np.ndarray:
    """MoE(x) = sum_{i in TopK(x)} g_i(x) E_i(x) with GELU experts.

    [L2] section 2, boxed equation: the gate multiplies the whole expert
    output, b2 included. No shared expert (the boxed form has none).
    ``w1[e]`` etc. give expert e's parameters.
    """
    x = _f64(x)
    idx = np.asarray(idx)
    gates = _f64(gates)
    y = np.zeros_like(x)
    for e in np.unique(idx):
        tok, slot = np.nonzero(idx == e)
        out = gelu_ffn(x[tok], w1[e], b1[e], w2[e], b2[e])
        np.add.at(y, tok, gates[tok, slot][:, None] * out)
    return y


def moe_forward_gelu(x, w_router, bias, w1, b1, w2, b2, k: int, gate_mode: int,
                     n_groups: int = 1, topk_groups: int = 1, route_scale: float = 1.0) -> np.ndarray:
    """Routing as in ``route`` followed by gated GELU experts ([L2] section 2)."""
    r = route(x, w_router, bias, k, gate_mode, n_groups, topk_groups, route_scale)
    return expert_outputs_gelu(x, r["idx"], r["gates"], w1, b1, w2, b2)


# ---------------------------------------------------------------------------
# Backward pass of the block (training). The expert choice is piecewise
# constant in the inputs, so gradients flow through the gates and the expert
# FFNs only; the selection bias receives none (it is moved by the balance
# step above, not by gradients: [CS] "Aux-loss-free balance loop").
# ---------------------------------------------------------------------------

def silu_grad(z) -> np.ndarray:
    """d/dz [z sigma(z)] = sigma(z) (1 + z (1 - sigma(z)))."""
    z = _f64(z)
    with np.errstate(over="ignore"):
        sig = 1.0 / (1.0 + np.exp(-z))
    return sig * (1.0 + z * (1.0 - sig))


def swiglu_ffn_backward(u, w1, w3, w2, dout):
    """Gradients of FFN(u) = W2 (SiLU(W1 u) * W3 u) for a batch of rows u.

    dout: (n, d), the gradient of the loss with respect to FFN(u).
    Returns (du (n, d), dw1 (f, d), dw3 (f, d), dw2 (d, f)).
    Chain rule through [DS]'s SwiGLU equation: a = W1 u, b = W3 u,
    h = SiLU(a) * b, out = W2 h.
    """
    u, w1, w3, w2, dout = (_f64(v) for v in (u, w1, w3, w2, dout))
    a = u @ w1.T
    b = u @ w3.T
    h = silu(a) * b
    dw2 = dout.T @ h
    dh = dout @ w2
    da = dh * b * silu_grad(a)
    db = dh * silu(a)
    du = da @ w1 + db @ w3
    return du, da.T @ u, db.T @ u, dw2


def gate_backward(logits, scores, idx, gates, dgates, gate_mode: int, route_scale: float) -> np.ndarray:
    """Gradient of the loss with respect to the router logits (T, E), given
    the gradient with respect to the k gates of every token.

    Sigmoid ([DS] "Routing"): g_j = rs * s_j / S with S the sum of the k
    selected s, s = sigmoid(l): dL/ds_j = rs * (dg_j / S - sum_i dg_i s_i / S^2),
    dL/dl_j = dL/ds_j * s_j (1 - s_j).
    Softmax ([CS] "The router in code"): g_j = rs * p_j, p = softmax over the
    k selected logits: dL/dl_j = rs * p_j (dg_j - sum_i p_i dg_i).
    Experts that were not selected get 0.
    """
    T, k = idx.shape
    E = _f64(logits).shape[1]
    rows = np.arange(T)[:, None]
    dg = _f64(dgates)
    dl = np.zeros((T, E))
    rs = float(route_scale)
    if gate_mode == GATE_SIGMOID:
        s = _f64(scores)[rows, idx]
        S = s.sum(axis=1, keepdims=True)
        ds = rs * (dg / S - (dg * s).sum(axis=1, keepdims=True) / S ** 2)
        dl[rows, idx] = ds * s * (1.0 - s)
    elif gate_mode == GATE_SOFTMAX:
        p = _f64(gates) / rs
        dl[rows, idx] = rs * p * (dg - (p * dg).sum(axis=1, keepdims=True))
    else:
        raise ValueError(f"unknown gate mode {gate_mode}")
    return dl


def moe_backward(x, w_router, bias, w1, w3, w2, k: int, gate_mode: int, dy,
                 n_groups: int = 1, topk_groups: int = 1, route_scale: float = 1.0,
                 ws1=None, ws3=None, ws2=None, idx=None) -> dict:
    """Gradients of <dy, MoE(x)> with respect to x and every weight.

    The forward is ``moe_forward``: y_t = sum_j g_tj FFN_{e_tj}(x_t) + FFN_s(x_t).
    Per token and slot: dL/dg_tj = <dy_t, FFN_{e_tj}(x_t)>, and the expert
    sees dout = g_tj dy_t. The router adds dL/dl @ w_router to dx and
    dL/dl^T x to its weight. Returns a dict with dx, dw_router, dw1, dw3, dw2
    (stacked per expert; zero for unchosen experts), dws1, dws3, dws2 (None
    without a shared expert), and the intermediates dgates, dlogits, idx, gates.

    ``idx`` (T, k), when given, fixes the expert choice (ascending ids per
    token) instead of this routing's own; the gates are then those of that
    choice. The gradient is defined for a fixed choice, so a caller whose
    selection differs only on near-tie tokens can compare against it.
    """
    x = _f64(x)
    dy = _f64(dy)
    r = route(x, w_router, bias, k, gate_mode, n_groups, topk_groups, route_scale)
    if idx is not None:
        r["idx"] = np.asarray(idx, dtype=np.int64)
        r["gates"] = gate_values(r["logits"], r["scores"], r["idx"], gate_mode, route_scale)
    idx, gates = r["idx"], r["gates"]
    dx = np.zeros_like(x)
    dgates = np.zeros_like(gates)
    # Expert matrices are read one expert at a time (w1[e]), so a caller may
    # pass lazily widened stacks; the weight gradients of chosen experts are
    # collected per expert and stacked (zeros elsewhere) for array inputs.
    g1s, g3s, g2s = {}, {}, {}
    for e in np.unique(idx):
        e = int(e)
        tok, slot = np.nonzero(idx == e)
        w1e, w3e, w2e = _f64(w1[e]), _f64(w3[e]), _f64(w2[e])
        out = swiglu_ffn(x[tok], w1e, w3e, w2e)
        dgates[tok, slot] = (dy[tok] * out).sum(axis=1)
        g = gates[tok, slot][:, None]
        du, g1s[e], g3s[e], g2s[e] = swiglu_ffn_backward(x[tok], w1e, w3e, w2e, g * dy[tok])
        np.add.at(dx, tok, du)
    if isinstance(w1, np.ndarray):
        dw1, dw3, dw2 = np.zeros(w1.shape), np.zeros(w3.shape), np.zeros(w2.shape)
        for e in g1s:
            dw1[e], dw3[e], dw2[e] = g1s[e], g3s[e], g2s[e]
    else:
        dw1, dw3, dw2 = g1s, g3s, g2s
    dws1 = dws3 = dws2 = None
    if ws1 is not None:
        du, dws1, dws3, dws2 = swiglu_ffn_backward(x, ws1, ws3, ws2, dy)
        dx += du
    dlogits = gate_backward(r["logits"], r["scores"], idx, gates, dgates, gate_mode, route_scale)
    dx += dlogits @ _f64(w_router)
    dw_router = dlogits.T @ x
    return dict(dx=dx, dw_router=dw_router, dw1=dw1, dw3=dw3, dw2=dw2, dws1=dws1, dws3=dws3,
                dws2=dws2, dgates=dgates, dlogits=dlogits, idx=idx, gates=gates)
