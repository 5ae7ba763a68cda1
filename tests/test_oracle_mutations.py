"""Plant plausible mistakes in the CPU oracle and check the pins catch each.

Every mutation replaces one oracle function (through the module's globals,
so the oracle's own callers see it) with a variant that carries one error:
a dropped term, a wrong sign or index, a transposed or swapped operand, a
missing step. The pins must fail (raise) for every one of them.
"""
import inspect

import numpy as np
import pytest

import oracle.moe_oracle as orc
import oracle_pins

_orig = {name: getattr(orc, name) for name in dir(orc) if callable(getattr(orc, name))}


def _swiglu_swapped(u, w1, w3, w2):
    return _orig["swiglu_ffn"](u, w3, w1, w2)


def _swiglu_no_silu(u, w1, w3, w2):
    u = np.asarray(u, np.float64)
    h = (u @ np.asarray(w1, np.float64).T) * (u @ np.asarray(w3, np.float64).T)
    return h @ np.asarray(w2, np.float64).T


def _swiglu_down_transposed(u, w1, w3, w2):
    return _orig["swiglu_ffn"](u, w1, w3, np.swapaxes(np.asarray(w2), -1, -2))


def _hidden_swapped(u, w1, w3):
    return _orig["swiglu_hidden"](u, w3, w1)


def _silu_dropped_z(z):
    return 1.0 / (1.0 + np.exp(-np.asarray(z, np.float64)))


def _sigmoid_wrong_sign(logits, gate_mode):
    if gate_mode == orc.GATE_SIGMOID:
        return 1.0 / (1.0 + np.exp(np.asarray(logits, np.float64)))
    return _orig["affinity"](logits, gate_mode)


def _router_transposed(x, w_router):
    x = np.asarray(x, np.float64)
    w = np.asarray(w_router, np.float64)
    if w.shape[0] == w.shape[1]:
        return x @ w
    return x @ w.T[:, ::-1]


def _route_gates_use_biased(x, w_router, bias, k, gate_mode, n_groups=1, topk_groups=1,
                            route_scale=1.0):
    r = _orig["route"](x, w_router, bias, k, gate_mode, n_groups, topk_groups, route_scale)
    r["gates"] = _orig["gate_values"](r["biased"], r["biased"], r["idx"], gate_mode, route_scale)
    return r


def _gates_no_renorm(logits, scores, idx, gate_mode, route_scale):
    if gate_mode == orc.GATE_SIGMOID:
        rows = np.arange(idx.shape[0])[:, None]
        return np.asarray(scores, np.float64)[rows, idx] * route_scale
    return _orig["gate_values"](logits, scores, idx, gate_mode, route_scale)


def _gates_no_scale(logits, scores, idx, gate_mode, route_scale):
    return _orig["gate_values"](logits, scores, idx, gate_mode, 1.0)


def _group_max(biased, n_groups):
    b = np.asarray(biased, np.float64)
    T, E = b.shape
    return b.reshape(T, n_groups, E // n_groups).max(axis=2)


def _select_ties_high(biased, eligible, k):
    masked = np.where(eligible, np.asarray(biased, np.float64), -np.inf)
    rev = masked[:, ::-1]
    win = np.argsort(-rev, axis=1, kind="stable")[:, :k]
    return np.sort(masked.shape[1] - 1 - win, axis=1)


def _select_biggest_last(biased, eligible, k):
    masked = np.where(eligible, np.asarray(biased, np.float64), -np.inf)
    win = np.argsort(-masked, axis=1, kind="stable")[:, 1:k + 1]
    return np.sort(win, axis=1)


def _outputs_no_shared(x, idx, gates, w1, w3, w2, ws1=None, ws3=None, ws2=None):
    return _orig["expert_outputs"](x, idx, gates, w1, w3, w2)


def _outputs_with_residual(x, idx, gates, w1, w3, w2, ws1=None, ws3=None, ws2=None):
    return _orig["expert_outputs"](x, idx, gates, w1, w3, w2, ws1, ws3, ws2) + np.asarray(x, np.float64)


def _outputs_slot_swapped(x, idx, gates, w1, w3, w2, ws1=None, ws3=None, ws2=None):
    return _orig["expert_outputs"](x, idx, np.asarray(gates)[:, ::-1], w1, w3, w2, ws1, ws3, ws2)


def _rows_reverse_tokens(idx, offsets):
    inv_row, perm_src = _orig["permutation_rows"](np.asarray(idx)[::-1], offsets)
    return inv_row[::-1], (len(idx) - 1 - perm_src)


def _counts_off_by_one(idx, E):
    counts, offsets = _orig["expert_counts_offsets"](idx, E)
    offsets = offsets.copy()
    offsets[1:-1] += 1
    return counts, offsets


def _near_tie_none(routed, k, n_groups=1, topk_groups=1, eps=1e-5):
    return np.zeros(routed["idx"].shape[0], dtype=bool)


def _loop_no_renorm(x, w_router, w1, w3, w2, k):
    # Dense-loop form that forgets to renormalise the kept probabilities.
    x = np.asarray(x, np.float64)
    lg = _orig["router_logits"](x, w_router)
    p = np.exp(lg - lg.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    idx = np.sort(np.argsort(-p, axis=1, kind="stable")[:, :k], axis=1)
    rows = np.arange(x.shape[0])[:, None]
    return _orig["expert_outputs"](x, idx, p[rows, idx], w1, w3, w2)


def _bias_update_wrong_sign(bias, counts, target, gamma):
    return _orig["update_bias"](bias, counts, target, -gamma)


def _entropy_log2(counts):
    return _orig["routing_entropy"](counts) / np.log(2.0)


def _target_no_k(T, k, E):
    return T / E


def _gelu_tanh(z):
    z = np.asarray(z, np.float64)
    return 0.5 * z * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (z + 0.044715 * z ** 3)))


def _gelu_cdf_only(z):
    return _orig["gelu"](z) / np.where(np.asarray(z, np.float64) == 0, 1.0, np.asarray(z, np.float64))


def _gelu_ffn_b1_outside(u, w1, b1, w2, b2):
    u = np.asarray(u, np.float64)
    h = orc.gelu(u @ np.asarray(w1, np.float64).T) + np.asarray(b1, np.float64)
    return h @ np.asarray(w2, np.float64).T + np.asarray(b2, np.float64)


def _gelu_ffn_no_b2(u, w1, b1, w2, b2):
    return _orig["gelu_ffn"](u, w1, b1, w2, np.zeros_like(np.asarray(b2, np.float64)))


def _gelu_ffn_down_transposed(u, w1, b1, w2, b2):
    return _orig["gelu_ffn"](u, w1, b1, np.swapaxes(np.asarray(w2), -1, -2), b2)


def _gelu_outputs_b2_ungated(x, idx, gates, w1, b1, w2, b2):
    # b2 added once per routed expert instead of scaled by its gate.
    y = _orig["expert_outputs_gelu"](x, idx, gates, w1, b1, w2, np.zeros_like(np.asarray(b2, np.float64)))
    for j in range(np.asarray(idx).shape[1]):
        y = y + np.asarray(b2, np.float64)[np.asarray(idx)[:, j]]
    return y


def _silu_grad_sigma_only(z):
    return 1.0 / (1.0 + np.exp(-np.asarray(z, np.float64)))


def _swiglu_bwd_da_db_swapped(u, w1, w3, w2, dout):
    du, g1, g3, g2 = _orig["swiglu_ffn_backward"](u, w1, w3, w2, dout)
    return du, g3, g1, g2


def _swiglu_bwd_no_up_factor(u, w1, w3, w2, dout):
    # da forgets the multiplier b = W3 u.
    u, w1, w3, w2, dout = (np.asarray(v, np.float64) for v in (u, w1, w3, w2, dout))
    a, b = u @ w1.T, u @ w3.T
    h = orc.silu(a) * b
    dh = dout @ w2
    da = dh * orc.silu_grad(a)
    db = dh * orc.silu(a)
    return da @ w1 + db @ w3, da.T @ u, db.T @ u, dout.T @ h


def _gate_bwd_no_sigmoid_factor(logits, scores, idx, gates, dgates, gate_mode, route_scale):
    dl = _orig["gate_backward"](logits, scores, idx, gates, dgates, gate_mode, route_scale)
    if gate_mode == orc.GATE_SIGMOID:
        s = np.asarray(scores, np.float64)
        with np.errstate(divide="ignore", invalid="ignore"):
            dl = np.where(dl != 0, dl / (s * (1 - s)), 0.0)
    return dl


def _gate_bwd_no_centering(logits, scores, idx, gates, dgates, gate_mode, route_scale):
    T = idx.shape[0]
    rows = np.arange(T)[:, None]
    dl = np.zeros(np.asarray(logits).shape)
    dl[rows, idx] = np.asarray(gates, np.float64) * np.asarray(dgates, np.float64)
    return dl


def _route_groups_from_unbiased(x, w_router, bias, k, gate_mode, n_groups=1, topk_groups=1,
                                route_scale=1.0):
    # Group scores from the unbiased affinities (the bias then moves only the
    # choice inside the kept groups).
    logits = _orig["router_logits"](x, w_router)
    scores = _orig["affinity"](logits, gate_mode)
    biased = _orig["biased_scores"](scores, bias)
    eligible = _orig["group_eligibility"](scores, n_groups, topk_groups)
    idx = _orig["select_experts"](biased, eligible, k)
    gates = _orig["gate_values"](logits, scores, idx, gate_mode, route_scale)
    return dict(idx=idx, gates=gates, logits=logits, scores=scores, biased=biased, eligible=eligible)


def _gate_bwd_no_route_scale(logits, scores, idx, gates, dgates, gate_mode, route_scale):
    if gate_mode == orc.GATE_SIGMOID:
        return _orig["gate_backward"](logits, scores, idx, gates, dgates, gate_mode, 1.0)
    return _orig["gate_backward"](logits, scores, idx, np.asarray(gates, np.float64) / route_scale, dgates,
                                  gate_mode, 1.0)


def _gate_bwd_softmax_over_all(logits, scores, idx, gates, dgates, gate_mode, route_scale):
    # Softmax Jacobian taken over all E logits instead of the k selected ones.
    if gate_mode != orc.GATE_SOFTMAX:
        return _orig["gate_backward"](logits, scores, idx, gates, dgates, gate_mode, route_scale)
    l = np.asarray(logits, np.float64)
    T, k = idx.shape
    rows = np.arange(T)[:, None]
    p_all = np.exp(l - l.max(axis=1, keepdims=True))
    p_all /= p_all.sum(axis=1, keepdims=True)
    dp = np.zeros_like(l)
    dp[rows, idx] = route_scale * np.asarray(dgates, np.float64)
    return p_all * (dp - (p_all * dp).sum(axis=1, keepdims=True))


def _biased_softmax_of_logits(scores, bias):
    # Softmax-mode bias added to softmax probabilities over all experts
    # instead of to the raw logit (sigmoid mode unchanged).
    sc = np.asarray(scores, np.float64)
    if bias is None:
        return sc.copy()
    p = np.exp(sc - sc.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    return p + np.asarray(bias, np.float64)[None, :]


def _gates_sigmoid_over_all(logits, scores, idx, gate_mode, route_scale):
    # Sigmoid gates renormalised over all E scores instead of the k selected.
    if gate_mode != orc.GATE_SIGMOID:
        return _orig["gate_values"](logits, scores, idx, gate_mode, route_scale)
    sc = np.asarray(scores, np.float64)
    rows = np.arange(idx.shape[0])[:, None]
    return sc[rows, idx] / sc.sum(axis=1, keepdims=True) * route_scale


def _near_tie_unbiased(routed, k, n_groups=1, topk_groups=1, eps=1e-5):
    # Gap measured on the unbiased scores instead of the selection scores.
    r = dict(routed)
    r["biased"] = routed["scores"]
    return _orig["near_tie_tokens"](r, k, n_groups, topk_groups, eps)


def _bias_update_proportional(bias, counts, target, gamma):
    # A step proportional to the miss instead of a fixed +-gamma.
    b = np.asarray(bias, np.float64).copy()
    return b - gamma * (np.asarray(counts, np.float64) - target)


def _moe_bwd_no_shared_dx(*a, **kw):
    g = _orig["moe_backward"](*a, **kw)
    bound = inspect.signature(_orig["moe_backward"]).bind(*a, **kw)
    bound.apply_defaults()
    ar = bound.arguments
    if ar["ws1"] is not None:
        du = _orig["swiglu_ffn_backward"](np.asarray(ar["x"], np.float64), ar["ws1"], ar["ws3"], ar["ws2"],
                                          np.asarray(ar["dy"], np.float64))[0]
        g["dx"] = g["dx"] - du
    return g


def _moe_bwd_shared_dw_swapped(*a, **kw):
    g = _orig["moe_backward"](*a, **kw)
    if g["dws1"] is not None:
        g["dws1"], g["dws3"] = g["dws3"], g["dws1"]
    return g


def _rows_slots_swapped(idx, offsets):
    # inv_row of a token's first two slots exchanged (perm_src unchanged).
    inv_row, perm_src = _orig["permutation_rows"](idx, offsets)
    if inv_row.shape[1] >= 2:
        inv_row = inv_row.copy()
        inv_row[:, [0, 1]] = inv_row[:, [1, 0]]
    return inv_row, perm_src


def _group_sum_all(biased, n_groups):
    b = np.asarray(biased, np.float64)
    T, E = b.shape
    return b.reshape(T, n_groups, E // n_groups).sum(axis=2)


def _silu_grad_no_sigma_term(z):
    # The derivative of z * sigma(z) without its first term sigma(z).
    z = np.asarray(z, np.float64)
    sig = 1.0 / (1.0 + np.exp(-z))
    return z * sig * (1.0 - sig)


def _outputs_first_slot_only(x, idx, gates, w1, w3, w2, ws1=None, ws3=None, ws2=None):
    idx = np.asarray(idx)
    return _orig["expert_outputs"](x, idx[:, :1], np.asarray(gates)[:, :1], w1, w3, w2, ws1, ws3, ws2)


def _swiglu_bwd_du_w1_only(u, w1, w3, w2, dout):
    # Input gradient through the W1 branch only (the W3 branch's da/db term dropped).
    du, dw1, dw3, dw2 = _orig["swiglu_ffn_backward"](u, w1, w3, w2, dout)
    u64, w1_, w3_, w2_, d64 = (np.asarray(v, np.float64) for v in (u, w1, w3, w2, dout))
    a = u64 @ w1_.T
    db = (d64 @ w2_) * _orig["silu"](a)
    return du - db @ w3_, dw1, dw3, dw2


def _select_descending(biased, eligible, k):
    # Winners left in descending-score order instead of ascending expert id.
    masked = np.where(eligible, np.asarray(biased, np.float64), -np.inf)
    return np.argsort(-masked, axis=1, kind="stable")[:, :k]


def _affinity_softmax_probs(logits, gate_mode):
    # Softmax mode scores as probabilities over all E instead of raw logits.
    if gate_mode != orc.GATE_SOFTMAX:
        return _orig["affinity"](logits, gate_mode)
    l = np.asarray(logits, np.float64)
    p = np.exp(l - l.max(axis=1, keepdims=True))
    return p / p.sum(axis=1, keepdims=True)


def _rows_slot_major(idx, offsets):
    # Packed rows filled slot by slot (all tokens' slot 0, then slot 1, ...).
    idx = np.asarray(idx)
    T, k = idx.shape
    nxt = np.asarray(offsets[:-1], dtype=np.int64).copy()
    inv_row = np.empty((T, k), dtype=np.int64)
    perm_src = np.full(int(offsets[-1]), -1, dtype=np.int64)
    for j in range(k):
        for t in range(T):
            e = idx[t, j]
            inv_row[t, j] = nxt[e]
            perm_src[nxt[e]] = t
            nxt[e] += 1
    return inv_row, perm_src


def _gelu_erf_without_sqrt2(z):
    from math import erf
    z = np.asarray(z, np.float64)
    return 0.5 * z * (1.0 + np.vectorize(erf)(z))


def _target_integer_division(T, k, E):
    return float((T * k) // E)


def _near_tie_pair_swap_only(routed, k, n_groups=1, topk_groups=1, eps=1e-5):
    # Group boundary checked by exchanging only the last kept and the first
    # dropped group.
    flags = _orig["near_tie_tokens"](routed, k, 1, 1, eps)
    if n_groups > 1 and topk_groups < n_groups:
        biased = routed["biased"]
        T, E = biased.shape
        gscore = orc.group_scores(biased, n_groups)
        order = np.argsort(-gscore, axis=1, kind="stable")
        size = E // n_groups
        for t in range(T):
            last, first_out = order[t, topk_groups - 1], order[t, topk_groups]
            if gscore[t, last] - gscore[t, first_out] >= eps:
                continue
            alt = np.zeros(E, dtype=bool)
            for g in list(order[t, :topk_groups - 1]) + [first_out]:
                alt[g * size:(g + 1) * size] = True
            if not np.array_equal(orc.select_experts(biased[t:t + 1], alt[None, :], k)[0], routed["idx"][t]):
                flags[t] = True
    return flags


def _near_tie_ignores_eligibility(routed, k, n_groups=1, topk_groups=1, eps=1e-5):
    # k-th / (k+1)-th gap taken over all experts, dropped groups included.
    r = dict(routed)
    r["eligible"] = np.ones_like(np.asarray(routed["eligible"]), dtype=bool)
    return _orig["near_tie_tokens"](r, k, n_groups, topk_groups, eps)


def _logits_with_bias_inside(x, w_router):
    # A constant offset folded into the router linear (as if the selection
    # bias were a linear-layer bias): shifts every logit by the same amount.
    return _orig["router_logits"](x, w_router) + 0.1


def _moe_bwd_dgate_with_gate(*a, **kw):
    # dL/dg taken as <dy, g * FFN(x)> instead of <dy, FFN(x)>: the logit
    # gradient is recomputed from the scaled dgates.
    g = _orig["moe_backward"](*a, **kw)
    bound = inspect.signature(_orig["moe_backward"]).bind(*a, **kw)
    bound.apply_defaults()
    ar = bound.arguments
    dg = g["dgates"] * g["gates"]
    r = _orig["route"](ar["x"], ar["w_router"], ar["bias"], ar["k"], ar["gate_mode"], ar["n_groups"],
                       ar["topk_groups"], ar["route_scale"])
    dl = _orig["gate_backward"](r["logits"], r["scores"], g["idx"], g["gates"], dg, ar["gate_mode"],
                                ar["route_scale"])
    x = np.asarray(ar["x"], np.float64)
    w = np.asarray(ar["w_router"], np.float64)
    g["dx"] = g["dx"] - g["dlogits"] @ w + dl @ w
    g["dw_router"] = dl.T @ x
    g["dgates"], g["dlogits"] = dg, dl
    return g


def _rows_first_row_of_expert(idx, offsets):
    # inv_row points at the expert's first packed row for every token.
    inv_row, perm_src = _orig["permutation_rows"](idx, offsets)
    idx = np.asarray(idx)
    return np.asarray(offsets)[idx].astype(np.int64), perm_src


def _hidden_both_gated(u, w1, w3):
    # SiLU applied to both branches.
    u = np.asarray(u, np.float64)
    return _orig["silu"](u @ np.asarray(w1, np.float64).T) * _orig["silu"](u @ np.asarray(w3, np.float64).T)


def _silu_wrong_sign(z):
    z = np.asarray(z, np.float64)
    return z / (1.0 + np.exp(z))


def _groups_keep_one_more(biased, n_groups, topk_groups):
    return _orig["group_eligibility"](biased, n_groups, min(n_groups, topk_groups + 1))


def _moe_bwd_no_router(*a, **kw):
    g = _orig["moe_backward"](*a, **kw)
    x = np.asarray(a[0], np.float64)
    g["dx"] = g["dx"] - g["dlogits"] @ np.asarray(a[1], np.float64)
    g["dw_router"] = np.zeros_like(g["dw_router"])
    return g


MUTATIONS = {
    "bias_update_wrong_sign": ("update_bias", _bias_update_wrong_sign),
    "entropy_in_bits": ("routing_entropy", _entropy_log2),
    "target_without_k": ("balance_target", _target_no_k),
    "swiglu_w1_w3_swapped": ("swiglu_ffn", _swiglu_swapped),
    "swiglu_no_silu": ("swiglu_ffn", _swiglu_no_silu),
    "swiglu_down_transposed": ("swiglu_ffn", _swiglu_down_transposed),
    "silu_drops_z": ("silu", _silu_dropped_z),
    "hidden_w1_w3_swapped": ("swiglu_hidden", _hidden_swapped),
    "sigmoid_wrong_sign": ("affinity", _sigmoid_wrong_sign),
    "router_transposed": ("router_logits", _router_transposed),
    "gates_from_biased": ("route", _route_gates_use_biased),
    "gates_not_renormalised": ("gate_values", _gates_no_renorm),
    "route_scale_dropped": ("gate_values", _gates_no_scale),
    "group_score_max": ("group_scores", _group_max),
    "ties_to_higher_index": ("select_experts", _select_ties_high),
    "topk_off_by_one": ("select_experts", _select_biggest_last),
    "shared_expert_dropped": ("expert_outputs", _outputs_no_shared),
    "residual_added": ("expert_outputs", _outputs_with_residual),
    "gate_slot_mismatch": ("expert_outputs", _outputs_slot_swapped),
    "rows_reverse_token_order": ("permutation_rows", _rows_reverse_tokens),
    "offsets_off_by_one": ("expert_counts_offsets", _counts_off_by_one),
    "near_ties_never_flagged": ("near_tie_tokens", _near_tie_none),
    "dense_loop_no_renorm": ("moe_forward_dense_loop", _loop_no_renorm),
    "gelu_tanh_approximation": ("gelu", _gelu_tanh),
    "gelu_drops_z": ("gelu", _gelu_cdf_only),
    "gelu_b1_outside_phi": ("gelu_ffn", _gelu_ffn_b1_outside),
    "gelu_b2_dropped": ("gelu_ffn", _gelu_ffn_no_b2),
    "gelu_down_transposed": ("gelu_ffn", _gelu_ffn_down_transposed),
    "gelu_b2_not_gated": ("expert_outputs_gelu", _gelu_outputs_b2_ungated),
    "silu_grad_sigma_only": ("silu_grad", _silu_grad_sigma_only),
    "swiglu_bwd_dw1_dw3_swapped": ("swiglu_ffn_backward", _swiglu_bwd_da_db_swapped),
    "swiglu_bwd_no_up_factor": ("swiglu_ffn_backward", _swiglu_bwd_no_up_factor),
    "gate_bwd_no_sigmoid_factor": ("gate_backward", _gate_bwd_no_sigmoid_factor),
    "gate_bwd_no_centering": ("gate_backward", _gate_bwd_no_centering),
    "backward_drops_router": ("moe_backward", _moe_bwd_no_router),
    "group_score_unbiased": ("route", _route_groups_from_unbiased),
    "gate_bwd_no_route_scale": ("gate_backward", _gate_bwd_no_route_scale),
    "gate_bwd_softmax_over_all": ("gate_backward", _gate_bwd_softmax_over_all),
    "softmax_bias_on_probabilities": ("biased_scores", _biased_softmax_of_logits),
    "sigmoid_gates_over_all_experts": ("gate_values", _gates_sigmoid_over_all),
    "near_tie_gap_unbiased": ("near_tie_tokens", _near_tie_unbiased),
    "bias_update_proportional": ("update_bias", _bias_update_proportional),
    "inv_row_slots_swapped": ("permutation_rows", _rows_slots_swapped),
    "silu_grad_no_sigma_term": ("silu_grad", _silu_grad_no_sigma_term),
    "winners_in_score_order": ("select_experts", _select_descending),
    "gelu_erf_without_sqrt2": ("gelu", _gelu_erf_without_sqrt2),
    "near_tie_ignores_group_mask": ("near_tie_tokens", _near_tie_ignores_eligibility),
    "near_tie_group_pair_swap_only": ("near_tie_tokens", _near_tie_pair_swap_only),
    "backward_dgate_includes_gate": ("moe_backward", _moe_bwd_dgate_with_gate),
    "hidden_silu_on_both_branches": ("swiglu_hidden", _hidden_both_gated),
    "silu_wrong_sign": ("silu", _silu_wrong_sign),
    "groups_keep_one_more": ("group_eligibility", _groups_keep_one_more),
    "inv_row_first_row_of_expert": ("permutation_rows", _rows_first_row_of_expert),
    "router_logits_offset": ("router_logits", _logits_with_bias_inside),
    "target_integer_division": ("balance_target", _target_integer_division),
    "softmax_scores_as_probabilities": ("affinity", _affinity_softmax_probs),
    "rows_filled_slot_major": ("permutation_rows", _rows_slot_major),
    "routed_sum_first_slot_only": ("expert_outputs", _outputs_first_slot_only),
    "swiglu_bwd_du_drops_w3_branch": ("swiglu_ffn_backward", _swiglu_bwd_du_w1_only),
    "group_score_sum_of_all": ("group_scores", _group_sum_all),
    "backward_drops_shared_dx": ("moe_backward", _moe_bwd_no_shared_dx),
    "backward_shared_dw1_dw3_swapped": ("moe_backward", _moe_bwd_shared_dw_swapped),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutation_is_caught(name, monkeypatch):
    attr, fn = MUTATIONS[name]
    monkeypatch.setattr(orc, attr, fn)
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin()
        except Exception as exc:  # AssertionError, or a shape error from a transposed operand
            caught.append((pin.__name__, type(exc).__name__))
    assert caught, f"mutation {name} passed every pin"
