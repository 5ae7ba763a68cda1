"""Pins of the CPU oracle to facts outside itself.

Each ``pin_*`` function raises AssertionError when the oracle disagrees with a
closed form, a hand-worked case, an invariant stated on the pages, a brute
force search, or an independent library routine. ``test_oracle_pins.py`` runs
them; ``test_oracle_mutations.py`` plants mistakes in the oracle and checks
that at least one pin catches each.

The hand cases use d = E = f = 2, an identity router and identity expert
matrices (expert 1's down projection doubled), so every value has a closed
form in the logistic function: SiLU(u) * u = u^2 * sigma(u) per coordinate,
and a 2-way softmax is sigma of the logit difference.
"""
from __future__ import annotations

import itertools
import math

import numpy as np
import torch

import oracle.moe_oracle as orc


def sigma(z: float) -> float:
    return 1.0 / (1.0 + math.exp(-z))


def _close(a, b, tol=1e-12):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, (a.shape, b.shape)
    err = np.max(np.abs(a - b)) if a.size else 0.0
    assert err <= tol * max(1.0, float(np.max(np.abs(b))) if b.size else 1.0), (a, b, err)


# ---------------------------------------------------------------- hand cases
HAND_X = np.array([[1.0, 0.0], [0.0, 1.0], [2.0, -1.0]])
HAND_WR = np.eye(2)
HAND_W1 = np.stack([np.eye(2), np.eye(2)])
HAND_W3 = np.stack([np.eye(2), np.eye(2)])
HAND_W2 = np.stack([np.eye(2), 2.0 * np.eye(2)])


def _ffn_closed(u, scale):
    """Identity-weight SwiGLU: scale * u^2 * sigma(u), per coordinate."""
    return np.array([scale * v * v * sigma(v) for v in u])


def _hand(k, gate_mode, bias, route_scale):
    r = orc.route(HAND_X, HAND_WR, bias, k, gate_mode, route_scale=route_scale)
    y = orc.moe_forward(HAND_X, HAND_WR, bias, HAND_W1, HAND_W3, HAND_W2, k, gate_mode,
                        route_scale=route_scale)
    return r, y


def pin_hand_softmax_k1():
    r, y = _hand(1, orc.GATE_SOFTMAX, None, 1.0)
    assert r["idx"].ravel().tolist() == [0, 1, 0]
    _close(r["gates"], np.ones((3, 1)))
    _close(y[0], _ffn_closed(HAND_X[0], 1.0))
    _close(y[1], _ffn_closed(HAND_X[1], 2.0))
    _close(y[2], _ffn_closed(HAND_X[2], 1.0))
    _close(y[0], [0.731059, 0.0], tol=1e-6)
    _close(y[2], [3.523188, 0.268941], tol=1e-6)


def pin_hand_softmax_k2():
    r, y = _hand(2, orc.GATE_SOFTMAX, None, 1.0)
    assert r["idx"].tolist() == [[0, 1]] * 3
    for t, u in enumerate(HAND_X):
        g0 = sigma(u[0] - u[1])            # two-way softmax of logits (u0, u1)
        _close(r["gates"][t], [g0, 1.0 - g0])
        _close(y[t], _ffn_closed(u, g0 * 1.0 + (1.0 - g0) * 2.0))
    _close(y[0], [0.927671, 0.0], tol=1e-6)
    _close(y[1], [0.0, 1.265505], tol=1e-6)


def pin_hand_sigmoid_bias_moves_selection():
    # Without bias token 0 picks expert 0 (sigma(1) > sigma(0)); a +0.3 bias on
    # expert 1 lifts sigma(0) + 0.3 = 0.8 above sigma(1) = 0.731: selection flips,
    # the single gate is still route_scale (renormalised over one winner).
    r0, y0 = _hand(1, orc.GATE_SIGMOID, np.array([0.0, 0.0]), 2.5)
    r1, y1 = _hand(1, orc.GATE_SIGMOID, np.array([0.0, 0.3]), 2.5)
    assert r0["idx"].ravel().tolist() == [0, 1, 0]
    assert r1["idx"].ravel().tolist() == [1, 1, 0]
    _close(r1["gates"], np.full((3, 1), 2.5))
    _close(y0[0], _ffn_closed(HAND_X[0], 2.5 * 1.0))
    _close(y1[0], _ffn_closed(HAND_X[0], 2.5 * 2.0))
    _close(y1[0], [3.655293, 0.0], tol=1e-6)
    _close(y1[2], [8.807971, 0.672354], tol=1e-6)


def pin_hand_sigmoid_k2_gates_ignore_bias():
    # k = E: both experts always win; the gates come from the raw sigmoid and
    # must not move with the bias.
    ra, ya = _hand(2, orc.GATE_SIGMOID, np.array([0.0, 0.0]), 2.5)
    rb, yb = _hand(2, orc.GATE_SIGMOID, np.array([0.0, 0.3]), 2.5)
    for t, u in enumerate(HAND_X):
        s0, s1 = sigma(u[0]), sigma(u[1])
        g = [2.5 * s0 / (s0 + s1), 2.5 * s1 / (s0 + s1)]
        _close(ra["gates"][t], g)
        _close(rb["gates"][t], g)
        _close(ya[t], _ffn_closed(u, g[0] + 2.0 * g[1]))
    _close(ya, yb)
    _close(ra["gates"][0], [1.484614, 1.015386], tol=1e-6)
    _close(ya[2], [10.86829, 0.829627], tol=1e-6)


def pin_tie_goes_to_lower_index():
    x = np.array([[1.0, 1.0], [0.5, 0.5]])
    for mode in (orc.GATE_SOFTMAX, orc.GATE_SIGMOID):
        r = orc.route(x, np.eye(2), None, 1, mode, route_scale=1.0)
        assert r["idx"].ravel().tolist() == [0, 0]
    # Group tie: two groups with identical scores, keep one -> the lower group.
    b = np.array([[0.5, 0.1, 0.5, 0.1]])
    el = orc.group_eligibility(b, 2, 1)
    assert el.tolist() == [[True, True, False, False]]


# ------------------------------------------------------------ closed forms
def pin_router_is_u_dot_e():
    # A permutation router: e_e = unit vector of coordinate perm[e], so the
    # logit of expert e is u[perm[e]]. A transposed operand gives perm^-1.
    perm = [2, 0, 3, 1]
    wr = np.zeros((4, 4))
    for e, c in enumerate(perm):
        wr[e, c] = 1.0
    x = np.array([[10.0, 20.0, 30.0, 40.0], [1.0, -2.0, 3.0, -4.0]])
    _close(orc.router_logits(x, wr), x[:, perm])
    # Non-square: E=3 experts over d=5 hidden.
    rng = np.random.default_rng(3)
    x = rng.standard_normal((4, 5))
    wr = rng.standard_normal((3, 5))
    expect = np.array([[sum(x[t, c] * wr[e, c] for c in range(5)) for e in range(3)]
                       for t in range(4)])
    _close(orc.router_logits(x, wr), expect, tol=1e-12)


def pin_sigmoid_values():
    l = np.array([[0.0, math.log(3.0), -math.log(3.0), 40.0, -40.0]])
    s = orc.affinity(l, orc.GATE_SIGMOID)
    _close(s[0, :3], [0.5, 0.75, 0.25])
    assert 1.0 - 1e-15 < s[0, 3] <= 1.0 and 0.0 <= s[0, 4] < 1e-17
    _close(orc.affinity(l, orc.GATE_SOFTMAX), l)


def pin_softmax_two_way_is_logistic():
    rng = np.random.default_rng(5)
    lg = rng.standard_normal((16, 6)) * 3
    idx = np.sort(np.stack([rng.choice(6, 2, replace=False) for _ in range(16)]), axis=1)
    g = orc.gate_values(lg, lg, idx, orc.GATE_SOFTMAX, 1.0)
    for t in range(16):
        a, b = lg[t, idx[t, 0]], lg[t, idx[t, 1]]
        _close(g[t], [sigma(a - b), sigma(b - a)])


# -------------------------------------------------------------- invariants
def _random_case(rng, T=12, d=6, E=8, f=5, shared=0):
    return dict(
        x=rng.standard_normal((T, d)),
        wr=rng.standard_normal((E, d)) / math.sqrt(d),
        w1=rng.standard_normal((E, f, d)) / math.sqrt(d),
        w3=rng.standard_normal((E, f, d)) / math.sqrt(d),
        w2=rng.standard_normal((E, d, f)) / math.sqrt(f),
        ws1=rng.standard_normal((shared, d)) if shared else None,
        ws3=rng.standard_normal((shared, d)) if shared else None,
        ws2=rng.standard_normal((d, shared)) if shared else None,
    )


def pin_gate_sums():
    rng = np.random.default_rng(11)
    c = _random_case(rng, T=40, E=16)
    bias = rng.uniform(-0.3, 0.3, 16)
    for k in (1, 2, 5, 16):
        r = orc.route(c["x"], c["wr"], bias, k, orc.GATE_SOFTMAX)
        _close(r["gates"].sum(axis=1), np.ones(40))
        assert np.all(r["gates"] > 0)
        for scale in (1.0, 2.5):
            r = orc.route(c["x"], c["wr"], bias, k, orc.GATE_SIGMOID, 4, 2 if k <= 8 else 4,
                          route_scale=scale)
            _close(r["gates"].sum(axis=1), np.full(40, scale))


def pin_bias_moves_selection_not_gates():
    rng = np.random.default_rng(12)
    c = _random_case(rng, T=50, E=8)
    for mode in (orc.GATE_SOFTMAX, orc.GATE_SIGMOID):
        base = orc.route(c["x"], c["wr"], None, 3, mode, route_scale=2.5)
        # A constant shift never changes the order: same winners, same gates.
        shifted = orc.route(c["x"], c["wr"], np.full(8, 0.7), 3, mode, route_scale=2.5)
        assert np.array_equal(base["idx"], shifted["idx"])
        _close(base["gates"], shifted["gates"])
        # A bias that changes selection: wherever a token keeps its winners,
        # its gates are unchanged; some tokens must move.
        b = np.zeros(8)
        b[7] = 5.0
        moved = orc.route(c["x"], c["wr"], b, 3, mode, route_scale=2.5)
        assert np.all(moved["idx"][:, -1] == 7)
        same = np.all(moved["idx"] == base["idx"], axis=1)
        assert same.sum() < 50
        _close(moved["gates"][same], base["gates"][same])
        # Gates of a moved token are the unbiased renormalisation over its winners.
        rows = np.arange(50)[:, None]
        if mode == orc.GATE_SIGMOID:
            s = moved["scores"][rows, moved["idx"]]
            _close(moved["gates"], 2.5 * s / s.sum(axis=1, keepdims=True))
        else:
            l = moved["logits"][rows, moved["idx"]]
            ex = np.exp(l - l.max(axis=1, keepdims=True))
            _close(moved["gates"], 2.5 * ex / ex.sum(axis=1, keepdims=True))


def pin_k_equals_E_bias_irrelevant():
    rng = np.random.default_rng(13)
    c = _random_case(rng, T=10, E=4)
    for mode in (orc.GATE_SOFTMAX, orc.GATE_SIGMOID):
        ya = orc.moe_forward(c["x"], c["wr"], None, c["w1"], c["w3"], c["w2"], 4, mode,
                             route_scale=2.5)
        yb = orc.moe_forward(c["x"], c["wr"], rng.uniform(-3, 3, 4), c["w1"], c["w3"],
                             c["w2"], 4, mode, route_scale=2.5)
        _close(ya, yb, tol=1e-12)


# ------------------------------------------------------------- brute force
def _brute_topk(vals, allowed, k):
    best, best_set = None, None
    for combo in itertools.combinations([e for e in range(len(vals)) if allowed[e]], k):
        s = math.fsum(vals[e] for e in combo)
        if best is None or s > best:
            best, best_set = s, combo
    return list(best_set)


def pin_brute_force_topk():
    rng = np.random.default_rng(21)
    for trial in range(60):
        E = int(rng.integers(2, 9))
        k = int(rng.integers(1, E + 1))
        vals = rng.integers(-3, 4, size=E).astype(np.float64)   # many exact ties
        got = orc.select_experts(vals[None, :], np.ones((1, E), bool), k)[0]
        assert got.tolist() == _brute_topk(vals.tolist(), [True] * E, k), (vals, k, got)


def _brute_group_route(vals, n_groups, topk_groups, k):
    E = len(vals)
    size = E // n_groups
    gscore = []
    for g in range(n_groups):
        mem = range(g * size, (g + 1) * size)
        gscore.append(max(vals[a] + vals[b] for a in mem for b in mem if a < b))
    kept = _brute_topk(gscore, [True] * n_groups, topk_groups)
    allowed = [e // size in kept for e in range(E)]
    return _brute_topk(vals, allowed, k)


def pin_brute_force_group_limited():
    # Hand case: expert 0 has the single best score but group 1 has the best
    # top-2 sum (0.6 + 0.5 > 0.9 + 0.0); keeping one group selects expert 2.
    b = np.array([[0.9, 0.0, 0.6, 0.5]])
    assert orc.select_experts(b, orc.group_eligibility(b, 2, 1), 1)[0].tolist() == [2]
    # Groups of three: the score counts the two best members only, so a weak
    # third member does not pull group 0 (0.9 + 0.8 = 1.7) below group 1
    # (0.5 + 0.5 = 1.0, whose three members would sum to 1.5 > -3.3).
    b = np.array([[0.9, 0.8, -5.0, 0.5, 0.5, 0.5]])
    assert np.allclose(orc.group_scores(b, 2)[0], [1.7, 1.0], rtol=0, atol=1e-15)
    assert orc.select_experts(b, orc.group_eligibility(b, 2, 1), 1)[0].tolist() == [0]
    rng = np.random.default_rng(22)
    for trial in range(60):
        n_groups = int(rng.choice([2, 4]))
        size = int(rng.choice([2, 3]))
        E = n_groups * size
        tg = int(rng.integers(1, n_groups + 1))
        k = int(rng.integers(1, tg * size + 1))
        vals = rng.integers(-4, 5, size=E).astype(np.float64) / 2
        got = orc.select_experts(vals[None, :], orc.group_eligibility(vals[None, :], n_groups, tg), k)
        assert got[0].tolist() == _brute_group_route(vals.tolist(), n_groups, tg, k), (vals, n_groups, tg, k)


def pin_group_score_uses_biased_scores():
    # The Sparse MoE FFN note's "Routing": the group score is the sum of the two
    # largest *biased* scores. Scores s = (0.4, 0.4 | 0.6, 0.5) in two groups of
    # two: unbiased, group 1 leads (1.1 > 0.8) and keeps expert 2; a +0.3 bias on
    # group 0 lifts its pair to 0.7 + 0.7 = 1.4 > 1.1, so the choice moves into
    # group 0 (the 0.7 / 0.7 tie goes to the lower id), and the gate is still
    # the unbiased score renormalised over the one selected expert, 1.
    s = np.array([[0.4, 0.4, 0.6, 0.5]])
    logits = np.log(s / (1.0 - s))                       # sigmoid(logits) = s
    eye = np.eye(4)
    r0 = orc.route(logits, eye, np.zeros(4), 1, orc.GATE_SIGMOID, 2, 1, 1.0)
    assert r0["idx"].tolist() == [[2]]
    r = orc.route(logits, eye, np.array([0.3, 0.3, 0.0, 0.0]), 1, orc.GATE_SIGMOID, 2, 1, 1.0)
    assert r["idx"].tolist() == [[0]]
    assert np.allclose(r["gates"], [[1.0]], rtol=0, atol=1e-15)
    assert r["eligible"][0].tolist() == [True, True, False, False]


# --------------------------------------------------- library special cases
def _torch_swiglu(u, w1, w3, w2):
    u, w1, w3, w2 = (torch.as_tensor(a, dtype=torch.float64) for a in (u, w1, w3, w2))
    return torch.nn.functional.linear(
        torch.nn.functional.silu(torch.nn.functional.linear(u, w1)) * torch.nn.functional.linear(u, w3),
        w2).numpy()


def pin_single_expert_is_dense_swiglu():
    rng = np.random.default_rng(31)
    T, d, f = 9, 7, 5
    x = rng.standard_normal((T, d))
    w1, w3 = rng.standard_normal((1, f, d)), rng.standard_normal((1, f, d))
    w2 = rng.standard_normal((1, d, f))
    y = orc.moe_forward(x, rng.standard_normal((1, d)), None, w1, w3, w2, 1, orc.GATE_SOFTMAX)
    _close(y, _torch_swiglu(x, w1[0], w3[0], w2[0]), tol=1e-12)
    _close(orc.swiglu_ffn(x, w1[0], w3[0], w2[0]), _torch_swiglu(x, w1[0], w3[0], w2[0]), tol=1e-12)
    # The inner activation alone: the down projection with W2 = I.
    _close(orc.swiglu_hidden(x, w1[0], w3[0]), _torch_swiglu(x, w1[0], w3[0], np.eye(f)), tol=1e-12)


def pin_shared_expert_added_no_residual():
    rng = np.random.default_rng(32)
    c = _random_case(rng, T=8, d=6, E=4, f=3, shared=10)
    zero_w2 = np.zeros_like(c["w2"])
    y = orc.moe_forward(c["x"], c["wr"], None, c["w1"], c["w3"], zero_w2, 2, orc.GATE_SIGMOID,
                        route_scale=2.5, ws1=c["ws1"], ws3=c["ws3"], ws2=c["ws2"])
    _close(y, _torch_swiglu(c["x"], c["ws1"], c["ws3"], c["ws2"]), tol=1e-12)
    # All-zero weights give a zero output: the block adds no residual.
    yz = orc.moe_forward(c["x"], c["wr"], None, np.zeros_like(c["w1"]), np.zeros_like(c["w3"]),
                         zero_w2, 2, orc.GATE_SOFTMAX, ws1=np.zeros_like(c["ws1"]),
                         ws3=np.zeros_like(c["ws3"]), ws2=np.zeros_like(c["ws2"]))
    _close(yz, np.zeros_like(c["x"]))
    # Shared + routed splits additively.
    yr = orc.moe_forward(c["x"], c["wr"], None, c["w1"], c["w3"], c["w2"], 2, orc.GATE_SIGMOID,
                         route_scale=2.5)
    ys = orc.moe_forward(c["x"], c["wr"], None, c["w1"], c["w3"], c["w2"], 2, orc.GATE_SIGMOID,
                         route_scale=2.5, ws1=c["ws1"], ws3=c["ws3"], ws2=c["ws2"])
    _close(ys - yr, _torch_swiglu(c["x"], c["ws1"], c["ws3"], c["ws2"]), tol=1e-12)


def pin_routed_sum_per_token_by_hand():
    rng = np.random.default_rng(33)
    c = _random_case(rng, T=6, d=5, E=5, f=4)
    r = orc.route(c["x"], c["wr"], None, 2, orc.GATE_SIGMOID, route_scale=2.5)
    y = orc.expert_outputs(c["x"], r["idx"], r["gates"], c["w1"], c["w3"], c["w2"])
    for t in range(6):
        acc = np.zeros(5)
        for j in range(2):
            e = r["idx"][t, j]
            acc += r["gates"][t, j] * _torch_swiglu(c["x"][t:t + 1], c["w1"][e], c["w3"][e], c["w2"][e])[0]
        _close(y[t], acc, tol=1e-12)


def pin_packed_equals_dense_loop():
    rng = np.random.default_rng(41)
    for E, k in ((4, 1), (6, 2), (8, 3), (5, 5)):
        c = _random_case(rng, T=15, d=6, E=E, f=4)
        packed = orc.moe_forward(c["x"], c["wr"], None, c["w1"], c["w3"], c["w2"], k, orc.GATE_SOFTMAX)
        loop = orc.moe_forward_dense_loop(c["x"], c["wr"], c["w1"], c["w3"], c["w2"], k)
        _close(packed, loop, tol=1e-11)


# ------------------------------------------------------------ packing
def pin_counts_offsets_rows():
    rng = np.random.default_rng(51)
    T, E, k = 37, 9, 3
    idx = np.sort(np.stack([rng.choice(E, k, replace=False) for _ in range(T)]), axis=1)
    counts, offsets = orc.expert_counts_offsets(idx, E)
    assert counts.sum() == T * k and offsets[0] == 0 and offsets[-1] == T * k
    for e in range(E):
        assert counts[e] == sum(int(e in idx[t]) for t in range(T))
        assert offsets[e] == sum(counts[:e])
    inv_row, perm_src = orc.permutation_rows(idx, offsets)
    # Independent statement: sort the (expert, token) pairs lexicographically;
    # a pair's position in that order is its packed row.
    pairs = sorted((idx[t, j], t, j) for t in range(T) for j in range(k))
    for row, (e, t, j) in enumerate(pairs):
        assert inv_row[t, j] == row and perm_src[row] == t
    assert sorted(perm_src.tolist()) == sorted([t for t in range(T) for _ in range(k)])


def pin_near_tie_flags():
    # Token 0: an exact tie between the 2nd and 3rd score (k = 2) -> flagged.
    # Token 1: wide gaps -> not flagged.
    lg = np.array([[3.0, 1.0, 1.0, -2.0], [3.0, 2.0, 0.0, -2.0]])
    r = orc.route(lg, np.eye(4), None, 2, orc.GATE_SOFTMAX)
    assert orc.near_tie_tokens(r, 2).tolist() == [True, False]
    # Group boundary tie that changes the selection is flagged; one that does
    # not (both candidate groups lose to the kept group's experts) is not.
    b = np.array([[0.9, 0.8, 0.5, 0.1, 0.5, 0.1], [0.9, 0.8, 0.5, 0.1, 0.5, 0.1]])
    r = orc.route(b, np.eye(6), None, 3, orc.GATE_SOFTMAX, n_groups=3, topk_groups=2)
    assert orc.near_tie_tokens(r, 3, 3, 2).tolist() == [True, True]
    r = orc.route(b, np.eye(6), None, 2, orc.GATE_SOFTMAX, n_groups=3, topk_groups=2)
    assert orc.near_tie_tokens(r, 2, 3, 2).tolist() == [False, False]


def pin_near_tie_three_groups_at_the_boundary():
    # Three groups within 1e-5 of one another, keep two, k = 1. Groups are
    # {0,1}, {2,3}, {4,5}; their scores (sums of both members) are 1.0,
    # 1.0 - 2e-6 and 1.0 - 4e-6, so groups 0 and 1 are kept and expert 0
    # (0.9) wins. Exchanging the last kept and first dropped group (1 and 2)
    # leaves expert 0 the winner, but another rounding could rank group 0
    # last and drop it, and then expert 4 (0.6) would win: a near tie.
    lg = np.array([[0.9, 0.1, 0.5, 0.5 - 2e-6, 0.6, 0.4 - 4e-6]])
    r = orc.route(lg, np.eye(6), None, 1, orc.GATE_SOFTMAX, n_groups=3, topk_groups=2)
    assert r["idx"].tolist() == [[0]]
    assert orc.near_tie_tokens(r, 1, 3, 2).tolist() == [True]
    # The same scores with group 0 well ahead (1.2): only groups 1 and 2 are
    # near the boundary, and either keeps expert 0 the winner: no near tie.
    lg2 = np.array([[0.9, 0.3, 0.5, 0.5 - 2e-6, 0.6, 0.4 - 4e-6]])
    r2 = orc.route(lg2, np.eye(6), None, 1, orc.GATE_SOFTMAX, n_groups=3, topk_groups=2)
    assert orc.near_tie_tokens(r2, 1, 3, 2).tolist() == [False]


def pin_near_tie_ignores_dropped_groups():
    # Top-k chooses among the experts of the kept groups only, so an expert of a
    # dropped group that ties the k-th winner cannot change the selection: not
    # a near tie. Groups {0,1} (1.0 + 0.9) and {2,3} (1.0 - 3.0), keep one,
    # k = 1: expert 0 wins against 0.9 inside its group; expert 2's 1.0 does
    # not count, and the group scores are far apart.
    lg = np.array([[1.0, 0.9, 1.0, -3.0]])
    r = orc.route(lg, np.eye(4), None, 1, orc.GATE_SOFTMAX, n_groups=2, topk_groups=1)
    assert r["idx"].tolist() == [[0]]
    assert orc.near_tie_tokens(r, 1, 2, 1).tolist() == [False]


def pin_near_tie_gap_is_on_biased_scores():
    # The near-tie rule measures the k-th / (k+1)-th gap of the selection
    # scores s + b, the values top-k ranks. Token 0: the raw scores tie (1, 1)
    # but the bias separates them (1.5 vs 1) -> not a near tie. Token 1: the
    # raw scores differ (0.5 vs 1) but the bias closes the gap (1 vs 1) -> a
    # near tie. k = 1, softmax mode (s = raw logit).
    lg = np.array([[1.0, 1.0, -1.0, -2.0], [0.5, 1.0, -1.0, -2.0]])
    r = orc.route(lg, np.eye(4), np.array([0.5, 0.0, 0.0, 0.0]), 1, orc.GATE_SOFTMAX)
    assert orc.near_tie_tokens(r, 1).tolist() == [False, True]


# ------------------------------------------------------- balance loop
def pin_entropy_closed_forms():
    for E in (1, 2, 7, 256):
        _close(orc.routing_entropy(np.full(E, 5)), math.log(E), tol=1e-14)
    _close(orc.routing_entropy([0, 0, 9, 0]), 0.0)
    _close(orc.routing_entropy([3, 1]), -(0.75 * math.log(0.75) + 0.25 * math.log(0.25)))
    _close(orc.routing_entropy([2, 0, 2]), math.log(2.0))
    assert orc.routing_entropy([0, 0]) == 0.0


def pin_bias_update_direction():
    # target = 12 * 2 / 4 = 6: experts at 9, 6, 3, 6 tokens.
    t = orc.balance_target(12, 2, 4)
    assert t == 6.0
    b = orc.update_bias([0.5, -0.25, 0.0, 1.0], [9, 6, 3, 6], t, 0.15)
    _close(b, [0.35, -0.25, 0.15, 1.0], tol=1e-15)


def pin_balance_target_is_not_rounded():
    # The cheat sheet's "Aux-loss-free balance loop", step 1: target usage =
    # n_tokens * top_k / n_experts, a real number. 10 tokens x top-3 over 4
    # experts target 7.5 each, so counts of 7 and 8 are under and over target
    # (none is on target) and every bias moves.
    t = orc.balance_target(10, 3, 4)
    assert t == 7.5
    b = orc.update_bias([0.0, 0.0, 0.0, 0.0], [7, 8, 8, 7], t, 0.25)
    assert np.array_equal(b, [0.25, -0.25, -0.25, 0.25])


def pin_balance_loop_raises_entropy():
    # The cheat sheet's loop: route with scores + bias, count, update with
    # gamma = 0.15, 10 iterations; entropy rises toward ln(E). A router whose
    # first experts are favoured starts far from uniform.
    rng = np.random.default_rng(61)
    T, d, E, k = 256, 16, 8, 2
    x = rng.standard_normal((T, d))
    wr = rng.standard_normal((E, d)) / math.sqrt(d)
    skew = np.linspace(1.5, -1.5, E)
    bias = np.zeros(E)
    ent = []
    for it in range(10):
        r = orc.route(x, wr, skew + bias, k, orc.GATE_SOFTMAX)
        counts, _ = orc.expert_counts_offsets(r["idx"], E)
        ent.append(orc.routing_entropy(counts))
        bias = orc.update_bias(bias, counts, orc.balance_target(T, k, E), 0.15)
    assert ent[-1] > ent[0] + 0.2, ent
    assert max(ent) <= math.log(E) + 1e-12
    assert ent[-1] > 0.95 * math.log(E), ent


# ------------------------------------------------ generic (GELU) experts
# Standard normal CDF values from the printed normal table (textbook values).
PHI_1 = 0.8413447460685429
PHI_2 = 0.9772498680518208


def pin_gelu_closed_forms():
    _close(orc.gelu([0.0, 1.0, -1.0, 2.0]), [0.0, PHI_1, -(1.0 - PHI_1), 2.0 * PHI_2], tol=1e-15)
    rng = np.random.default_rng(61)
    z = rng.standard_normal(50) * 3
    # Phi(-z) = 1 - Phi(z) gives GELU(z) - GELU(-z) = z.
    _close(orc.gelu(z) - orc.gelu(-z), z, tol=1e-14)
    # Far tails: GELU(z) -> z for z >> 0 and -> 0 for z << 0.
    _close(orc.gelu([12.0, -12.0]), [12.0, 0.0], tol=1e-15)


def pin_gelu_is_torch_exact_gelu():
    rng = np.random.default_rng(62)
    z = rng.standard_normal(200) * 4
    ref = torch.nn.functional.gelu(torch.as_tensor(z, dtype=torch.float64), approximate="none").numpy()
    _close(orc.gelu(z), ref, tol=1e-14)
    tanh_form = torch.nn.functional.gelu(torch.as_tensor(z, dtype=torch.float64), approximate="tanh").numpy()
    assert np.max(np.abs(orc.gelu(z) - tanh_form)) > 1e-5   # the erf form, not the tanh one


def _torch_gelu_ffn(u, w1, b1, w2, b2):
    u, w1, b1, w2, b2 = (torch.as_tensor(a, dtype=torch.float64) for a in (u, w1, b1, w2, b2))
    F = torch.nn.functional
    return F.linear(F.gelu(F.linear(u, w1, b1)), w2, b2).numpy()


def pin_gelu_single_expert_is_dense_ffn():
    rng = np.random.default_rng(63)
    T, d, f = 9, 7, 5
    x = rng.standard_normal((T, d))
    w1, b1 = rng.standard_normal((1, f, d)), rng.standard_normal((1, f))
    w2, b2 = rng.standard_normal((1, d, f)), rng.standard_normal((1, d))
    ref = _torch_gelu_ffn(x, w1[0], b1[0], w2[0], b2[0])
    _close(orc.gelu_ffn(x, w1[0], b1[0], w2[0], b2[0]), ref, tol=1e-12)
    y = orc.moe_forward_gelu(x, rng.standard_normal((1, d)), None, w1, b1, w2, b2, 1, orc.GATE_SOFTMAX)
    _close(y, ref, tol=1e-12)


def pin_gelu_hand_case():
    # Identity router and weights, expert 1 doubled; expert 1 has b1 = (1, -1)
    # and b2 = (0.5, 0.5). Softmax, k = 1: tokens go to experts 0, 1, 0.
    b1 = np.array([[0.0, 0.0], [1.0, -1.0]])
    b2 = np.array([[0.0, 0.0], [0.5, 0.5]])
    y = orc.moe_forward_gelu(HAND_X, HAND_WR, None, HAND_W1, b1, HAND_W2, b2, 1, orc.GATE_SOFTMAX)
    want = np.array([
        [PHI_1, 0.0],                             # GELU(1, 0)
        [2.0 * PHI_1 + 0.5, 0.5],                 # 2 GELU((0, 1) + (1, -1)) + b2
        [2.0 * PHI_2, -(1.0 - PHI_1)],            # GELU(2, -1)
    ])
    _close(y, want, tol=1e-15)


def pin_gelu_b2_is_gated():
    # The gate multiplies the whole expert output: shifting every b2 by c
    # moves y by (sum of the token's gates) * c: route_scale * c in sigmoid
    # mode, c in softmax mode.
    rng = np.random.default_rng(64)
    T, d, E, f = 10, 6, 8, 5
    x = rng.standard_normal((T, d))
    wr = rng.standard_normal((E, d))
    w1, b1 = rng.standard_normal((E, f, d)), rng.standard_normal((E, f))
    w2, b2 = rng.standard_normal((E, d, f)), rng.standard_normal((E, d))
    c = rng.standard_normal(d)
    for mode, scale in ((orc.GATE_SOFTMAX, 1.0), (orc.GATE_SIGMOID, 2.5)):
        y0 = orc.moe_forward_gelu(x, wr, None, w1, b1, w2, b2, 3, mode, route_scale=scale)
        y1 = orc.moe_forward_gelu(x, wr, None, w1, b1, w2, b2 + c, 3, mode, route_scale=scale)
        _close(y1 - y0, np.tile(scale * c, (T, 1)), tol=1e-12)


# ---------------------------------------------------------------- backward
def _bwd_case(rng, gate_mode, T=7, d=5, E=6, k=2, f=3, shared=4, n_groups=1, topk_groups=1):
    c = _random_case(rng, T=T, d=d, E=E, f=f, shared=shared)
    c.update(bias=rng.uniform(-0.2, 0.2, E), dy=rng.standard_normal((T, d)), k=k, mode=gate_mode,
             n_groups=n_groups, topk_groups=topk_groups, rs=2.5 if gate_mode == orc.GATE_SIGMOID else 1.0)
    return c


def _loss(c, **override):
    a = dict(c)
    a.update(override)
    y = orc.moe_forward(a["x"], a["wr"], a["bias"], a["w1"], a["w3"], a["w2"], a["k"], a["mode"],
                        a["n_groups"], a["topk_groups"], a["rs"], a["ws1"], a["ws3"], a["ws2"])
    idx = orc.route(a["x"], a["wr"], a["bias"], a["k"], a["mode"], a["n_groups"], a["topk_groups"],
                    a["rs"])["idx"]
    return float((np.asarray(a["dy"]) * y).sum()), idx


def _bwd(c):
    return orc.moe_backward(c["x"], c["wr"], c["bias"], c["w1"], c["w3"], c["w2"], c["k"], c["mode"], c["dy"],
                            c["n_groups"], c["topk_groups"], c["rs"], c["ws1"], c["ws3"], c["ws2"])


def pin_backward_finite_differences():
    # Central differences of the (pinned) forward: the gradient's definition,
    # exact up to O(h^2) while the expert choice does not move.
    h = 1e-5
    for seed, mode, ng, tg in ((71, orc.GATE_SIGMOID, 3, 2), (72, orc.GATE_SOFTMAX, 1, 1)):
        rng = np.random.default_rng(seed)
        c = _bwd_case(rng, mode, n_groups=ng, topk_groups=tg)
        g = _bwd(c)
        _, idx0 = _loss(c)
        names = {"x": "dx", "wr": "dw_router", "w1": "dw1", "w3": "dw3", "w2": "dw2",
                 "ws1": "dws1", "ws3": "dws3", "ws2": "dws2"}
        for p, gname in names.items():
            base = np.asarray(c[p], dtype=np.float64)
            num = np.zeros_like(base)
            for pos in np.ndindex(base.shape):
                plus, minus = base.copy(), base.copy()
                plus[pos] += h
                minus[pos] -= h
                lp, ip = _loss(c, **{p: plus})
                lm, im = _loss(c, **{p: minus})
                assert np.array_equal(ip, idx0) and np.array_equal(im, idx0), (p, pos)
                num[pos] = (lp - lm) / (2 * h)
            _close(g[gname], num, tol=1e-7)


def _torch_moe_loss(c, idx):
    """Independent fp64 torch statement of <dy, MoE(x)> for a fixed expert choice."""
    t = lambda a: torch.tensor(np.asarray(a, dtype=np.float64), requires_grad=True)
    P = {n: t(c[n]) for n in ("x", "wr", "w1", "w3", "w2", "ws1", "ws3", "ws2")}
    F = torch.nn.functional
    logits = P["x"] @ P["wr"].T
    ii = torch.as_tensor(idx)
    sel = torch.gather(logits, 1, ii)
    if c["mode"] == orc.GATE_SIGMOID:
        s = torch.sigmoid(sel)
        gates = c["rs"] * s / s.sum(dim=1, keepdim=True)
    else:
        gates = c["rs"] * torch.softmax(sel, dim=1)
    y = F.linear(F.silu(F.linear(P["x"], P["ws1"])) * F.linear(P["x"], P["ws3"]), P["ws2"])
    for t_ in range(idx.shape[0]):
        for j in range(idx.shape[1]):
            e = int(idx[t_, j])
            u = P["x"][t_]
            o = P["w2"][e] @ (F.silu(P["w1"][e] @ u) * (P["w3"][e] @ u))
            y = y + F.pad((gates[t_, j] * o)[None, :], (0, 0, t_, idx.shape[0] - t_ - 1))
    loss = (torch.as_tensor(np.asarray(c["dy"])) * y).sum()
    loss.backward()
    return {n: P[n].grad.numpy() for n in P}


def pin_backward_matches_torch_autograd():
    names = {"x": "dx", "wr": "dw_router", "w1": "dw1", "w3": "dw3", "w2": "dw2",
             "ws1": "dws1", "ws3": "dws3", "ws2": "dws2"}
    for seed, mode in ((73, orc.GATE_SIGMOID), (74, orc.GATE_SOFTMAX)):
        rng = np.random.default_rng(seed)
        c = _bwd_case(rng, mode, T=9, d=6, E=8, k=3, f=4, shared=5)
        g = _bwd(c)
        ref = _torch_moe_loss(c, g["idx"])
        for p, gname in names.items():
            _close(g[gname], ref[p], tol=1e-12)


def pin_silu_grad():
    z = np.linspace(-8, 8, 41)
    zt = torch.tensor(z, requires_grad=True)
    torch.nn.functional.silu(zt).sum().backward()
    _close(orc.silu_grad(z), zt.grad.numpy(), tol=1e-14)
    _close(orc.silu_grad([0.0]), [0.5], tol=1e-15)


def pin_constant_gate_gradient_moves_no_logit():
    # Gates of a token sum to route_scale whatever the logits (both modes), so
    # a gate gradient equal on all k slots has zero logit gradient.
    rng = np.random.default_rng(75)
    for mode, rs in ((orc.GATE_SIGMOID, 2.5), (orc.GATE_SOFTMAX, 1.0)):
        c = _random_case(rng, T=10, E=8)
        r = orc.route(c["x"], c["wr"], None, 3, mode, route_scale=rs)
        dg = np.repeat(rng.standard_normal((10, 1)), 3, axis=1)
        dl = orc.gate_backward(r["logits"], r["scores"], r["idx"], r["gates"], dg, mode, rs)
        _close(dl, np.zeros_like(dl), tol=1e-14)


def pin_single_expert_backward_is_dense():
    # E = 1, k = 1, softmax: the gate is identically 1, the router gets no
    # gradient and dx is the dense SwiGLU's input gradient (torch autograd).
    rng = np.random.default_rng(76)
    T, d, f = 6, 5, 4
    x, dy = rng.standard_normal((T, d)), rng.standard_normal((T, d))
    w1, w3, w2 = rng.standard_normal((1, f, d)), rng.standard_normal((1, f, d)), rng.standard_normal((1, d, f))
    g = orc.moe_backward(x, rng.standard_normal((1, d)), None, w1, w3, w2, 1, orc.GATE_SOFTMAX, dy)
    _close(g["dw_router"], np.zeros((1, d)), tol=1e-15)
    xt = torch.tensor(x, requires_grad=True)
    ws = [torch.tensor(w[0], requires_grad=True) for w in (w1, w3, w2)]
    F = torch.nn.functional
    y = F.linear(F.silu(F.linear(xt, ws[0])) * F.linear(xt, ws[1]), ws[2])
    (torch.as_tensor(dy) * y).sum().backward()
    _close(g["dx"], xt.grad.numpy(), tol=1e-12)
    _close(g["dw1"][0], ws[0].grad.numpy(), tol=1e-12)
    _close(g["dw3"][0], ws[1].grad.numpy(), tol=1e-12)
    _close(g["dw2"][0], ws[2].grad.numpy(), tol=1e-12)


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_") and callable(v)]
