"""Pins of the fp64 oracle against facts fixed outside the oracle itself:
numbers the pages print, brute force on tiny inputs, structural identities
the pages state (segmentation, shared-expert fusion, dense ceiling), closed
forms and invariances. Each is chosen so a plausible slip in the oracle (a
dropped term, a wrong sign or index, a transposed operand, the bias leaking
into the gates) fails at least one of them."""
import itertools
import json
import math
import os

import numpy as np
import pytest

import oracle
from oracle import RouterCfg

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def _rng(seed):
    return np.random.default_rng(seed)


def _experts(rng, N, d, F, scale=1.0):
    W1 = rng.standard_normal((N, F, d)) * scale / math.sqrt(d)
    W3 = rng.standard_normal((N, F, d)) * scale / math.sqrt(d)
    W2 = rng.standard_normal((N, d, F)) * scale / math.sqrt(F)
    return W1, W3, W2


# ------------------------------------------------------- printed numbers ----

def test_printed_v3_parameter_counts():
    g = _gold("v3_block_params.json")
    d, N, ns = g["d"], g["n_routed"], g["n_shared"]
    d_ff = g["routed_expert_each"] // (3 * d)
    assert d_ff * 3 * d == g["routed_expert_each"] and d_ff == 2048
    assert oracle.expert_params(d, d_ff) == g["routed_expert_each"] == g["shared_expert"]
    assert oracle.router_params(d, N) == g["router"]
    assert N * oracle.expert_params(d, d_ff) == g["routed_experts_total"]
    assert oracle.block_params(d, d_ff, N, ns) == g["block_total"]
    assert g["n_moe_blocks"] * oracle.block_params(d, d_ff, N, ns) == g["all_blocks_total"]


def test_printed_team_counts():
    g = _gold("team_counts.json")
    for n, k, v in g["exact"]:
        assert oracle.routing_combinations(n, k) == v
    for n, k, trillions in g["approx_trillions"]:
        assert round(oracle.routing_combinations(n, k) / 1e12) == trillions
    # the walkthrough's hand count for top-2 of 16: 16 * 15 / 2
    assert oracle.routing_combinations(16, 2) == 16 * 15 // 2


def test_segmentation_keeps_params_and_flops():
    # N experts of width F -> mN experts of width F/m with top-mk: same params, same FLOPs
    for (N, k, d, F, m) in [(16, 2, 1280, 3584, 4), (16, 2, 256, 512, 8)]:
        assert N * oracle.expert_params(d, F) == m * N * oracle.expert_params(d, F // m)
        assert oracle.flops_per_token(d, F, k, 0) == oracle.flops_per_token(d, F // m, m * k, 0)


# ------------------------------------------------------ closed forms ----

def test_score_and_activation_closed_forms():
    z = np.linspace(-30, 30, 241)
    s = oracle.sigmoid(z)
    np.testing.assert_allclose(s + oracle.sigmoid(-z), 1.0, rtol=0, atol=1e-15)
    assert oracle.sigmoid(np.array([0.0]))[0] == 0.5
    # silu(g) - silu(-g) = g(sigma(g) + sigma(-g)) = g ; silu(0) = 0
    np.testing.assert_allclose(oracle.silu(z) - oracle.silu(-z), z, rtol=1e-14, atol=1e-13)
    assert oracle.silu(np.array([0.0]))[0] == 0.0
    # softmax: positive, sums to 1, invariant to a shift of all logits
    rng = _rng(1)
    Z = rng.standard_normal((7, 19)) * 5
    P = oracle.softmax(Z)
    assert (P > 0).all()
    np.testing.assert_allclose(P.sum(axis=1), 1.0, rtol=0, atol=1e-14)
    np.testing.assert_allclose(oracle.softmax(Z + 123.25), P, rtol=1e-13, atol=0)
    # two-way softmax equals the logistic function of the logit difference
    a, b = Z[:, 0], Z[:, 1]
    P2 = oracle.softmax(Z[:, :2])
    np.testing.assert_allclose(P2[:, 0], 1.0 / (1.0 + np.exp(b - a)), rtol=1e-14)


def test_score_value_pins():
    # values, not only symmetries: sigma(ln 3) = 1 / (1 + 1/3) = 3/4, sigma(-ln 3) = 1/4,
    # silu(ln 3) = (3/4) ln 3 (a wrong slope such as 1/(1+exp(-2z)) gives 9/10 instead);
    # softmax of (ln 1, ln 2, ln 3) = (1, 2, 3) / 6
    l3 = math.log(3.0)
    assert abs(oracle.sigmoid(np.array([l3]))[0] - 0.75) < 1e-15
    assert abs(oracle.sigmoid(np.array([-l3]))[0] - 0.25) < 1e-15
    assert abs(oracle.silu(np.array([l3]))[0] - 0.75 * l3) < 1e-15
    np.testing.assert_allclose(oracle.softmax(np.log(np.array([[1.0, 2.0, 3.0]]))), [[1 / 6, 2 / 6, 3 / 6]],
                               rtol=1e-15)


def test_router_logits_is_x_times_router_rows():
    # z_e is the dot product of the token with centroid e (walkthrough Step 2)
    rng = _rng(2)
    x = rng.standard_normal((5, 7))
    W = rng.standard_normal((4, 7))
    z = oracle.router_logits(x, W)
    for t in range(5):
        for e in range(4):
            assert abs(z[t, e] - sum(x[t, j] * W[e, j] for j in range(7))) < 1e-12


def test_swiglu_bilinear_identity():
    # FFN(W1) - FFN(-W1) = W2 ((W1 x) * (W3 x)) because silu(g) - silu(-g) = g:
    # pins the activation, its position (on g, not u) and the operand orientation.
    rng = _rng(3)
    n, d, F = 6, 12, 20
    x = rng.standard_normal((n, d))
    W1, W3, W2 = (a[0] for a in _experts(rng, 1, d, F))
    lhs = oracle.expert_ffn(x, W1, W3, W2) - oracle.expert_ffn(x, -W1, W3, W2)
    rhs = ((x @ W1.T) * (x @ W3.T)) @ W2.T
    np.testing.assert_allclose(lhs, rhs, rtol=1e-12, atol=1e-12)
    # the output is linear in W2 and in W3, and vanishes with W3 = 0
    np.testing.assert_allclose(oracle.expert_ffn(x, W1, W3, 3 * W2), 3 * oracle.expert_ffn(x, W1, W3, W2),
                               rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(oracle.expert_ffn(x, W1, -W3, W2), -oracle.expert_ffn(x, W1, W3, W2),
                               rtol=1e-12, atol=1e-12)
    assert np.abs(oracle.expert_ffn(x, W1, 0 * W3, W2)).max() == 0.0
    with pytest.raises(ValueError):
        oracle.expert_ffn(x, W1, W3, W2.T)  # a transposed W2 does not fit [d, d_ff]


# ---------------------------------------------------------- brute force ----

def _brute_topk(keys, allowed, k):
    cand = [e for e in range(len(keys)) if allowed[e]]
    best, best_set = -np.inf, None
    for sub in itertools.combinations(cand, k):
        v = sum(keys[e] for e in sub)
        if v > best:
            best, best_set = v, set(sub)
    return best_set


@pytest.mark.parametrize("score,N,k,bias", [("softmax", 16, 2, False), ("sigmoid", 10, 3, True),
                                            ("softmax", 9, 9, False), ("sigmoid", 12, 1, True)])
def test_topk_matches_brute_force(score, N, k, bias):
    rng = _rng(10 + N + k)
    T, d = 40, 8
    x = rng.standard_normal((T, d))
    W = rng.standard_normal((N, d)) / math.sqrt(d)
    b = rng.uniform(-0.1, 0.1, N) if bias else None
    cfg = RouterCfg(n_routed=N, top_k=k, score=score)
    r = oracle.route(x, W, b, cfg)
    for t in range(T):
        assert set(r.idx[t].tolist()) == _brute_topk(r.keys[t], [True] * N, k)
        ks = r.keys[t, r.idx[t]]
        assert (np.diff(ks) <= 0).all()  # slots in descending key order
    # C(16,2) = 120 candidate teams were searched for the GShard case
    if (N, k) == (16, 2):
        assert len(list(itertools.combinations(range(N), k))) == 120


@pytest.mark.parametrize("gscore", ["top2_sum", "max"])
def test_group_limited_topk_matches_brute_force(gscore):
    # N=16 in G=4 groups of 4, keep the top TG=2 groups, then top k=4:
    # enumerate the C(4,2) group pairs, then the C(8,4) expert subsets.
    rng = _rng(20)
    N, G, TG, k, T, d = 16, 4, 2, 4, 60, 8
    x = rng.standard_normal((T, d))
    W = rng.standard_normal((N, d)) / math.sqrt(d)
    b = rng.uniform(-0.1, 0.1, N)
    cfg = RouterCfg(n_routed=N, top_k=k, score="sigmoid", n_groups=G, topk_groups=TG, normalize=True,
                    route_scale=2.5, group_score=gscore)
    r = oracle.route(x, W, b, cfg)
    S = N // G
    for t in range(T):
        key = r.keys[t]
        gsc = []
        for g in range(G):
            members = range(g * S, (g + 1) * S)
            if gscore == "max":
                gsc.append(max(key[e] for e in members))
            else:
                gsc.append(max(key[i] + key[j] for i, j in itertools.combinations(members, 2)))
        best_pair = max(itertools.combinations(range(G), TG), key=lambda p: sum(gsc[g] for g in p))
        allowed = [e // S in best_pair for e in range(N)]
        assert set(r.idx[t].tolist()) == _brute_topk(key, allowed, k)
        assert list(r.allowed[t]) == allowed


def test_tie_flags():
    # two experts with identical router rows tie exactly; a clear winner does not
    d, N = 6, 5
    W = np.zeros((N, d))
    W[0, 0] = 3.0
    W[1, 1] = 2.0
    W[2, 1] = 2.0  # experts 1 and 2 tie whenever x[1] != 0
    W[3, 2] = 1.0
    x = np.array([[1.0, 1.0, 0, 0, 0, 0],   # logits 3, 2, 2, 0, 0
                  [1.0, 0.0, 1.0, 0, 0, 0]])  # logits 3, 0, 0, 1, 0
    r = oracle.route(x, W, None, RouterCfg(n_routed=N, top_k=2, score="sigmoid"))
    assert r.sel_tie[0] and not r.sel_tie[1]
    assert r.idx[0].tolist() == [0, 1]  # lower index wins the tie
    assert r.idx[1].tolist() == [0, 3]
    r3 = oracle.route(x, W, None, RouterCfg(n_routed=N, top_k=3, score="sigmoid"))
    assert not r3.sel_tie[0] and r3.order_tie[0]  # both tied experts inside: only the order is tied


# ---------------------------------------------------------------- gates ----

def test_normalized_gates_sum_to_route_scale():
    rng = _rng(30)
    N, T, d = 32, 50, 16
    x = rng.standard_normal((T, d))
    W = rng.standard_normal((N, d)) / math.sqrt(d)
    b = rng.uniform(-0.1, 0.1, N)
    cfg = RouterCfg(n_routed=N, top_k=8, score="sigmoid", n_groups=8, topk_groups=4, normalize=True,
                    route_scale=2.5)
    r = oracle.route(x, W, b, cfg)
    np.testing.assert_allclose(r.gates.sum(axis=1), 2.5, rtol=0, atol=1e-12)
    assert (r.gates > 0).all()


def test_bias_steers_selection_but_not_gates():
    rng = _rng(31)
    N, T, d = 16, 64, 8
    x = rng.standard_normal((T, d))
    W = rng.standard_normal((N, d)) / math.sqrt(d)
    b = rng.uniform(-0.1, 0.1, N)
    cfg = RouterCfg(n_routed=N, top_k=4, score="sigmoid", normalize=True, route_scale=2.5)
    r = oracle.route(x, W, b, cfg)
    # a constant added to every bias changes neither the selection nor the gates
    r_c = oracle.route(x, W, b + 0.37, cfg)
    assert (r_c.idx == r.idx).all()
    np.testing.assert_allclose(r_c.gates, r.gates, rtol=1e-14)
    # a tiny rescale of the bias that keeps every selection keeps the gates too
    r_s = oracle.route(x, W, b * (1 + 1e-9), cfg)
    same = (r_s.idx == r.idx).all(axis=1)
    assert same.mean() > 0.9
    np.testing.assert_allclose(r_s.gates[same], r.gates[same], rtol=1e-14)
    # a large bias on one expert forces it in, and its gate still follows its unbiased score
    bb = b.copy()
    bb[5] = 10.0
    r_f = oracle.route(x, W, bb, cfg)
    assert (r_f.idx[:, 0] == 5).all()
    r_nob = oracle.route(x, W, None, cfg)
    s5 = r_nob.scores[:, 5]
    assert np.all(r_f.gates[:, 0] < 1.5)  # a biased key (about 10) would push it near 2.5
    np.testing.assert_allclose(r_f.scores[:, 5], s5, rtol=1e-15)


def test_gates_for_hand_example():
    # scores 0.1 .. 0.4, selection (3, 1): normalised gates 2.5 * (0.4, 0.2) / 0.6 = (5/3, 5/6);
    # raw gates are route_scale times the selected scores
    s = np.array([[0.1, 0.2, 0.3, 0.4]])
    idx = np.array([[3, 1]])
    cfg_n = RouterCfg(n_routed=4, top_k=2, score="sigmoid", normalize=True, route_scale=2.5)
    np.testing.assert_allclose(oracle.gates_for(s, idx, cfg_n), [[5 / 3, 5 / 6]], rtol=1e-15)
    cfg_r = RouterCfg(n_routed=4, top_k=2, score="softmax", route_scale=2.0)
    np.testing.assert_allclose(oracle.gates_for(s, idx, cfg_r), [[0.8, 0.4]], rtol=1e-15)


@pytest.mark.parametrize("score,normalize,scale,G,TG", [("sigmoid", True, 2.5, 8, 4), ("softmax", False, 1.0, 1, 1),
                                                       ("sigmoid", False, 1.5, 4, 2), ("softmax", True, 1.0, 1, 1)])
def test_gates_for_reproduces_router_gates(score, normalize, scale, G, TG):
    # the gates the parity checker recomputes for a given selection equal the
    # router's own gates when handed the router's own selection, bit for bit
    rng = _rng(32)
    N, T, d = 32, 64, 16
    x = rng.standard_normal((T, d))
    W = rng.standard_normal((N, d)) / math.sqrt(d)
    b = rng.uniform(-0.1, 0.1, N)
    cfg = RouterCfg(n_routed=N, top_k=6, score=score, n_groups=G, topk_groups=TG, normalize=normalize,
                    route_scale=scale)
    r = oracle.route(x, W, b, cfg)
    assert np.array_equal(oracle.gates_for(r.scores, r.idx, cfg), r.gates)


# ------------------------------------------------------------ layer level ----

def _layer(rng, T, d, F, N, k, score, ns=0, normalize=False, route_scale=1.0, G=1, TG=1, bias=False):
    x = rng.standard_normal((T, d))
    W_r = rng.standard_normal((N, d)) / math.sqrt(d)
    b = rng.uniform(-0.1, 0.1, N) if bias else None
    W1, W3, W2 = _experts(rng, N, d, F)
    shared = None
    if ns:
        shared = tuple(a[0] for a in _experts(rng, 1, d, ns * F))
    cfg = RouterCfg(n_routed=N, top_k=k, score=score, normalize=normalize, route_scale=route_scale,
                    n_groups=G, topk_groups=TG)
    return x, W_r, b, (W1, W3, W2), shared, cfg


def test_dense_ceiling_identical_experts():
    # k = N with softmax: every expert on, gates are all the probabilities, which sum to 1;
    # with identical experts the routed output is the plain FFN ("all experts on" ceiling)
    rng = _rng(40)
    T, d, F, N = 20, 10, 14, 6
    x, W_r, b, (W1, W3, W2), _, cfg = _layer(rng, T, d, F, N, N, "softmax")
    y, r, idx, gates = oracle.forward(x, W_r, b, cfg, lambda e: (W1[0], W3[0], W2[0]))
    np.testing.assert_allclose(gates.sum(axis=1), 1.0, atol=1e-14)
    np.testing.assert_allclose(y, oracle.expert_ffn(x, W1[0], W3[0], W2[0]), rtol=1e-12, atol=1e-12)


def test_identical_experts_normalized_gates_give_route_scale_times_ffn_plus_shared():
    rng = _rng(41)
    T, d, F, N = 30, 12, 16, 32
    x, W_r, b, (W1, W3, W2), shared, cfg = _layer(rng, T, d, F, N, 8, "sigmoid", ns=1, normalize=True,
                                                  route_scale=2.5, G=8, TG=4, bias=True)
    y, *_ = oracle.forward(x, W_r, b, cfg, lambda e: (W1[3], W3[3], W2[3]), shared)
    want = 2.5 * oracle.expert_ffn(x, W1[3], W3[3], W2[3]) + oracle.expert_ffn(x, *shared)
    np.testing.assert_allclose(y, want, rtol=1e-12, atol=1e-12)
    # dropping the shared term must show
    y0, *_ = oracle.forward(x, W_r, b, cfg, lambda e: (W1[3], W3[3], W2[3]), None)
    assert np.abs(y - y0).max() > 1e-3


def test_idx_override_with_own_selection_is_plain_forward():
    # re-evaluating a layer with the router's own selection changes nothing (bitwise)
    rng = _rng(48)
    T, d, F, N = 24, 12, 10, 16
    x, W_r, b, (W1, W3, W2), shared, cfg = _layer(rng, T, d, F, N, 4, "sigmoid", ns=1, normalize=True,
                                                  route_scale=2.5, G=4, TG=2, bias=True)
    ex = lambda e: (W1[e], W3[e], W2[e])  # noqa: E731
    y, r, idx, gates = oracle.forward(x, W_r, b, cfg, ex, shared)
    y2, r2, idx2, gates2 = oracle.forward(x, W_r, b, cfg, ex, shared, idx_override=r.idx)
    assert np.array_equal(y2, y) and np.array_equal(idx2, idx) and np.array_equal(gates2, gates)
    # a shuffled slot order of the same selection is the same layer output
    perm = np.stack([rng.permutation(4) for _ in range(T)])
    y3, *_ = oracle.forward(x, W_r, b, cfg, ex, shared, idx_override=np.take_along_axis(r.idx, perm, axis=1))
    np.testing.assert_allclose(y3, y, rtol=1e-13, atol=1e-14)


def test_exact_tie_swapped_selection_hand_computed():
    # d = 2, d_ff = 1, three experts, top-1, sigmoid, raw gates. Experts 1 and 2
    # have the same router row (ln 3, 0), expert 0 a zero row, so for x = (1, 0)
    # the scores are (1/2, 3/4, 3/4): an exact tie between 1 and 2, which the
    # router resolves toward the lower index. Both experts have W1 = (ln 3, 0),
    # so g = ln 3 and silu(g) = (3/4) ln 3; W3 = (2, 0) / (4, 0) and
    # W2 = (1, 0)^T / (0, 1)^T give E_1 = (1.5 ln 3, 0) and E_2 = (0, 3 ln 3).
    # Gate 3/4: y = (9/8 ln 3, 0) with expert 1, (0, 9/4 ln 3) with expert 2.
    l3 = math.log(3.0)
    W_r = np.array([[0.0, 0.0], [l3, 0.0], [l3, 0.0]])
    W1 = np.array([[[l3, 0.0]], [[l3, 0.0]], [[l3, 0.0]]])
    W3 = np.array([[[1.0, 0.0]], [[2.0, 0.0]], [[4.0, 0.0]]])
    W2 = np.array([[[1.0], [1.0]], [[1.0], [0.0]], [[0.0], [1.0]]])
    x = np.array([[1.0, 0.0], [1.0, 0.0]])
    cfg = RouterCfg(n_routed=3, top_k=1, score="sigmoid")
    ex = lambda e: (W1[e], W3[e], W2[e])  # noqa: E731
    y, r, idx, gates = oracle.forward(x, W_r, None, cfg, ex)
    assert r.sel_tie.all() and idx.tolist() == [[1], [1]]
    np.testing.assert_allclose(gates, [[0.75], [0.75]], rtol=1e-15)
    np.testing.assert_allclose(y, [[9 / 8 * l3, 0.0], [9 / 8 * l3, 0.0]], rtol=1e-14, atol=1e-15)
    # the other valid selection for token 1 only
    y2, _, idx2, gates2 = oracle.forward(x, W_r, None, cfg, ex, routing=r, idx_override=np.array([[1], [2]]))
    np.testing.assert_allclose(gates2, [[0.75], [0.75]], rtol=1e-15)
    np.testing.assert_allclose(y2, [[9 / 8 * l3, 0.0], [0.0, 9 / 4 * l3]], rtol=1e-14, atol=1e-15)


def test_segmentation_identity_single_expert():
    rng = _rng(42)
    d, F, m = 16, 24, 4
    x = rng.standard_normal((9, d))
    W1, W3, W2 = (a[0] for a in _experts(rng, 1, d, F))
    parts = oracle.segment_expert(W1, W3, W2, m)
    total = sum(oracle.expert_ffn(x, *p) for p in parts)
    np.testing.assert_allclose(total, oracle.expert_ffn(x, W1, W3, W2), rtol=1e-12, atol=1e-12)


def test_segmentation_identity_whole_layer():
    # N experts, top-k, normalised softmax gates == mN slices with each parent's router
    # row replicated m times and top-mk ("The DeepSeekMoE Architecture.", Idea 1). Each
    # slice then scores s_e / m, so the slices of one parent share its gate only with a
    # route scale of m: the segmented layer with route_scale m equals the original.
    rng = _rng(43)
    T, d, F, N, k, m = 25, 10, 12, 8, 2, 3
    x, W_r, b, (W1, W3, W2), _, cfg = _layer(rng, T, d, F, N, k, "softmax", normalize=True)
    y, r, *_ = oracle.forward(x, W_r, None, cfg, lambda e: (W1[e], W3[e], W2[e]))
    sl = [oracle.segment_expert(W1[e], W3[e], W2[e], m) for e in range(N)]
    W_r_seg = np.repeat(W_r, m, axis=0)
    cfg_seg = RouterCfg(n_routed=m * N, top_k=m * k, score="softmax", normalize=True, route_scale=m)
    y_seg, r_seg, idx_seg, _ = oracle.forward(x, W_r_seg, None, cfg_seg, lambda e: sl[e // m][e % m])
    np.testing.assert_allclose(y_seg, y, rtol=1e-11, atol=1e-12)
    for t in range(T):
        assert set((idx_seg[t] // m).tolist()) == set(r.idx[t].tolist())


def test_shared_fusion_identity():
    # n_s shared experts equal one MLP of width n_s * d_ff (the excerpt's fused shared MLP)
    rng = _rng(44)
    d, F, ns = 10, 8, 3
    x = rng.standard_normal((7, d))
    parts = [tuple(a[0] for a in _experts(rng, 1, d, F)) for _ in range(ns)]
    fused = (np.concatenate([p[0] for p in parts]), np.concatenate([p[1] for p in parts]),
             np.concatenate([p[2] for p in parts], axis=1))
    np.testing.assert_allclose(oracle.expert_ffn(x, *fused), sum(oracle.expert_ffn(x, *p) for p in parts),
                               rtol=1e-12, atol=1e-12)


def test_gshard_two_experts_closed_form():
    # m=1, no shared expert, softmax top-2 of 2 experts, unnormalised: gate of expert 0 is
    # sigma(z0 - z1), so y = sigma(z0-z1) FFN_0 + sigma(z1-z0) FFN_1
    rng = _rng(45)
    T, d, F = 12, 6, 9
    x, W_r, b, (W1, W3, W2), _, cfg = _layer(rng, T, d, F, 2, 2, "softmax")
    y, r, idx, gates = oracle.forward(x, W_r, None, cfg, lambda e: (W1[e], W3[e], W2[e]))
    z = x @ W_r.T
    p0 = 1.0 / (1.0 + np.exp(z[:, 1] - z[:, 0]))
    want = p0[:, None] * oracle.expert_ffn(x, W1[0], W3[0], W2[0]) + \
        (1 - p0)[:, None] * oracle.expert_ffn(x, W1[1], W3[1], W2[1])
    np.testing.assert_allclose(y, want, rtol=1e-11, atol=1e-12)


def test_expert_and_token_permutation_equivariance():
    rng = _rng(46)
    T, d, F, N = 40, 12, 10, 16
    x, W_r, b, (W1, W3, W2), shared, cfg = _layer(rng, T, d, F, N, 4, "sigmoid", ns=1, normalize=True,
                                                  route_scale=2.5, bias=True)
    y, r, *_ = oracle.forward(x, W_r, b, cfg, lambda e: (W1[e], W3[e], W2[e]), shared)
    # relabel experts: new label j holds old expert pi[j]
    pi = rng.permutation(N)
    y2, r2, *_ = oracle.forward(x, W_r[pi], b[pi], cfg, lambda j: (W1[pi[j]], W3[pi[j]], W2[pi[j]]), shared)
    np.testing.assert_allclose(y2, y, rtol=1e-12, atol=1e-12)
    assert (pi[r2.idx] == r.idx).all()
    # reorder tokens
    sigma = rng.permutation(T)
    y3, *_ = oracle.forward(x[sigma], W_r, b, cfg, lambda e: (W1[e], W3[e], W2[e]), shared)
    np.testing.assert_allclose(y3, y[sigma], rtol=1e-12, atol=1e-12)


def test_permutation_against_sorted_pairs():
    rng = _rng(47)
    T, N, k = 300, 24, 5
    idx = np.stack([rng.choice(N, size=k, replace=False) for _ in range(T)])
    counts, offsets, perm = oracle.permutation(idx, N)
    pairs = sorted((int(idx[t, s]), t, s) for t in range(T) for s in range(k))
    assert [t * k + s for (_, t, s) in pairs] == perm.tolist()
    assert counts.tolist() == [sum(1 for p in pairs if p[0] == e) for e in range(N)]
    assert offsets[0] == 0 and offsets[-1] == T * k


# --------------------------------------------------- bias update (balancing) --

def test_bias_update_hand_example():
    # N = 4 experts, T = 6 tokens, k = 2: mean load 3 pairs per expert.
    # counts 5 (over), 3 (at the mean), 2 and 2 (under) -> -g, 0, +g, +g
    b = np.array([0.25, -0.5, 0.0, 1.0])
    got = oracle.bias_update(b, np.array([5, 3, 2, 2]), T=6, k=2, gamma=0.125)
    assert np.array_equal(got, [0.125, -0.5, 0.125, 1.125])


def test_bias_update_properties():
    rng = np.random.default_rng(7)
    for _ in range(20):
        N, T, k = 16, int(rng.integers(1, 64)), int(rng.integers(1, 5))
        # a random assignment of T*k pairs to experts
        counts = np.bincount(rng.integers(0, N, size=T * k), minlength=N)
        b = rng.normal(size=N)
        new = oracle.bias_update(b, counts, T, k, 1e-3)
        step = new - b
        mean = T * k / N
        assert np.all(step[counts > mean] < 0) and np.all(step[counts < mean] > 0)
        assert np.all(step[counts == mean] == 0)
        assert np.allclose(np.abs(step[counts != mean]), 1e-3)
    # a perfectly balanced batch leaves the bias alone
    assert np.array_equal(oracle.bias_update(np.ones(8), np.full(8, 3), T=12, k=2, gamma=0.5), np.ones(8))


# ------------------------------------------------------- FP8 weights ----

def test_e4m3_code_values_from_the_format_definition():
    # values fixed by the OCP FP8 E4M3 definition: zero, the smallest
    # subnormal 2^-9, the largest subnormal 7 * 2^-9, the smallest normal
    # 2^-6, one, 1.5, two, the largest finite 448, signs, NaN
    table = {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x38: 1.0, 0x3C: 1.5,
             0x40: 2.0, 0x7E: 448.0, 0xFE: -448.0, 0xB8: -1.0, 0x80: -0.0,
             0x4B: 5.5}  # 0x4B: exponent field 9 (2^2), mantissa 3 -> 1.375 * 4
    for code, want in table.items():
        got = oracle.e4m3_value(np.array([code], dtype=np.uint8))[0]
        assert got == want and np.signbit(got) == np.signbit(want), (hex(code), got, want)
    assert np.isnan(oracle.e4m3_value(np.array([0x7F, 0xFF], dtype=np.uint8))).all()
    # the 127 non-negative finite codes are strictly increasing, spaced by the
    # 3-bit mantissa step of their binade
    v = oracle.e4m3_value(np.arange(0, 0x7F, dtype=np.uint8))
    assert (np.diff(v) > 0).all()
    assert np.allclose(np.diff(v)[:8], 2.0 ** -9)
    # sign symmetry
    pos = np.arange(0, 0x7F, dtype=np.uint8)
    assert np.array_equal(oracle.e4m3_value(pos | 0x80), -v)


def test_fp8_block_dequant_hand_example():
    # a 128 x 256 matrix: two 128 x 128 blocks with scale bytes 127 (x1) and
    # 125 (x1/4); code 0x40 (2.0) becomes 2.0 and 0.5, code 0xB8 (-1.0) becomes
    # -1.0 and -0.25
    codes = np.full((128, 256), 0x40, dtype=np.uint8)
    codes[5, 7] = codes[9, 200] = 0xB8
    scales = np.array([[127, 125]], dtype=np.uint8)
    w = oracle.dequant_fp8(codes, scales)
    assert w.shape == (128, 256)
    assert w[0, 0] == 2.0 and w[127, 127] == 2.0 and w[0, 128] == 0.5 and w[127, 255] == 0.5
    assert w[5, 7] == -1.0 and w[9, 200] == -0.25
    # a 256 x 128 matrix with row blocks scaled by 2^3 and 2^-10
    codes2 = np.full((256, 128), 0x38, dtype=np.uint8)
    w2 = oracle.dequant_fp8(codes2, np.array([[130], [117]], dtype=np.uint8))
    assert (w2[:128] == 8.0).all() and (w2[128:] == 2.0 ** -10).all()
