"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Each check is chosen so that a plausible slip in the oracle (a dropped term, a
wrong sign or index, a transposed operand, a swapped gate/up matrix) fails at
least one of them. None re-types the oracle's own formula: they use values the
pages print, closed forms, brute force or a differently shaped evaluation.
"""
import itertools
import math

import numpy as np
import pytest

from oracle import moe_oracle as O
from tests.conftest import load_golden


def _floats(v):
    return [float(s) for s in (v if isinstance(v, list) else [v])]


# --- worked examples printed on the pages -----------------------------------

def test_worked_example_top2_gates():
    g = load_golden("worked_example_top2.txt")
    r = np.array([_floats(g["logits"])])
    k = int(g["k"])
    idx = O.top_k(r, k)
    assert sorted(idx[0].tolist()) == [int(s) for s in g["topk"]]
    gates = O.gates_softmax_topk(r, idx)[0]
    want = dict(zip([int(s) for s in g["topk"]], _floats(g["gates"])))
    for e, ge in zip(idx[0], gates):
        assert round(ge, int(g["decimals"])) == pytest.approx(want[int(e)], abs=1e-12)


def test_kevinluzbetak_softmax_topk_renormalise():
    g = load_golden("kevinluzbetak_routing.txt")
    r = np.array([_floats(g["logits"])])
    dec = int(g["decimals"])
    p = O.softmax_all(r)[0]
    assert [round(v, dec) for v in p] == pytest.approx(_floats(g["softmax"]), abs=1e-12)
    idx = O.top_k(r, int(g["k"]))
    assert idx[0].tolist() == [int(s) for s in g["topk"]]
    gates = O.gates_renormalised(O.softmax_all(r), idx)[0]
    assert [round(v, dec) for v in gates] == pytest.approx(_floats(g["gates"]), abs=1e-12)


def test_moatlab_router_two_of_sixty_four():
    g = load_golden("moatlab_router.txt")
    E = int(g["E"])
    r = np.full((1, E), -5.0)
    a, b = int(g["expert_a"]), int(g["expert_b"])
    r[0, a], r[0, b] = float(g["logit_a"]), float(g["logit_b"])
    idx = O.top_k(r, int(g["k"]))
    assert idx[0].tolist() == [a, b]
    gates = O.gates_softmax_topk(r, idx)[0]
    assert [round(v, int(g["decimals"])) for v in gates] == pytest.approx(_floats(g["gates"]))


def test_capacity_worked_example():
    g = load_golden("capacity_example.txt")
    T, E, k = int(g["T"]), int(g["E"]), int(g["k"])
    C = O.capacity_limit(float(g["capacity_factor"]), T, k, E)
    assert C == int(g["capacity"])
    # expert 0 is chosen by the first `chosen` tokens; the rest spread elsewhere
    chosen = int(g["chosen"])
    idx = np.zeros((T, k), dtype=np.int64)
    for t in range(T):
        idx[t] = [0, 1] if t < chosen else [2, 3]
    keep = O.capacity_keep(idx, E, C)
    dropped_e0 = int(((idx == 0) & ~keep).sum())
    assert dropped_e0 == int(g["overflow"])
    # the survivors are the earliest tokens
    assert keep[:C, 0].all() and not keep[C:chosen, 0].any()


def test_parameter_counts_exact():
    g = load_golden("param_counts.txt")
    for model in ("mixtral", "deepseek_v3"):
        cfg = {key.split(".", 1)[1]: int(v) for key, v in g.items() if key.startswith(model + ".")}
        cfg["tied"] = bool(cfg["tied"])
        total, active = O.moe_param_count(cfg)
        assert total == cfg["total"], model
        assert active == cfg["active"], model
        assert 3 * cfg["d"] * cfg["d_e"] == cfg["one_expert"]
        one_layer = dict(cfg, L=1, n_dense=0, V=0)
        t1, a1 = O.moe_param_count(one_layer)
        assert t1 - cfg["d"] == cfg["layer_total"]
        assert a1 - cfg["d"] == cfg["layer_active"]


def test_flop_accounting_matches_page():
    g = load_golden("flops_per_token.txt")
    d, E, de = int(g["d"]), int(g["E"]), int(g["d_e"])
    tol = float(g["rounding_millions"])
    router = 2 * d * E
    assert abs(router / 1e6 - float(g["router_flops_millions"])) < 0.05 + 1e-9
    nine = O.active_flops(int(g["experts_per_token"]), d, de)
    assert abs(nine / 1e6 - float(g["expert_flops_millions"])) <= tol


# --- closed forms -------------------------------------------------------------

def test_two_way_gate_is_sigmoid_of_gap():
    rng = np.random.default_rng(1)
    r = rng.normal(size=(50, 6))
    idx = O.top_k(r, 2)
    g = O.gates_softmax_topk(r, idx)
    ra = np.take_along_axis(r, idx, 1)
    assert np.allclose(g[:, 0], 1.0 / (1.0 + np.exp(-(ra[:, 0] - ra[:, 1]))), atol=1e-15)


def test_top1_renormalised_gate_is_one():
    rng = np.random.default_rng(2)
    r = rng.normal(size=(20, 8))
    g = O.gates_softmax_topk(r, O.top_k(r, 1))
    assert np.all(g == 1.0)


def test_silu_and_swiglu_scalar_closed_form():
    # d = d_e = 1: FFN(x) = SiLU(x w_g) * (x w_u) * w_d; SiLU(1) = sigma(1) = 0.7311
    # (the same sigmoid value the worked example prints for g_0).
    y = O.swiglu_ffn(np.array([[1.0]]), np.array([[1.0]]), np.array([[2.0]]), np.array([[3.0]]))
    assert y[0, 0] == pytest.approx(6.0 / (1.0 + math.exp(-1.0)), rel=1e-15)
    # swapping gate and up would give SiLU(2)*1*3
    assert abs(y[0, 0] - 3.0 * 2.0 / (1.0 + math.exp(-2.0))) > 0.5
    assert O.silu(np.array([0.0]))[0] == 0.0
    assert O.silu(np.array([-1000.0]))[0] == pytest.approx(0.0, abs=1e-300)


def test_swiglu_shapes_follow_linear_layout():
    # x [n,d], W_g/W_u [d_e,d], W_d [d,d_e]; a one-hot x selects column j of
    # W_g/W_u, so the output is W_d[:, h] weighted per hidden unit h.
    d, de = 3, 2
    Wg = np.arange(de * d, dtype=float).reshape(de, d) / 10
    Wu = np.ones((de, d))
    Wd = np.arange(d * de, dtype=float).reshape(d, de)
    x = np.array([[0.0, 1.0, 0.0]])
    y = O.swiglu_ffn(x, Wg, Wu, Wd)[0]
    a = Wg[:, 1]  # x W_g for the one-hot x
    h = a / (1 + np.exp(-a)) * 1.0
    assert np.allclose(y, [sum(Wd[i, j] * h[j] for j in range(de)) for i in range(d)], atol=1e-15)


# --- brute force and invariants ------------------------------------------------

def test_topk_brute_force_tiny():
    rng = np.random.default_rng(3)
    for E, k in [(4, 2), (5, 3), (6, 1), (6, 6)]:
        r = rng.normal(size=(30, E))
        idx = O.top_k(r, k)
        for t in range(30):
            best = max(itertools.combinations(range(E), k), key=lambda c: sum(r[t, list(c)]))
            assert sorted(idx[t].tolist()) == sorted(best)
            assert all(r[t, idx[t, s]] >= r[t, idx[t, s + 1]] for s in range(k - 1))


def test_topk_ties_go_to_lower_index():
    r = np.zeros((3, 8))
    assert O.top_k(r, 3).tolist() == [[0, 1, 2]] * 3
    r2 = np.array([[1.0, 3.0, 3.0, 0.0, 3.0]])
    assert O.top_k(r2, 2).tolist() == [[1, 2]]


def test_gates_sum_to_one_over_distinct_experts():
    rng = np.random.default_rng(4)
    r = rng.normal(size=(200, 16)) * 3
    for k in (1, 2, 4, 8):
        idx = O.top_k(r, k)
        g = O.gates_softmax_topk(r, idx)
        assert np.allclose(g.sum(1), 1.0, atol=1e-14)
        assert all(len(set(row)) == k for row in idx.tolist())
        assert np.all(g > 0)


def test_softmax_then_renormalise_equals_softmax_over_topk():
    rng = np.random.default_rng(5)
    r = rng.normal(size=(300, 32)) * 4
    for k in (1, 2, 8):
        idx = O.top_k(r, k)
        a = O.gates_softmax_topk(r, idx)
        b = O.gates_renormalised(O.softmax_all(r), idx)
        assert np.max(np.abs(a - b)) < 1e-14


def test_aux_is_exactly_one_for_uniform_router():
    # W_r = 0: every logit is 0, P_i = 1/E, top-k ties give experts 0..k-1,
    # and f sums to one, so E * sum f_i P_i = 1 exactly for E a power of two.
    rng = np.random.default_rng(6)
    for E, k in [(8, 2), (64, 1), (16, 4)]:
        x = rng.normal(size=(32, 16))
        res = O.moe_forward(x, np.zeros((E, 16)), lambda e: None, k, rows=np.array([], dtype=int))
        assert res.aux == 1.0
        assert res.counts.tolist() == [32] * k + [0] * (E - k)


def test_aux_extremes():
    # uniform f and P: 1; all tokens to one expert with P -> 1 there: -> E
    E, T, k = 8, 40, 1
    assert O.aux_statistic(np.full(E, T * k // E), np.full(E, T / E), T, k) == pytest.approx(1.0)
    counts = np.zeros(E)
    counts[3] = T
    probsum = np.zeros(E)
    probsum[3] = T
    assert O.aux_statistic(counts, probsum, T, k) == pytest.approx(E)


def _tiny_layer(rng, T=12, d=6, E=4, de=5, ds=0):
    x = rng.normal(size=(T, d))
    Wr = rng.normal(size=(E, d))
    Wg = rng.normal(size=(E, de, d))
    Wu = rng.normal(size=(E, de, d))
    Wd = rng.normal(size=(E, d, de))
    sh = None
    if ds:
        sh = (rng.normal(size=(ds, d)), rng.normal(size=(ds, d)), rng.normal(size=(d, ds)))
    return x, Wr, Wg, Wu, Wd, sh


def _dense_masked(x, Wr, Wg, Wu, Wd, k, sh=None, keep=None):
    """Run every expert on every token and weight it by a dense gate vector
    that is zero off the top-k (the check the worked example describes)."""
    T, E = x.shape[0], Wr.shape[0]
    r = (x @ Wr.T).astype(np.float32).astype(np.float64)
    y = np.zeros_like(x)
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-r[t, e], e))[:k]
        z = np.exp(np.array([r[t, e] for e in order]) - max(r[t, e] for e in order))
        dense_g = np.zeros(E)
        for j, e in enumerate(order):
            if keep is None or keep[t, j]:
                dense_g[e] = z[j] / z.sum()
        for e in range(E):
            a = x[t] @ Wg[e].T
            b = x[t] @ Wu[e].T
            h = a * (1 / (1 + np.exp(-a))) * b
            y[t] += dense_g[e] * (Wd[e] @ h)
        if sh is not None:
            a = x[t] @ sh[0].T
            y[t] += sh[2] @ (a * (1 / (1 + np.exp(-a))) * (x[t] @ sh[1].T))
    return y


@pytest.mark.parametrize("k,ds", [(1, 0), (2, 0), (3, 4), (4, 0)])
def test_sparse_loop_equals_dense_run_all_and_mask(k, ds):
    rng = np.random.default_rng(7 + k)
    x, Wr, Wg, Wu, Wd, sh = _tiny_layer(rng, ds=ds)
    res = O.moe_forward(x, Wr, lambda e: (Wg[e], Wu[e], Wd[e]), k, shared_weights=sh)
    ref = _dense_masked(x, Wr, Wg, Wu, Wd, k, sh)
    assert np.max(np.abs(res.y - ref)) < 1e-12


def test_capacity_drops_match_dense_mask_and_are_zero():
    rng = np.random.default_rng(11)
    T, E, k = 16, 4, 2
    x, Wr, Wg, Wu, Wd, _ = _tiny_layer(rng, T=T, E=E)
    Wr[0] += 3.0 * x.mean(0)  # skew toward expert 0 so the cut bites
    res = O.moe_forward(x, Wr, lambda e: (Wg[e], Wu[e], Wd[e]), k, capacity_factor=0.75)
    assert res.capacity == 6
    assert (~res.keep).any()
    ref = _dense_masked(x, Wr, Wg, Wu, Wd, k, keep=res.keep)
    assert np.max(np.abs(res.y - ref)) < 1e-12
    # a token whose every assignment is dropped gets exactly 0
    gone = ~res.keep.any(axis=1)
    assert np.all(res.y[gone] == 0.0)
    # with every assignment dropped the whole output is 0
    none = O.moe_forward(x, Wr, lambda e: (Wg[e], Wu[e], Wd[e]), k, capacity_factor=1e-9)
    assert none.capacity == 0 and np.all(none.y == 0.0)


def test_drop_order_hand_built_case():
    # T=8, E=2, k=1, cf=0.5 -> C = 2; the two lowest token indices per expert stay.
    idx = np.array([[1], [0], [1], [1], [0], [0], [1], [0]])
    C = O.capacity_limit(0.5, 8, 1, 2)
    assert C == 2
    keep = O.capacity_keep(idx, 2, C)[:, 0]
    assert keep.tolist() == [True, True, True, False, True, False, False, False]


def test_wide_ffn_is_sum_of_expert_blocks():
    # An MoE layer is a wide FFN with blocks switched off: summing every expert
    # with weight 1 equals one SwiGLU of width E*d_e with concatenated weights.
    rng = np.random.default_rng(12)
    x, _, Wg, Wu, Wd, _ = _tiny_layer(rng, E=3, de=4)
    blocks = sum(O.swiglu_ffn(x, Wg[e], Wu[e], Wd[e]) for e in range(3))
    wide_g = np.concatenate(list(Wg), axis=0)       # [E*d_e, d]
    wide_u = np.concatenate(list(Wu), axis=0)
    wide_d = np.concatenate(list(Wd), axis=1)       # [d, E*d_e]
    a = x @ wide_g.T
    wide = ((a / (1 + np.exp(-a))) * (x @ wide_u.T)) @ wide_d.T
    assert np.max(np.abs(blocks - wide)) < 1e-12


def test_router_logits_are_float32_rounded_exact_dot():
    rng = np.random.default_rng(13)
    x = rng.normal(size=(5, 64)).astype(np.float32)
    W = rng.normal(size=(3, 64)).astype(np.float32)
    r = O.router_logits(x, W)
    # brute force: exact rational sum via math.fsum, then one rounding to fp32
    for t in range(5):
        for e in range(3):
            exact = math.fsum(float(a) * float(b) for a, b in zip(x[t], W[e]))
            assert r[t, e] == float(np.float32(exact))
    bias = np.array([0.5, -1.0, 2.0], dtype=np.float32)
    rb = O.router_logits(x, W, bias)
    for t in range(5):
        for e in range(3):
            exact = math.fsum([float(a) * float(b) for a, b in zip(x[t], W[e])] + [float(bias[e])])
            assert rb[t, e] == float(np.float32(exact))


def test_aux_top1_variant_agrees_at_k1():
    rng = np.random.default_rng(14)
    x, Wr, Wg, Wu, Wd, _ = _tiny_layer(rng, T=40, E=4)
    res = O.moe_forward(x, Wr, lambda e: (Wg[e], Wu[e], Wd[e]), 1)
    assert res.aux == pytest.approx(O.aux_statistic_top1(res.idx, res.probs), rel=1e-14)


def test_dropped_fraction_from_counts():
    assert O.dropped_fraction(np.array([3000, 2000, 1500, 1692]), 2560, 4096, 2) == pytest.approx(440 / 8192)
    assert O.dropped_fraction(np.array([5, 5]), None, 5, 2) == 0.0


# --- the routing margin that decides which tokens parity compares ----------

def _separation_brute(row, k):
    """The largest gap by which some k-subset of `row` sits above the rest:
    max over k-subsets S of (min over S) - (max outside S). The top-k set
    attains it, so it is the k-th/(k+1)-th gap, found without sorting."""
    n = len(row)
    if k >= n:
        return math.inf
    best = -math.inf
    for S in itertools.combinations(range(n), k):
        inside = min(row[i] for i in S)
        outside = max(row[j] for j in range(n) if j not in S)
        best = max(best, inside - outside)
    return best


def test_topk_margin_brute_force_tiny():
    rng = np.random.default_rng(40)
    for E in (2, 3, 5, 7):
        r = rng.normal(size=(25, E))
        r[:5] = np.round(r[:5], 1)  # repeated values, ties at the cut included
        for k in range(1, E + 1):
            got = O.topk_margin(r, k)
            want = np.array([_separation_brute(list(row), k) for row in r])
            assert np.array_equal(got, want), (E, k)


def test_topk_margin_hand_cases():
    r = np.array([[5.0, 4.0, 2.0, 1.0],    # k=2: 4 - 2, not 2 - 1 nor 5 - 4
                  [1.0, 3.0, 3.0, 0.0],    # k=1: a tie at the cut gives 0
                  [0.5, 0.5, 0.5, 0.5]])
    assert O.topk_margin(r, 2).tolist() == [2.0, 2.0, 0.0]
    assert O.topk_margin(r, 1).tolist() == [1.0, 0.0, 0.0]
    assert np.isinf(O.topk_margin(r, 4)).all()


def test_group_gap_and_selection_gap_brute_force():
    # group scores and the kept groups by hand; both gaps by the subset brute force
    rng = np.random.default_rng(41)
    E, n_group, topk_group, k = 12, 4, 2, 3
    gsize = E // n_group
    sel = rng.normal(size=(50, E))
    sel[:6] = np.round(sel[:6], 1)
    el, gap = O.group_eligible(sel, n_group, topk_group)
    idx, kgap = O.select_experts(sel, k, el)
    for t in range(50):
        gbest = [max(sel[t, g * gsize:(g + 1) * gsize]) for g in range(n_group)]
        assert gap[t] == _separation_brute(gbest, topk_group)
        groups = sorted(range(n_group), key=lambda g: (-gbest[g], g))[:topk_group]
        allowed = [e for e in range(E) if e // gsize in groups]
        assert el[t].tolist() == [e in allowed for e in range(E)]
        assert kgap[t] == _separation_brute([sel[t, e] for e in allowed], k)
    # every group kept, or one pick per allowed expert: no gap can matter
    assert np.isinf(O.group_eligible(sel, n_group, n_group)[1]).all()
    _, kg = O.select_experts(sel, topk_group * gsize, el)
    assert np.isinf(kg).all()


def test_layer_margin_is_the_smaller_gap_on_the_selection_scores():
    # the layer's margin is taken on what the top-k ranks (affinity + selection
    # bias in sigmoid mode), and is the smaller of the group and the expert gap
    rng = np.random.default_rng(42)
    T, d, E, k, ng, tg = 30, 8, 8, 2, 4, 2
    x = rng.normal(size=(T, d))
    Wr = rng.normal(size=(E, d))
    b = rng.normal(scale=0.05, size=E)
    res = O.moe_forward(x, Wr, lambda e: None, k, rows=np.array([], dtype=int),
                        gate_mode=O.GATE_SIGMOID, selection_bias=b, n_group=ng, topk_group=tg)
    gsize = E // ng
    for t in range(T):
        s = [1.0 / (1.0 + math.exp(-res.logits[t, e])) + b[e] for e in range(E)]
        gbest = [max(s[g * gsize:(g + 1) * gsize]) for g in range(ng)]
        groups = sorted(range(ng), key=lambda g: (-gbest[g], g))[:tg]
        allowed = [s[e] for e in range(E) if e // gsize in groups]
        want = min(_separation_brute(gbest, tg), _separation_brute(allowed, k))
        assert res.margin[t] == pytest.approx(want, rel=1e-12, abs=1e-15)
    # with plain renormalised routing it is the logit gap
    res0 = O.moe_forward(x, Wr, lambda e: None, k, rows=np.array([], dtype=int))
    want0 = [_separation_brute(list(res0.logits[t]), k) for t in range(T)]
    assert res0.margin.tolist() == want0
