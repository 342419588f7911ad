"""Pins of the oracle's routing variants: raw softmax gates (Switch), the
selection-only bias (DeepSeek-V3 balancing), sigmoid affinities normalised over
the chosen experts and group-limited selection (DeepSeek-V3)."""
import itertools
import math

import numpy as np
import pytest

from oracle import moe_oracle as O
from tests.conftest import load_golden


def _floats(v):
    return [float(s) for s in (v if isinstance(v, list) else [v])]


def test_raw_gates_are_the_printed_softmax():
    # kevinluzbetak worked example: without renormalisation the top-2 gates are
    # the printed softmax values of experts 1 and 2 (indices 0, 1).
    g = load_golden("kevinluzbetak_routing.txt")
    r = np.array([_floats(g["logits"])])
    dec = int(g["decimals"])
    idx = O.top_k(r, 2)
    raw = O.gates_for_mode(r, idx, O.GATE_RAW)[0]
    assert [round(v, dec) for v in raw] == pytest.approx(_floats(g["softmax"])[:2])
    # Switch top-1: the kept gate is the largest probability itself
    top1 = O.gates_for_mode(r, O.top_k(r, 1), O.GATE_RAW)[0, 0]
    assert top1 == pytest.approx(math.exp(2.0) / sum(math.exp(v) for v in _floats(g["logits"])))


def test_sigmoid_gates_closed_form():
    r = np.array([[0.0, math.log(3.0)]])  # affinities 1/2 and 3/4
    idx = O.select_experts(O.selection_scores(r, O.GATE_SIGMOID), 2, np.ones((1, 2), bool))[0]
    assert idx.tolist() == [[1, 0]]
    g = O.gates_for_mode(r, idx, O.GATE_SIGMOID)[0]
    assert g.tolist() == pytest.approx([0.6, 0.4], abs=1e-15)
    g1 = O.gates_for_mode(r, idx[:, :1], O.GATE_SIGMOID)
    assert g1[0, 0] == 1.0


def test_selection_bias_changes_choice_not_weights():
    r = np.array([[1.0, 0.9]])
    b = np.array([0.0, 0.2])
    sel = O.selection_scores(r, O.GATE_RENORM, b)
    idx1, _ = O.select_experts(sel, 1, np.ones((1, 2), bool))
    assert idx1.tolist() == [[1]]  # 0.9 + 0.2 beats 1.0
    assert O.gates_for_mode(r, idx1, O.GATE_RENORM)[0, 0] == 1.0
    idx2, _ = O.select_experts(sel, 2, np.ones((1, 2), bool))
    g = O.gates_for_mode(r, idx2, O.GATE_RENORM)[0]
    # weights come from the unbiased logits: sigma(-0.1), sigma(0.1)
    assert g.tolist() == pytest.approx([1 / (1 + math.exp(0.1)), 1 / (1 + math.exp(-0.1))])
    # and the balance probabilities ignore the selection bias
    assert np.allclose(O.balance_probs(r, O.GATE_RENORM), O.softmax_all(r))


def test_group_limit_special_cases():
    rng = np.random.default_rng(20)
    sel = rng.normal(size=(40, 16))
    # every group kept: plain top-k
    el, gm = O.group_eligible(sel, 4, 4)
    assert el.all() and np.isinf(gm).all()
    idx, _ = O.select_experts(sel, 5, el)
    assert (idx == O.top_k(sel, 5)).all()
    # one expert per group, as many groups as picks: the plain top-k again
    el, _ = O.group_eligible(sel, 16, 5)
    idx, _ = O.select_experts(sel, 5, el)
    assert (idx == O.top_k(sel, 5)).all()


def test_group_limit_brute_force():
    rng = np.random.default_rng(21)
    E, n_group, topk_group, k = 12, 4, 2, 3
    gsize = E // n_group
    sel = rng.normal(size=(60, E))
    el, _ = O.group_eligible(sel, n_group, topk_group)
    idx, _ = O.select_experts(sel, k, el)
    for t in range(60):
        gbest = [max(sel[t, g * gsize:(g + 1) * gsize]) for g in range(n_group)]
        groups = sorted(range(n_group), key=lambda g: (-gbest[g], g))[:topk_group]
        allowed = [e for e in range(E) if e // gsize in groups]
        best = max(itertools.combinations(allowed, k), key=lambda c: sum(sel[t, list(c)]))
        assert sorted(idx[t].tolist()) == sorted(best)


def test_deepseek_v3_group_configuration():
    g = load_golden("deepseek_v3_routing.txt")
    E, k, ng, tg = (int(g[n]) for n in ("E", "k", "n_group", "topk_group"))
    rng = np.random.default_rng(22)
    r = rng.normal(size=(100, E))
    sel = O.selection_scores(r, O.GATE_SIGMOID, rng.normal(scale=0.05, size=E))
    el, _ = O.group_eligible(sel, ng, tg)
    idx, _ = O.select_experts(sel, k, el)
    gsize = E // ng
    for t in range(100):
        assert len({e // gsize for e in idx[t]}) <= tg
        assert len(set(idx[t].tolist())) == k
    gates = O.gates_for_mode(r, idx, O.GATE_SIGMOID)
    assert np.allclose(gates.sum(axis=1), 1.0, atol=1e-14) and (gates > 0).all()


def test_sigmoid_mode_aux_is_one_for_uniform_router():
    x = np.random.default_rng(23).normal(size=(32, 8))
    res = O.moe_forward(x, np.zeros((16, 8)), lambda e: None, 4, rows=np.array([], dtype=int),
                        gate_mode=O.GATE_SIGMOID, n_group=4, topk_group=2)
    assert res.aux == 1.0
    assert res.counts.tolist() == [32] * 4 + [0] * 12


def test_variant_layer_matches_dense_masked_evaluation():
    # the sparse loop with every variant on equals running all experts and
    # weighting them by a dense gate vector built from the chosen set
    rng = np.random.default_rng(24)
    T, d, E, de, k = 10, 6, 8, 5, 3
    x = rng.normal(size=(T, d))
    Wr = rng.normal(size=(E, d))
    Wg, Wu, Wd = rng.normal(size=(E, de, d)), rng.normal(size=(E, de, d)), rng.normal(size=(E, d, de))
    b = rng.normal(scale=0.3, size=E)
    for mode in (O.GATE_RENORM, O.GATE_RAW, O.GATE_SIGMOID):
        res = O.moe_forward(x, Wr, lambda e: (Wg[e], Wu[e], Wd[e]), k, gate_mode=mode,
                            selection_bias=b, n_group=4, topk_group=2)
        dense = np.zeros((T, E))
        np.put_along_axis(dense, res.idx, res.gates, axis=1)
        ref = np.zeros((T, d))
        for e in range(E):
            ref += dense[:, e:e + 1] * O.swiglu_ffn(x, Wg[e], Wu[e], Wd[e])
        assert np.max(np.abs(res.y - ref)) < 1e-12
