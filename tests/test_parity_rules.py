"""The near-tie bookkeeping of the parity tests (tests/parity_util.py), on CPU.

Where a token's k-th/(k+1)-th selection gap is below the comparison margin,
the layer may pick either expert set. Under a capacity limit that can move
the cut of the two contested experts by one rank for every later token of
theirs, and of no other expert. These cases check that exactly the tokens
whose kept/dropped status is then uncertain are left out of the comparison,
and that every other token is compared."""
import itertools

import numpy as np

from oracle import moe_oracle as O
from sparse_mixture_experts_aux_b200.inputs import Workload
from tests.parity_util import MARGIN, contested_experts, unaffected_tokens


def _ref(logits, k, C):
    r = np.asarray(logits, dtype=np.float64)
    idx = O.top_k(r, k)
    return O.OracleResult(logits=r, idx=idx, margin=O.topk_margin(r, k), capacity=C,
                          keep=O.capacity_keep(idx, r.shape[1], C))


def test_hand_built_switch_case():
    # E=2, k=1, C=2; token 1 ties between experts 0 and 1
    eps = MARGIN / 4
    r = [[1, 0], [eps, 0], [1, 0], [1, 0], [0, 1], [0, 1]]
    ref = _ref(r, 1, 2)
    w = Workload("hand", 6, 2, 2, 2, 1)
    con = contested_experts(ref, w)
    assert list(con) == [1] and con[1].tolist() == [True, True]
    ok = unaffected_tokens(ref, con)
    # t0 before the tie; t2 (rank 2 of expert 0) kept if token 1 moved away;
    # t3 (rank 3) dropped either way; t4 (rank 0 of expert 1) kept either way;
    # t5 (rank 1 of expert 1) dropped if token 1 moved there
    assert ok.tolist() == [True, False, False, True, True, False]


def test_other_experts_are_untouched():
    # the tie is between experts 0 and 1; expert 2's cut cannot move
    eps = MARGIN / 4
    r = [[eps, 0, -5], [0, 0, 5], [0, 0, 5], [0, 0, 5], [1, 0, -5]]
    ref = _ref(r, 1, 2)
    con = contested_experts(ref, Workload("hand", 5, 2, 3, 2, 1))
    assert con[0].tolist() == [True, True, False]
    ok = unaffected_tokens(ref, con)
    # tokens 1..3 go to expert 2, the third one over C: no near-tie contests it.
    # Token 4 (expert 0, rank 1) can only move down to rank 0 if token 0 leaves
    # expert 0, so it is kept either way.
    assert ok.tolist() == [False, True, True, True, True]
    assert ref.keep[:, 0].tolist() == [True, True, True, False, True]


def test_exclusion_is_exact_against_every_alternative_choice():
    # brute force: let every near-tie token pick any expert of its contested band
    # and recompute the keep mask; tokens whose status never changes must be the
    # ones marked unaffected (among those that are not near-ties themselves)
    rng = np.random.default_rng(7)
    for trial in range(30):
        T, E, C = 14, 3, 3
        r = rng.normal(size=(T, E)).round(0)  # many exact ties
        ref = _ref(r, 1, C)
        con = contested_experts(ref, Workload("bf", T, 2, E, 2, 1))
        near = sorted(con)
        options = [np.nonzero(con[t])[0].tolist() for t in near]
        statuses = set()
        stable = np.ones(T, dtype=bool)
        base = None
        for pick in itertools.product(*options):
            idx = ref.idx.copy()
            for t, e in zip(near, pick):
                idx[t, 0] = e
            keep = O.capacity_keep(idx, E, C)[:, 0]
            if base is None:
                base = keep
            stable &= keep == base
        ok = unaffected_tokens(ref, con)
        clear = ref.margin > MARGIN
        assert (ok <= (stable & clear)).all()          # never compares an uncertain token
        assert (ok == (stable & clear)).all(), trial   # and drops no certain one (k = 1)


def test_exclusion_never_compares_an_uncertain_token_k2():
    rng = np.random.default_rng(8)
    for trial in range(30):
        T, E, C, k = 10, 4, 4, 2
        r = rng.normal(size=(T, E)).round(0)
        ref = _ref(r, k, C)
        con = contested_experts(ref, Workload("bf", T, 2, E, 2, k))
        near = sorted(con)
        options = []
        for t in near:
            band = np.nonzero(con[t])[0].tolist()
            above = [e for e in ref.idx[t] if e not in band]
            options.append([tuple(above) + c for c in
                            itertools.combinations(band, k - len(above))])
        stable = np.ones(T, dtype=bool)
        base = None
        for pick in itertools.product(*options):
            idx = ref.idx.copy()
            for t, choice in zip(near, pick):
                idx[t] = sorted(choice)
            keep = O.capacity_keep(idx, E, C)
            if base is None:
                base = keep
            stable &= (keep == base).all(axis=1)
        ok = unaffected_tokens(ref, con)
        assert (ok <= (stable & (ref.margin > MARGIN))).all(), trial
