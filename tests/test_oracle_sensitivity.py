"""Pins of the sensitivity score and the bit allocation.

KronQ summary (hyper.ai), "Method", Eq. 14: s = tr(H_G) tr(H_X) after BiIP;
Q, K, V share H_X, so tr(H_X) alone cannot separate them while the joint
score can.
"""

import numpy as np

from oracle import biip, sensitivity as S
from synth import get_config


def _spd(r, d, scale=1.0):
    A = r.standard_normal((d, 2 * d)) * scale
    return A @ A.T / (2 * d)


def test_score_is_trace_product_and_rotation_invariant():
    r = np.random.default_rng(1)
    m, n = 8, 16
    HX, HG = _spd(r, n), _spd(r, m, 3.0)
    W = r.standard_normal((m, n))
    su = (1 - 2 * r.integers(0, 2, m)).astype(np.int8)
    sv = (1 - 2 * r.integers(0, 2, n)).astype(np.int8)
    Wr, HXr, HGr, _, _ = biip.rescale(W, HX, HG, 0.25, "full")
    _, HXt, HGt = biip.rotate(Wr, HXr, HGr, su, sv)
    # tr is unchanged by the orthogonal step; only the rescale moves it
    np.testing.assert_allclose(np.trace(HXt), np.trace(HXr), rtol=1e-13)
    np.testing.assert_allclose(S.sensitivity(HXt, HGt), np.trace(HXr) * np.trace(HGr), rtol=1e-13)
    assert S.sensitivity(np.eye(3), 2 * np.eye(5)) == 30.0


def test_shared_input_tie_broken_by_gradients():
    r = np.random.default_rng(2)
    HX = _spd(r, 16)
    scores = [S.sensitivity(HX, _spd(r, 8, s)) for s in (1.0, 3.0, 0.5)]   # q, k, v
    assert len(set(scores)) == 3
    assert S.ranking(scores) == [1, 0, 2]
    assert [np.trace(HX)] * 3 == [np.trace(HX)] * 3   # tr(H_X) alone: a three-way tie


def test_ranking_ties_keep_decoder_order():
    assert S.ranking([1.0, 2.0, 2.0, 0.5]) == [1, 2, 0, 3]


def test_allocation_hand_example():
    # params 4, 4, 2; target average 3 -> budget 30 bit-params, base 20
    # order by score: idx 2 (+2 -> cost 4, used 24), idx 0 (+2 -> 32 > 30, +1 -> 28), idx 1 (+2 no, +1 no... 32 > 30)
    bits = S.allocate_bits([5.0, 1.0, 9.0], [4, 4, 2], 3.0)
    assert bits == [3, 2, 4]


def test_allocation_on_llama3_block_sizes_mixes_2_3_4():
    cfg = get_config("llama3-8b-block")
    params = [s.m * s.n for s in cfg.sublayers]
    r = np.random.default_rng(3)
    for _ in range(20):
        scores = list(r.permutation(len(params)).astype(float))
        bits = S.allocate_bits(scores, params, 3.0)
        avg = sum(b * p for b, p in zip(bits, params)) / sum(params)
        assert avg <= 3.0 + 1e-12
        assert set(bits) <= {2, 3, 4}
        # the most sensitive sublayer always gets the top width
        assert bits[S.ranking(scores)[0]] == 4
    # with the MLP on top the greedy rule reaches a genuine three-way mix
    scores = [1, 2, 3, 4, 7, 6, 5]        # q k v o gate up down
    bits = S.allocate_bits(scores, params, 3.0)
    assert set(bits) == {2, 3, 4}


def test_score_from_diagonals_equals_score_after_biip():
    r = np.random.default_rng(3)
    m, n = 24, 56
    HX, HG = _spd(r, n), _spd(r, m, 2.0)
    W = r.standard_normal((m, n)) * np.exp(r.uniform(-1, 1, n))[None, :]
    su = (1 - 2 * r.integers(0, 2, m)).astype(np.int8)
    sv = (1 - 2 * r.integers(0, 2, n)).astype(np.int8)
    for mode in ("full", "sv_only", "su_only", "no_rescale"):
        _, HXt, HGt, SX, SG = biip.biip(W, HX, HG, su, sv, 0.25, mode)
        np.testing.assert_allclose(S.sensitivity_from_diagonals(np.diag(HX), np.diag(HG), SX, SG),
                                   S.sensitivity(HXt, HGt), rtol=1e-12)


def test_oracle_allocation_is_the_lexicographic_maximum():
    """The greedy rule equals an exhaustive search: among all vectors in
    {2,3,4}^k whose parameter-weighted average stays at or below the target,
    the largest when read in descending score order."""
    import itertools
    r = np.random.default_rng(12)
    for _ in range(200):
        k = int(r.integers(1, 6))
        params = [int(p) for p in r.integers(1, 30, k)]
        scores = [float(s) for s in r.integers(0, 4, k)]
        target = float(r.choice([2.5, 3.0, 3.4]))
        order = S.ranking(scores)
        budget = round(target * sum(params))
        feas = [b for b in itertools.product((2, 3, 4), repeat=k)
                if sum(x * p for x, p in zip(b, params)) <= budget]
        best = max(feas, key=lambda b: tuple(b[i] for i in order))
        assert S.allocate_bits(scores, params, target) == list(best)
