"""The product's 2/3/4-bit allocation (post_quantization_02_b200.alloc),
pinned on its own: hand-worked budgets, and an exhaustive search that
defines the rule independently of any greedy loop (the chosen bit vector,
read in descending score order, is the lexicographically largest of all
vectors in {2,3,4}^k whose parameter-weighted average stays at or below the
target).  KronQ summary (hyper.ai), "Method" (Eq. 14): more bits for larger
s = tr(H_G) tr(H_X)."""

import itertools

import numpy as np
import pytest

from post_quantization_02_b200 import alloc


def _lex_max(scores, params, target):
    order = sorted(range(len(scores)), key=lambda i: (-scores[i], i))
    budget = round(target * sum(params))
    best = None
    for bits in itertools.product((2, 3, 4), repeat=len(scores)):
        if sum(b * p for b, p in zip(bits, params)) > budget:
            continue
        key = tuple(bits[i] for i in order)
        if best is None or key > best[0]:
            best = (key, list(bits))
    return best[1]


def test_hand_worked_budget():
    # params 4, 4, 2 at an average of 3: 30 bit-params, 20 at the base width,
    # 10 spare.  Index 2 (score 9) takes +2 (4 spent, 6 left); index 0 takes
    # +1 (4 more would need 8); index 1 finds 2 left, less than its 4 params.
    assert alloc.allocate_bits([5.0, 1.0, 9.0], [4, 4, 2], 3.0) == [3, 2, 4]


def test_a_plus_two_jump_and_an_exact_fit():
    # 10 spare over params 5, 5: the first takes +2 (10), nothing is left.
    assert alloc.allocate_bits([1.0, 2.0], [5, 5], 3.0) == [2, 4]
    # 3 params x 3 = 9 spare; +2 on 3 leaves 3 for the next: exactly +1.
    assert alloc.allocate_bits([3.0, 2.0, 1.0], [3, 3, 3], 3.0) == [4, 3, 2]


def test_ties_keep_the_given_order():
    assert alloc.rank([1.0, 2.0, 2.0, 0.5]) == [1, 2, 0, 3]
    assert alloc.allocate_bits([1.0, 1.0, 1.0], [4, 4, 4], 3.0) == [4, 3, 2]


def test_single_sublayer_and_extremes():
    assert alloc.allocate_bits([7.0], [100], 3.0) == [3]
    assert alloc.allocate_bits([7.0, 1.0], [100, 100], 2.0) == [2, 2]
    assert alloc.allocate_bits([7.0, 1.0], [100, 100], 4.0) == [4, 4]
    with pytest.raises(ValueError):
        alloc.allocate_bits([1.0], [10], 1.5)


def test_equals_the_exhaustive_lexicographic_maximum():
    r = np.random.default_rng(11)
    for _ in range(300):
        k = int(r.integers(1, 7))
        params = [int(p) for p in r.integers(1, 40, k)]
        scores = [float(s) for s in r.integers(0, 5, k)]       # many ties
        target = float(r.choice([2.25, 2.5, 3.0, 3.3, 3.75]))
        assert alloc.allocate_bits(scores, params, target) == _lex_max(scores, params, target)


def test_llama3_block_sizes_reach_a_real_mix():
    # q k v o gate up down of the LLaMA-3-8B-shaped block, MLP most sensitive
    params = [4096 * 4096, 1024 * 4096, 1024 * 4096, 4096 * 4096, 14336 * 4096, 14336 * 4096,
              4096 * 14336]
    bits = alloc.allocate_bits([1, 2, 3, 4, 7, 6, 5], params, 3.0)
    assert set(bits) == {2, 3, 4}
    assert sum(b * p for b, p in zip(bits, params)) <= 3 * sum(params)
