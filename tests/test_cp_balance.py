"""Host logic of the sparsity-aware chunk assignment (no GPU): the longest-first
assignment is a valid partition with equal chunks per rank, never worse than
dual-chunk on skewed costs, optimal on small cases checked by brute force, and
chunk costs from the oracle's per-chunk counts add up to the mask's pairs."""
import itertools

import numpy as np
import pytest

import oracle
import synth
from mask_aware_flash_b200 import cp_balance as cb


def test_partition_and_order():
    r = np.random.default_rng(1)
    cost = r.integers(0, 1000, 32)
    a = cb.assign_longest_first(cost, 16, 2)
    assert sorted(c for x in a for c in x) == list(range(32))
    assert all(len(x) == 2 and x == sorted(x) for x in a)
    assert cb.dual_chunk(8) == [[0, 7], [1, 6], [2, 5], [3, 4]]
    with pytest.raises(ValueError):
        cb.assign_longest_first(cost, 15, 2)


def _best(cost, ranks, per_rank):
    """Brute force: the minimum max-work over all partitions into equal groups (tiny sizes)."""
    n = len(cost)
    best = None

    def rec(left, groups):
        nonlocal best
        if not left:
            m = max(sum(cost[c] for c in g) for g in groups)
            best = m if best is None else min(best, m)
            return
        first = left[0]
        for rest in itertools.combinations(left[1:], per_rank - 1):
            g = (first,) + rest
            rec([c for c in left if c not in g], groups + [g])

    rec(list(range(n)), [])
    return best


def test_longest_first_near_optimal_small():
    r = np.random.default_rng(2)
    for _ in range(30):
        cost = [int(x) for x in r.integers(0, 100, 8)]
        a = cb.assign_longest_first(cost, 4, 2)
        got = max(sum(cost[c] for c in x) for x in a)
        opt = _best(cost, 4, 2)
        assert got <= opt * 4 / 3 + 1e-9  # the LPT bound (Graham) for identical machines


def test_costs_from_oracle_and_skewed_masks():
    N, chunk = 4096, 256
    spec = synth.mask_causal_document(N, synth.draw_docs(synth.Rng(7), N, 256, 2048))
    v = spec.vectors()
    # per query chunk: localize it as its own rank, count its pairs over all keys
    cost = []
    for c in range(N // chunk):
        loc = [oracle.localize(x, [c * chunk], [chunk]) for x in v]
        cost.append(int(oracle.kv_chunk_pairs(chunk, N, N, *loc).sum()))
    assert sum(cost) == oracle.count_unmasked_dense(N, N, *v)
    dual = cb.imbalance(cost, cb.dual_chunk(len(cost)))
    lpt = cb.imbalance(cost, cb.assign_longest_first(cost, len(cost) // 2, 2))
    assert lpt <= dual + 1e-12
    assert lpt < 1.1
