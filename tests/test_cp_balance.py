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


def _max_work(cost, a):
    return max(sum(int(cost[c]) for c in x) for x in a)


def test_swap_refinement_valid_and_never_worse():
    r = np.random.default_rng(3)
    for trial in range(200):
        ranks, per = int(r.integers(2, 9)), int(r.integers(1, 4))
        cost = r.integers(0, 10 ** int(r.integers(1, 7)), ranks * per)
        lpt = cb.assign_longest_first(cost, ranks, per)
        ref = cb.refine_by_swaps(cost, lpt)
        assert sorted(c for x in ref for c in x) == list(range(ranks * per))
        assert all(len(x) == per and x == sorted(x) for x in ref)
        assert _max_work(cost, ref) <= _max_work(cost, lpt)
        # a local optimum: no single exchange with the heaviest rank lowers the pair below the max
        w = [sum(int(cost[c]) for c in x) for x in ref]
        hi = int(np.argmax(w))
        for rr in range(ranks):
            if rr != hi:
                for a in ref[hi]:
                    for b in ref[rr]:
                        d = int(cost[a]) - int(cost[b])
                        assert d <= 0 or max(w[hi] - d, w[rr] + d) >= w[hi]


def test_swap_refinement_reaches_optimum_small():
    """Brute force on 8 chunks, 4 ranks x 2: the refined assignment is optimal in most draws and
    within the LPT bound in all."""
    r = np.random.default_rng(4)
    hits = 0
    for _ in range(40):
        cost = [int(x) for x in r.integers(0, 100, 8)]
        ref = cb.refine_by_swaps(cost, cb.assign_longest_first(cost, 4, 2))
        opt = _best(cost, 4, 2)
        got = _max_work(cost, ref)
        assert got <= opt * 4 / 3 + 1e-9
        hits += got == opt
    assert hits >= 30


def test_swap_refinement_on_document_mask_costs():
    """Per-chunk work of a long-document mask (32 chunks, 16 ranks x 2), from the oracle's counts:
    dual-chunk >= longest-first >= refined, and the refined maximum is within 5% of the lower bound
    max(total / ranks, largest chunk + smallest chunk) (the rank holding the largest chunk holds
    one more)."""
    N, chunk = 32768, 1024
    spec = synth.mask_causal_document(N, synth.draw_docs(synth.Rng(11), N, 512, 16384))
    v = spec.vectors()
    cost = []
    for c in range(N // chunk):
        loc = [oracle.localize(x, [c * chunk], [chunk]) for x in v]
        cost.append(int(oracle.kv_chunk_pairs(chunk, N, N, *loc).sum()))
    dual = cb.imbalance(cost, cb.dual_chunk(len(cost)))
    lpt_a = cb.assign_longest_first(cost, 16, 2)
    lpt = cb.imbalance(cost, lpt_a)
    ref = cb.imbalance(cost, cb.refine_by_swaps(cost, lpt_a))
    assert ref <= lpt <= dual + 1e-12
    srt = sorted(cost)
    bound = max(sum(cost) / 16, srt[-1] + srt[0]) / (sum(cost) / 16)
    assert ref <= bound * 1.05, (dual, lpt, ref, bound)


def test_balance_report_keys_and_order():
    """The report the bench prints: bound <= refined <= longest-first <= dual-chunk on skewed costs."""
    r = np.random.default_rng(9)
    cost = (r.pareto(1.5, 32) * 1e6).astype(np.int64)
    rep = cb.balance_report(cost, 16, 2)
    assert set(rep) == {"ranks", "chunks_per_rank", "dual_chunk_max_over_mean", "longest_first_max_over_mean",
                        "refined_max_over_mean", "lower_bound_max_over_mean"}
    assert rep["lower_bound_max_over_mean"] <= rep["refined_max_over_mean"] <= rep["longest_first_max_over_mean"]
    assert rep["longest_first_max_over_mean"] <= rep["dual_chunk_max_over_mean"] + 1e-4
    rep4 = cb.balance_report(cost, 8, 4)
    assert "dual_chunk_max_over_mean" not in rep4 and rep4["lower_bound_max_over_mean"] <= rep4["refined_max_over_mean"]
