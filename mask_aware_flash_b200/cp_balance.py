"""Sparsity-aware assignment of query chunks to context-parallel ranks.

FlashMask-3 explainer (learnaivisually.com), across-ranks paragraph: under
expressive masks the work no longer grows smoothly with position, so the paper
adds a sparsity-aware load balancer (HCC-IPO) to avoid stragglers; the pages
give no algorithm for it.  Here the cost of a query chunk is its exact number
of unmasked (row, key) pairs, measured on the GPU by localizing every chunk as
a rank of its own (clip-shift-max) and summing that rank's KV-chunk pair
counts; an assignment is then scored by max / mean work over the ranks.

`assign_longest_first` is longest-processing-time-first with a fixed number of
chunks per rank (every rank holds the same number of tokens, as under the
dual-chunk assignment): chunks in descending cost, each to the currently
lightest rank that still has room (ties: lowest rank).  `refine_by_swaps`
then exchanges chunks between the heaviest rank and another one while that
lowers the maximum (pairwise interchange, a standard local search for
equal-cardinality partitioning).  Chunks of one rank are returned in
increasing global order, as fm_localize requires.
"""
from __future__ import annotations

import heapq

import numpy as np


def dual_chunk(n_chunks: int):
    """Rank r owns chunks r and n_chunks - 1 - r (n_chunks even)."""
    if n_chunks % 2:
        raise ValueError("dual-chunk assignment needs an even number of chunks")
    return [[r, n_chunks - 1 - r] for r in range(n_chunks // 2)]


def assign_longest_first(cost, ranks: int, per_rank: int):
    """cost: per-chunk work (len = ranks * per_rank).  Returns a list of `ranks` sorted chunk lists."""
    cost = np.asarray(cost)
    if cost.size != ranks * per_rank:
        raise ValueError("need exactly ranks * per_rank chunks")
    order = sorted(range(cost.size), key=lambda c: (-int(cost[c]), c))
    heap = [(0, r) for r in range(ranks)]  # (work, rank); ranks that are full leave the heap
    owned = [[] for _ in range(ranks)]
    for c in order:
        w, r = heapq.heappop(heap)
        owned[r].append(c)
        if len(owned[r]) < per_rank:
            heapq.heappush(heap, (w + int(cost[c]), r))
    return [sorted(x) for x in owned]


def refine_by_swaps(cost, assignment, max_rounds: int = 10000):
    """Pairwise-interchange local search on an assignment with equal chunks per rank: while some
    exchange of one chunk of the heaviest rank with one chunk of another rank lowers the heavier
    of the two ranks below the current maximum, make the exchange that lowers it most (ties: lowest
    rank, then lowest chunk ids).  Ranks keep their chunk counts, the maximum work never grows,
    and the result is returned as sorted chunk lists like the input."""
    cost = np.asarray(cost, dtype=np.int64)
    owned = [sorted(int(c) for c in x) for x in assignment]
    work = [int(cost[x].sum()) if x else 0 for x in owned]
    for _ in range(max_rounds):
        hi = max(range(len(owned)), key=lambda r: (work[r], -r))
        best = None  # (new max of the pair, rank, chunk out of hi, chunk in from rank)
        for r in range(len(owned)):
            if r == hi:
                continue
            for a in owned[hi]:
                for b in owned[r]:
                    d = int(cost[a]) - int(cost[b])  # work moved from hi to r
                    if d <= 0:
                        continue
                    pair_max = max(work[hi] - d, work[r] + d)
                    if pair_max < work[hi] and (best is None or (pair_max, r, a, b) < best):
                        best = (pair_max, r, a, b)
        if best is None:
            break
        _, r, a, b = best
        d = int(cost[a]) - int(cost[b])
        owned[hi].remove(a)
        owned[hi].append(b)
        owned[r].remove(b)
        owned[r].append(a)
        work[hi] -= d
        work[r] += d
    return [sorted(x) for x in owned]


def imbalance(cost, assignment) -> float:
    """max / mean of the per-rank work of an assignment."""
    work = np.array([sum(int(cost[c]) for c in chunks) for chunks in assignment], dtype=np.float64)
    return float(work.max() / work.mean()) if work.mean() > 0 else 1.0


def balance_report(cost, ranks: int, per_rank: int) -> dict:
    """max / mean per-rank work of the dual-chunk, longest-first and refined assignments of
    `cost` (ranks * per_rank chunks), with the lower bound that no assignment with per_rank
    chunks per rank can beat: max(mean, the largest chunk plus the per_rank - 1 smallest)."""
    cost = np.asarray(cost, dtype=np.int64)
    mean = float(cost.sum()) / ranks
    lpt = assign_longest_first(cost, ranks, per_rank)
    srt = np.sort(cost)
    bound = max(mean, float(srt[-1] + srt[:per_rank - 1].sum()))
    out = {"ranks": ranks, "chunks_per_rank": per_rank}
    if per_rank == 2:
        out["dual_chunk_max_over_mean"] = round(imbalance(cost, dual_chunk(len(cost))), 4)
    out["longest_first_max_over_mean"] = round(imbalance(cost, lpt), 4)
    out["refined_max_over_mean"] = round(imbalance(cost, refine_by_swaps(cost, lpt)), 4)
    out["lower_bound_max_over_mean"] = round(bound / mean, 4) if mean > 0 else 1.0
    return out


def chunk_costs(fm, vecs, chunk_len: int):
    """Per query chunk of `chunk_len` rows: unmasked (row, key) pairs over all keys, measured with
    the library's passes (one fm_localize launch treating every chunk as a rank, then
    fm_kv_chunk_pairs).  vecs: 4 int32 CUDA tensors [1, 1, N]; returns int64 numpy [N / chunk_len]."""
    N = vecs[0].shape[-1]
    if N % chunk_len:
        raise ValueError("chunk_len must divide the sequence length")
    n_ch = N // chunk_len
    starts = [[c * chunk_len] for c in range(n_ch)]
    lens = [[chunk_len]] * n_ch
    loc = fm.fm_localize(vecs, starts, lens)
    pairs = fm.fm_kv_chunk_pairs(loc, [chunk_len] * n_ch, chunk_len)
    return pairs.sum(dim=(1, 2, 3)).cpu().numpy()
