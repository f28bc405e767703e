"""The range form of the tile rule that both metadata kernels use, checked on the CPU against the
oracle's classes and column lists.

For a fixed key tile the query tile's rows are r0 = 128 qt and r1 = min(r0 + 128, n_q), which never
decrease as qt grows, so each term of the rule flips at most once: "x <= r0" holds from
qt = first_le_r0(x) on and "y >= r1" holds for qt < count_ge_r1(y).  Skip is then qt in two ranges
(from max LTS / min LTE and max UTS / min UTE), and a non-skip tile is partial on two more ranges
(min LTS / max LTE, min UTS / max UTE).  The key-tile pass writes its column list as the runs
outside the skip ranges; the query-tile pass of large launches reads the same ranges as bits.
This file restates that arithmetic (the kernels' `first_le_r0`, `count_ge_r1`, run emission) in
numpy and compares it with `oracle.tile_meta`, which applies the rule pair by pair."""
import numpy as np
import pytest

import oracle

I32_MIN, I32_MAX = -2**31, 2**31 - 1


def first_le_r0(x, T):
    if x <= 0:
        return 0
    return min(x // 128 + (1 if x % 128 else 0), T)


def count_ge_r1(y, n_q, T):
    if y >= n_q:
        return T
    if y < 0:
        return 0
    return min(y // 128, T)


def column_list(mm, n_q):
    """One key tile's column list from its min/max (minLTS, maxLTS, minLTE, maxLTE, minUTS, ...)."""
    T = (n_q + 127) // 128
    a0, a1 = first_le_r0(mm[1], T), count_ge_r1(mm[2], n_q, T)
    b0, b1 = first_le_r0(mm[5], T), count_ge_r1(mm[6], n_q, T)
    if a1 <= a0:
        a0 = a1 = T
    if b1 <= b0:
        b0 = b1 = T
    if b0 < a0:
        a0, a1, b0, b1 = b0, b1, a0, a1
    runs = [(0, a0)] + ([(max(a1, b1), T)] if b0 <= a1 else [(a1, b0), (b1, T)])
    p0, p1 = count_ge_r1(mm[0], n_q, T), first_le_r0(mm[3], T)
    u0, u1 = count_ge_r1(mm[4], n_q, T), first_le_r0(mm[7], T)
    out = []
    for lo, hi in runs:
        for q in range(lo, hi):
            out.append((q << 1) | int(p0 <= q < p1 or u0 <= q < u1))
    return out


def classes_from_ranges(mm, n_q):
    """Class of every (qt, kt) pair from the ranges (the bit-mask form of the query-tile pass)."""
    T = (n_q + 127) // 128
    cls = np.zeros((T, mm.shape[0]), np.uint8)
    for kt, m in enumerate(mm):
        sk = [(first_le_r0(m[1], T), count_ge_r1(m[2], n_q, T)), (first_le_r0(m[5], T), count_ge_r1(m[6], n_q, T))]
        pr = [(count_ge_r1(m[0], n_q, T), first_le_r0(m[3], T)), (count_ge_r1(m[4], n_q, T), first_le_r0(m[7], T))]
        for qt in range(T):
            if any(lo <= qt < hi for lo, hi in sk):
                cls[qt, kt] = 0
            else:
                cls[qt, kt] = 1 if any(lo <= qt < hi for lo, hi in pr) else 2
    return cls


def _vectors(rng, n_q, n_k):
    """Random bounds per column, plus whole key tiles set to one edge value (so that a tile's min
    or max lands exactly on a tile boundary, one off it, on n_q, or on an int32 extreme)."""
    def edge():
        k = int(rng.integers(0, n_q // 128 + 2))
        return int(rng.choice([128 * k - 1, 128 * k, 128 * k + 1, n_q, n_q - 1, n_q + 1, 0, -1, I32_MIN, I32_MAX]))
    vecs = []
    for _ in range(4):
        v = rng.integers(-200, n_q + 200, n_k).astype(np.int64)
        for t0 in range(0, n_k, 128):
            if rng.random() < 0.4:
                v[t0:t0 + 128] = edge()
            elif rng.random() < 0.3:
                v[t0:t0 + 128][rng.random(min(128, n_k - t0)) < 0.5] = edge()
        vecs.append(np.clip(v, I32_MIN, I32_MAX).astype(np.int32))
    return vecs


@pytest.mark.parametrize("n_q,n_k,seed", [(1000, 640, 1), (128, 384, 2), (300, 1000, 3), (4096, 512, 4), (5, 256, 5)])
def test_range_form_equals_oracle_rule(n_q, n_k, seed):
    rng = np.random.default_rng(seed)
    for _ in range(12):
        vecs = _vectors(rng, n_q, n_k)
        ref = oracle.tile_meta(n_q, n_k, *vecs)
        mm = ref["minmax"]
        np.testing.assert_array_equal(classes_from_ranges(mm, n_q), ref["cls"])
        for kt in range(mm.shape[0]):
            cc = int(ref["col_count"][kt])
            assert column_list(mm[kt], n_q) == list(ref["col_entries"][kt, :cc])


@pytest.mark.parametrize("n", [2048, 1000, 300])
def test_range_form_on_sweep_families(n):
    import synth
    for fam in synth.SWEEP_FAMILIES:
        vecs = synth.make_family(fam, n, 11).vectors()
        ref = oracle.tile_meta(n, n, *vecs)
        np.testing.assert_array_equal(classes_from_ranges(ref["minmax"], n), ref["cls"])
        for kt in range(ref["minmax"].shape[0]):
            cc = int(ref["col_count"][kt])
            assert column_list(ref["minmax"][kt], n) == list(ref["col_entries"][kt, :cc])
