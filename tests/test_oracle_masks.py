"""Pins for the oracle's mask semantics, tile metadata and localization
(CPU only).  Each check compares the oracle with something other than itself:
hand-worked examples, closed forms, independent dense predicates, brute force.
"""
import json
import os

import numpy as np
import pytest

import oracle
import synth
from oracle import families

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


# ---- the pages' byte arithmetic -------------------------------------------
def test_mask_bytes_128k():
    g = _load("mask_bytes_128k.json")
    n = g["n"]
    assert n * n == g["dense_bytes"]               # one byte per (row, key) entry
    assert 4 * n * 4 == g["vector_bytes"]           # four int32 vectors of n keys
    assert g["dense_bytes"] // g["vector_bytes"] == g["ratio"]
    m = synth.mask_causal(n)
    assert sum(x.nbytes for x in m.vectors()) == g["vector_bytes"]


# ---- hand-worked example ----------------------------------------------------
def test_hand_example_dense_and_count():
    g = _load("causal_doc_n8.json")
    n = g["n"]
    spec = synth.mask_causal_document(n, [tuple(d) for d in g["docs"]])
    for name in ("lts", "lte", "uts", "ute"):
        assert getattr(spec, name).tolist() == g[name]
    allowed = np.array([[c == "1" for c in row] for row in g["allowed_rows"]])
    dm = oracle.dense_mask(n, n, *spec.vectors())
    np.testing.assert_array_equal(~dm, allowed)
    assert oracle.count_unmasked_dense(n, n, *spec.vectors()) == g["unmasked_pairs"]
    assert oracle.count_unmasked(n, n, *spec.vectors()) == g["unmasked_pairs"]


def test_hand_example_localization():
    g = _load("causal_doc_n8.json")
    st, ln = g["rank_chunks"]["starts"], g["rank_chunks"]["lens"]
    for name in ("lts", "lte", "uts", "ute"):
        for formula in ("clip_shift_max", "count"):
            got = oracle.localize(np.array(g[name]), st, ln, formula)
            assert got.tolist() == g["local"][name], (name, formula)


# ---- family encodings vs independent dense predicates ------------------------
@pytest.mark.parametrize("family", synth.SWEEP_FAMILIES)
@pytest.mark.parametrize("n", [64, 200, 384])
def test_family_vectors_match_dense_predicate(family, n):
    for seed in range(8):
        spec = synth.make_family(family, n, seed)
        dm = oracle.dense_mask(n, n, *spec.vectors())
        allowed = families.allowed_from_spec(spec)
        np.testing.assert_array_equal(~dm, allowed, err_msg=f"{family} n={n} seed={seed}")


@pytest.mark.parametrize("seed", range(40))
def test_document_families_many_seeds(seed):
    n = 96 + seed * 7
    rng = synth.Rng(seed)
    docs = synth.draw_docs(rng, n, 1, 40)
    prefixes = [rng.randint(0, b - a) for (a, b) in docs]
    for spec in (synth.mask_causal_document(n, docs), synth.mask_bidir_document(n, docs),
                 synth.mask_prefix_lm_document(n, docs, prefixes)):
        np.testing.assert_array_equal(~oracle.dense_mask(n, n, *spec.vectors()),
                                      families.allowed_from_spec(spec))
    groups = synth.draw_share_question(rng, n, 3, 20, (2, 6), 1, 10)
    spec = synth.mask_share_question(n, groups)
    np.testing.assert_array_equal(~oracle.dense_mask(n, n, *spec.vectors()), families.allowed_from_spec(spec))


def test_config1_document_cut():
    rng = synth.Rng(1000)
    docs = synth.cut_segments(rng, 256, 3)
    assert len(docs) == 3 and docs[0][0] == 0 and docs[-1][1] == 256
    assert all(b > a for a, b in docs)


# ---- unmasked-pair closed forms ---------------------------------------------
@pytest.mark.parametrize("n", [1, 7, 128, 300])
def test_unmasked_closed_forms(n):
    assert oracle.count_unmasked_dense(n, n, *synth.mask_full(n).vectors()) == n * n
    assert oracle.count_unmasked_dense(n, n, *synth.mask_causal(n).vectors()) == n * (n + 1) // 2
    for w in sorted({1, min(3, n), n}):  # closed form holds for w <= n
        exp = w * (w + 1) // 2 + (n - w) * w
        assert oracle.count_unmasked_dense(n, n, *synth.mask_sliding_window(n, w).vectors()) == exp


def test_unmasked_interval_count_matches_dense_random():
    r = np.random.default_rng(0)
    for _ in range(50):
        n_q, n_k = int(r.integers(1, 70)), int(r.integers(1, 70))
        v = [r.integers(-5, n_q + 5, n_k) for _ in range(4)]
        assert oracle.count_unmasked(n_q, n_k, *v) == oracle.count_unmasked_dense(n_q, n_k, *v)


def test_null_vectors_mean_empty():
    n_q, n_k = 37, 19
    dm = oracle.dense_mask(n_q, n_k, None, None, None, None)
    assert not dm.any()
    e = synth.canonical_empty(n_q, n_k)
    assert not oracle.dense_mask(n_q, n_k, *e).any()


# ---- tile classification ----------------------------------------------------
def _check_sound(n_q, n_k, vecs, tq, tk):
    dm = oracle.dense_mask(n_q, n_k, *vecs)
    meta = oracle.tile_meta(n_q, n_k, *vecs, tile_q=tq, tile_k=tk)
    cls = meta["cls"]
    T_q, T_k = cls.shape
    for qt in range(T_q):
        for kt in range(T_k):
            blk = dm[qt * tq:(qt + 1) * tq, kt * tk:(kt + 1) * tk]
            if cls[qt, kt] == 0:
                assert blk.all(), (qt, kt)
            elif cls[qt, kt] == 2:
                assert not blk.any(), (qt, kt)
    # minmax vs numpy reductions of the columns
    for kt in range(T_k):
        cols = slice(kt * tk, min((kt + 1) * tk, n_k))
        for c, vec in enumerate(vecs):
            assert meta["minmax"][kt, 2 * c] == np.min(vec[cols])
            assert meta["minmax"][kt, 2 * c + 1] == np.max(vec[cols])
    # lists are the ascending non-skip tiles with the partial bit
    for qt in range(T_q):
        want = [(kt << 1) | int(cls[qt, kt] == 1) for kt in range(T_k) if cls[qt, kt]]
        assert meta["row_count"][qt] == len(want)
        assert meta["row_entries"][qt, :len(want)].tolist() == want
    for kt in range(T_k):
        want = [(qt << 1) | int(cls[qt, kt] == 1) for qt in range(T_q) if cls[qt, kt]]
        assert meta["col_count"][kt] == len(want)
        assert meta["col_entries"][kt, :len(want)].tolist() == want
    return meta


@pytest.mark.parametrize("family", synth.SWEEP_FAMILIES)
def test_classification_sound_families(family):
    n = 256
    spec = synth.make_family(family, n, 3)
    _check_sound(n, n, spec.vectors(), 16, 16)
    _check_sound(n, n, spec.vectors(), 32, 64)


def test_classification_sound_random_vectors():
    r = np.random.default_rng(1)
    for _ in range(30):
        n_q, n_k = int(r.integers(1, 90)), int(r.integers(1, 90))
        v = [r.integers(-10, n_q + 10, n_k).astype(np.int32) for _ in range(4)]
        _check_sound(n_q, n_k, v, int(r.integers(1, 17)), int(r.integers(1, 17)))


@pytest.mark.parametrize("T", [1, 2, 5, 16])
def test_classification_causal_closed_form(T):
    n = 128 * T
    meta = oracle.tile_meta(n, n, *synth.mask_causal(n).vectors())
    cls = meta["cls"]
    assert (cls == 0).sum() == T * (T - 1) // 2
    assert (cls == 1).sum() == T
    assert (cls == 2).sum() == T * (T - 1) // 2
    assert all(cls[t, t] == 1 for t in range(T))
    meta = oracle.tile_meta(n, n, *synth.mask_full(n).vectors())
    assert (meta["cls"] == 2).all()


def test_classification_exact_tile_cover():
    # a key tile fully masked for one query tile by the lower interval only
    n = 256
    lts = np.full(n, 128, np.int32)
    lte = np.full(n, 256, np.int32)
    uts = np.zeros(n, np.int32)
    ute = np.zeros(n, np.int32)
    meta = oracle.tile_meta(n, n, lts, lte, uts, ute)
    assert meta["cls"].tolist() == [[2, 2], [0, 0]]


# ---- localization -------------------------------------------------------------
def _random_chunks(r, N, max_chunks):
    C = int(r.integers(1, max_chunks + 1))
    cuts = np.sort(r.choice(np.arange(0, N + 1), size=2 * C, replace=True))
    starts, lens = [], []
    for k in range(C):
        a, b = int(cuts[2 * k]), int(cuts[2 * k + 1])
        if b > a and (not starts or a >= starts[-1] + lens[-1]):
            starts.append(a)
            lens.append(b - a)
    if not starts:
        starts, lens = [0], [N]
    return starts, lens


def test_localize_formulas_agree_random():
    r = np.random.default_rng(2)
    for _ in range(300):
        N = int(r.integers(1, 200))
        starts, lens = _random_chunks(r, N, 5)
        v = r.integers(-20, N + 20, 64).astype(np.int32)
        a = oracle.localize(v, starts, lens, "clip_shift_max")
        b = oracle.localize(v, starts, lens, "count")
        np.testing.assert_array_equal(a, b)
        assert a.min() >= 0 and a.max() <= sum(lens)


def _theorem1(vecs, N, starts, lens):
    loc = [oracle.localize(v, starts, lens) for v in vecs]
    rows = np.concatenate([np.arange(s, s + L) for s, L in zip(starts, lens)])
    n_loc = rows.size
    glob = oracle.dense_mask(N, N, *vecs)
    local = oracle.dense_mask(n_loc, N, *loc)
    np.testing.assert_array_equal(local, glob[rows, :])


def test_theorem1_families_random_chunkings():
    r = np.random.default_rng(3)
    for family in synth.SWEEP_FAMILIES:
        N = 192
        spec = synth.make_family(family, N, 5)
        for _ in range(6):
            starts, lens = _random_chunks(r, N, 4)
            _theorem1(spec.vectors(), N, starts, lens)


def test_theorem1_random_vectors():
    r = np.random.default_rng(4)
    for _ in range(60):
        N = int(r.integers(2, 80))
        vecs = [r.integers(-3, N + 3, N).astype(np.int32) for _ in range(4)]
        starts, lens = _random_chunks(r, N, 4)
        _theorem1(vecs, N, starts, lens)


def test_localize_identity_and_shift():
    N = 100
    v = np.arange(-5, N + 5, dtype=np.int32)
    np.testing.assert_array_equal(oracle.localize(v, [0], [N]), np.clip(v, 0, N))
    got = oracle.localize(v, [30], [40])
    np.testing.assert_array_equal(got, np.clip(v - 30, 0, 40))


def test_dual_chunk_tile_classes_match_global():
    # 128-aligned chunks: every local query tile has the class row of its global tile
    N, chunk = 2048, 256
    nchunks = N // chunk
    spec = synth.make_family("causal_document", N, 11)
    gm = oracle.tile_meta(N, N, *spec.vectors())
    for rank in range(nchunks // 2):
        ids = [rank, nchunks - 1 - rank]
        starts = [c * chunk for c in ids]
        loc = [oracle.localize(v, starts, [chunk, chunk]) for v in spec.vectors()]
        lm = oracle.tile_meta(2 * chunk, N, *loc)
        grows = np.concatenate([np.arange(s // 128, (s + chunk) // 128) for s in starts])
        np.testing.assert_array_equal(lm["cls"], gm["cls"][grows])


# ---- KV-chunk pruning counts ------------------------------------------------
def test_kv_chunk_pairs_dense_brute_force():
    """Per-chunk unmasked pairs equal the dense mask's count over each chunk's keys
    (random vectors with out-of-range and empty stretches, ragged last chunk)."""
    r = np.random.default_rng(21)
    for _ in range(120):
        n_q, n_k = int(r.integers(1, 90)), int(r.integers(1, 120))
        vecs = [r.integers(-5, n_q + 5, n_k).astype(np.int32) for _ in range(4)]
        cl = int(r.integers(1, n_k + 3))
        got = oracle.kv_chunk_pairs(n_q, n_k, cl, *vecs)
        unm = ~oracle.dense_mask(n_q, n_k, *vecs)
        want = np.add.reduceat(unm.sum(0), np.arange(0, n_k, cl)).astype(np.int64)
        np.testing.assert_array_equal(got, want)


def test_kv_chunk_pairs_null_and_causal_closed_form():
    N, cl = 1000, 128
    full = oracle.kv_chunk_pairs(N, N, cl, None, None, None, None)
    np.testing.assert_array_equal(full, [N * min(cl, N - c * cl) for c in range(-(-N // cl))])
    spec = synth.mask_causal(N)  # key j is seen by rows j .. N-1
    got = oracle.kv_chunk_pairs(N, N, cl, *spec.vectors())
    want = [sum(N - j for j in range(c * cl, min((c + 1) * cl, N))) for c in range(-(-N // cl))]
    np.testing.assert_array_equal(got, want)


def test_kv_chunk_pairs_ranks_partition_global():
    """Ranks whose chunks partition the query rows: by Theorem 1 their local pairs
    per KV chunk add up to the global mask's, and a chunk is pruned for a rank
    exactly when the rank's rows of the global dense mask are all masked there."""
    r = np.random.default_rng(22)
    N, nch, cl = 512, 8, 64
    chunk = N // nch
    pruned = 0
    for family in ("causal_document", "share_question", "sliding_window_2k", "prefix_lm_document", "random_eviction"):
        spec = synth.make_family(family, N, 23)
        vecs = spec.vectors()
        glob = oracle.kv_chunk_pairs(N, N, cl, *vecs)
        dense = oracle.dense_mask(N, N, *vecs)
        perm = r.permutation(nch)
        total = np.zeros_like(glob)
        for rank in range(nch // 2):
            ids = sorted(perm[2 * rank: 2 * rank + 2])
            starts, lens = [c * chunk for c in ids], [chunk, chunk]
            loc = [oracle.localize(v, starts, lens) for v in vecs]
            pr = oracle.kv_chunk_pairs(2 * chunk, N, cl, *loc)
            rows = np.concatenate([np.arange(s, s + chunk) for s in starts])
            seen = (~dense[rows]).reshape(rows.size, -1, cl).any(axis=(0, 2))
            np.testing.assert_array_equal(pr > 0, seen)
            pruned += int((pr == 0).sum())
            total += pr
        np.testing.assert_array_equal(total, glob)
        assert glob.sum() == oracle.count_unmasked_dense(N, N, *vecs)
    assert pruned > 0  # the cases include chunks some ranks never need


def _varlen_predicate(cu, N, causal):
    """Plain definition of a packed batch: (i, j) is visible iff both lie in the same sequence
    and, when causal, j <= i; every other pair (other sequence, padding) is masked."""
    seq = np.full(N, -1)
    for s in range(len(cu) - 1):
        seq[cu[s]:cu[s + 1]] = s
    i, j = np.arange(N)[:, None], np.arange(N)[None, :]
    visible = (seq[:, None] == seq[None, :]) & (seq[:, None] >= 0)
    if causal:
        visible &= j <= i
    return ~visible


@pytest.mark.parametrize("causal", [True, False])
def test_varlen_vectors_match_packed_predicate(causal):
    r = np.random.default_rng(41)
    for N in (1, 7, 130, 300, 517):
        for _ in range(20):
            n_seq = int(r.integers(1, 9))
            cuts = np.sort(r.integers(0, N + 1, n_seq))  # repeated cuts = empty sequences
            cu = np.concatenate([[0], cuts])
            vecs = oracle.varlen_vectors(cu, N, causal)
            np.testing.assert_array_equal(oracle.dense_mask(N, N, *vecs), _varlen_predicate(cu, N, causal))


def test_varlen_single_sequence_is_causal_or_full():
    """One sequence over all N positions: the causal mask (UTE = j) or no mask at all."""
    N = 300
    lts, lte, uts, ute = oracle.varlen_vectors([0, N], N, True)
    assert oracle.count_unmasked(N, N, lts, lte, uts, ute) == N * (N + 1) // 2
    np.testing.assert_array_equal(ute, np.arange(N))
    assert oracle.count_unmasked(N, N, *oracle.varlen_vectors([0, N], N, False)) == N * N
