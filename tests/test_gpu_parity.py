"""GPU parity: the CUDA path (through the C ABI) against the oracle on the same
seeded inputs.  Bit-exact for tile metadata and localized vectors; for the
attention: O max-abs <= 1e-2, LSE abs <= 1e-3 on live rows (exactly -inf and
O exactly 0 on fully masked rows), dQ/dK/dV max-abs error relative to the
oracle's max-abs <= 2e-2 per (b, h).

fp32 inputs go through tf32 tensor-core products, which keep 10 of the 23
mantissa bits of each operand (truncation, relative error < 2^-10 per operand).
A score then moves by at most scale * sum_d |q_d k_d| * 2^-9, and the LSE, a
smooth maximum over the row's scores, by at most the largest such move in its
row; that bound (over all keys of the row) is added to the LSE tolerance."""
import math

import numpy as np
import pytest

import oracle
import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

O_TOL, LSE_TOL, G_TOL = 1e-2, 1e-3, 2e-2


@pytest.fixture(scope="module")
def fm():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from mask_aware_flash_b200 import _build
    _build.build()
    import mask_aware_flash_b200 as m
    m.lib()
    return m


def _bf16_tensor(bits):
    t = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)
    return t.cuda()


def _inputs(B, n_q, n_k, H, D, seed):
    qb = synth.normal_bf16_bits(seed, 1, (B, n_q, H, D))
    kb = synth.normal_bf16_bits(seed, 2, (B, n_k, H, D))
    vb = synth.normal_bf16_bits(seed, 3, (B, n_k, H, D))
    db = synth.normal_bf16_bits(seed, 4, (B, n_q, H, D))
    host = [synth.bf16_bits_to_f32(x) for x in (qb, kb, vb, db)]
    dev = [_bf16_tensor(x) for x in (qb, kb, vb, db)]
    return host, dev


def _vec_tensors(vecs, B, Hm, n_k):
    """1-D (or [B, Hm, n_k]) int32 vectors -> CUDA tensors [B, Hm, n_k]; None stays None."""
    return [None if v is None else
            torch.from_numpy(np.broadcast_to(np.asarray(v, np.int32), (B, Hm, n_k)).copy()).cuda()
            for v in vecs]


def _host_vecs(vt):
    return [None if v is None else v.cpu().numpy() for v in vt]


# ---------------------------------------------------------------------------- metadata
def _check_meta(fm, vt, n_q, n_k):
    meta = fm.fm_build_mask_meta(*vt, n_q=n_q)
    torch.cuda.synchronize()
    hv = _host_vecs(vt)
    B, Hm = meta.desc.B, meta.desc.Hm
    for b in range(B):
        for hm in range(Hm):
            ref = oracle.tile_meta(n_q, n_k, *[None if v is None else v[b, hm] for v in hv])
            np.testing.assert_array_equal(meta.tile_minmax[b, hm].cpu().numpy(), ref["minmax"])
            np.testing.assert_array_equal(meta.tile_class[b, hm].cpu().numpy(), ref["cls"])
            rc = meta.row_count[b, hm].cpu().numpy()
            np.testing.assert_array_equal(rc, ref["row_count"])
            re_ = meta.row_entries[b, hm].cpu().numpy()
            for qt in range(len(rc)):
                np.testing.assert_array_equal(re_[qt, :rc[qt]], ref["row_entries"][qt, :rc[qt]])
            cc = meta.col_count[b, hm].cpu().numpy()
            np.testing.assert_array_equal(cc, ref["col_count"])
            ce = meta.col_entries[b, hm].cpu().numpy()
            for kt in range(len(cc)):
                np.testing.assert_array_equal(ce[kt, :cc[kt]], ref["col_entries"][kt, :cc[kt]])
            # dispatch orders: longest first, ties by ascending index (stable sort on -cost); past
            # 4096 tiles either way (sizes the attention kernels do not take) the identity order
            rcp = np.concatenate([ref["row_count"], [0]])[: 2 * ((len(rc) + 1) // 2)].reshape(-1, 2).sum(1)
            big = len(rc) > 4096 or len(cc) > 4096
            np.testing.assert_array_equal(meta.fwd_order[b, hm].cpu().numpy(),
                                          np.arange(len(rcp)) if big else np.argsort(-rcp, kind="stable"))
            np.testing.assert_array_equal(meta.bwd_order[b, hm].cpu().numpy(),
                                          np.arange(len(cc)) if big else np.argsort(-ref["col_count"], kind="stable"))
    return meta


@pytest.mark.parametrize("family", synth.SWEEP_FAMILIES)
def test_meta_bitexact_families(fm, family):
    n = 2048
    spec = synth.make_family(family, n, 77)
    vt = _vec_tensors(spec.vectors(), 2, 1, n)
    _check_meta(fm, vt, n, n)


def test_meta_bitexact_random_ragged(fm):
    r = np.random.default_rng(5)
    for (n_q, n_k, B, Hm) in [(300, 517, 2, 3), (128, 1000, 1, 1), (1001, 129, 3, 2), (5000, 4500, 1, 2)]:
        vecs = [r.integers(-50, n_q + 50, (B, Hm, n_k)).astype(np.int32) for _ in range(4)]
        vt = [torch.from_numpy(v).cuda() for v in vecs]
        _check_meta(fm, vt, n_q, n_k)


@pytest.mark.parametrize("n_k", [13000, 12800])
def test_meta_bitexact_batched(fm, n_k):
    # more than 148 x 32 query-tile lists in one launch: the query-tile pass takes four lists per warp
    # (bit masks from each key tile's skip / partial ranges) instead of four warps per list; with
    # n_k = 12800 (100 key tiles, a multiple of 4) its class bytes go out as packed 4-byte stores
    r = np.random.default_rng(11)
    B, Hm, n_q = 2, 24, 16300
    fams = list(synth.SWEEP_FAMILIES)
    vecs = [np.empty((B, Hm, n_k), np.int32) for _ in range(4)]
    for b in range(B):
        for hm in range(Hm):
            if (b * Hm + hm) % 3 == 2:  # random bounds, out-of-range values and int32 extremes included
                for c in range(4):
                    vecs[c][b, hm] = r.integers(-300, n_q + 300, n_k).astype(np.int32)
                vecs[0][b, hm, :6] = [-2**31, 2**31 - 1, 0, n_q, n_q - 1, 128]
                vecs[3][b, hm, 6:12] = [2**31 - 1, -2**31, n_q + 1, 127, 129, -1]
            else:  # a sweep family laid out over n_k keys, rows clipped to n_q
                spec = synth.make_family(fams[(b * Hm + hm) % len(fams)], n_k, 900 + b * Hm + hm)
                for c, v in enumerate(spec.vectors()):
                    vecs[c][b, hm] = v
    assert B * Hm * ((n_q + 127) // 128) > 148 * 32
    _check_meta(fm, [torch.from_numpy(v).cuda() for v in vecs], n_q, n_k)


@pytest.mark.parametrize("n_q", [1000, 606300])
def test_meta_unstaged_key_tiles(fm, n_q):
    # more than 4096 key tiles: the query-tile pass reads the min/max from global memory instead of a
    # shared-memory copy (n_q = 1000: four warps per list; 606300: 4737 query tiles, four lists per warp)
    r = np.random.default_rng(12)
    n_k = 530000
    vecs = [r.integers(-100, n_q + 100, (1, 1, n_k)).astype(np.int32) for _ in range(4)]
    vecs[1][0, 0, : n_k // 2] = n_q  # half the keys: lower interval to the end, so skip tiles exist
    vecs[0][0, 0, : n_k // 2] = r.integers(0, n_q, n_k // 2)
    _check_meta(fm, [torch.from_numpy(v).cuda() for v in vecs], n_q, n_k)


def test_meta_null_vectors(fm):
    n = 512
    spec = synth.mask_causal(n)
    vt = [None, None, None] + _vec_tensors([spec.ute], 1, 1, n)
    meta = _check_meta(fm, vt, n, n)
    assert int(meta.tile_class.eq(1).sum()) == 4


@pytest.mark.parametrize("Hm", [1, 8])
def test_meta_causal_128k_closed_form(fm, Hm):
    # Hm = 8: 8192 query-tile lists, the four-lists-per-warp form of the query-tile pass
    n = 131072
    T = n // 128
    spec = synth.mask_causal(n)
    meta = fm.fm_build_mask_meta(*_vec_tensors(spec.vectors(), 1, Hm, n), n_q=n)
    for hm in range(Hm):
        cls = meta.tile_class[0, hm]
        assert int(cls.eq(0).sum()) == T * (T - 1) // 2
        assert int(cls.eq(1).sum()) == T
        assert int(cls.eq(2).sum()) == T * (T - 1) // 2
        assert int(meta.row_count[0, hm].sum()) == T * (T + 1) // 2
        assert int(meta.col_count[0, hm].sum()) == T * (T + 1) // 2


# ---------------------------------------------------------------------------- localization
def test_localize_bitexact(fm):
    N, nch = 4096, 16
    chunk = N // nch
    R = nch // 2
    starts = [[r * chunk, (nch - 1 - r) * chunk] for r in range(R)]
    lens = [[chunk, chunk]] * R
    r = np.random.default_rng(9)
    vecs = [r.integers(-100, N + 100, (2, 1, N)).astype(np.int32) for _ in range(4)]
    spec = synth.make_family("causal_document", N, 3)
    vecs[0][1, 0] = spec.lts  # one batch row with a real mask
    vecs[3][1, 0] = spec.ute
    out = fm.fm_localize([torch.from_numpy(v).cuda() for v in vecs], starts, lens)
    torch.cuda.synchronize()
    for c in range(4):
        got = out[c].cpu().numpy()
        for rr in range(R):
            for b in range(2):
                exp = oracle.localize(vecs[c][b, 0], starts[rr], lens[rr])
                np.testing.assert_array_equal(got[rr, b, 0], exp)


def test_kv_chunk_pairs_bitexact(fm):
    """Per-rank unmasked pairs per KV chunk (KV-chunk pruning) on localized vectors: bit-exact
    against the oracle for random vectors and a document mask, a ragged last chunk, null vectors,
    and ranks owning different numbers of rows."""
    N, nch = 4096, 16
    chunk = N // nch
    r = np.random.default_rng(19)
    vecs = [r.integers(-100, N + 100, (2, 1, N)).astype(np.int32) for _ in range(4)]
    spec = synth.make_family("causal_document", N, 13)
    for c in range(4):
        vecs[c][1, 0] = spec.vectors()[c]
    # 5 ranks: dual chunks, a single chunk and three chunks
    starts = [[0, 15 * chunk], [chunk, 14 * chunk], [2 * chunk, 13 * chunk], [3 * chunk, 5 * chunk],
              [6 * chunk, 9 * chunk]]
    lens = [[chunk, chunk], [chunk, chunk], [chunk, chunk], [2 * chunk, 4 * chunk], [3 * chunk, 4 * chunk]]
    n_loc = [sum(x) for x in lens]
    loc = fm.fm_localize([torch.from_numpy(v).cuda() for v in vecs], starts, lens)
    for cl in (chunk, 1000):  # aligned chunks and a ragged last chunk
        got = fm.fm_kv_chunk_pairs(loc, n_loc, cl).cpu().numpy()
        for rr in range(len(starts)):
            for b in range(2):
                lv = [x[rr, b, 0].cpu().numpy() for x in loc]
                np.testing.assert_array_equal(got[rr, b, 0], oracle.kv_chunk_pairs(n_loc[rr], N, cl, *lv))
    # null vectors = canonical empty: every pair of the rank is unmasked
    nul = fm.fm_kv_chunk_pairs([None, None, None, loc[3]], n_loc, chunk).cpu().numpy()
    for rr in range(len(starts)):
        lv = loc[3][rr, 0, 0].cpu().numpy()
        np.testing.assert_array_equal(nul[rr, 0, 0], oracle.kv_chunk_pairs(n_loc[rr], N, chunk, None, None, None, lv))


def test_chunk_costs_and_balanced_assignment(fm):
    """Per-query-chunk work measured by the GPU passes equals the oracle's counts; the
    longest-first assignment balances a document mask at least as well as dual-chunk."""
    from mask_aware_flash_b200 import cp_balance as cb
    N, chunk = 8192, 256
    spec = synth.mask_causal_document(N, synth.draw_docs(synth.Rng(71), N, 256, 2048))
    vt = [torch.from_numpy(np.ascontiguousarray(x[None, None])).cuda() for x in spec.vectors()]
    cost = cb.chunk_costs(fm, vt, chunk)
    want = []
    for c in range(N // chunk):
        loc = [oracle.localize(x, [c * chunk], [chunk]) for x in spec.vectors()]
        want.append(int(oracle.kv_chunk_pairs(chunk, N, N, *loc).sum()))
    np.testing.assert_array_equal(cost, want)
    assert cb.imbalance(cost, cb.assign_longest_first(cost, N // chunk // 2, 2)) <= \
        cb.imbalance(cost, cb.dual_chunk(N // chunk)) + 1e-12


# ---------------------------------------------------------------------------- attention
def _run_attention(fm, B, H, n_q, n_k, D, vecs_np, Hm, seed, scale=None, bwd=True, det=False):
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    host, dev = _inputs(B, n_q, n_k, H, D, seed)
    vt = [None if v is None else torch.from_numpy(np.ascontiguousarray(v, np.int32)).cuda() for v in vecs_np]
    meta = fm.fm_build_mask_meta(*vt, n_q=n_q)
    o, lse = fm.fm_attn_fwd(dev[0], dev[1], dev[2], meta, vt, scale)
    res = {"o": o, "lse": lse, "host": host, "meta": meta, "vt": vt, "scale": scale}
    if bwd:
        dq, dk, dv = fm.fm_attn_bwd(dev[0], dev[1], dev[2], o, lse, dev[3], meta, vt, scale, deterministic=det)
        res.update(dq=dq, dk=dk, dv=dv, dev=dev)
    torch.cuda.synchronize()
    assert fm.fm_get_device_status() == 0
    return res


def _compare(res, vecs_np, Hm, heads=None, rows=None, cols=None, bwd=True):
    q, k, v, do = res["host"]
    B, n_q, H, D = q.shape
    o = res["o"].float().cpu().numpy()
    lse = res["lse"].cpu().numpy()
    if bwd:
        dq, dk, dv = (res[x].float().cpu().numpy() for x in ("dq", "dk", "dv"))
    heads = [(b, h) for b in range(B) for h in range(H)] if heads is None else heads
    for (b, h) in heads:
        ref = oracle.attention_head(q, k, v, vecs_np, b, h, res["scale"], rows=rows,
                                    cols=(np.arange(k.shape[1]) if (cols is None and bwd) else cols),
                                    dout=do if bwd else None, Hm=Hm)
        rr = ref["rows"]
        live = np.isfinite(ref["lse"])
        err_o = np.abs(o[b, rr, h] - ref["o"]).max()
        assert err_o <= O_TOL, f"O max-abs {err_o} at (b={b}, h={h})"
        if live.any():
            tol = LSE_TOL + (res["lse_slack"][b, h, rr][live] if "lse_slack" in res else 0.0)
            err_l = np.abs(lse[b, h, rr][live] - ref["lse"][live])
            assert np.all(err_l <= tol), f"LSE {err_l.max()} (tolerance {np.min(tol)}..)"
        assert np.all(np.isneginf(lse[b, h, rr][~live])), "dead rows need LSE = -inf"
        assert np.all(o[b, rr, h][~live] == 0.0), "dead rows need O = 0"
        if bwd:
            for name, got, exp in (("dq", dq[b, rr, h], ref["dq"]), ("dk", dk[b, ref["cols"], h], ref["dk"]),
                                   ("dv", dv[b, ref["cols"], h], ref["dv"])):
                scale = max(np.abs(exp).max(), 1e-30)
                err = np.abs(got - exp).max() / scale
                assert err <= G_TOL, f"{name} rel-to-max error {err} at (b={b}, h={h})"


def _vec_stack(spec, B, Hm):
    return [np.ascontiguousarray(np.broadcast_to(x, (B, Hm, x.shape[-1]))) for x in spec.vectors()]


@pytest.mark.parametrize("D", [64, 128])
def test_tiny_causal_document(fm, D):
    """B=1, H=2, n=256, 3 seeded documents, causal inside each."""
    n = 256
    docs = synth.cut_segments(synth.Rng(1000), n, 3)
    spec = synth.mask_causal_document(n, docs)
    vecs = _vec_stack(spec, 1, 1)
    res = _run_attention(fm, 1, 2, n, n, D, vecs, 1, seed=1000)
    _compare(res, vecs, 1)


@pytest.mark.parametrize("n,family", [(256, "causal_document"), (640, "full"), (640, "sliding_window_2k"),
                                      (1000, "random_eviction"), (388, "share_question"), (1536, "global_sliding")])
def test_head_dim_256_forward(fm, n, family):
    """D = 256 (one query tile per CTA, K / V streamed in 64-key halves): the forward against the
    oracle on every row of both heads, ragged lengths included."""
    vecs = _vec_stack(synth.make_family(family, n, 71), 1, 1)
    res = _run_attention(fm, 1, 2, n, n, 256, vecs, 1, seed=72, bwd=False)
    _compare(res, vecs, 1, bwd=False)


@pytest.mark.parametrize("n,family", [(256, "causal_document"), (640, "full"), (1000, "random_eviction"),
                                      (388, "share_question"), (1536, "global_sliding")])
def test_head_dim_256_backward(fm, n, family):
    """D = 256 backward (dK, dV and dQ accumulated one 128-column half per launch, S^T and dP^T over
    all 256 columns in both): every row and column of both heads against the oracle."""
    vecs = _vec_stack(synth.make_family(family, n, 73), 1, 1)
    res = _run_attention(fm, 1, 2, n, n, 256, vecs, 1, seed=74)
    _compare(res, vecs, 1)


def _run_fp32(fm, B, H, n, vecs, seed):
    """fp32 inputs and outputs (tf32 tensor-core products), D = 64."""
    D = 64
    host = [synth.normal_f32(seed, t, (B, n, H, D)) for t in (1, 2, 3, 4)]
    dev = [torch.from_numpy(x).cuda() for x in host]
    vt = [torch.from_numpy(np.ascontiguousarray(np.broadcast_to(v, (B, 1, n)), np.int32)).cuda() for v in vecs]
    scale = 1.0 / math.sqrt(D)
    meta = fm.fm_build_mask_meta(*vt, n_q=n)
    o, lse = fm.fm_attn_fwd(dev[0], dev[1], dev[2], meta, vt, scale)
    dq, dk, dv = fm.fm_attn_bwd(dev[0], dev[1], dev[2], o, lse, dev[3], meta, vt, scale)
    torch.cuda.synchronize()
    assert fm.fm_get_device_status() == 0
    assert o.dtype == torch.float32 and dq.dtype == torch.float32 and dk.dtype == torch.float32
    q64, k64 = np.abs(host[0].astype(np.float64)), np.abs(host[1].astype(np.float64))
    slack = scale * 2.0 ** -9 * np.einsum("bihd,bjhd->bhij", q64, k64).max(axis=3)  # [B, H, n_q]
    return {"o": o, "lse": lse, "dq": dq, "dk": dk, "dv": dv, "host": host, "scale": scale, "lse_slack": slack}


def test_tiny_causal_document_fp32(fm):
    """B=1, H=2, n=256, D=64, three seeded documents, fp32 in and out."""
    n, seed = 256, 1000
    docs = synth.cut_segments(synth.Rng(seed), n, 3)
    vecs = _vec_stack(synth.mask_causal_document(n, docs), 1, 1)
    _compare(_run_fp32(fm, 1, 2, n, vecs, seed), vecs, 1)


@pytest.mark.parametrize("family", ["full", "causal", "share_question", "random_eviction"])
def test_fp32_families_n640(fm, family):
    """fp32 over five tiles: the V ring, both Q/dO stages and the in-place operand transposes wrap."""
    n = 640
    vecs = _vec_stack(synth.make_family(family, n, 41), 2, 1)
    _compare(_run_fp32(fm, 2, 2, n, vecs, 43), vecs, 1)


@pytest.mark.parametrize("family", ["full", "causal", "sliding_window_2k", "share_question", "random_eviction",
                                    "global_sliding", "prefix_lm_document", "causal_blockwise"])
def test_families_n640(fm, family):
    n = 640  # five tiles: full, partial and skipped tiles
    spec = synth.make_family(family, n, 31)
    vecs = _vec_stack(spec, 1, 1)
    res = _run_attention(fm, 1, 2, n, n, 128, vecs, 1, seed=2)
    _compare(res, vecs, 1)


@pytest.mark.parametrize("n,D,family", [(200, 128, "causal_document"), (388, 64, "share_question"), (4, 128, "full"),
                                         (1000, 128, "sliding_window_2k"), (132, 128, "random_eviction"),
                                         (676, 64, "prefix_lm_document")])
def test_ragged_lengths(fm, n, D, family):
    """Lengths that are not multiples of 128: zero-filled tail rows of the last tiles, the last key
    tile always interval-tested, padded backward rows; every real row and column compared."""
    vecs = _vec_stack(synth.make_family(family, n, 61), 1, 1)
    res = _run_attention(fm, 1, 2, n, n, D, vecs, 1, seed=62)
    _compare(res, vecs, 1)


def test_ragged_cross_lengths(fm):
    n_q, n_k = 77, 516
    r = np.random.default_rng(63)
    vecs = [r.integers(-10, n_q + 10, n_k).astype(np.int32)[None, None] for _ in range(4)]
    res = _run_attention(fm, 2, 2, n_q, n_k, 128, [np.broadcast_to(v, (2, 1, n_k)).copy() for v in vecs], 1,
                         seed=64)
    _compare(res, [np.broadcast_to(v, (2, 1, n_k)).copy() for v in vecs], 1)


def test_ragged_fp32(fm):
    n = 200
    docs = synth.cut_segments(synth.Rng(65), n, 3)
    vecs = _vec_stack(synth.mask_causal_document(n, docs), 1, 1)
    _compare(_run_fp32(fm, 1, 2, n, vecs, 66), vecs, 1)


@pytest.mark.parametrize("H,H_kv,Hm,D,det", [(4, 2, 1, 128, False), (4, 1, 1, 64, False), (6, 2, 6, 128, False),
                                             (8, 8, 1, 64, False), (6, 2, 6, 128, True)])
def test_grouped_query_heads(fm, H, H_kv, Hm, D, det):
    """Grouped-query attention: K / V have H_kv heads, query head h reads K/V head h // (H / H_kv).
    The oracle sees K / V repeated to H heads; the reference dK / dV of a K/V head is the sum over
    its query heads of their gradients (the plain chain rule through the repetition)."""
    n, seed, g = 640, 81, H // H_kv
    fams = ["causal_document", "share_question", "sliding_window_2k", "prefix_lm", "random_eviction", "full"]
    if Hm == 1:
        vecs = _vec_stack(synth.make_family("causal_document", n, seed), 1, 1)
    else:
        specs = [synth.make_family(fams[h % len(fams)], n, seed + h) for h in range(H)]
        vecs = [np.stack([sp.vectors()[c] for sp in specs])[None] for c in range(4)]  # [1, H, n]
    bits = [synth.normal_bf16_bits(seed, t, (1, n, hh, D)) for t, hh in ((1, H), (2, H_kv), (3, H_kv), (4, H))]
    host = [synth.bf16_bits_to_f32(x) for x in bits]
    dev = [_bf16_tensor(x) for x in bits]
    vt = [torch.from_numpy(np.ascontiguousarray(v, np.int32)).cuda() for v in vecs]
    scale = 1.0 / math.sqrt(D)
    meta = fm.fm_build_mask_meta(*vt, n_q=n)
    o, lse = fm.fm_attn_fwd(dev[0], dev[1], dev[2], meta, vt, scale)
    dq, dk, dv = fm.fm_attn_bwd(dev[0], dev[1], dev[2], o, lse, dev[3], meta, vt, scale, deterministic=det)
    torch.cuda.synchronize()
    assert fm.fm_get_device_status() == 0
    assert dk.shape == (1, n, H_kv, D)
    k_exp, v_exp = np.repeat(host[1], g, axis=2), np.repeat(host[2], g, axis=2)
    dk_ref = np.zeros((n, H_kv, D))
    dv_ref = np.zeros((n, H_kv, D))
    o_np, lse_np, dq_np = o.float().cpu().numpy(), lse.cpu().numpy(), dq.float().cpu().numpy()
    for h in range(H):
        ref = oracle.attention_head(host[0], k_exp, v_exp, vecs, 0, h, scale, cols=np.arange(n), dout=host[3],
                                    Hm=Hm)
        live = np.isfinite(ref["lse"])
        assert np.abs(o_np[0, :, h] - ref["o"]).max() <= O_TOL
        if live.any():
            assert np.abs(lse_np[0, h][live] - ref["lse"][live]).max() <= LSE_TOL
        assert np.abs(dq_np[0, :, h] - ref["dq"]).max() <= G_TOL * max(np.abs(ref["dq"]).max(), 1e-30)
        dk_ref[:, h // g] += ref["dk"]
        dv_ref[:, h // g] += ref["dv"]
    for name, got, exp in (("dk", dk, dk_ref), ("dv", dv, dv_ref)):
        for hk in range(H_kv):
            e = exp[:, hk]
            err = np.abs(got.float().cpu().numpy()[0, :, hk] - e).max() / max(np.abs(e).max(), 1e-30)
            assert err <= G_TOL, f"{name} head {hk}: rel-to-max {err}"


@pytest.mark.parametrize("family,n,B,H,D", [("causal_document", 1000, 2, 3, 128), ("global_sliding", 2048, 1, 2, 64),
                                             ("random_eviction", 1536, 1, 4, 128)])
def test_fixed_order_dq(fm, family, n, B, H, D):
    """deterministic=1: dQ matches the oracle, and three backward calls on the same inputs give
    bitwise identical dQ, dK and dV (each query tile takes its key tiles' contributions in
    ascending key-tile order)."""
    vecs = _vec_stack(synth.make_family(family, n, 93), B, 1)
    res = _run_attention(fm, B, H, n, n, D, vecs, 1, seed=94, det=True)
    _compare(res, vecs, 1)
    q, k, v, do = res["dev"]
    for _ in range(2):
        again = fm.fm_attn_bwd(q, k, v, res["o"], res["lse"], do, res["meta"], res["vt"], res["scale"],
                               deterministic=True)
        torch.cuda.synchronize()
        assert fm.fm_get_device_status() == 0
        for name, a, b in zip(("dq", "dk", "dv"), (res["dq"], res["dk"], res["dv"]), again):
            assert torch.equal(a.view(torch.int16), b.view(torch.int16)), f"{name} differs between calls"


def test_fully_masked_key_tile(fm):
    """Keys 128..255 masked for every row: that key tile has an empty column list (no MMA work),
    its dK / dV are exactly 0, and the other tiles still match the oracle."""
    n_q, n_k = 256, 512
    lts = np.full(n_k, n_q, np.int32)
    lte = np.full(n_k, n_q, np.int32)
    lts[128:256], lte[128:256] = 0, n_q
    uts = np.zeros(n_k, np.int32)
    ute = np.minimum(np.arange(n_k), n_q).astype(np.int32)  # causal on the remaining keys
    vecs = [x[None, None] for x in (lts, lte, uts, ute)]
    res = _run_attention(fm, 1, 2, n_q, n_k, 128, vecs, 1, seed=91)
    assert int(res["meta"].col_count[0, 0, 1].item()) == 0
    _compare(res, vecs, 1)
    assert np.all(res["dk"].float().cpu().numpy()[0, 128:256] == 0.0)
    assert np.all(res["dv"].float().cpu().numpy()[0, 128:256] == 0.0)


def test_dead_rows_and_cross_lengths(fm):
    n_q, n_k = 256, 512
    r = np.random.default_rng(3)
    lts = r.integers(0, n_q, n_k).astype(np.int32)
    lte = r.integers(0, n_q + 1, n_k).astype(np.int32)
    uts = np.zeros(n_k, np.int32)
    ute = r.integers(0, n_q, n_k).astype(np.int32)
    lts[:] = np.minimum(lts, 100)   # rows 100..139 are masked by every key
    lte[:] = np.maximum(lte, 140)
    vecs = [x[None, None] for x in (lts, lte, uts, ute)]
    res = _run_attention(fm, 1, 2, n_q, n_k, 128, vecs, 1, seed=4)
    _compare(res, vecs, 1)
    assert np.all(res["dq"].float().cpu().numpy()[0, 100:140] == 0.0)


def test_per_head_vectors_and_null(fm):
    n, H = 384, 2
    a, b_ = synth.mask_causal(n), synth.make_family("bidir_document", n, 5)
    vecs = [np.stack([x, y])[None] for x, y in zip(a.vectors(), b_.vectors())]  # [1, 2, n]
    res = _run_attention(fm, 1, H, n, n, 128, vecs, 2, seed=6)
    _compare(res, vecs, 2)
    vecs_null = [None, None, None, synth.mask_causal(n).ute[None, None]]
    res = _run_attention(fm, 1, H, n, n, 128, vecs_null, 1, seed=7)
    _compare(res, vecs_null, 1)


def test_forward_deterministic(fm):
    n = 1024
    spec = synth.make_family("causal_document", n, 8)
    vecs = _vec_stack(spec, 1, 1)
    r1 = _run_attention(fm, 1, 4, n, n, 128, vecs, 1, seed=9, bwd=False)
    r2 = _run_attention(fm, 1, 4, n, n, 128, vecs, 1, seed=9, bwd=False)
    assert torch.equal(r1["o"], r2["o"]) and torch.equal(r1["lse"], r2["lse"])


def _sample(n, count, seed, extra=()):
    rng = synth.Rng(seed)
    idx = set(rng.sample_distinct(0, n - 1, min(count, n)))
    idx.update(extra)
    return np.array(sorted(idx), dtype=np.int32)


@pytest.mark.parametrize("mask", ["sliding_window", "causal_document"])
def test_n8192_sampled(fm, mask):
    """B=2, H=16, n=8192, D=128: (a) causal sliding window w=1024, (b) causal
    documents with lengths ~ U[512, 4096]; checked on seeded samples of 512 rows
    and 512 columns for two heads."""
    n, B, H, D = 8192, 2, 16, 128
    if mask == "sliding_window":
        spec = synth.mask_sliding_window(n, 1024)
    else:
        spec = synth.mask_causal_document(n, synth.draw_docs(synth.Rng(2001), n, 512, 4096))
    vecs = _vec_stack(spec, B, 1)
    res = _run_attention(fm, B, H, n, n, D, vecs, 1, seed=2000 + (mask == "causal_document"))
    rows = _sample(n, 512, 11, extra=(0, n - 1))
    cols = _sample(n, 512, 12, extra=(0, n - 1))
    _compare(res, vecs, 1, heads=[(0, 0), (1, 15)], rows=rows, cols=cols)


def test_localized_forward_equals_global_rows(fm):
    """Clip-shift-max + rank-local forward: each simulated rank's output rows are
    bitwise equal to the corresponding rows of the global forward."""
    N, nch, H, D = 4096, 8, 2, 128
    chunk = N // nch
    spec = synth.mask_causal_document(N, synth.draw_docs(synth.Rng(5), N, 256, 1024))
    host, dev = _inputs(1, N, N, H, D, 50)
    vt = [torch.from_numpy(np.ascontiguousarray(x[None, None])).cuda() for x in spec.vectors()]
    scale = 1.0 / math.sqrt(D)
    gmeta = fm.fm_build_mask_meta(*vt, n_q=N)
    go, glse = fm.fm_attn_fwd(dev[0], dev[1], dev[2], gmeta, vt, scale)
    R = nch // 2
    starts = [[r * chunk, (nch - 1 - r) * chunk] for r in range(R)]
    lens = [[chunk, chunk]] * R
    loc = fm.fm_localize(vt, starts, lens)
    for r in range(R):
        rows = torch.cat([torch.arange(s, s + chunk) for s in starts[r]]).cuda()
        ql = dev[0][:, rows].contiguous()
        lv = [x[r].contiguous() for x in loc]
        lmeta = fm.fm_build_mask_meta(*lv, n_q=2 * chunk)
        lo, llse = fm.fm_attn_fwd(ql, dev[1], dev[2], lmeta, lv, scale)
        torch.cuda.synchronize()
        assert torch.equal(lo, go[:, rows]), f"rank {r}: O differs"
        assert torch.equal(llse, glse[:, :, rows]), f"rank {r}: LSE differs"
    assert fm.fm_get_device_status() == 0


@pytest.mark.parametrize("causal", [True, False])
def test_varlen_packed_batch(fm, causal):
    """A packed variable-length batch (one empty sequence, a padding tail past the last one):
    fm_varlen_mask matches the oracle's vectors bit for bit, the packed attention matches the
    oracle, and each sequence's rows match the same sequence run on its own (causal or unmasked),
    so the packing is invisible to the result."""
    N, H, D = 1500, 2, 128
    cu = np.array([0, 200, 712, 712, 1000, 1392], np.int32)  # sequence 2 is empty; keys 1392.. pad
    vecs_dev = fm.fm_varlen_mask(torch.from_numpy(cu).cuda(), N, causal=causal)
    torch.cuda.synchronize()
    ref_vecs = oracle.varlen_vectors(cu, N, causal)
    for got, exp in zip(vecs_dev, ref_vecs):
        np.testing.assert_array_equal(got.cpu().numpy()[0, 0], exp)
    vecs = [x[None, None] for x in ref_vecs]
    res = _run_attention(fm, 1, H, N, N, D, vecs, 1, seed=95)
    _compare(res, vecs, 1)
    assert np.all(np.isneginf(res["lse"].cpu().numpy()[0, :, 1392:]))  # padding rows see no key
    q, k, v, do = res["dev"]
    for s in range(len(cu) - 1):
        a, b = int(cu[s]), int(cu[s + 1])
        if a == b:
            continue
        L = b - a
        alone = [np.full(L, L), np.full(L, L), np.zeros(L), np.arange(L) if causal else np.zeros(L)]
        vt = [torch.from_numpy(x.astype(np.int32)[None, None]).cuda() for x in alone]
        meta = fm.fm_build_mask_meta(*vt, n_q=L)
        qs, ks, vs, dos = (x[:, a:b].contiguous() for x in (q, k, v, do))
        o, lse = fm.fm_attn_fwd(qs, ks, vs, meta, vt, res["scale"])
        dq, dk, dv = fm.fm_attn_bwd(qs, ks, vs, o, lse, dos, meta, vt, res["scale"])
        torch.cuda.synchronize()
        assert fm.fm_get_device_status() == 0
        assert (o.float() - res["o"][:, a:b].float()).abs().max().item() <= O_TOL
        assert (lse - res["lse"][:, :, a:b]).abs().max().item() <= LSE_TOL
        for name, alone, packed in (("dq", dq, res["dq"]), ("dk", dk, res["dk"]), ("dv", dv, res["dv"])):
            p = packed[:, a:b].float()
            err = (alone.float() - p).abs().max().item() / max(p.abs().max().item(), 1e-30)
            assert err <= G_TOL, f"{name} of sequence {s}: {err}"
