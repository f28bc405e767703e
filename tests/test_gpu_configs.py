"""GPU parity at the full workload sizes, in the launch configuration bench.py
times, on seeded samples the oracle can compute one by one:
  * n=32768, B=1, H=32, D=128: prefix-LM (P ~ U[n/8, n/2]) and share-question;
  * n=131072, B=1, H=16, D=128: the 12-mask sweep, 512 sampled query rows
    (O, LSE, dQ) of the first, middle and last head of every mask; 512 sampled
    key columns (dK, dV) of the same heads for the masks whose oracle all-rows
    statistics pass is affordable at 131072 tokens (sliding window 2K and 8K,
    share-question, global + sliding window);
  * n=32768, B=1, H=32, D=128: the other eight sweep masks (full, causal,
    prefix-LM, causal blockwise, random eviction and the three document masks),
    where the same column samples are affordable: 512 rows and 512 columns of
    three heads each, through the same kernel paths;
  * global n=262144, H=8: causal documents (L ~ U[4096, 65536]) localized by
    clip-shift-max to 16 simulated context-parallel ranks (32 chunks of 8192,
    rank r owns chunks r and 31-r); every rank's forward rows equal the global
    forward's rows bitwise, and the global forward matches the oracle.
Tolerances as in test_gpu_parity: O max-abs 1e-2, LSE 1e-3 (live rows), dQ/dK/dV
max-abs error / max-abs reference 2e-2; fully masked rows exact.  At 131072
tokens the dense masks' dK / dV are also checked through properties that hold
at any size (sum_j dV_j = sum over live rows of dO_i, sum_j dK_j = 0), as an
extra beside the element-wise checks at 32768."""
import math

import numpy as np
import pytest

import oracle
import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

O_TOL, LSE_TOL, G_TOL = 1e-2, 1e-3, 2e-2
N_SAMPLE = 512


@pytest.fixture(scope="module")
def fm():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from mask_aware_flash_b200 import _build
    _build.build()
    import mask_aware_flash_b200 as m
    m.lib()
    return m


def _sample(n, count, seed, extra=()):
    rng = synth.Rng(seed)
    idx = set(rng.sample_distinct(0, n - 1, min(count, n)))
    idx.update(int(x) for x in extra)
    return np.array(sorted(idx), dtype=np.int32)


def _inputs(B, n, H, D, seed):
    bits = [synth.normal_bf16_bits(seed, t, (B, n, H, D)) for t in (1, 2, 3, 4)]
    dev = [torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).cuda() for b in bits]
    host = [synth.bf16_bits_to_f32(b) for b in bits]
    return host, dev


def _check_rows(res_o, res_lse, res_dq, ref, b, h):
    rr = ref["rows"]
    live = np.isfinite(ref["lse"])
    o = res_o[b, rr, h].float().cpu().numpy()
    err = np.abs(o - ref["o"]).max()
    assert err <= O_TOL, f"O max-abs {err} (b={b}, h={h})"
    lse = res_lse[b, h, rr].cpu().numpy()
    if live.any():
        assert np.abs(lse[live] - ref["lse"][live]).max() <= LSE_TOL
    assert np.all(np.isneginf(lse[~live])) and np.all(o[~live] == 0.0)
    if res_dq is not None:
        dq = res_dq[b, rr, h].float().cpu().numpy()
        rel = np.abs(dq - ref["dq"]).max() / max(np.abs(ref["dq"]).max(), 1e-30)
        assert rel <= G_TOL, f"dQ rel {rel} (b={b}, h={h})"


def _check_cols(dk, dv, ref, b, h):
    cols = ref["cols"]
    for name, got, exp in (("dK", dk[b, cols, h], ref["dk"]), ("dV", dv[b, cols, h], ref["dv"])):
        g = got.float().cpu().numpy()
        rel = np.abs(g - exp).max() / max(np.abs(exp).max(), 1e-30)
        assert rel <= G_TOL, f"{name} rel {rel} (b={b}, h={h})"


SUM_EPS = 2.0 ** -8  # per-element relative error allowed in the sum checks (bf16 output rounding is 2^-9)


def _check_sums(dk, dv, do_host, lse, b, h):
    """sum_j dV_j = sum_{live i} dO_i and sum_j dK_j = 0 (bf16 outputs summed in fp64).  If every
    element carries a relative error of at most eps, the sum's error is at most eps * sum_j |x_j|:
    that is the bound, with eps = 2^-8.  (At 131072 keys the measured gap is ~1.5e-4 of the sum,
    of one sign: the fp32 accumulation over 8192 MMA steps shrinks magnitudes slightly.)"""
    live = torch.isfinite(lse[b, h]).cpu().numpy()
    sdv = dv[b, :, h].double().sum(0).cpu().numpy()
    want = do_host[b, live, h].astype(np.float64).sum(0)
    scale_v = dv[b, :, h].double().abs().sum(0).cpu().numpy()
    assert np.all(np.abs(sdv - want) <= SUM_EPS * scale_v), "sum dV"
    sdk = dk[b, :, h].double().sum(0).cpu().numpy()
    scale_k = dk[b, :, h].double().abs().sum(0).cpu().numpy()
    assert np.all(np.abs(sdk) <= SUM_EPS * scale_k), "sum dK"


def _heads(H):
    """First, middle and last head."""
    return sorted({0, H // 2, H - 1})


def _run(fm, dev, vecs, n, scale):
    vt = [torch.from_numpy(np.ascontiguousarray(v)).cuda() for v in vecs]
    meta = fm.fm_build_mask_meta(*vt, n_q=n)
    o, lse = fm.fm_attn_fwd(dev[0], dev[1], dev[2], meta, vt, scale)
    dq, dk, dv = fm.fm_attn_bwd(dev[0], dev[1], dev[2], o, lse, dev[3], meta, vt, scale)
    torch.cuda.synchronize()
    assert fm.fm_get_device_status() == 0
    return o, lse, dq, dk, dv


@pytest.mark.parametrize("mask", ["prefix_lm", "share_question"])
def test_n32768_masks(fm, mask):
    n, B, H, D = 32768, 1, 32, 128
    seed = 3000 + (mask == "share_question")
    spec = synth.make_family(mask, n, seed)
    vecs = [x[None, None] for x in spec.vectors()]
    host, dev = _inputs(B, n, H, D, seed)
    scale = 1.0 / math.sqrt(D)
    o, lse, dq, dk, dv = _run(fm, dev, vecs, n, scale)
    rows = _sample(n, N_SAMPLE, seed + 1, extra=[0, n - 1])
    cols = _sample(n, N_SAMPLE, seed + 2, extra=[0, n - 1])
    for h in _heads(H):
        ref = oracle.attention_head(*host[:3], vecs, 0, h, scale, rows=rows, cols=cols, dout=host[3])
        _check_rows(o, lse, dq, ref, 0, h)
        _check_cols(dk, dv, ref, 0, h)


# sweep masks whose oracle all-rows pass is affordable at 128K: column samples there; the others get
# their column samples at 32K (test_n32768_sweep_columns) and the gradient-sum properties at 128K
SPARSE_128K = {"sliding_window_2k", "sliding_window_8k", "share_question", "global_sliding"}
DENSE_SWEEP = [m for m in synth.SWEEP_FAMILIES if m not in SPARSE_128K]


@pytest.fixture(scope="module")
def inputs_128k():
    n, B, H, D = 131072, 1, 16, 128
    return _inputs(B, n, H, D, 4000)


@pytest.mark.parametrize("mask", synth.SWEEP_FAMILIES)
def test_n131072_sweep(fm, inputs_128k, mask):
    n, B, H, D = 131072, 1, 16, 128
    host, dev = inputs_128k
    m_idx = synth.SWEEP_FAMILIES.index(mask)
    spec = synth.make_family(mask, n, 4000 + m_idx)
    vecs = [x[None, None] for x in spec.vectors()]
    scale = 1.0 / math.sqrt(D)
    o, lse, dq, dk, dv = _run(fm, dev, vecs, n, scale)
    rows = _sample(n, N_SAMPLE, 4100 + m_idx, extra=[0, n - 1])
    cols = _sample(n, N_SAMPLE, 4200 + m_idx, extra=[0, n - 1]) if mask in SPARSE_128K else None
    for h in _heads(H):
        ref = oracle.attention_head(*host[:3], vecs, 0, h, scale, rows=rows, cols=cols, dout=host[3])
        _check_rows(o, lse, dq, ref, 0, h)
        if cols is not None:
            _check_cols(dk, dv, ref, 0, h)
        else:
            _check_sums(dk, dv, host[3], lse, 0, h)


@pytest.fixture(scope="module")
def inputs_32k():
    n, B, H, D = 32768, 1, 32, 128
    return _inputs(B, n, H, D, 4500)


@pytest.mark.parametrize("mask", DENSE_SWEEP)
def test_n32768_sweep_columns(fm, inputs_32k, mask):
    """The sweep masks whose 131072-token column check is out of the oracle's reach, at 32768 tokens
    with H = 32: 512 rows (O, LSE, dQ) and 512 columns (dK, dV) of the first, middle and last head."""
    n, B, H, D = 32768, 1, 32, 128
    host, dev = inputs_32k
    m_idx = synth.SWEEP_FAMILIES.index(mask)
    spec = synth.make_family(mask, n, 4500 + m_idx)
    vecs = [x[None, None] for x in spec.vectors()]
    scale = 1.0 / math.sqrt(D)
    o, lse, dq, dk, dv = _run(fm, dev, vecs, n, scale)
    rows = _sample(n, N_SAMPLE, 4600 + m_idx, extra=[0, n - 1])
    cols = _sample(n, N_SAMPLE, 4700 + m_idx, extra=[0, n - 1])
    for h in _heads(H):
        ref = oracle.attention_head(*host[:3], vecs, 0, h, scale, rows=rows, cols=cols, dout=host[3])
        _check_rows(o, lse, dq, ref, 0, h)
        _check_cols(dk, dv, ref, 0, h)


def test_localization_262144_16_ranks(fm):
    N, H, D, nch = 262144, 8, 128, 32
    chunk = N // nch
    R = nch // 2
    seed = 5000
    docs = synth.draw_docs(synth.Rng(seed), N, 4096, 65536)
    spec = synth.mask_causal_document(N, docs)
    vecs = [x[None, None] for x in spec.vectors()]
    host, dev = _inputs(1, N, H, D, seed)
    scale = 1.0 / math.sqrt(D)
    vt = [torch.from_numpy(np.ascontiguousarray(v)).cuda() for v in vecs]
    gmeta = fm.fm_build_mask_meta(*vt, n_q=N)
    go, glse = fm.fm_attn_fwd(dev[0], dev[1], dev[2], gmeta, vt, scale)
    starts = [[r * chunk, (nch - 1 - r) * chunk] for r in range(R)]
    lens = [[chunk, chunk]] * R
    loc = fm.fm_localize(vt, starts, lens)  # all 16 ranks in one launch
    torch.cuda.synchronize()
    # localized vectors: bit-exact vs the oracle (both formulas), sampled keys
    keys = _sample(N, 4096, seed + 3, extra=[0, N - 1])
    for c in range(4):
        got = loc[c][:, 0, 0, keys].cpu().numpy()
        for r in range(R):
            np.testing.assert_array_equal(got[r], oracle.localize(spec.vectors()[c][keys], starts[r], lens[r]))
    # KV-chunk pruning: per-rank unmasked pairs per KV chunk, bit-exact; over the ranks (which
    # partition the rows) they add up to the global mask's pairs per chunk
    pairs = fm.fm_kv_chunk_pairs(loc, [2 * chunk] * R, chunk).cpu().numpy()[:, 0, 0]
    for r in range(R):
        lv = [x[r, 0, 0].cpu().numpy() for x in loc]
        np.testing.assert_array_equal(pairs[r], oracle.kv_chunk_pairs(2 * chunk, N, chunk, *lv))
    np.testing.assert_array_equal(pairs.sum(0), oracle.kv_chunk_pairs(N, N, chunk, *spec.vectors()))
    assert (pairs == 0).sum() > 0  # documents: every rank skips some KV chunks
    for r in range(R):
        rows = torch.cat([torch.arange(s, s + chunk) for s in starts[r]]).cuda()
        lv = [x[r].contiguous() for x in loc]
        lmeta = fm.fm_build_mask_meta(*lv, n_q=2 * chunk)
        lo, llse = fm.fm_attn_fwd(dev[0][:, rows].contiguous(), dev[1], dev[2], lmeta, lv, scale)
        torch.cuda.synchronize()
        assert torch.equal(lo, go[:, rows]), f"rank {r}: O differs from the global rows"
        assert torch.equal(llse, glse[:, :, rows]), f"rank {r}: LSE differs from the global rows"
    # the global forward itself against the oracle on sampled rows of two heads
    rows = _sample(N, N_SAMPLE, seed + 4, extra=[0, N - 1])
    for h in (0, H - 1):
        ref = oracle.attention_head(*host[:3], vecs, 0, h, scale, rows=rows)
        _check_rows(go, glse, None, ref, 0, h)
    assert fm.fm_get_device_status() == 0


def test_maximum_tile_count_524288(fm):
    """The largest length the row / column lists hold: 4096 tiles of 128 (n = 524288).  Global +
    sliding window (128 global tokens, band 512): query tile 0 sees every key tile and key tile 0 is
    seen by every query tile, so both a row list and a column list hold all 4096 entries, while the
    oracle's all-rows pass stays affordable.  Sampled rows (O, LSE, dQ) and sampled columns (dK, dV)
    against the oracle; one tile more is rejected on the host (test_abi)."""
    n, B, H, D = 524288, 1, 1, 128
    host, dev = _inputs(B, n, H, D, 7000)
    spec = synth.mask_global_sliding(n, 128, 512)
    vecs = [x[None, None] for x in spec.vectors()]
    scale = 1.0 / math.sqrt(D)
    vt = [torch.from_numpy(np.ascontiguousarray(v)).cuda() for v in vecs]
    meta = fm.fm_build_mask_meta(*vt, n_q=n)
    o, lse = fm.fm_attn_fwd(dev[0], dev[1], dev[2], meta, vt, scale)
    dq, dk, dv = fm.fm_attn_bwd(dev[0], dev[1], dev[2], o, lse, dev[3], meta, vt, scale)
    torch.cuda.synchronize()
    assert fm.fm_get_device_status() == 0
    assert int(meta.row_count[0, 0, 0].item()) == 4096 and int(meta.col_count[0, 0, 0].item()) == 4096
    rows = _sample(n, N_SAMPLE, 7001, extra=[0, 127, 128, n - 129, n - 1])
    cols = _sample(n, N_SAMPLE, 7002, extra=[0, 127, 128, n - 1])
    ref = oracle.attention_head(*host[:3], vecs, 0, 0, scale, rows=rows, cols=cols, dout=host[3])
    _check_rows(o, lse, dq, ref, 0, 0)
    _check_cols(dk, dv, ref, 0, 0)
