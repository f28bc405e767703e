"""Seeded synthetic inputs for the mask-aware attention path.

This module is shared by the tests, the bench and the oracle's tests.  It
holds no attention arithmetic: it produces (a) N(0,1) tensors from a
counter-based generator (see ``csrc/synth.c`` for the exact definition) and
(b) the four key-indexed boundary vectors (LTS, LTE, UTS, UTE) of the
structured mask families the FlashMask-3 pages name (document, prefix-LM,
share-question, sliding-window, block-sparse / causal-blockwise) plus the
families of the 12-mask sweep.

Mask convention (half-open, 0-based): key column j masks query row i iff
``LTS[j] <= i < LTE[j]`` or ``UTS[j] <= i < UTE[j]``.  "Four numbers per
avenue": each key has at most two masked stretches of query rows
(learnaivisually.com explainer, "four-vector sparse attention masks").

The vector encodings below are the input a user of the method would build;
the oracle checks each one against an independent dense predicate.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libfm_synth.so")
_lib = None

MASK = (1 << 64) - 1


def build(force: bool = False) -> str:
    """Compile csrc/synth.c into libfm_synth.so (plain C, OpenMP)."""
    src = os.path.join(_HERE, "csrc", "synth.c")
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(src):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", src, "-o", _LIB_PATH, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        u64, i64, vp = ctypes.c_uint64, ctypes.c_int64, ctypes.c_void_p
        lib.synth_splitmix64.restype = u64
        lib.synth_splitmix64.argtypes = [u64]
        lib.synth_normal_f32.argtypes = [u64, u64, u64, i64, vp]
        lib.synth_normal_bf16.argtypes = [u64, u64, u64, i64, vp]
        lib.synth_bf16_to_f32.argtypes = [vp, i64, vp]
        lib.synth_f32_to_bf16.argtypes = [vp, i64, vp]
        _lib = lib
    return _lib


# ----------------------------------------------------------------------------
# tensors
# ----------------------------------------------------------------------------
TENSOR_IDS = {"q": 1, "k": 2, "v": 3, "do": 4}


def normal_f32(seed: int, tensor_id: int, shape, offset: int = 0) -> np.ndarray:
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.float32)
    _load().synth_normal_f32(seed & MASK, tensor_id & MASK, offset, n, out.ctypes.data)
    return out.reshape(shape)


def normal_bf16_bits(seed: int, tensor_id: int, shape, offset: int = 0) -> np.ndarray:
    """N(0,1) rounded to bf16; returned as uint16 bit patterns."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    _load().synth_normal_bf16(seed & MASK, tensor_id & MASK, offset, n, out.ctypes.data)
    return out.reshape(shape)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    out = np.empty(bits.shape, dtype=np.float32)
    _load().synth_bf16_to_f32(bits.ctypes.data, bits.size, out.ctypes.data)
    return out


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint16)
    _load().synth_f32_to_bf16(x.ctypes.data, x.size, out.ctypes.data)
    return out


def splitmix64(x: int) -> int:
    """Pure-Python SplitMix64 mix (same constants as csrc/synth.c)."""
    z = (x + 0x9E3779B97F4A7C15) & MASK
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK
    return z ^ (z >> 31)


class Rng:
    """Sequential SplitMix64 stream for mask parameters (lengths, prefixes)."""

    def __init__(self, seed: int):
        self.state = splitmix64(seed & MASK)

    def next_u64(self) -> int:
        self.state = (self.state + 0x9E3779B97F4A7C15) & MASK
        z = self.state
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK
        return z ^ (z >> 31)

    def randint(self, lo: int, hi: int) -> int:
        """Uniform integer in [lo, hi] (inclusive)."""
        assert hi >= lo
        return lo + self.next_u64() % (hi - lo + 1)

    def sample_distinct(self, lo: int, hi: int, count: int) -> list:
        """``count`` distinct integers from [lo, hi], sorted (Fisher-Yates prefix)."""
        pool = list(range(lo, hi + 1))
        for t in range(count):
            r = t + self.next_u64() % (len(pool) - t)
            pool[t], pool[r] = pool[r], pool[t]
        return sorted(pool[:count])


# ----------------------------------------------------------------------------
# mask families: parameters and the four boundary vectors
# ----------------------------------------------------------------------------
@dataclass
class MaskSpec:
    family: str
    n: int                      # query rows = key columns for the families
    params: dict = field(default_factory=dict)
    lts: np.ndarray = None
    lte: np.ndarray = None
    uts: np.ndarray = None
    ute: np.ndarray = None

    def vectors(self):
        return self.lts, self.lte, self.uts, self.ute


def draw_segments(rng: Rng, n: int, lo: int, hi: int) -> list:
    """Segment lengths ~ U[lo, hi] drawn until they cover n; the last is cut to end at n.
    Returns a list of [start, end) pairs."""
    segs, s = [], 0
    while s < n:
        L = rng.randint(lo, hi)
        e = min(s + L, n)
        segs.append((s, e))
        s = e
    return segs


def cut_segments(rng: Rng, n: int, ndocs: int) -> list:
    """``ndocs`` documents from ndocs-1 distinct seeded cut points in [1, n-1]."""
    cuts = rng.sample_distinct(1, n - 1, ndocs - 1)
    edges = [0] + cuts + [n]
    return [(edges[t], edges[t + 1]) for t in range(ndocs)]


def _doc_arrays(n: int, docs: list):
    s = np.empty(n, dtype=np.int64)
    e = np.empty(n, dtype=np.int64)
    for (a, b) in docs:
        s[a:b] = a
        e[a:b] = b
    return s, e


def _pack(spec: MaskSpec, lts, lte, uts, ute) -> MaskSpec:
    spec.lts = np.ascontiguousarray(lts, dtype=np.int32)
    spec.lte = np.ascontiguousarray(lte, dtype=np.int32)
    spec.uts = np.ascontiguousarray(uts, dtype=np.int32)
    spec.ute = np.ascontiguousarray(ute, dtype=np.int32)
    return spec


def mask_full(n: int) -> MaskSpec:
    j = np.arange(n)
    return _pack(MaskSpec("full", n), np.full(n, n), np.full(n, n), np.zeros(n), np.zeros(n))


def mask_causal(n: int) -> MaskSpec:
    j = np.arange(n)
    return _pack(MaskSpec("causal", n), np.full(n, n), np.full(n, n), np.zeros(n), j)


def mask_sliding_window(n: int, w: int) -> MaskSpec:
    """Causal sliding window: key j is seen by rows j <= i < j + w (LTS stored clipped to n)."""
    j = np.arange(n)
    return _pack(MaskSpec("sliding_window", n, {"w": w}),
                 np.minimum(j + w, n), np.full(n, n), np.zeros(n), j)


def mask_causal_document(n: int, docs: list) -> MaskSpec:
    j = np.arange(n)
    s, e = _doc_arrays(n, docs)
    return _pack(MaskSpec("causal_document", n, {"docs": docs}), e, np.full(n, n), np.zeros(n), j)


def mask_bidir_document(n: int, docs: list) -> MaskSpec:
    s, e = _doc_arrays(n, docs)
    return _pack(MaskSpec("bidir_document", n, {"docs": docs}), e, np.full(n, n), np.zeros(n), s)


def mask_prefix_lm(n: int, prefix: int) -> MaskSpec:
    j = np.arange(n)
    ute = np.where(j < prefix, 0, j)
    return _pack(MaskSpec("prefix_lm", n, {"prefix": prefix}), np.full(n, n), np.full(n, n), np.zeros(n), ute)


def mask_prefix_lm_document(n: int, docs: list, prefixes: list) -> MaskSpec:
    j = np.arange(n)
    s, e = _doc_arrays(n, docs)
    pend = np.empty(n, dtype=np.int64)
    for (a, b), p in zip(docs, prefixes):
        pend[a:b] = a + p
    ute = np.where(j < pend, s, j)
    return _pack(MaskSpec("prefix_lm_document", n, {"docs": docs, "prefixes": prefixes}),
                 e, np.full(n, n), np.zeros(n), ute)


def mask_share_question(n: int, groups: list) -> MaskSpec:
    """groups: list of (question (s, e), [answers (s, e), ...]).  A question key is
    seen causally by every row of its group; an answer key causally inside its answer."""
    j = np.arange(n)
    lts = np.full(n, n, dtype=np.int64)
    for (qs, qe), answers in groups:
        gend = answers[-1][1] if answers else qe
        lts[qs:qe] = gend
        for (a, b) in answers:
            lts[a:b] = b
    return _pack(MaskSpec("share_question", n, {"groups": groups}), lts, np.full(n, n), np.zeros(n), j)


def mask_causal_blockwise(n: int, block: int = 64) -> MaskSpec:
    j = np.arange(n)
    return _pack(MaskSpec("causal_blockwise", n, {"block": block}),
                 np.full(n, n), np.full(n, n), np.zeros(n), (j // block) * block)


def mask_global_sliding(n: int, g: int, w: int) -> MaskSpec:
    """First g tokens global (see and are seen by all); others a symmetric band |i-j| < w."""
    j = np.arange(n)
    glob = j < g
    lts = np.where(glob, n, np.minimum(j + w, n))
    uts = np.where(glob, 0, g)
    ute = np.where(glob, 0, np.maximum(g, j - w + 1))
    return _pack(MaskSpec("global_sliding", n, {"g": g, "w": w}), lts, np.full(n, n), uts, ute)


def mask_random_eviction(n: int, evict: np.ndarray) -> MaskSpec:
    """Causal, and key j is evicted from row evict[j] on (evict[j] in [j+1, n])."""
    j = np.arange(n)
    return _pack(MaskSpec("random_eviction", n, {"evict": evict}),
                 evict, np.full(n, n), np.zeros(n), j)


# ---- seeded parameter draws -------------------------------------------------
def draw_docs(rng: Rng, n: int, lo: int, hi: int) -> list:
    return draw_segments(rng, n, lo, hi)


def draw_share_question(rng: Rng, n: int, q_lo=1024, q_hi=4096, a_cnt=(2, 6), a_lo=256, a_hi=2048) -> list:
    groups, s = [], 0
    while s < n:
        qe = min(s + rng.randint(q_lo, q_hi), n)
        answers, a = [], qe
        cnt = rng.randint(*a_cnt)
        for _ in range(cnt):
            if a >= n:
                break
            b = min(a + rng.randint(a_lo, a_hi), n)
            answers.append((a, b))
            a = b
        groups.append(((s, qe), answers))
        s = a
    return groups


SWEEP_FAMILIES = ["full", "causal", "sliding_window_2k", "sliding_window_8k", "causal_document",
                  "bidir_document", "prefix_lm", "prefix_lm_document", "share_question",
                  "causal_blockwise", "global_sliding", "random_eviction"]


def make_family(name: str, n: int, seed: int) -> MaskSpec:
    """One of the 12 sweep masks at length n, parameters drawn from ``seed``.
    Document lengths ~ U[4096, 65536] scaled down for short n (min(n/2, .)) so that
    small test sizes still hold several documents."""
    rng = Rng(seed)
    dlo, dhi = min(4096, max(n // 8, 16)), min(65536, max(n // 2, 32))
    if name == "full":
        return mask_full(n)
    if name == "causal":
        return mask_causal(n)
    if name == "sliding_window_2k":
        return mask_sliding_window(n, min(2048, max(n // 4, 1)))
    if name == "sliding_window_8k":
        return mask_sliding_window(n, min(8192, max(n // 2, 1)))
    if name == "causal_document":
        return mask_causal_document(n, draw_docs(rng, n, dlo, dhi))
    if name == "bidir_document":
        return mask_bidir_document(n, draw_docs(rng, n, dlo, dhi))
    if name == "prefix_lm":
        return mask_prefix_lm(n, rng.randint(n // 8, n // 2))
    if name == "prefix_lm_document":
        docs = draw_docs(rng, n, dlo, dhi)
        prefixes = [rng.randint(-(-(b - a) // 8), max((b - a) // 2, -(-(b - a) // 8))) for (a, b) in docs]
        return mask_prefix_lm_document(n, docs, prefixes)
    if name == "share_question":
        if n >= 32768:
            groups = draw_share_question(rng, n)
        else:  # shrink the question/answer lengths for short test sequences
            f = max(n / 32768.0, 1.0 / 64)
            groups = draw_share_question(rng, n, max(int(1024 * f), 4), max(int(4096 * f), 8), (2, 6),
                                         max(int(256 * f), 2), max(int(2048 * f), 4))
        return mask_share_question(n, groups)
    if name == "causal_blockwise":
        return mask_causal_blockwise(n, 64)
    if name == "global_sliding":
        return mask_global_sliding(n, min(1024, max(n // 16, 1)), min(2048, max(n // 8, 1)))
    if name == "random_eviction":
        ev = np.array([rng.randint(j + 1, n) for j in range(n)], dtype=np.int64)
        return mask_random_eviction(n, ev)
    raise ValueError(name)


def canonical_empty(n_q: int, n_k: int):
    """Vectors that mask nothing: lower LTS=LTE=n_q, upper UTS=UTE=0."""
    return (np.full(n_k, n_q, np.int32), np.full(n_k, n_q, np.int32),
            np.zeros(n_k, np.int32), np.zeros(n_k, np.int32))
