"""Oracle for the mask-aware attention hot path -- TEST INFRASTRUCTURE ONLY.

Plain, slow, fp64 CPU implementation (``fm_oracle.cpp``) of what the CUDA
library computes: dense expansion of the four boundary vectors, per-tile
min/max + classification + block lists, clip-shift-max localization, and exact
masked softmax attention forward/backward.  Only ``tests/``, the smoke check
and the bench's CPU-baseline leg may import this package; the library never
does, and this package never imports the library.

Each wrapper names the passage it follows (FlashMask-3 pages):
  [abstract]  acceptodds.com, FlashMask-3 paper abstract
  [explainer] learnaivisually.com, "Four-vector sparse attention masks"
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libfm_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile fm_oracle.cpp (plain C++17 + OpenMP; no CUDA)."""
    src = os.path.join(_HERE, "fm_oracle.cpp")
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(src):
        subprocess.run(["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-fopenmp", src, "-o", _LIB_PATH],
                       check=True)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        i32, i64, vp, f64 = ctypes.c_int32, ctypes.c_int64, ctypes.c_void_p, ctypes.c_double
        L.orc_dense_mask.argtypes = [i32, i32, vp, vp, vp, vp, vp]
        L.orc_count_unmasked_dense.argtypes = [i32, i32, vp, vp, vp, vp]
        L.orc_count_unmasked_dense.restype = i64
        L.orc_count_unmasked_intervals.argtypes = [i32, i32, vp, vp, vp, vp]
        L.orc_count_unmasked_intervals.restype = i64
        L.orc_kv_chunk_pairs.argtypes = [i32, i32, i32, vp, vp, vp, vp, vp]
        L.orc_tile_meta.argtypes = [i32, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
        L.orc_localize_clip_shift_max.argtypes = [i64, vp, i32, vp, vp, vp]
        L.orc_localize_count.argtypes = [i64, vp, i32, vp, vp, vp]
        L.orc_attention_head.argtypes = [i32, i32, i32, i32, i32, i32, f64, vp, vp, vp, vp, vp, vp, vp, vp,
                                         i32, i32, i32, vp, i32, vp, vp, vp, vp, vp, vp, i32]
        L.orc_attention_head.restype = ctypes.c_int
        L.orc_max_threads.restype = ctypes.c_int
        _lib = L
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data


def _i32(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.int32)


def max_threads() -> int:
    return _load().orc_max_threads()


# ---- masks ------------------------------------------------------------------
def dense_mask(n_q, n_k, lts, lte, uts, ute) -> np.ndarray:
    """[explainer] "four numbers per avenue": True where (i, j) is masked
    (half-open intervals [LTS, LTE) and [UTS, UTE) of query rows per key j)."""
    v = [_i32(x) for x in (lts, lte, uts, ute)]
    out = np.empty((n_q, n_k), dtype=np.uint8)
    _load().orc_dense_mask(n_q, n_k, *[_ptr(x) for x in v], out.ctypes.data)
    return out.astype(bool)


def count_unmasked_dense(n_q, n_k, lts, lte, uts, ute) -> int:
    v = [_i32(x) for x in (lts, lte, uts, ute)]
    return int(_load().orc_count_unmasked_dense(n_q, n_k, *[_ptr(x) for x in v]))


def count_unmasked(n_q, n_k, lts, lte, uts, ute) -> int:
    """Unmasked pairs from interval lengths (O(n_k)); equals the dense count."""
    v = [_i32(x) for x in (lts, lte, uts, ute)]
    return int(_load().orc_count_unmasked_intervals(n_q, n_k, *[_ptr(x) for x in v]))


def kv_chunk_pairs(n_q, n_k, chunk_len, lts, lte, uts, ute) -> np.ndarray:
    """[explainer] across-ranks paragraph ("skips key-value chunks that are fully
    masked"): unmasked (row, key) pairs of rows [0, n_q) per chunk of chunk_len
    keys; a zero entry is a chunk no row attends to."""
    v = [None if x is None else _i32(x) for x in (lts, lte, uts, ute)]
    out = np.empty(-(-n_k // chunk_len), np.int64)
    _load().orc_kv_chunk_pairs(n_q, n_k, chunk_len, *[None if x is None else _ptr(x) for x in v], out.ctypes.data)
    return out


def varlen_vectors(cu_seqlens, N, causal) -> list:
    """[explainer] document masks: sequences packed end to end, each attending
    only within itself (causal or bidirectional).  Sequence s owns positions
    [cu[s], cu[s+1]).  Its keys mask the rows after the sequence through the lower
    stretch [cu[s+1], N) and, through the upper stretch [0, UTE), the rows before
    the key (causal: UTE = j) or before the sequence (UTE = cu[s]).  Reading:
    keys past cu[-1] (padding) mask every row ([0, N) as the lower stretch)."""
    cu = [int(x) for x in cu_seqlens]
    lts = np.zeros(N, np.int32)
    lte = np.full(N, N, np.int32)
    uts = np.zeros(N, np.int32)
    ute = np.zeros(N, np.int32)
    for s in range(len(cu) - 1):
        for j in range(cu[s], cu[s + 1]):
            lts[j] = cu[s + 1]
            ute[j] = j if causal else cu[s]
    return [lts, lte, uts, ute]


def tile_meta(n_q, n_k, lts, lte, uts, ute, tile_q=128, tile_k=128) -> dict:
    """[explainer] tile paragraph: per-key-tile min/max of the four vectors,
    class of every (query tile, key tile) pair (0 skip, 1 partial, 2 full) and
    the compacted row / column block lists."""
    v = [_i32(x) for x in (lts, lte, uts, ute)]
    T_q, T_k = -(-n_q // tile_q), -(-n_k // tile_k)
    mm = np.empty((T_k, 8), np.int32)
    cls = np.empty((T_q, T_k), np.uint8)
    rc = np.empty(T_q, np.int32)
    re = np.zeros((T_q, T_k), np.int32)
    cc = np.empty(T_k, np.int32)
    ce = np.zeros((T_k, T_q), np.int32)
    _load().orc_tile_meta(n_q, n_k, tile_q, tile_k, *[_ptr(x) for x in v], mm.ctypes.data, cls.ctypes.data,
                          rc.ctypes.data, re.ctypes.data, cc.ctypes.data, ce.ctypes.data)
    return {"minmax": mm, "cls": cls, "row_count": rc, "row_entries": re, "col_count": cc, "col_entries": ce}


def localize(vec, starts, lens, formula: str = "clip_shift_max") -> np.ndarray:
    """[explainer] clip-shift-max paragraph; [abstract] "zero-communication
    clip-shift-max on the boundary vectors".  Maps one global vector onto a rank
    owning chunks [starts[k], starts[k]+lens[k]) (increasing order)."""
    vec = _i32(vec)
    g, L = _i32(starts), _i32(lens)
    out = np.empty_like(vec)
    fn = _load().orc_localize_clip_shift_max if formula == "clip_shift_max" else _load().orc_localize_count
    fn(vec.size, vec.ctypes.data, len(g), g.ctypes.data, L.ctypes.data, out.ctypes.data)
    return out


# ---- attention --------------------------------------------------------------
def attention_head(q, k, v, vecs, b, h, scale, rows=None, cols=None, dout=None, Hm=1, nthreads=0):
    """Exact fp64 masked attention for head (b, h).

    q, dout: float32 [B, n_q, H, D]; k, v: float32 [B, n_k, H, D];
    vecs: 4 arrays [B, Hm, n_k] (or None = canonical empty).
    rows: query rows to return (O, LSE, and dQ if dout given); cols: key columns
    for dK, dV (needs dout).  Returns a dict of float64 arrays."""
    B, n_q, H, D = q.shape
    n_k = k.shape[1]
    if not (0 <= b < B and 0 <= h < H) or Hm not in (1, H):
        raise ValueError("oracle: bad arguments")
    # The C++ code reads only head (b, h): hand it that head as contiguous [1, n, 1, D] copies (and
    # the head's vector rows), so that its key loop walks memory in order.  Same values, same
    # arithmetic; only the layout of the input changes.
    hm = 0 if Hm == 1 else h
    q = np.ascontiguousarray(q[b:b + 1, :, h:h + 1], np.float32)
    k = np.ascontiguousarray(k[b:b + 1, :, h:h + 1], np.float32)
    v = np.ascontiguousarray(v[b:b + 1, :, h:h + 1], np.float32)
    dd = None if dout is None else np.ascontiguousarray(dout[b:b + 1, :, h:h + 1], np.float32)
    vv = [None if x is None else _i32(np.asarray(x)[b:b + 1, hm:hm + 1]) for x in vecs]
    B, H, Hm, b, h = 1, 1, 1, 0, 0
    rows = np.arange(n_q, dtype=np.int32) if rows is None else _i32(rows)
    cols = np.zeros(0, np.int32) if cols is None else _i32(cols)
    if cols.size and dd is None:
        raise ValueError("column outputs need dout")
    o = np.zeros((rows.size, D))
    lse = np.zeros(rows.size)
    dq = np.zeros((rows.size, D)) if dd is not None else None
    dk = np.zeros((cols.size, D))
    dv = np.zeros((cols.size, D))
    rc = _load().orc_attention_head(B, H, Hm, n_q, n_k, D, float(scale), q.ctypes.data, k.ctypes.data,
                                    v.ctypes.data, _ptr(dd), *[_ptr(x) for x in vv], b, h, rows.size,
                                    rows.ctypes.data, cols.size, cols.ctypes.data, o.ctypes.data,
                                    lse.ctypes.data, _ptr(dq), dk.ctypes.data, dv.ctypes.data, nthreads)
    if rc != 0:
        raise ValueError("oracle: bad arguments")
    out = {"o": o, "lse": lse, "rows": rows}
    if dd is not None:
        out["dq"] = dq
    if cols.size:
        out.update({"dk": dk, "dv": dv, "cols": cols})
    return out
