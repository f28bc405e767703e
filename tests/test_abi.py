"""CPU-only checks of the C-ABI library: it builds, loads, exports every symbol
include/fm.h declares, and rejects bad arguments on the host before any CUDA
call (no compute is launched here)."""
import ctypes
import os
import re

import pytest

import mask_aware_flash_b200 as fm
from mask_aware_flash_b200 import _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def torch_cuda_present():
    import torch
    return torch.cuda.is_available()


@pytest.fixture(scope="module")
def L():
    _build.build()
    return fm.lib()


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "fm.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(fm_[a-z_0-9]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = _declared_functions()
    for want in ("fm_build_mask_meta", "fm_localize", "fm_attn_fwd", "fm_attn_bwd", "fm_mask_meta_workspace_bytes",
                 "fm_attn_bwd_workspace_bytes", "fm_get_device_status", "fm_status_string"):
        assert want in names


def test_library_exports_every_declared_symbol(L):
    for name in _declared_functions():
        assert hasattr(L, name), name


def test_status_strings(L):
    for code in range(7):
        assert fm.status_string(code) and fm.status_string(code) != "unknown status"
    assert fm.status_string(99) == "unknown status"


def test_meta_workspace_bytes(L):
    d = fm.MaskDesc(2, 1, 1024, 2048, 128, 128)
    n = L.fm_mask_meta_workspace_bytes(ctypes.byref(d))
    T_q, T_k = 8, 16
    assert n >= 2 * (T_k * 8 * 4 + T_q * 4 + T_q * T_k * 4 + T_k * 4 + T_k * T_q * 4 + T_q * T_k + (T_q // 2) * 4
                     + T_k * 4)
    assert n % 256 == 0
    bad = fm.MaskDesc(2, 1, 1024, 2048, 64, 128)
    assert L.fm_mask_meta_workspace_bytes(ctypes.byref(bad)) == 0
    assert L.fm_mask_meta_workspace_bytes(None) == 0


def test_build_meta_rejects_bad_args(L):
    c = fm.MaskMetaC()
    bad = fm.MaskDesc(1, 1, 0, 128, 128, 128)
    assert L.fm_build_mask_meta(ctypes.byref(bad), None, None, None, None, None, 0, ctypes.byref(c), None) == \
        fm.FM_ERR_INVALID_ARG
    good = fm.MaskDesc(1, 1, 128, 128, 128, 128)
    assert L.fm_build_mask_meta(ctypes.byref(good), None, None, None, None, None, 0, ctypes.byref(c), None) == \
        fm.FM_ERR_WORKSPACE
    assert L.fm_build_mask_meta(ctypes.byref(good), None, None, None, None, ctypes.c_void_p(0x1001), 1 << 20,
                                ctypes.byref(c), None) == fm.FM_ERR_WORKSPACE  # misaligned
    assert L.fm_build_mask_meta(ctypes.byref(good), None, None, None, None, ctypes.c_void_p(0x1000), 16,
                                ctypes.byref(c), None) == fm.FM_ERR_WORKSPACE  # too small


def _loc(L, starts, lens, N=1024, R=None, C=None, null_in=False):
    import numpy as np
    st = np.asarray(starts, np.int32)
    ln = np.asarray(lens, np.int32)
    fake = ctypes.c_void_p(0x10000)
    vin = fm.VecArray(*([None] * 4 if null_in else [0x10000] * 4))
    vout = fm.VecArray(*[0x20000] * 4)
    R = R if R is not None else st.shape[0]
    C = C if C is not None else st.shape[1]
    return L.fm_localize(1, 1, N, vin, R, C, st.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                         ln.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), vout, None)


def test_localize_rejects_bad_chunks(L):
    assert _loc(L, [[512, 0]], [[128, 128]]) == fm.FM_ERR_INVALID_ARG          # decreasing
    assert _loc(L, [[0, 100]], [[128, 128]]) == fm.FM_ERR_INVALID_ARG          # overlapping
    assert _loc(L, [[0, 1000]], [[128, 128]]) == fm.FM_ERR_INVALID_ARG         # past N
    assert _loc(L, [[0, 256]], [[0, 128]]) == fm.FM_ERR_INVALID_ARG            # empty chunk
    assert _loc(L, [[0, 256]], [[128, 128]], null_in=True) == fm.FM_ERR_INVALID_ARG
    assert _loc(L, [[0]] * 2, [[8]] * 2, R=300, C=1) == fm.FM_ERR_INVALID_ARG  # too many chunks


def _attn(L, n_q=256, n_k=256, D=128, dtype=0, meta_nq=None, Hm=1, H=2):
    a = fm.AttnArgs(1, H, n_q, n_k, D, dtype, 0.125, 0x10000, 0x20000, 0x30000)
    m = fm.MaskMetaC()
    m.d = fm.MaskDesc(1, Hm, meta_nq or n_q, n_k, 128, 128)
    m.row_count = m.row_entries = m.col_count = m.col_entries = m.tile_minmax = 0x40000
    m.tile_class = m.fwd_order = m.bwd_order = 0x40000
    return a, m


def test_fwd_rejects_before_launch(L):
    vec = fm.VecArray(None, None, None, None)
    o, lse = ctypes.c_void_p(0x50000), ctypes.c_void_p(0x60000)
    a, m = _attn(L, n_k=202)  # key length not a multiple of 4 (ragged lengths otherwise allowed)
    assert L.fm_attn_fwd(ctypes.byref(a), ctypes.byref(m), vec, o, lse, None) == fm.FM_ERR_UNSUPPORTED
    a, m = _attn(L, n_q=4097 * 128)  # one query tile more than the lists hold
    assert L.fm_attn_fwd(ctypes.byref(a), ctypes.byref(m), vec, o, lse, None) == fm.FM_ERR_UNSUPPORTED
    a, m = _attn(L, n_k=4097 * 128)
    assert L.fm_attn_fwd(ctypes.byref(a), ctypes.byref(m), vec, o, lse, None) == fm.FM_ERR_UNSUPPORTED
    a, m = _attn(L, D=96)
    assert L.fm_attn_fwd(ctypes.byref(a), ctypes.byref(m), vec, o, lse, None) == fm.FM_ERR_UNSUPPORTED
    a, m = _attn(L, dtype=1)
    assert L.fm_attn_fwd(ctypes.byref(a), ctypes.byref(m), vec, o, lse, None) == fm.FM_ERR_UNSUPPORTED
    a, m = _attn(L, meta_nq=384)
    assert L.fm_attn_fwd(ctypes.byref(a), ctypes.byref(m), vec, o, lse, None) == fm.FM_ERR_INVALID_ARG
    a, m = _attn(L, Hm=3)
    assert L.fm_attn_fwd(ctypes.byref(a), ctypes.byref(m), vec, o, lse, None) == fm.FM_ERR_INVALID_ARG
    a, m = _attn(L)
    assert L.fm_attn_fwd(ctypes.byref(a), ctypes.byref(m), vec, ctypes.c_void_p(0x50008), lse, None) == \
        fm.FM_ERR_INVALID_ARG  # misaligned output
    vec_bad = fm.VecArray(0x70004, None, None, None)
    assert L.fm_attn_fwd(ctypes.byref(a), ctypes.byref(m), vec_bad, o, lse, None) == fm.FM_ERR_INVALID_ARG
    a, m = _attn(L)
    m.fwd_order = None  # metadata without its dispatch orders
    assert L.fm_attn_fwd(ctypes.byref(a), ctypes.byref(m), vec, o, lse, None) == fm.FM_ERR_INVALID_ARG


def test_bwd_rejects_before_launch(L):
    vec = fm.VecArray(None, None, None, None)
    a, m = _attn(L)
    need = L.fm_attn_bwd_workspace_bytes(ctypes.byref(a))
    assert need >= 1 * 2 * 256 * 128 * 4
    p = [ctypes.c_void_p(0x100000 * (t + 1)) for t in range(6)]
    assert L.fm_attn_bwd(ctypes.byref(a), ctypes.byref(m), vec, *p, ctypes.c_void_p(0x900000), need - 1, None) == \
        fm.FM_ERR_WORKSPACE
    assert L.fm_attn_bwd(ctypes.byref(a), ctypes.byref(m), vec, *p, None, need, None) == fm.FM_ERR_WORKSPACE
    a, m = _attn(L, n_k=130)
    assert L.fm_attn_bwd(ctypes.byref(a), ctypes.byref(m), vec, *p, ctypes.c_void_p(0x900000), need, None) == \
        fm.FM_ERR_UNSUPPORTED


def test_deterministic_flag(L):
    """Fixed-order dQ: the flag is 0 or 1, and its workspace adds the turn table (2 bytes per
    (b, h, key tile, query tile)) and one int32 counter per (b, h, query tile), each 256-aligned."""
    vec = fm.VecArray(None, None, None, None)
    p = [ctypes.c_void_p(0x100000 * (t + 1)) for t in range(6)]
    a, m = _attn(L, n_q=384, n_k=640, H=2)
    base = L.fm_attn_bwd_workspace_bytes(ctypes.byref(a))
    a.deterministic = 1
    det = L.fm_attn_bwd_workspace_bytes(ctypes.byref(a))
    al = lambda x: (x + 255) // 256 * 256
    assert det - base == al(1 * 2 * 5 * 3 * 2) + al(1 * 2 * 3 * 4)
    assert L.fm_attn_bwd(ctypes.byref(a), ctypes.byref(m), vec, *p, ctypes.c_void_p(0x900000), base, None) == \
        fm.FM_ERR_WORKSPACE  # the deterministic call needs the larger workspace
    a.deterministic = 2
    assert L.fm_attn_bwd(ctypes.byref(a), ctypes.byref(m), vec, *p, ctypes.c_void_p(0x900000), det, None) == \
        fm.FM_ERR_INVALID_ARG
    assert L.fm_attn_fwd(ctypes.byref(a), ctypes.byref(m), vec, ctypes.c_void_p(0x50000),
                         ctypes.c_void_p(0x60000), None) == fm.FM_ERR_INVALID_ARG


def test_no_oracle_import_in_library():
    """The product path must not reach the oracle or any CPU fallback."""
    pkg = os.path.join(ROOT, "mask_aware_flash_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                txt = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in txt and "from oracle" not in txt, f
                assert "fm_oracle" not in txt, f


def test_kv_chunk_pairs_rejects_bad_args(L):
    import numpy as np
    vec = fm.VecArray(0x10000, 0x20000, 0x30000, 0x40000)
    nl = np.array([64, 64], np.int32)
    p_nl = nl.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
    out = ctypes.c_void_p(0x50000)
    assert L.fm_kv_chunk_pairs(1, 1, 256, 2, vec, p_nl, 0, out, None) == fm.FM_ERR_INVALID_ARG  # chunk_len
    assert L.fm_kv_chunk_pairs(1, 1, 256, 0, vec, p_nl, 64, out, None) == fm.FM_ERR_INVALID_ARG  # no ranks
    assert L.fm_kv_chunk_pairs(1, 1, 256, 2, vec, p_nl, 64, ctypes.c_void_p(0x50004), None) == \
        fm.FM_ERR_INVALID_ARG  # misaligned int64 output
    assert L.fm_kv_chunk_pairs(1, 1, 256, 2, vec, None, 64, out, None) == fm.FM_ERR_INVALID_ARG
    bad = np.array([64, -1], np.int32)
    assert L.fm_kv_chunk_pairs(1, 1, 256, 2, vec, bad.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), 64, out,
                               None) == fm.FM_ERR_INVALID_ARG
    many = np.full(256, 64, np.int32)
    assert L.fm_kv_chunk_pairs(300, 1, 256, 256, vec, many.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), 64, out,
                               None) == fm.FM_ERR_UNSUPPORTED  # 256 ranks x 300 rows > 65535


def test_varlen_mask_rejects_bad_args(L):
    cu, o = ctypes.c_void_p(0x10000), [ctypes.c_void_p(0x20000 * (t + 1)) for t in range(4)]
    assert L.fm_varlen_mask(None, 2, 100, 1, *o, None) == fm.FM_ERR_INVALID_ARG
    assert L.fm_varlen_mask(cu, 0, 100, 1, *o, None) == fm.FM_ERR_INVALID_ARG        # no sequence
    assert L.fm_varlen_mask(cu, 2, 0, 1, *o, None) == fm.FM_ERR_INVALID_ARG          # empty pack
    assert L.fm_varlen_mask(cu, 2, 100, 2, *o, None) == fm.FM_ERR_INVALID_ARG        # causal flag
    assert L.fm_varlen_mask(cu, 2, 100, 1, o[0], o[1], ctypes.c_void_p(0x60002), o[3], None) == \
        fm.FM_ERR_INVALID_ARG  # misaligned int32 output


def test_varlen_binding_rejects_non_int32():
    torch = pytest.importorskip("torch")
    with pytest.raises(fm.FmError):
        fm.fm_varlen_mask(torch.zeros(3, dtype=torch.int64), 10)
    with pytest.raises(fm.FmError):
        fm.fm_varlen_mask(torch.zeros((2, 2), dtype=torch.int32), 10)


def test_binding_needs_one_vector_for_the_shape():
    with pytest.raises(fm.FmError):
        fm.fm_build_mask_meta(None, None, None, None, n_q=128)
    with pytest.raises(fm.FmError):
        fm.fm_kv_chunk_pairs([None] * 4, [64], 64)
    with pytest.raises(fm.FmError):
        fm.fm_localize([None] * 4, [[0]], [[64]])


@pytest.mark.skipif(torch_cuda_present(), reason="hands made-up device addresses to an entry point that can launch")
def test_noalloc_rejects_oversize(L):
    """fm_attn_bwd_noalloc: a problem beyond its fixed scratch fails on the host, before any CUDA call."""
    L.fm_attn_bwd_noalloc.argtypes = [ctypes.POINTER(fm.AttnArgs), ctypes.POINTER(fm.MaskMetaC), fm.VecArray] + \
        [ctypes.c_void_p] * 7
    L.fm_attn_bwd_noalloc.restype = ctypes.c_int
    D, H = 128, 16
    n = 8192  # B*H*n_q = 131072 rows of fp32 dQ accumulator: 64 MiB > 32 MiB
    a = fm.AttnArgs(1, H, n, n, D, 0, 0.1, 0x10000, 0x20000, 0x30000)
    m = fm.MaskMetaC()
    m.d = fm.MaskDesc(1, 1, n, n, 128, 128)
    m.row_count = m.row_entries = m.col_count = m.col_entries = m.tile_minmax = 0x40000
    m.tile_class = m.fwd_order = m.bwd_order = 0x40000
    p = [ctypes.c_void_p(0x100000 * (t + 1)) for t in range(6)]
    rc = L.fm_attn_bwd_noalloc(ctypes.byref(a), ctypes.byref(m), fm.VecArray(None, None, None, None), *p, None)
    assert rc == fm.FM_ERR_WORKSPACE


@pytest.mark.skipif(torch_cuda_present(), reason="hands made-up device addresses to an entry point that can launch")
def test_head_dim_256_fixed_order_rejected(L):
    """D = 256 runs the backward in two launches over the two halves of d; the fixed-order dQ mode is
    not offered there: FM_ERR_UNSUPPORTED on the host."""
    vec = fm.VecArray(None, None, None, None)
    p = [ctypes.c_void_p(0x100000 * (t + 1)) for t in range(6)]
    a, m = _attn(L, n_q=384, n_k=640, H=2)
    a.D = 256
    a.deterministic = 1
    assert L.fm_attn_bwd_workspace_bytes(ctypes.byref(a)) > 0
    assert L.fm_attn_bwd(ctypes.byref(a), ctypes.byref(m), vec, *p, ctypes.c_void_p(0x900000), 1 << 30, None) == \
        fm.FM_ERR_UNSUPPORTED
