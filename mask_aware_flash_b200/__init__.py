"""Python binding of the B200 mask-aware attention library (libfm_b200.so).

Argument marshalling only: every step of the hot path runs in the CUDA
kernels behind the C ABI declared in ``include/fm.h``.  PyTorch supplies device
memory (the caller's tensors and the workspaces allocated here) and the
current CUDA stream.  There is no CPU fallback: if the library is missing or
cannot be loaded, ``lib()`` raises.

Entry points (same names as the C ABI):
  fm_build_mask_meta(lts, lte, uts, ute, n_q)      -> MaskMeta
  fm_localize(vecs, chunk_start, chunk_len)         -> 4 tensors [R, B, Hm, N]
  fm_kv_chunk_pairs(loc_vecs, n_loc, chunk_len)     -> int64 [R, B, Hm, n_chunks]
  fm_varlen_mask(cu_seqlens, N, causal)             -> 4 tensors [1, 1, N]
  fm_attn_fwd(q, k, v, meta, vecs, scale)           -> (o, lse)
  fm_attn_bwd(q, k, v, o, lse, do, meta, vecs, scale, deterministic=False) -> (dq, dk, dv)
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# FM_DEBUG=1 in the environment loads the checking build (device-side index checks and shared-memory
# canaries; failures come back as FM_ERR_DEVICE_CHECK from fm_get_device_status)
LIB_PATH = os.path.join(_HERE, "libfm_b200_debug.so" if os.environ.get("FM_DEBUG") == "1" else "libfm_b200.so")
_lib = None

FM_OK, FM_ERR_INVALID_ARG, FM_ERR_UNSUPPORTED, FM_ERR_WORKSPACE, FM_ERR_CUDA, FM_ERR_DEVICE_TIMEOUT, \
    FM_ERR_DEVICE_CHECK = range(7)
TILE = 128
META_LAUNCHES = 2  # kernels one fm_build_mask_meta call launches
BWD_LAUNCHES = 3   # kernels one fm_attn_bwd call launches (one more with deterministic=True)


class FmError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {status_string(code)} (status {code})")


class MaskDesc(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("Hm", ctypes.c_int32), ("n_q", ctypes.c_int32), ("n_k", ctypes.c_int32),
                ("tile_q", ctypes.c_int32), ("tile_k", ctypes.c_int32)]


class MaskMetaC(ctypes.Structure):
    _fields_ = [("d", MaskDesc), ("tile_minmax", ctypes.c_void_p), ("row_count", ctypes.c_void_p),
                ("row_entries", ctypes.c_void_p), ("col_count", ctypes.c_void_p),
                ("col_entries", ctypes.c_void_p), ("tile_class", ctypes.c_void_p),
                ("fwd_order", ctypes.c_void_p), ("bwd_order", ctypes.c_void_p)]


class AttnArgs(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("n_q", ctypes.c_int32), ("n_k", ctypes.c_int32),
                ("D", ctypes.c_int32), ("dtype", ctypes.c_int32), ("scale", ctypes.c_float),
                ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("H_kv", ctypes.c_int32),
                ("deterministic", ctypes.c_int32)]


VecArray = ctypes.c_void_p * 4


def lib():
    """Load the CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with mask_aware_flash_b200._build.build()")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
        L.fm_mask_meta_workspace_bytes.argtypes = [ctypes.POINTER(MaskDesc)]
        L.fm_mask_meta_workspace_bytes.restype = sz
        L.fm_build_mask_meta.argtypes = [ctypes.POINTER(MaskDesc), vp, vp, vp, vp, vp, sz, ctypes.POINTER(MaskMetaC),
                                         vp]
        L.fm_build_mask_meta.restype = ctypes.c_int
        L.fm_localize.argtypes = [i32, i32, i32, VecArray, i32, i32, ctypes.POINTER(ctypes.c_int32),
                                  ctypes.POINTER(ctypes.c_int32), VecArray, vp]
        L.fm_localize.restype = ctypes.c_int
        L.fm_kv_chunk_pairs.argtypes = [i32, i32, i32, i32, VecArray, ctypes.POINTER(ctypes.c_int32), i32, vp, vp]
        L.fm_kv_chunk_pairs.restype = ctypes.c_int
        L.fm_varlen_mask.argtypes = [vp, i32, i32, i32, vp, vp, vp, vp, vp]
        L.fm_varlen_mask.restype = ctypes.c_int
        L.fm_attn_fwd.argtypes = [ctypes.POINTER(AttnArgs), ctypes.POINTER(MaskMetaC), VecArray, vp, vp, vp]
        L.fm_attn_fwd.restype = ctypes.c_int
        L.fm_attn_bwd_workspace_bytes.argtypes = [ctypes.POINTER(AttnArgs)]
        L.fm_attn_bwd_workspace_bytes.restype = sz
        L.fm_attn_bwd.argtypes = [ctypes.POINTER(AttnArgs), ctypes.POINTER(MaskMetaC), VecArray, vp, vp, vp, vp, vp,
                                  vp, vp, sz, vp]
        L.fm_attn_bwd.restype = ctypes.c_int
        L.fm_get_device_status.argtypes = [vp]
        L.fm_get_device_status.restype = ctypes.c_int
        L.fm_selftest_wait_timeout.argtypes = [vp]
        L.fm_selftest_wait_timeout.restype = ctypes.c_int
        L.fm_status_string.argtypes = [ctypes.c_int]
        L.fm_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().fm_status_string(int(code)).decode()


def _check(code: int, what: str):
    if code != FM_OK:
        raise FmError(code, what)


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _vecs(vecs):
    return VecArray(*[None if v is None else v.data_ptr() for v in vecs])


def _check_tensors(what, device, items):
    """The C ABI sees raw pointers only: reject here host tensors, tensors of another device,
    non-contiguous views and wrong element types or shapes.  items: (name, tensor or None,
    dtype or None, shape or None); None entries are skipped (NULL vectors are legal)."""
    for name, t, dtype, shape in items:
        if t is None:
            continue
        if not t.is_cuda or t.device != device:
            raise FmError(FM_ERR_INVALID_ARG, f"{what}: {name} must be a CUDA tensor on {device}")
        if not t.is_contiguous():
            raise FmError(FM_ERR_INVALID_ARG, f"{what}: {name} must be contiguous")
        if dtype is not None and t.dtype != dtype:
            raise FmError(FM_ERR_INVALID_ARG, f"{what}: {name} must be {dtype}, not {t.dtype}")
        if shape is not None and tuple(t.shape) != tuple(shape):
            raise FmError(FM_ERR_INVALID_ARG, f"{what}: {name} must have shape {tuple(shape)}, not {tuple(t.shape)}")


def _check_qkv(what, q, k, v):
    """q [B, n_q, H, D] and k, v [B, n_k, H_kv, D] of one element type (bf16 or fp32)."""
    if q.dim() != 4 or k.dim() != 4 or v.dim() != 4:
        raise FmError(FM_ERR_INVALID_ARG, f"{what}: q, k, v must be 4-D [B, n, heads, D]")
    if q.dtype not in (torch.bfloat16, torch.float32):
        raise FmError(FM_ERR_INVALID_ARG, f"{what}: q must be bfloat16 or float32, not {q.dtype}")
    B, _, _, D = q.shape
    kv_shape = (B, k.shape[1], k.shape[2], D)
    _check_tensors(what, q.device, [("q", q, None, None), ("k", k, q.dtype, kv_shape), ("v", v, q.dtype, kv_shape)])
    return tuple(q.shape), kv_shape


def _first_vector(vecs, what):
    """The first non-None vector (it gives the shape); all None is an invalid call."""
    ref = next((v for v in vecs if v is not None), None)
    if ref is None:
        raise FmError(FM_ERR_INVALID_ARG, f"{what}: at least one vector must be given (it sets the shape)")
    return ref


class MaskMeta:
    """Tile metadata (views into an owned workspace tensor)."""

    def __init__(self, desc: MaskDesc, ws: torch.Tensor, c: MaskMetaC):
        self.desc, self.ws, self.c = desc, ws, c
        B, Hm, n_q, n_k = desc.B, desc.Hm, desc.n_q, desc.n_k
        self.T_q, self.T_k = -(-n_q // TILE), -(-n_k // TILE)
        base = ws.data_ptr()

        def view(ptr, dtype, shape):
            n = 1
            for s in shape:
                n *= s
            off = ptr - base
            itemsize = torch.empty(0, dtype=dtype).element_size()
            return ws[off:off + n * itemsize].view(dtype).view(*shape)

        self.tile_minmax = view(c.tile_minmax, torch.int32, (B, Hm, self.T_k, 8))
        self.row_count = view(c.row_count, torch.int32, (B, Hm, self.T_q))
        self.row_entries = view(c.row_entries, torch.int32, (B, Hm, self.T_q, self.T_k))
        self.col_count = view(c.col_count, torch.int32, (B, Hm, self.T_k))
        self.col_entries = view(c.col_entries, torch.int32, (B, Hm, self.T_k, self.T_q))
        self.tile_class = view(c.tile_class, torch.uint8, (B, Hm, self.T_q, self.T_k))
        self.fwd_order = view(c.fwd_order, torch.int32, (B, Hm, (self.T_q + 1) // 2))
        self.bwd_order = view(c.bwd_order, torch.int32, (B, Hm, self.T_k))


def fm_mask_meta_workspace_bytes(B, Hm, n_q, n_k) -> int:
    d = MaskDesc(B, Hm, n_q, n_k, TILE, TILE)
    return int(lib().fm_mask_meta_workspace_bytes(ctypes.byref(d)))


def fm_build_mask_meta(lts, lte, uts, ute, n_q: int, stream=None, ws=None) -> MaskMeta:
    """Vectors: int32 CUDA tensors [B, Hm, n_k] (or None = canonical empty).  ws: optional uint8 CUDA
    workspace of at least fm_mask_meta_workspace_bytes (allocated here when None)."""
    ref = _first_vector((lts, lte, uts, ute), "fm_build_mask_meta")
    if ref.dim() != 3:
        raise FmError(FM_ERR_INVALID_ARG, "fm_build_mask_meta: vectors must be [B, Hm, n_k]")
    B, Hm, n_k = ref.shape
    _check_tensors("fm_build_mask_meta", ref.device,
                   [(nm, t, torch.int32, ref.shape) for nm, t in zip(("lts", "lte", "uts", "ute"), (lts, lte, uts, ute))])
    d = MaskDesc(B, Hm, n_q, n_k, TILE, TILE)
    nbytes = lib().fm_mask_meta_workspace_bytes(ctypes.byref(d))
    if nbytes == 0:
        raise FmError(FM_ERR_INVALID_ARG, "fm_mask_meta_workspace_bytes")
    if ws is None:
        ws = torch.empty(nbytes, dtype=torch.uint8, device=ref.device)
    _check_tensors("fm_build_mask_meta", ref.device, [("ws", ws, torch.uint8, None)])
    if ws.numel() < nbytes:
        raise FmError(FM_ERR_WORKSPACE, "fm_build_mask_meta: workspace too small")
    c = MaskMetaC()
    _check(lib().fm_build_mask_meta(ctypes.byref(d), _ptr(lts), _ptr(lte), _ptr(uts), _ptr(ute), _ptr(ws), nbytes,
                                    ctypes.byref(c), _stream(stream)), "fm_build_mask_meta")
    return MaskMeta(d, ws, c)


def fm_localize(vecs, chunk_start, chunk_len, out=None, stream=None):
    """vecs: 4 int32 CUDA tensors [B, Hm, N]; chunk_start / chunk_len: [R, C] host ints.
    Returns 4 int32 tensors [R, B, Hm, N] (written into `out` when given)."""
    import numpy as np
    cs = np.ascontiguousarray(np.asarray(chunk_start, dtype=np.int32))
    cl = np.ascontiguousarray(np.asarray(chunk_len, dtype=np.int32))
    R, C = cs.shape
    ref = _first_vector(vecs, "fm_localize")
    if ref.dim() != 3:
        raise FmError(FM_ERR_INVALID_ARG, "fm_localize: vectors must be [B, Hm, N]")
    B, Hm, N = ref.shape
    outs = out if out is not None else [torch.empty((R, B, Hm, N), dtype=torch.int32, device=ref.device)
                                        for _ in range(4)]
    _check_tensors("fm_localize", ref.device,
                   [(f"vecs[{c}]", vecs[c], torch.int32, ref.shape) for c in range(4)] +
                   [(f"out[{c}]", outs[c], torch.int32, (R, B, Hm, N)) for c in range(4)])
    _check(lib().fm_localize(B, Hm, N, _vecs(vecs), R, C, cs.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                             cl.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), _vecs(outs), _stream(stream)),
           "fm_localize")
    return outs


def fm_kv_chunk_pairs(loc_vecs, n_loc, chunk_len: int, out=None, stream=None):
    """loc_vecs: 4 int32 CUDA tensors [R, B, Hm, N] (fm_localize's output; None = canonical empty);
    n_loc: R host ints.  Returns int64 [R, B, Hm, ceil(N / chunk_len)] unmasked-pair counts per KV chunk."""
    import numpy as np
    ref = _first_vector(loc_vecs, "fm_kv_chunk_pairs")
    if ref.dim() != 4:
        raise FmError(FM_ERR_INVALID_ARG, "fm_kv_chunk_pairs: vectors must be [R, B, Hm, N]")
    R, B, Hm, N = ref.shape
    nl = np.ascontiguousarray(np.asarray(n_loc, dtype=np.int32))
    if nl.shape != (R,):
        raise FmError(FM_ERR_INVALID_ARG, "fm_kv_chunk_pairs: n_loc must hold one row count per rank")
    if int(chunk_len) < 1:
        raise FmError(FM_ERR_INVALID_ARG, "fm_kv_chunk_pairs: chunk_len must be >= 1")
    if out is None:
        out = torch.empty((R, B, Hm, -(-N // chunk_len)), dtype=torch.int64, device=ref.device)
    _check_tensors("fm_kv_chunk_pairs", ref.device,
                   [(f"loc_vecs[{c}]", loc_vecs[c], torch.int32, ref.shape) for c in range(4)] +
                   [("out", out, torch.int64, (R, B, Hm, -(-N // chunk_len)))])
    _check(lib().fm_kv_chunk_pairs(B, Hm, N, R, _vecs(loc_vecs), nl.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                                   int(chunk_len), _ptr(out), _stream(stream)), "fm_kv_chunk_pairs")
    return out


def fm_varlen_mask(cu_seqlens, N: int, causal: bool = True, out=None, stream=None):
    """Packed variable-length batch -> the four mask vectors, each int32 [1, 1, N] on the device.
    cu_seqlens: int32 CUDA tensor [n_seq + 1] of sequence boundaries (0 first, non-decreasing)."""
    if cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1 or not cu_seqlens.is_contiguous():
        raise FmError(FM_ERR_INVALID_ARG, "fm_varlen_mask: cu_seqlens must be a contiguous int32 vector")
    if out is None:
        out = [torch.empty((1, 1, N), dtype=torch.int32, device=cu_seqlens.device) for _ in range(4)]
    _check_tensors("fm_varlen_mask", cu_seqlens.device,
                   [("cu_seqlens", cu_seqlens, None, None)] + [(f"out[{c}]", out[c], torch.int32, (1, 1, N))
                                                             for c in range(4)])
    _check(lib().fm_varlen_mask(_ptr(cu_seqlens), cu_seqlens.numel() - 1, int(N), 1 if causal else 0,
                                *[_ptr(x) for x in out], _stream(stream)), "fm_varlen_mask")
    return out


def _args(q, k, v, scale, deterministic=False) -> AttnArgs:
    B, n_q, H, D = q.shape
    dtype = 1 if q.dtype == torch.float32 else 0
    return AttnArgs(B, H, n_q, k.shape[1], D, dtype, float(scale), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                    k.shape[2], 1 if deterministic else 0)


def fm_attn_fwd(q, k, v, meta: MaskMeta, vecs, scale, o=None, lse=None, stream=None):
    """q [B, n_q, H, D], k/v [B, n_k, H_kv, D] CUDA tensors (bf16, or fp32 with D=64; H % H_kv == 0)
    -> o (same dtype), lse [B, H, n_q] fp32."""
    q_shape, _ = _check_qkv("fm_attn_fwd", q, k, v)
    B, n_q, H, D = q_shape
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, n_q), dtype=torch.float32, device=q.device)
    d = meta.desc
    _check_tensors("fm_attn_fwd", q.device, [("o", o, q.dtype, q_shape), ("lse", lse, torch.float32, (B, H, n_q))] +
                   [(f"vecs[{c}]", vecs[c], torch.int32, (d.B, d.Hm, d.n_k)) for c in range(4)])
    a = _args(q, k, v, scale)
    _check(lib().fm_attn_fwd(ctypes.byref(a), ctypes.byref(meta.c), _vecs(vecs), _ptr(o), _ptr(lse),
                             _stream(stream)), "fm_attn_fwd")
    return o, lse


def fm_attn_bwd_workspace_bytes(q, k, v, scale=1.0, deterministic=False) -> int:
    a = _args(q, k, v, scale, deterministic)
    return int(lib().fm_attn_bwd_workspace_bytes(ctypes.byref(a)))


def fm_attn_bwd(q, k, v, o, lse, do, meta: MaskMeta, vecs, scale, dq=None, dk=None, dv=None, ws=None,
                stream=None, deterministic=False):
    """Gradients (dtype of q) of the masked attention; ws: optional uint8 CUDA workspace.
    deterministic: add the key tiles' dQ contributions in a fixed order (bitwise repeatable dQ)."""
    q_shape, kv_shape = _check_qkv("fm_attn_bwd", q, k, v)
    B, n_q, H, D = q_shape
    a = _args(q, k, v, scale, deterministic)
    nbytes = lib().fm_attn_bwd_workspace_bytes(ctypes.byref(a))
    if ws is None:
        ws = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    dq = torch.empty_like(q) if dq is None else dq  # dk, dv: the shape of k, v ([B, n_k, H_kv, D])
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    d = meta.desc
    _check_tensors("fm_attn_bwd", q.device,
                   [("o", o, q.dtype, q_shape), ("lse", lse, torch.float32, (B, H, n_q)), ("do", do, q.dtype, q_shape),
                    ("dq", dq, q.dtype, q_shape), ("dk", dk, q.dtype, kv_shape), ("dv", dv, q.dtype, kv_shape),
                    ("ws", ws, None, None)] +
                   [(f"vecs[{c}]", vecs[c], torch.int32, (d.B, d.Hm, d.n_k)) for c in range(4)])
    _check(lib().fm_attn_bwd(ctypes.byref(a), ctypes.byref(meta.c), _vecs(vecs), _ptr(o), _ptr(lse), _ptr(do),
                             _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "fm_attn_bwd")
    return dq, dk, dv


def fm_selftest_wait_timeout(stream=None):
    """Enqueue the bounded-wait self-test (a wait that runs out after ~2 s and records
    FM_ERR_DEVICE_TIMEOUT for the next fm_get_device_status)."""
    _check(lib().fm_selftest_wait_timeout(_stream(stream)), "fm_selftest_wait_timeout")


def fm_get_device_status(stream=None) -> int:
    return int(lib().fm_get_device_status(_stream(stream)))
