"""fm_attn_bwd_noalloc: the backward for callers that cannot allocate device
memory at call time (engine plug-ins that plan every buffer ahead, loops that
must not pay cudaMalloc's implicit synchronisation).  Its scratch is a fixed
array inside the library.  Checked through the C ABI against fm_attn_bwd on
the same inputs, on two calls in a row (the array keeps the previous call's
contents, so the second call also checks that the entry point clears what it
must).  Kept in its own file, collected last."""
import ctypes
import math

import numpy as np
import pytest

import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

G_TOL = 2e-2  # dQ/dK/dV max-abs error relative to the reference's max-abs


@pytest.fixture(scope="module")
def fm():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from mask_aware_flash_b200 import _build
    _build.build()
    import mask_aware_flash_b200 as m
    L = m.lib()
    L.fm_attn_bwd_noalloc.argtypes = [ctypes.POINTER(m.AttnArgs), ctypes.POINTER(m.MaskMetaC), m.VecArray] + \
        [ctypes.c_void_p] * 7
    L.fm_attn_bwd_noalloc.restype = ctypes.c_int
    return m


def _bf16(bits):
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()


def _rel(got, ref):
    return float((got.float() - ref.float()).abs().max() / ref.float().abs().max().clamp_min(1e-30))


def test_noalloc_matches_workspace_backward_twice(fm):
    B, H, n, D, seed = 1, 4, 1024, 128, 4242
    docs = synth.draw_docs(synth.Rng(seed), n, 100, 400)
    spec = synth.mask_causal_document(n, docs)
    q, k, v, do = (_bf16(synth.normal_bf16_bits(seed, t, (B, n, H, D))) for t in (1, 2, 3, 4))
    vt = [torch.from_numpy(np.ascontiguousarray(x[None, None])).cuda() for x in spec.vectors()]
    scale = 1.0 / math.sqrt(D)
    meta = fm.fm_build_mask_meta(*vt, n_q=n)
    o, lse = fm.fm_attn_fwd(q, k, v, meta, vt, scale)
    ref = fm.fm_attn_bwd(q, k, v, o, lse, do, meta, vt, scale)
    a = fm._args(q, k, v, scale)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        dq, dk, dv = torch.full_like(q, float("nan")), torch.full_like(k, float("nan")), torch.full_like(v, float("nan"))
        rc = fm.lib().fm_attn_bwd_noalloc(ctypes.byref(a), ctypes.byref(meta.c), fm._vecs(vt), o.data_ptr(),
                                          lse.data_ptr(), do.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                                          dv.data_ptr(), stream)
        assert rc == fm.FM_OK, fm.status_string(rc)
        torch.cuda.synchronize()
        for name, got, exp in (("dq", dq, ref[0]), ("dk", dk, ref[1]), ("dv", dv, ref[2])):
            assert torch.isfinite(got.float()).all(), f"call {call}: {name} has non-finite values"
            err = _rel(got, exp)
            assert err <= G_TOL, f"call {call}: {name} differs from fm_attn_bwd by {err}"
    assert fm.fm_get_device_status() == 0


def test_noalloc_rejects_oversize(fm):
    """Beyond the fixed scratch the call fails on the host, before any launch."""
    D, H = 128, 16
    n = 8192  # B*H*n_q = 131072 rows of fp32 dQ accumulator: 64 MiB > 32 MiB
    a = fm.AttnArgs(1, H, n, n, D, 0, 0.1, 0x10000, 0x20000, 0x30000)
    m = fm.MaskMetaC()
    m.d = fm.MaskDesc(1, 1, n, n, 128, 128)
    m.row_count = m.row_entries = m.col_count = m.col_entries = m.tile_minmax = 0x40000
    m.tile_class = m.fwd_order = m.bwd_order = 0x40000
    p = [ctypes.c_void_p(0x100000 * (t + 1)) for t in range(6)]
    rc = fm.lib().fm_attn_bwd_noalloc(ctypes.byref(a), ctypes.byref(m), fm.VecArray(None, None, None, None), *p,
                                      None)
    assert rc == fm.FM_ERR_WORKSPACE
