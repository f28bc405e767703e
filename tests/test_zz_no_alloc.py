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


@pytest.mark.parametrize("deterministic", [False, True])
def test_noalloc_matches_workspace_backward_twice(fm, deterministic):
    """Two calls in a row against fm_attn_bwd.  With the fixed-order dQ the array also holds the turn
    table and the per-query-tile counters that the first call leaves non-zero; the second call must
    clear them, and then both calls give exactly fm_attn_bwd's dQ, dK and dV."""
    B, H, n, D, seed = 1, 4, 1024, 128, 4242
    docs = synth.draw_docs(synth.Rng(seed), n, 100, 400)
    spec = synth.mask_causal_document(n, docs)
    q, k, v, do = (_bf16(synth.normal_bf16_bits(seed, t, (B, n, H, D))) for t in (1, 2, 3, 4))
    vt = [torch.from_numpy(np.ascontiguousarray(x[None, None])).cuda() for x in spec.vectors()]
    scale = 1.0 / math.sqrt(D)
    meta = fm.fm_build_mask_meta(*vt, n_q=n)
    o, lse = fm.fm_attn_fwd(q, k, v, meta, vt, scale)
    ref = fm.fm_attn_bwd(q, k, v, o, lse, do, meta, vt, scale, deterministic=deterministic)
    a = fm._args(q, k, v, scale, deterministic)
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
            if deterministic:
                assert torch.equal(got, exp), f"call {call}: fixed-order {name} is not bitwise fm_attn_bwd's"
    assert fm.fm_get_device_status() == 0
