"""Device-side checks of the FM_DEBUG build fire on bad metadata and leave the context usable.
Runs only against libfm_b200_debug.so (FM_DEBUG=1; test_gpu_debug_build runs this file in such a
subprocess): in the release build nothing would stop the bad entry, so there the test is skipped.

The last entry of one query tile's row list is rewritten to name a key tile past the end.  The
forward's load warp checks every entry before it issues a copy for it: the check records
FM_ERR_DEVICE_CHECK, raises the CTA's abort flag so every role stops waiting, and the copy is
never issued.  The same call with intact metadata then matches the oracle."""
import math

import numpy as np
import pytest

import oracle
import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fm():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import mask_aware_flash_b200 as m
    if not m.LIB_PATH.endswith("libfm_b200_debug.so"):
        pytest.skip("needs the FM_DEBUG build (FM_DEBUG=1)")
    m.lib()
    return m


def test_bad_list_entry_is_caught(fm):
    n, H, D, seed = 512, 2, 64, 81
    spec = synth.make_family("causal", n, seed)
    vt = [torch.from_numpy(np.ascontiguousarray(x[None, None])).cuda() for x in spec.vectors()]
    bits = [synth.normal_bf16_bits(seed, t, (1, n, H, D)) for t in (1, 2, 3)]
    q, k, v = (torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).cuda() for b in bits)
    scale = 1.0 / math.sqrt(D)
    assert fm.fm_get_device_status() == fm.FM_OK
    meta = fm.fm_build_mask_meta(*vt, n_q=n)
    qt = 2
    cnt = int(meta.row_count[0, 0, qt].item())
    meta.row_entries[0, 0, qt, cnt - 1] = ((meta.T_k + 3) << 1) | 1  # a key tile past the end
    fm.fm_attn_fwd(q, k, v, meta, vt, scale)
    torch.cuda.synchronize()
    assert fm.fm_get_device_status() == fm.FM_ERR_DEVICE_CHECK
    # the context still computes: fresh metadata, the oracle's rows
    meta = fm.fm_build_mask_meta(*vt, n_q=n)
    o, lse = fm.fm_attn_fwd(q, k, v, meta, vt, scale)
    torch.cuda.synchronize()
    assert fm.fm_get_device_status() == fm.FM_OK
    host = [synth.bf16_bits_to_f32(b) for b in bits]
    vecs = [x[None, None] for x in spec.vectors()]
    ref = oracle.attention_head(*host, vecs, 0, 1, scale)
    assert np.abs(o[0, :, 1].float().cpu().numpy() - ref["o"]).max() <= 1e-2
