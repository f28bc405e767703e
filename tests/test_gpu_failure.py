"""Failure detection on the GPU without a fault: a kernel wait that nothing
completes runs out (bounded, ~2 s), the kernel records FM_ERR_DEVICE_TIMEOUT in
the per-device status word and returns; the host reads (and clears) the status,
and the same context then computes attention correctly."""
import math
import time

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
    from mask_aware_flash_b200 import _build
    _build.build()
    import mask_aware_flash_b200 as m
    m.lib()
    return m


def test_bounded_wait_reports_timeout_and_context_survives(fm):
    assert fm.fm_get_device_status() == fm.FM_OK
    t0 = time.monotonic()
    fm.fm_selftest_wait_timeout()
    status = fm.fm_get_device_status()  # synchronises the stream, then reads and clears the word
    waited = time.monotonic() - t0
    assert status == fm.FM_ERR_DEVICE_TIMEOUT
    assert 1.5 < waited < 60.0, waited
    assert fm.fm_get_device_status() == fm.FM_OK  # cleared by the read

    # the context is still healthy: a small causal-document forward matches the oracle
    n, H, D = 256, 2, 64
    spec = synth.mask_causal_document(n, synth.cut_segments(synth.Rng(1000), n, 3))
    bits = [synth.normal_bf16_bits(7, t, (1, n, H, D)) for t in (1, 2, 3)]
    host = [synth.bf16_bits_to_f32(x) for x in bits]
    dev = [torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda() for x in bits]
    vt = [torch.from_numpy(np.ascontiguousarray(x[None, None])).cuda() for x in spec.vectors()]
    scale = 1.0 / math.sqrt(D)
    meta = fm.fm_build_mask_meta(*vt, n_q=n)
    o, lse = fm.fm_attn_fwd(dev[0], dev[1], dev[2], meta, vt, scale)
    torch.cuda.synchronize()
    assert fm.fm_get_device_status() == fm.FM_OK
    vecs = [x[None, None] for x in spec.vectors()]
    for h in range(H):
        ref = oracle.attention_head(*host, vecs, 0, h, scale)
        assert np.abs(o.float().cpu().numpy()[0, :, h] - ref["o"]).max() <= 1e-2
        live = np.isfinite(ref["lse"])
        assert np.abs(lse.cpu().numpy()[0, h][live] - ref["lse"][live]).max() <= 1e-3
