"""CPU check of the autograd wrapper's plumbing: with the library's forward and
backward replaced by dense fp64 stand-ins (the oracle's mask and plain torch
attention), the wrapper must return the forward's O and route the backward's
dq, dk, dv to q, k, v for the upstream gradient it receives, with no gradient
for the mask vectors."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
import oracle  # noqa: E402
import synth  # noqa: E402
from mask_aware_flash_b200 import autograd as fa  # noqa: E402


def _dense(q, k, v, vecs, scale):
    """O of masked attention, [B, n_q, H, D], in plain torch (differentiable); vectors [B, 1, n_k]."""
    B, n_q, H, D = q.shape
    n_k = k.shape[1]
    out = []
    for b in range(B):
        vv = [None if x is None else x[b, 0].numpy() for x in vecs]
        masked = torch.from_numpy(oracle.dense_mask(n_q, n_k, *vv))
        s = torch.einsum("ihd,jhd->hij", q[b], k[b]) * scale
        s = s.masked_fill(masked[None], float("-inf"))
        p = torch.softmax(s, dim=-1)
        out.append(torch.einsum("hij,jhd->ihd", p, v[b]))
    return torch.stack(out)


@pytest.fixture
def standins(monkeypatch):
    calls = []

    def meta(*vecs, n_q):
        calls.append("meta")
        return ("meta", n_q)

    def fwd(q, k, v, meta, vecs, scale):
        calls.append("fwd")
        o = _dense(q, k, v, vecs, scale)
        return o.detach(), torch.zeros(q.shape[0], q.shape[2], q.shape[1], dtype=torch.float64)

    def bwd(q, k, v, o, lse, do, meta, vecs, scale, deterministic=False):
        calls.append(("bwd", deterministic))
        with torch.enable_grad():
            qq, kk, vv = (x.detach().requires_grad_() for x in (q, k, v))
            ref = _dense(qq, kk, vv, vecs, scale)
            return torch.autograd.grad(ref, (qq, kk, vv), do)

    monkeypatch.setattr(fa, "fm_build_mask_meta", meta)
    monkeypatch.setattr(fa, "fm_attn_fwd", fwd)
    monkeypatch.setattr(fa, "fm_attn_bwd", bwd)
    return calls


def test_wrapper_routes_gradients(standins):
    B, n, H, D = 2, 40, 2, 8
    spec = synth.mask_causal_document(n, synth.cut_segments(synth.Rng(3), n, 3))
    vecs = [torch.from_numpy(np.broadcast_to(x, (B, 1, n)).copy()) for x in spec.vectors()]
    g = torch.Generator().manual_seed(0)
    q, k, v = (torch.randn(B, n, H, D, dtype=torch.float64, generator=g, requires_grad=True) for _ in range(3))
    w = torch.randn(B, n, H, D, dtype=torch.float64, generator=g)
    o = fa.flashmask_attention(q, k, v, *vecs, deterministic=True)
    (o * w).sum().backward()
    qr, kr, vr = (x.detach().clone().requires_grad_() for x in (q, k, v))
    ref = _dense(qr, kr, vr, vecs, 1.0 / np.sqrt(D))
    (ref * w).sum().backward()
    assert torch.allclose(o, ref)
    for got, exp in ((q.grad, qr.grad), (k.grad, kr.grad), (v.grad, vr.grad)):
        assert torch.allclose(got, exp)
    assert standins == ["meta", "fwd", ("bwd", True)]
    assert all(x.grad is None for x in vecs)


def test_wrapper_null_vectors_and_default_scale(standins):
    B, n, H, D = 1, 24, 1, 16
    ute = torch.arange(n, dtype=torch.int32).reshape(1, 1, n)  # causal through the upper stretch only
    q, k, v = (torch.randn(B, n, H, D, dtype=torch.float64, requires_grad=True) for _ in range(3))
    o = fa.flashmask_attention(q, k, v, None, None, None, ute)
    o.sum().backward()
    ref = _dense(q.detach(), k.detach(), v.detach(), [None, None, None, ute], 0.25)
    assert torch.allclose(o, ref)
    assert standins == ["meta", "fwd", ("bwd", False)]
