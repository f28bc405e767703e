"""Pins for the oracle's fp64 masked attention (CPU only).

The oracle is checked against: PyTorch's CPU fp64 scaled_dot_product_attention
+ autograd with a dense boolean mask (a library special case), central finite
differences, closed forms (constant scores), and invariants that hold for any
masked softmax attention.  Mistakes such as a dropped term in dS, a wrong sign,
a transposed operand or a wrong LSE base fail at least one of these.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth


def _inputs(B, n_q, n_k, H, D, seed):
    q = synth.normal_f32(seed, 1, (B, n_q, H, D))
    k = synth.normal_f32(seed, 2, (B, n_k, H, D))
    v = synth.normal_f32(seed, 3, (B, n_k, H, D))
    do = synth.normal_f32(seed, 4, (B, n_q, H, D))
    return q, k, v, do


def _full(q, k, v, do, vecs, b, h, scale, Hm=1):
    return oracle.attention_head(q, k, v, vecs, b, h, scale, rows=None,
                                 cols=np.arange(k.shape[1]), dout=do, Hm=Hm)


def _torch_ref(q, k, v, do, allowed, b, h, scale):
    """SDPA in fp64 + autograd; rows with no allowed key are dropped from the loss
    (SDPA returns NaN there)."""
    Q = torch.tensor(q[b, :, h, :], dtype=torch.float64, requires_grad=True)
    K = torch.tensor(k[b, :, h, :], dtype=torch.float64, requires_grad=True)
    V = torch.tensor(v[b, :, h, :], dtype=torch.float64, requires_grad=True)
    dO = torch.tensor(do[b, :, h, :], dtype=torch.float64)
    live = allowed.any(axis=1)
    am = torch.tensor(allowed)
    am[~torch.tensor(live)] = True  # keep SDPA finite on dead rows; they are excluded below
    O = torch.nn.functional.scaled_dot_product_attention(Q[None, None], K[None, None], V[None, None],
                                                         attn_mask=am[None, None], scale=scale)[0, 0]
    lv = torch.tensor(live)
    loss = (O[lv] * dO[lv]).sum()
    loss.backward()
    return O.detach().numpy(), Q.grad.numpy(), K.grad.numpy(), V.grad.numpy(), live


@pytest.mark.parametrize("family", ["full", "causal", "causal_document", "share_question", "global_sliding",
                                    "random_eviction", "prefix_lm_document"])
def test_vs_torch_sdpa(family):
    n, H, D = 96, 2, 16
    spec = synth.make_family(family, n, 21)
    q, k, v, do = _inputs(1, n, n, H, D, 5)
    vecs = [x[None, None, :] for x in spec.vectors()]
    allowed = ~oracle.dense_mask(n, n, *spec.vectors())
    scale = 1.0 / math.sqrt(D)
    for h in range(H):
        r = _full(q, k, v, do, vecs, 0, h, scale)
        O, dQ, dK, dV, live = _torch_ref(q, k, v, do, allowed, 0, h, scale)
        np.testing.assert_allclose(r["o"][live], O[live], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(r["dq"], dQ, rtol=1e-9, atol=1e-11)
        np.testing.assert_allclose(r["dk"], dK, rtol=1e-9, atol=1e-11)
        np.testing.assert_allclose(r["dv"], dV, rtol=1e-9, atol=1e-11)


def test_vs_torch_sdpa_random_vectors_with_dead_rows():
    n_q, n_k, H, D = 40, 56, 1, 8
    r = np.random.default_rng(7)
    vecs = [r.integers(-4, n_q + 4, n_k).astype(np.int32) for _ in range(4)]
    vecs[0][:] = np.minimum(vecs[0], 10)   # lower interval starts early ...
    vecs[1][:] = np.maximum(vecs[1], 14)   # ... and covers rows 10..13 for every key
    q, k, v, do = _inputs(1, n_q, n_k, H, D, 9)
    allowed = ~oracle.dense_mask(n_q, n_k, *vecs)
    assert (~allowed.any(axis=1)).sum() >= 4
    scale = 0.3
    res = _full(q, k, v, do, [x[None, None] for x in vecs], 0, 0, scale)
    O, dQ, dK, dV, live = _torch_ref(q, k, v, do, allowed, 0, 0, scale)
    np.testing.assert_allclose(res["o"][live], O[live], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(res["dq"], dQ, rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(res["dk"], dK, rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(res["dv"], dV, rtol=1e-9, atol=1e-11)
    # fully masked rows: O = 0, LSE = -inf, dQ = 0
    dead = ~live
    assert np.all(res["o"][dead] == 0.0)
    assert np.all(np.isneginf(res["lse"][dead]))
    assert np.all(res["dq"][dead] == 0.0)


def test_lse_closed_form_constant_scores():
    """All keys equal -> every unmasked score of row i is the same s_i, so
    LSE_i = s_i + ln|U_i| and O_i is the mean of v_j over U_i."""
    n, D = 64, 8
    spec = synth.make_family("causal_document", n, 4)
    q, k, v, do = _inputs(1, n, n, 1, D, 3)
    k[:] = k[:, :1]  # every key row = key row 0
    scale = 0.7
    res = oracle.attention_head(q, k, v, [x[None, None] for x in spec.vectors()], 0, 0, scale)
    allowed = ~oracle.dense_mask(n, n, *spec.vectors())
    for i in range(n):
        U = np.nonzero(allowed[i])[0]
        s = scale * float(np.dot(q[0, i, 0].astype(np.float64), k[0, 0, 0].astype(np.float64)))
        assert res["lse"][i] == pytest.approx(s + math.log(len(U)), rel=1e-12, abs=1e-12)
        np.testing.assert_allclose(res["o"][i], v[0, U, 0].astype(np.float64).mean(axis=0), rtol=1e-11,
                                   atol=1e-13)


def test_finite_differences():
    n, D = 12, 4
    spec = synth.make_family("prefix_lm", n, 2)
    q, k, v, do = _inputs(1, n, n, 1, D, 13)
    q, k, v, do = (x.astype(np.float64) for x in (q, k, v, do))
    vecs = [x[None, None] for x in spec.vectors()]
    scale = 0.5

    def loss(qq, kk, vv):
        o = oracle.attention_head(qq.astype(np.float32), kk.astype(np.float32), vv.astype(np.float32), vecs,
                                  0, 0, scale)["o"]
        return float((o * do[0, :, 0]).sum())

    # work on fp32-exact perturbations: choose h so x +- h is exact in fp32
    h = 2.0 ** -12
    res = _full(q.astype(np.float32), k.astype(np.float32), v.astype(np.float32), do.astype(np.float32), vecs,
                0, 0, scale)
    for name, arr, grad in (("q", q, res["dq"]), ("k", k, res["dk"]), ("v", v, res["dv"])):
        for (i, d) in [(0, 0), (3, 1), (7, 2), (11, 3), (5, 0)]:
            plus, minus = arr.copy(), arr.copy()
            plus[0, i, 0, d] += h
            minus[0, i, 0, d] -= h
            args_p = {"q": q, "k": k, "v": v}
            args_m = dict(args_p)
            args_p[name], args_m[name] = plus, minus
            fd = (loss(args_p["q"], args_p["k"], args_p["v"]) - loss(args_m["q"], args_m["k"], args_m["v"])) / (2 * h)
            assert fd == pytest.approx(grad[i, d], rel=2e-5, abs=2e-7), (name, i, d)


def test_invariants_gradient_sums_and_shift():
    n, H, D = 80, 1, 16
    spec = synth.make_family("share_question", n, 8)
    q, k, v, do = _inputs(1, n, n, H, D, 17)
    vecs = [x[None, None] for x in spec.vectors()]
    scale = 0.25
    r = _full(q, k, v, do, vecs, 0, 0, scale)
    live = np.isfinite(r["lse"])
    # sum_j dS_ij = 0  =>  sum_j dK_j = 0 ;  sum_j dV_j = sum over live rows of dO_i
    np.testing.assert_allclose(r["dk"].sum(axis=0), 0.0, atol=1e-11)
    np.testing.assert_allclose(r["dv"].sum(axis=0), do[0, live, 0].astype(np.float64).sum(axis=0), atol=1e-10)
    # softmax shift invariance: k_j += c for all j leaves O unchanged
    c = synth.normal_f32(99, 5, (D,))
    k2 = (k + c[None, None, None, :] * 0.5).astype(np.float32)
    r2 = oracle.attention_head(q, k2, v, vecs, 0, 0, scale)
    np.testing.assert_allclose(r2["o"], r["o"], atol=1e-6)  # k2 rounded to fp32 -> tiny differences


def test_sampled_rows_and_cols_equal_full():
    n, H, D = 70, 2, 8
    spec = synth.make_family("causal_document", n, 1)
    q, k, v, do = _inputs(2, n, n, H, D, 23)
    vecs = [np.stack([x, x])[:, None, :] for x in spec.vectors()]  # B=2, Hm=1
    scale = 0.4
    full = _full(q, k, v, do, vecs, 1, 1, scale)
    rows = np.array([0, 5, 33, 69])
    cols = np.array([1, 2, 60])
    s = oracle.attention_head(q, k, v, vecs, 1, 1, scale, rows=rows, cols=cols, dout=do)
    np.testing.assert_array_equal(s["o"], full["o"][rows])
    np.testing.assert_array_equal(s["dq"], full["dq"][rows])
    np.testing.assert_array_equal(s["dk"], full["dk"][cols])
    np.testing.assert_array_equal(s["dv"], full["dv"][cols])


def test_per_head_vectors():
    """Hm = H: head h reads its own vector row."""
    n, H, D = 32, 2, 8
    q, k, v, do = _inputs(1, n, n, H, D, 31)
    m0, m1 = synth.mask_causal(n), synth.mask_full(n)
    vecs = [np.stack([a, b])[None] for a, b in zip(m0.vectors(), m1.vectors())]  # [1, 2, n]
    r0 = oracle.attention_head(q, k, v, vecs, 0, 0, 0.3, Hm=2)
    r1 = oracle.attention_head(q, k, v, vecs, 0, 1, 0.3, Hm=2)
    c0 = oracle.attention_head(q, k, v, [x[None, None] for x in m0.vectors()], 0, 0, 0.3)
    c1 = oracle.attention_head(q, k, v, [None] * 4, 0, 1, 0.3)
    np.testing.assert_array_equal(r0["o"], c0["o"])
    np.testing.assert_array_equal(r1["o"], c1["o"])


@pytest.mark.parametrize("family", ["causal_document", "global_sliding"])
def test_grouped_query_reading_vs_torch_sdpa(family):
    """Grouped-query attention as the GPU tests check it: the oracle run on K / V repeated to H
    heads (query head h reads K/V head h // (H / H_kv)), dK / dV of a K/V head summed over its query
    heads, equals PyTorch's fp64 SDPA with enable_gqa=True + autograd."""
    n, H, H_kv, D = 64, 6, 2, 16
    g = H // H_kv
    spec = synth.make_family(family, n, 31)
    q, _, _, do = _inputs(1, n, n, H, D, 8)
    _, k, v, _ = _inputs(1, n, n, H_kv, D, 9)
    vecs = [x[None, None, :] for x in spec.vectors()]
    allowed = ~oracle.dense_mask(n, n, *spec.vectors())
    assert allowed.any(axis=1).all()  # no dead rows, so SDPA stays finite everywhere
    scale = 1.0 / math.sqrt(D)
    k_rep, v_rep = np.repeat(k, g, axis=2), np.repeat(v, g, axis=2)
    dk = np.zeros((n, H_kv, D))
    dv = np.zeros((n, H_kv, D))
    rows = []
    for h in range(H):
        r = _full(q, k_rep, v_rep, do, vecs, 0, h, scale)
        rows.append(r)
        dk[:, h // g] += r["dk"]
        dv[:, h // g] += r["dv"]
    Q = torch.tensor(q[0].transpose(1, 0, 2), dtype=torch.float64, requires_grad=True)  # [H, n, D]
    K = torch.tensor(k[0].transpose(1, 0, 2), dtype=torch.float64, requires_grad=True)  # [H_kv, n, D]
    V = torch.tensor(v[0].transpose(1, 0, 2), dtype=torch.float64, requires_grad=True)
    O = torch.nn.functional.scaled_dot_product_attention(Q[None], K[None], V[None],
                                                         attn_mask=torch.tensor(allowed)[None, None], scale=scale,
                                                         enable_gqa=True)[0]
    (O * torch.tensor(do[0].transpose(1, 0, 2), dtype=torch.float64)).sum().backward()
    for h in range(H):
        np.testing.assert_allclose(rows[h]["o"], O[h].detach().numpy(), rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(rows[h]["dq"], Q.grad[h].numpy(), rtol=1e-9, atol=1e-11)
    for hk in range(H_kv):
        np.testing.assert_allclose(dk[:, hk], K.grad[hk].numpy(), rtol=1e-9, atol=1e-11)
        np.testing.assert_allclose(dv[:, hk], V.grad[hk].numpy(), rtol=1e-9, atol=1e-11)


@pytest.mark.parametrize("causal", [True, False])
def test_varlen_packing_vs_torch_sdpa_per_sequence(causal):
    """A packed batch under the varlen vectors: every sequence's rows of O / dQ and keys of dK / dV
    equal PyTorch's fp64 SDPA (+ autograd) on that sequence alone (causal or unmasked); padding
    rows are dead (LSE = -inf) and padding keys get zero gradients."""
    cu = [0, 13, 40, 40, 57]
    N, H, D = 64, 1, 8
    q, k, v, do = _inputs(1, N, N, H, D, 12)
    vecs = [x[None, None, :] for x in oracle.varlen_vectors(cu, N, causal)]
    r = _full(q, k, v, do, vecs, 0, 0, 0.3)
    for s in range(len(cu) - 1):
        a, b = cu[s], cu[s + 1]
        if a == b:
            continue
        Q, K, V = (torch.tensor(x[0, a:b, 0], dtype=torch.float64, requires_grad=True) for x in (q, k, v))
        O = torch.nn.functional.scaled_dot_product_attention(Q[None], K[None], V[None], is_causal=causal,
                                                             scale=0.3)[0]
        (O * torch.tensor(do[0, a:b, 0], dtype=torch.float64)).sum().backward()
        np.testing.assert_allclose(r["o"][a:b], O.detach().numpy(), rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(r["dq"][a:b], Q.grad.numpy(), rtol=1e-9, atol=1e-11)
        np.testing.assert_allclose(r["dk"][a:b], K.grad.numpy(), rtol=1e-9, atol=1e-11)
        np.testing.assert_allclose(r["dv"][a:b], V.grad.numpy(), rtol=1e-9, atol=1e-11)
    assert np.all(np.isneginf(r["lse"][cu[-1]:]))
    assert np.all(r["dk"][cu[-1]:] == 0) and np.all(r["dv"][cu[-1]:] == 0)
