"""Context parallelism (mask_aware_flash_b200.cp): the exchange logic on CPU with gloo ranks, the
attention replaced by the oracle through the module's operations interface; and the kernel path on
one GPU through NCCL.

Each CPU rank holds the rows of its chunks (dual-chunk plan), localizes the global vectors, gathers
only the K/V chunks its rows attend to, and runs the oracle over them; the backward returns dK / dV
contributions to the chunk owners.  Every rank's O, LSE and dQ rows and every owner's dK / dV must
equal the global oracle (fp64 on both sides, so only summation order differs), and the masks used
leave some (rank, chunk) pairs out of the exchange."""
import os
import pickle
import socket
import sys

import numpy as np
import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import oracle  # noqa: E402
import synth  # noqa: E402
from mask_aware_flash_b200 import cp  # noqa: E402


class OracleOps:
    """The cp module's operations on CPU tensors, computed by the oracle (fp64 outputs)."""

    def localize(self, vecs, starts, lens):
        out = []
        for v in vecs:
            a = v.numpy()
            out.append(torch.from_numpy(np.stack([[oracle.localize(a[b, hm], starts, lens) for hm in range(a.shape[1])]
                                                  for b in range(a.shape[0])])))
        return out

    def chunk_pairs(self, loc, n_loc, chunk_len):
        B, Hm, N = loc[0].shape
        return torch.from_numpy(np.stack([[oracle.kv_chunk_pairs(n_loc, N, chunk_len, *[x[b, hm].numpy() for x in loc])
                                           for hm in range(Hm)] for b in range(B)]))

    def _run(self, q, k, v, vecs, scale, do=None):
        B, n_q, H, D = q.shape
        n_k, H_kv = k.shape[1], k.shape[2]
        g = H // H_kv  # query heads per K/V head
        k, v = k.repeat_interleave(g, dim=2), v.repeat_interleave(g, dim=2)
        Hm = vecs[0].shape[1]
        vv = [x.numpy() for x in vecs]
        o = np.zeros((B, n_q, H, D))
        lse = np.zeros((B, H, n_q))
        dq, dk, dv = np.zeros((B, n_q, H, D)), np.zeros((B, n_k, H, D)), np.zeros((B, n_k, H, D))
        for b in range(B):
            for h in range(H):
                r = oracle.attention_head(q.float().numpy(), k.float().numpy(), v.float().numpy(), vv, b, h, scale,
                                          cols=None if do is None else np.arange(n_k),
                                          dout=None if do is None else do.float().numpy(), Hm=Hm)
                o[b, :, h], lse[b, h] = r["o"], r["lse"]
                if do is not None:
                    dq[b, :, h], dk[b, :, h], dv[b, :, h] = r["dq"], r["dk"], r["dv"]
        if g > 1:  # the gradient of a shared K/V head is the sum over its query heads
            dk, dv = dk.reshape(B, n_k, H_kv, g, D).sum(3), dv.reshape(B, n_k, H_kv, g, D).sum(3)
        return o, lse, dq, dk, dv

    def attn_fwd(self, q, k, v, vecs, scale):
        o, lse, *_ = self._run(q, k, v, vecs, scale)
        return torch.from_numpy(o), torch.from_numpy(lse), None

    def attn_bwd(self, q, k, v, o, lse, do, vecs, scale, state):
        _, _, dq, dk, dv = self._run(q, k, v, vecs, scale, do)
        return torch.from_numpy(dq), torch.from_numpy(dk), torch.from_numpy(dv)


def _problem(N, B, H, D, mask, seed):
    if mask == "middle_rows_dead":  # rows [N/4, 3N/4) masked for every key: rank 1 of a 2-rank dual plan
        lts, lte = np.full(N, N // 4, np.int32), np.full(N, 3 * N // 4, np.int32)
        uts, ute = np.zeros(N, np.int32), np.arange(N, dtype=np.int32)  # causal elsewhere
        raw = [lts, lte, uts, ute]
    else:
        raw = synth.make_family(mask, N, seed).vectors()
    vecs = [np.broadcast_to(x, (B, 1, N)).copy() for x in raw]
    q, k, v, do = (synth.bf16_bits_to_f32(synth.normal_bf16_bits(seed, t, (B, N, H, D))) for t in (1, 2, 3, 4))
    return vecs, q, k, v, do


def _problem_multi(N, seed):
    """B = 2, H = 4 query heads over H_kv = 2 K/V heads, per-head masks (Hm = H): a different
    family per (b, h), so the need matrix is the union over every (b, mask head)."""
    B, H, H_kv, D = 2, 4, 2, 16
    fams = ["causal_document", "sliding_window_2k", "share_question", "prefix_lm_document"]
    vecs = [np.empty((B, H, N), np.int32) for _ in range(4)]
    for b in range(B):
        for h in range(H):
            for c, x in enumerate(synth.make_family(fams[(b + h) % 4], N, seed + 10 * b + h).vectors()):
                vecs[c][b, h] = x
    q, do = (synth.bf16_bits_to_f32(synth.normal_bf16_bits(seed, t, (B, N, H, D))) for t in (1, 4))
    k, v = (synth.bf16_bits_to_f32(synth.normal_bf16_bits(seed, t, (B, N, H_kv, D))) for t in (2, 3))
    return vecs, q, k, v, do


def _rank_multi(rank, world, port, out_dir, N, seed):
    import datetime
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        vecs, q, k, v, do = _problem_multi(N, seed)
        plan = cp.ChunkPlan.dual(N, world)
        rows = plan.rows(rank).numpy()
        t = lambda a: torch.from_numpy(np.ascontiguousarray(a[:, rows])).double()  # noqa: E731
        o, lse, ctx = cp.cp_attention_forward(t(q), t(k), t(v), [torch.from_numpy(x) for x in vecs], plan, 0.25,
                                              ops=OracleOps())
        dq, dk, dv = cp.cp_attention_backward(t(do), ctx)
        with open(os.path.join(out_dir, f"m{rank}.pkl"), "wb") as f:
            pickle.dump({"rows": rows, "o": o.numpy(), "lse": lse.numpy(), "dq": dq.numpy(), "dk": dk.numpy(),
                         "dv": dv.numpy(), "need": ctx.need.numpy()}, f)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_cp_batched_per_head_masks_grouped_query(tmp_path):
    N, seed, world = 512, 57, 2
    mp.start_processes(_rank_multi, args=(world, _free_port(), str(tmp_path), N, seed), nprocs=world,
                       start_method="spawn", join=True)
    vecs, q, k, v, do = _problem_multi(N, seed)
    ref = OracleOps()._run(*(torch.from_numpy(x) for x in (q, k, v)), [torch.from_numpy(x) for x in vecs], 0.25,
                           torch.from_numpy(do))
    o_ref, lse_ref, dq_ref, dk_ref, dv_ref = ref
    tol = 1e-12 * max(np.abs(dq_ref).max(), np.abs(dk_ref).max(), np.abs(dv_ref).max())
    plan = cp.ChunkPlan.dual(N, world)
    for r in range(world):
        res = pickle.load(open(tmp_path / f"m{r}.pkl", "rb"))
        rows = res["rows"]
        np.testing.assert_allclose(res["o"], o_ref[:, rows], rtol=0, atol=1e-12)
        np.testing.assert_allclose(res["lse"], lse_ref[:, :, rows], rtol=0, atol=1e-12)
        np.testing.assert_allclose(res["dq"], dq_ref[:, rows], rtol=0, atol=tol)
        np.testing.assert_allclose(res["dk"], dk_ref[:, rows], rtol=0, atol=tol)
        np.testing.assert_allclose(res["dv"], dv_ref[:, rows], rtol=0, atol=tol)
        # need: any (b, mask head) of this rank's rows with unmasked pairs in the chunk
        any_pairs = np.zeros(plan.n_chunks, bool)
        for b in range(2):
            for hm in range(4):
                loc = [oracle.localize(x[b, hm], *plan.starts_lens(r)) for x in vecs]
                any_pairs |= oracle.kv_chunk_pairs(2 * plan.chunk_len, N, plan.chunk_len, *loc) > 0
        np.testing.assert_array_equal(res["need"][r], any_pairs.astype(np.uint8))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir, N, mask, seed):
    import datetime
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        B, H, D = 1, 2, 16
        vecs, q, k, v, do = _problem(N, B, H, D, mask, seed)
        plan = cp.ChunkPlan.dual(N, world)
        rows = plan.rows(rank).numpy()
        t = lambda a: torch.from_numpy(np.ascontiguousarray(a[:, rows])).double()  # noqa: E731
        vt = [torch.from_numpy(x) for x in vecs]
        o, lse, ctx = cp.cp_attention_forward(t(q), t(k), t(v), vt, plan, 0.25, ops=OracleOps())
        dq, dk, dv = cp.cp_attention_backward(t(do), ctx)
        with open(os.path.join(out_dir, f"r{rank}.pkl"), "wb") as f:
            pickle.dump({"rows": rows, "o": o.numpy(), "lse": lse.numpy(), "dq": dq.numpy(), "dk": dk.numpy(),
                         "dv": dv.numpy(), "need": ctx.need.numpy(), "chunks": ctx.chunks}, f)
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,mask", [(2, "causal_document"), (3, "sliding_window_2k"), (2, "full"),
                                        (2, "middle_rows_dead")])
def test_cp_exchange_matches_global_oracle(tmp_path, world, mask):
    N, seed = 768, 31
    port = _free_port()
    mp.start_processes(_rank_main, args=(world, port, str(tmp_path), N, mask, seed), nprocs=world,
                       start_method="spawn", join=True)
    B, H, D = 1, 2, 16
    vecs, q, k, v, do = _problem(N, B, H, D, mask, seed)
    ref = {h: oracle.attention_head(q, k, v, vecs, 0, h, 0.25, cols=np.arange(N), dout=do) for h in range(H)}
    res = [pickle.load(open(tmp_path / f"r{r}.pkl", "rb")) for r in range(world)]
    need = res[0]["need"]
    for r in res:
        np.testing.assert_array_equal(r["need"], need)  # every rank saw the same need matrix
        rows = r["rows"]
        for h in range(H):
            scale_g = max(np.abs(ref[h]["dk"]).max(), np.abs(ref[h]["dv"]).max(), np.abs(ref[h]["dq"]).max())
            np.testing.assert_allclose(r["o"][0, :, h], ref[h]["o"][rows], rtol=0, atol=1e-12)
            np.testing.assert_allclose(r["lse"][0, h], ref[h]["lse"][rows], rtol=0, atol=1e-12)
            np.testing.assert_allclose(r["dq"][0, :, h], ref[h]["dq"][rows], rtol=0, atol=1e-12 * scale_g)
            np.testing.assert_allclose(r["dk"][0, :, h], ref[h]["dk"][rows], rtol=0, atol=1e-12 * scale_g)
            np.testing.assert_allclose(r["dv"][0, :, h], ref[h]["dv"][rows], rtol=0, atol=1e-12 * scale_g)
    # the need matrix is the oracle's: rank r needs chunk c iff its rows have unmasked pairs in c
    plan = cp.ChunkPlan.dual(N, world)
    for r in range(world):
        loc = [oracle.localize(x[0, 0], *plan.starts_lens(r)) for x in vecs]
        pairs = oracle.kv_chunk_pairs(plan.chunk_len * 2, N, plan.chunk_len, *loc)
        np.testing.assert_array_equal(need[r], (pairs > 0).astype(np.uint8))
    if mask == "full":
        assert need.sum() == need.size
    else:
        assert need.sum() < need.size  # chunks left out of the exchange
    if mask == "middle_rows_dead":  # rank 1 gathers nothing: its rows are O = 0, LSE = -inf, dQ = 0
        assert need[1].sum() == 0 and res[1]["chunks"] == []
        assert np.all(res[1]["o"] == 0) and np.all(np.isneginf(res[1]["lse"])) and np.all(res[1]["dq"] == 0)


def test_chunk_plan_checks():
    plan = cp.ChunkPlan.dual(1024, 4)
    assert plan.owned == [[0, 7], [1, 6], [2, 5], [3, 4]] and plan.chunk_len == 128
    assert plan.owner[6] == 1
    assert plan.rows(1).tolist() == list(range(128, 256)) + list(range(768, 896))
    with pytest.raises(ValueError):
        cp.ChunkPlan(1024, 128, [[0, 1], [2, 3]])  # chunks 4..7 unowned
    with pytest.raises(ValueError):
        cp.ChunkPlan(1000, 125, [[0, 1, 2, 3], [4, 5, 6, 7]])  # chunk length not a multiple of 4


def _rank_bad_args(rank, world, port, out_dir):
    import datetime
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        plan = cp.ChunkPlan.dual(256, world)
        q = torch.zeros(1, 128, 2, 16, dtype=torch.float64)
        vt = [torch.zeros(1, 1, 256, dtype=torch.int32) for _ in range(4)]
        errs = []
        for args in ((q, q[:, :64], q, vt), (q, q, q, [x[..., :128] for x in vt]), (q, q, q, vt[:3])):
            try:
                cp.cp_attention_forward(*args, plan=plan, scale=0.25, ops=OracleOps())
                errs.append("accepted")
            except ValueError:
                errs.append("rejected")
        with pytest.raises(ValueError):  # a plan for another number of ranks
            cp.cp_attention_forward(q, q, q, vt, cp.ChunkPlan.dual(256, world + 1), 0.25, ops=OracleOps())
        with open(os.path.join(out_dir, f"e{rank}.txt"), "w") as f:
            f.write(",".join(errs))
    finally:
        dist.destroy_process_group()


def test_cp_rejects_bad_arguments(tmp_path):
    # every check fires on the host before any collective, on every rank
    world = 2
    mp.start_processes(_rank_bad_args, args=(world, _free_port(), str(tmp_path)), nprocs=world, start_method="spawn",
                       join=True)
    for r in range(world):
        assert open(tmp_path / f"e{r}.txt").read() == "rejected,rejected,rejected"


@pytest.mark.gpu
def test_cp_kernels_one_rank_nccl():
    """The kernel path through NCCL with one rank: the exchange degenerates to copies, and the
    result equals one call of the kernels on the whole sequence."""
    import datetime
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import mask_aware_flash_b200 as fm
    torch.cuda.set_device(0)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60))
    try:
        N, B, H, D = 4096, 1, 4, 128
        vecs, q, k, v, do = _problem(N, B, H, D, "causal_document", 41)
        dev = torch.device("cuda", 0)
        bf = lambda a: torch.from_numpy(a).to(dev).bfloat16()  # noqa: E731
        qt, kt, vt_, dot = bf(q), bf(k), bf(v), bf(do)
        vt = [torch.from_numpy(x).to(dev) for x in vecs]
        plan = cp.ChunkPlan.dual(N, 1)
        o, lse, ctx = cp.cp_attention_forward(qt, kt, vt_, vt, plan, 1 / np.sqrt(D))
        dq, dk, dv = cp.cp_attention_backward(dot, ctx)
        meta = fm.fm_build_mask_meta(*vt, n_q=N)
        o1, lse1 = fm.fm_attn_fwd(qt, kt, vt_, meta, vt, 1 / np.sqrt(D))
        dq1, dk1, dv1 = fm.fm_attn_bwd(qt, kt, vt_, o1, lse1, dot, meta, vt, 1 / np.sqrt(D))
        torch.cuda.synchronize()
        assert fm.fm_get_device_status() == fm.FM_OK
        assert torch.equal(o, o1) and torch.equal(lse, lse1)
        assert torch.equal(dk, dk1) and torch.equal(dv, dv1)
        assert (dq.float() - dq1.float()).abs().max().item() <= 1e-2 * dq1.float().abs().max().item()
    finally:
        dist.destroy_process_group()
