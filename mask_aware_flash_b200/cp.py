"""Context parallelism: one sequence sharded over ranks in chunks, K/V exchanged only where the
mask needs it.

FlashMask-3 explainer (learnaivisually.com), across-ranks paragraph, and the paper abstract
("zero-communication clip-shift-max" on the boundary vectors; "mask-driven communication
pruning"): every rank holds the rows of its chunks and the key-indexed boundary vectors of the
whole sequence.  Each rank

  1. localizes the vectors to its own rows without communication (`fm_localize`, clip-shift-max:
     a row bound becomes the number of this rank's rows below it);
  2. counts, per global KV chunk, the unmasked (row, key) pairs of its rows (`fm_kv_chunk_pairs`);
     a chunk with a zero count holds no key that any of its rows attends to;
  3. exchanges one byte per chunk with every rank (all-gather), so that each owner knows which
     ranks need which of its chunks, and the K/V chunks then move only to the ranks that need
     them (one all-to-all with per-peer sizes);
  4. runs the attention kernels over the gathered keys in ascending global order, with the
     localized vectors of those keys.  Every key left out is masked for every local row, so the
     outputs equal the global attention of the local rows;
  5. in the backward, sends each gathered chunk's dK / dV contribution back to the chunk's owner
     (the same all-to-all reversed); the owner sums the contributions in fp32 (fp64 for fp64 inputs).

The pages give no exchange protocol; the chunk granularity, the byte-per-chunk need vector and
the all-to-all are this module's reading.  The collectives are torch.distributed's (NCCL on
GPUs, where the exchange crosses NVLink); payloads move as bytes, so any dtype travels.  The
attention itself runs in the library's CUDA kernels (`KernelOps`); a caller may pass other
operations with the same signatures.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch
import torch.distributed as dist


@dataclass
class ChunkPlan:
    """Global sequence of N tokens in chunks of `chunk_len`; `owned[r]` = rank r's chunks, ascending."""
    N: int
    chunk_len: int
    owned: list

    def __post_init__(self):
        n_ch = self.N // self.chunk_len
        if self.N % self.chunk_len or self.chunk_len % 4:
            raise ValueError("chunk_len must divide N and be a multiple of 4")
        flat = sorted(c for cs in self.owned for c in cs)
        if flat != list(range(n_ch)):
            raise ValueError("every chunk must be owned by exactly one rank")
        self.owned = [sorted(int(c) for c in cs) for cs in self.owned]
        self.owner = [0] * n_ch
        for r, cs in enumerate(self.owned):
            for c in cs:
                self.owner[c] = r

    @property
    def n_chunks(self) -> int:
        return self.N // self.chunk_len

    @property
    def ranks(self) -> int:
        return len(self.owned)

    def starts_lens(self, r: int):
        return [c * self.chunk_len for c in self.owned[r]], [self.chunk_len] * len(self.owned[r])

    def rows(self, r: int) -> torch.Tensor:
        """Global row indices of rank r's rows, in local order."""
        L = self.chunk_len
        return torch.cat([torch.arange(c * L, (c + 1) * L) for c in self.owned[r]])

    @staticmethod
    def dual(N: int, ranks: int) -> "ChunkPlan":
        """2 * ranks chunks; rank r owns chunks r and 2 * ranks - 1 - r (balanced for causal masks)."""
        n_ch = 2 * ranks
        return ChunkPlan(N, N // n_ch, [[r, n_ch - 1 - r] for r in range(ranks)])


class KernelOps:
    """The library's kernels (CUDA tensors)."""

    def __init__(self, fm=None):
        if fm is None:
            import mask_aware_flash_b200 as fm
        self.fm = fm

    def localize(self, vecs, starts, lens):
        return [x[0] for x in self.fm.fm_localize(vecs, [starts], [lens])]  # 4 x [B, Hm, N]

    def chunk_pairs(self, loc, n_loc: int, chunk_len: int):
        return self.fm.fm_kv_chunk_pairs([x[None] for x in loc], [n_loc], chunk_len)[0]  # [B, Hm, n_chunks]

    def attn_fwd(self, q, k, v, vecs, scale):
        meta = self.fm.fm_build_mask_meta(*vecs, n_q=q.shape[1])
        o, lse = self.fm.fm_attn_fwd(q, k, v, meta, vecs, scale)
        return o, lse, meta

    def attn_bwd(self, q, k, v, o, lse, do, vecs, scale, state):
        return self.fm.fm_attn_bwd(q, k, v, o, lse, do, state, vecs, scale)


@dataclass
class CpContext:
    """What the backward needs from the forward on one rank."""
    plan: ChunkPlan
    rank: int
    need: torch.Tensor          # [R, n_chunks] uint8 (host): rank r's rows attend to chunk c
    chunks: list                # chunks gathered here, ascending
    q: torch.Tensor
    k: torch.Tensor             # gathered keys [B, n_g, H_kv, D]
    v: torch.Tensor
    vecs: list                  # localized vectors of the gathered keys, 4 x [B, Hm, n_g]
    o: torch.Tensor
    lse: torch.Tensor
    scale: float
    state: object = None
    group: object = None
    ops: object = field(default=None, repr=False)


def _bytes(t: torch.Tensor) -> torch.Tensor:
    return t.contiguous().view(torch.uint8).reshape(-1)


def _exchange(send_pieces, send_to, recv_from_counts, piece_bytes, device, group):
    """send_pieces: list of byte tensors of piece_bytes each, grouped by destination rank in rank
    order (send_to[i] = destination of piece i); recv_from_counts[s] = pieces arriving from rank s.
    Returns the received bytes, grouped by source rank in rank order."""
    R = len(recv_from_counts)
    send_counts = [0] * R
    for d in send_to:
        send_counts[d] += 1
    send = torch.cat(send_pieces) if send_pieces else torch.empty(0, dtype=torch.uint8, device=device)
    recv = torch.empty(sum(recv_from_counts) * piece_bytes, dtype=torch.uint8, device=device)
    dist.all_to_all_single(recv, send, [c * piece_bytes for c in recv_from_counts],
                           [c * piece_bytes for c in send_counts], group=group)
    return recv


def cp_attention_forward(q, k, v, vecs, plan: ChunkPlan, scale: float, group=None, ops=None):
    """One rank's forward.  q: [B, n_loc, H, D], k, v: [B, n_loc, H_kv, D] (this rank's rows, its
    chunks in ascending order); vecs: the four global key-indexed vectors [B, Hm, N] (int32; the
    same on every rank).  Returns (o [B, n_loc, H, D], lse [B, H, n_loc], context)."""
    ops = ops or KernelOps()
    rank = dist.get_rank(group)
    R = dist.get_world_size(group)
    if R != plan.ranks:
        raise ValueError("the plan's rank count differs from the group's")
    L, n_ch = plan.chunk_len, plan.n_chunks
    n_loc = L * len(plan.owned[rank])
    if q.dim() != 4 or k.shape != v.shape or q.shape[1] != n_loc or k.shape[1] != n_loc or q.shape[0] != k.shape[0]:
        raise ValueError("q [B, n_loc, H, D] and k, v [B, n_loc, H_kv, D] must hold this rank's rows")
    if len(vecs) != 4 or any(x.dim() != 3 or x.shape[0] != q.shape[0] or x.shape[2] != plan.N for x in vecs):
        raise ValueError("vecs must be the four global vectors [B, Hm, N] of the plan's sequence")
    if any(x.device != q.device for x in (k, v, *vecs)):
        raise ValueError("all tensors must be on the same device")
    B, _, H_kv, D = k.shape
    dev = q.device
    starts, lens = plan.starts_lens(rank)
    loc = ops.localize(vecs, starts, lens)                     # 4 x [B, Hm, N], rows local
    pairs = ops.chunk_pairs(loc, n_loc, L)                     # [B, Hm, n_chunks]
    mine = (pairs.reshape(-1, n_ch) > 0).any(dim=0).to(torch.uint8)
    gathered = [torch.empty_like(mine) for _ in range(R)]
    dist.all_gather(gathered, mine, group=group)               # one byte per chunk from each rank
    need = torch.stack(gathered).cpu()                         # [R, n_chunks]
    # K/V chunks to the ranks that need them: [K chunk | V chunk] per piece, by destination
    kv_loc = torch.stack([k, v])                               # [2, B, n_loc, H_kv, D]
    piece_bytes = _bytes(kv_loc[:, :, :L]).numel()
    my_pos = {c: i for i, c in enumerate(plan.owned[rank])}
    pieces, send_to = [], []
    for d in range(R):
        for c in plan.owned[rank]:
            if need[d, c]:
                i = my_pos[c]
                pieces.append(_bytes(kv_loc[:, :, i * L:(i + 1) * L]))
                send_to.append(d)
    chunks = [c for c in range(n_ch) if need[rank, c]]
    from_counts = [sum(1 for c in chunks if plan.owner[c] == s) for s in range(R)]
    recv = _exchange(pieces, send_to, from_counts, piece_bytes, dev, group)
    # received pieces are grouped by source rank, each source's chunks ascending: index them
    offset, at = 0, {}
    for s in range(R):
        for c in chunks:
            if plan.owner[c] == s:
                at[c] = offset
                offset += piece_bytes
    shape = (2, B, L, H_kv, D)
    if chunks:
        kv_g = torch.cat([recv[at[c]:at[c] + piece_bytes].view(k.dtype).reshape(shape) for c in chunks], dim=2)
        key_ids = torch.cat([torch.arange(c * L, (c + 1) * L, device=dev) for c in chunks])
        vecs_g = [x.index_select(-1, key_ids).contiguous() for x in loc]
    else:  # no local row attends to any key: the kernels run over one fully masked chunk
        kv_g = torch.zeros((2, B, L, H_kv, D), dtype=k.dtype, device=dev)
        vecs_g = [torch.zeros_like(loc[0][..., :L]) for _ in range(4)]
        vecs_g[1].fill_(n_loc)  # lower interval [0, n_loc): every row masked
    k_g, v_g = kv_g[0].contiguous(), kv_g[1].contiguous()
    o, lse, state = ops.attn_fwd(q, k_g, v_g, vecs_g, scale)
    ctx = CpContext(plan, rank, need, chunks, q, k_g, v_g, vecs_g, o, lse, scale, state, group, ops)
    return o, lse, ctx


def cp_attention_backward(do, ctx: CpContext):
    """One rank's backward.  do: [B, n_loc, H, D].  Returns (dq, dk, dv) for this rank's rows and
    keys: dK / dV summed over every rank whose rows attend to this rank's keys."""
    plan, rank, group = ctx.plan, ctx.rank, ctx.group
    R, L = plan.ranks, plan.chunk_len
    dq, dk_g, dv_g = ctx.ops.attn_bwd(ctx.q, ctx.k, ctx.v, ctx.o, ctx.lse, do, ctx.vecs, ctx.scale, ctx.state)
    B, _, H_kv, D = ctx.k.shape
    dev = do.device
    chunks = ctx.chunks
    grads = torch.stack([dk_g, dv_g])                          # [2, B, n_g, H_kv, D]
    piece_bytes = _bytes(grads[:, :, :L]).numel()
    pieces, send_to = [], []
    for d in range(R):                                         # back to each chunk's owner
        for i, c in enumerate(chunks):
            if plan.owner[c] == d:
                pieces.append(_bytes(grads[:, :, i * L:(i + 1) * L]))
                send_to.append(d)
    from_counts = [sum(1 for c in plan.owned[rank] if ctx.need[s, c]) for s in range(R)]
    recv = _exchange(pieces, send_to, from_counts, piece_bytes, dev, group)
    n_loc = L * len(plan.owned[rank])
    acc_dtype = torch.float64 if dk_g.dtype == torch.float64 else torch.float32
    acc = torch.zeros((2, B, n_loc, H_kv, D), dtype=acc_dtype, device=dev)
    my_pos = {c: i for i, c in enumerate(plan.owned[rank])}
    offset = 0
    for s in range(R):
        for c in plan.owned[rank]:
            if ctx.need[s, c]:
                i = my_pos[c]
                part = recv[offset:offset + piece_bytes].view(dk_g.dtype).reshape(2, B, L, H_kv, D)
                acc[:, :, i * L:(i + 1) * L] += part.to(acc_dtype)
                offset += piece_bytes
    return dq, acc[0].to(dk_g.dtype), acc[1].to(dv_g.dtype)
