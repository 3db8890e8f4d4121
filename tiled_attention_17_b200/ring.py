"""Ring attention (context parallelism) over torch.distributed.

The sequence is split into contiguous shards, one per rank: rank r holds the
queries, keys and values of positions [r n, (r + 1) n).  The K/V shards travel
around a logical ring, one hop per step: at hop h rank r holds the shard that
started on rank (r - h) mod P, computes its queries' attention over it with
attn_fwd while the next shard is already on its way, and merges the partial
result into an fp32 accumulator by log-sum-exp (LLM-inference article,
section 4.1: queries sharded by rows, K/V passed around a ring, communication
overlapped with the local block; the merge is the block-order exactness of the
FlashAttention optimisation article, section 3.2.2).

With a causal mask the shards from later ranks are entirely masked (skipped),
the rank's own shard is the causal diagonal, and earlier shards are fully
visible.  Every rank still forwards every shard, so all ranks take the same
communication steps in the same order.

With a causal mask, contiguous shards give rank r about r + 1/2 shards of
visible work, so the last rank does most of it.  The zig-zag layout
(layout="zigzag") cuts the sequence into 2P chunks and gives rank r chunks r
and 2P - 1 - r: every rank then holds 2P chunk-pairs of visible work.  The
K/V of both chunks travel together; each (query chunk, key chunk) pair is full,
diagonal or skipped by chunk index, and each local query chunk keeps its own
accumulator.

The attention, merge and finish steps are the library's CUDA kernels; they are
parameters only so that the schedule itself can be exercised with other
implementations (tests on CPU ranks).
"""
from __future__ import annotations


def _cuda_attend(q, k, v, causal, scale):
    from . import binding
    return binding.attention(q, k, v, causal, scale)


class _CudaAccumulator:
    """fp32 output and lse accumulated across hops by attn_lse_merge."""

    def __init__(self, q):
        import torch
        B, H, n, d = q.shape
        self.rows, self.d = B * H * n, d
        self.shape = q.shape
        self.o = torch.empty((B, H, n, d), dtype=torch.float32, device=q.device)
        self.lse = torch.empty((B, H, n), dtype=torch.float32, device=q.device)
        self.first = True

    def merge(self, o_part, lse_part):
        from . import binding
        binding.attn_lse_merge(self.o, self.lse, o_part, lse_part, self.rows, self.d, int(self.first))
        self.first = False

    def finish(self):
        import torch
        from . import binding
        out = torch.empty(self.shape, dtype=torch.bfloat16, device=self.o.device)
        if self.first:   # no visible key at all
            out.zero_()
            self.lse.fill_(float("-inf"))
            return out, self.lse
        binding.attn_lse_merge_finish(self.o, out, self.rows, self.d)
        return out, self.lse


def hop_mask(rank: int, src: int, causal: bool):
    """How rank `rank`'s queries see the shard that started on rank `src`:
    None (fully masked, skipped), "causal" (the diagonal) or "full"."""
    if not causal or src < rank:
        return "full"
    if src == rank:
        return "causal"
    return None


def zigzag_chunks(rank: int, world: int):
    """The two sequence chunks (of 2 * world) that rank `rank` holds in the
    zig-zag layout, in the order they are stored: (rank, 2 * world - 1 - rank)."""
    return rank, 2 * world - 1 - rank


def zigzag_shard(x, rank: int, world: int, dim: int = 2):
    """Rank `rank`'s zig-zag shard of a whole-sequence array or tensor (the
    sequence along `dim`, its length a multiple of 2 * world): its two chunks,
    concatenated."""
    import numpy as np
    n = x.shape[dim]
    if n % (2 * world):
        raise ValueError("sequence length must divide into 2 * world chunks")
    c = n // (2 * world)
    parts = []
    for ch in zigzag_chunks(rank, world):
        idx = [slice(None)] * x.ndim
        idx[dim] = slice(ch * c, (ch + 1) * c)
        parts.append(x[tuple(idx)])
    if isinstance(x, np.ndarray):
        return np.concatenate(parts, axis=dim)
    import torch
    return torch.cat(parts, dim=dim)


def chunk_mask(q_chunk: int, k_chunk: int, causal: bool):
    """How query chunk `q_chunk` sees key chunk `k_chunk` (equal-length chunks
    of one sequence): None (fully masked), "causal" (the diagonal) or "full"."""
    if not causal or k_chunk < q_chunk:
        return "full"
    if k_chunk == q_chunk:
        return "causal"
    return None


def visible_chunk_pairs(rank: int, world: int, causal: bool, layout: str = "contiguous") -> float:
    """Attention work rank `rank` does over the whole ring, in units of
    (chunk x chunk) query-key blocks of the zig-zag chunk size, a diagonal block
    counting one half.  Host arithmetic only (load-balance bookkeeping)."""
    w = {"full": 1.0, "causal": 0.5, None: 0.0}
    if layout == "zigzag":
        mine = zigzag_chunks(rank, world)
        return sum(w[chunk_mask(qc, kc, causal)] for qc in mine for src in range(world)
                   for kc in zigzag_chunks(src, world))
    # a contiguous shard is two chunks: 2r and 2r + 1
    mine = (2 * rank, 2 * rank + 1)
    return sum(w[chunk_mask(qc, kc, causal)] for qc in mine for kc in range(2 * world))


def ring_attention(q, k, v, causal: bool, scale: float | None = None, group=None, attend=None,
                   accumulator=None, layout: str = "contiguous"):
    """This rank's attention output over the whole (sharded) sequence.

    q [B, Hq, n, d], k/v [B, Hkv, n, d]: this rank's shard (same n on every
    rank).  layout "contiguous": positions [r n, (r + 1) n); "zigzag": chunks r
    and 2P - 1 - r of length n / 2 (see zigzag_shard).  Returns (o [B, Hq, n, d]
    bf16, lse [B, Hq, n] fp32) in the shard's own row order.
    """
    if layout == "zigzag":
        return _ring_attention_zigzag(q, k, v, causal, scale, group, attend, accumulator)
    if layout != "contiguous":
        raise ValueError(f"unknown layout {layout!r}")
    import torch
    import torch.distributed as dist
    if scale is None:
        scale = q.shape[-1] ** -0.5
    attend = attend or _cuda_attend
    acc = (accumulator or _CudaAccumulator)(q)
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    to_rank = lambda r: dist.get_global_rank(group, r) if group is not None else r
    nxt, prv = to_rank((rank + 1) % world), to_rank((rank - 1) % world)
    cur = (k.contiguous(), v.contiguous())
    for h in range(world):
        src = (rank - h) % world
        reqs = []
        if h + 1 < world:
            # post this hop's transfer first so it overlaps the local block
            nk, nv = torch.empty_like(cur[0]), torch.empty_like(cur[1])
            ops = [dist.P2POp(dist.isend, cur[0], nxt, group), dist.P2POp(dist.isend, cur[1], nxt, group),
                   dist.P2POp(dist.irecv, nk, prv, group), dist.P2POp(dist.irecv, nv, prv, group)]
            reqs = dist.batch_isend_irecv(ops)
        mode = hop_mask(rank, src, causal)
        if mode is not None:
            o_part, lse_part = attend(q, cur[0], cur[1], mode == "causal", scale)
            acc.merge(o_part, lse_part)
        for r in reqs:
            r.wait()
        if h + 1 < world:
            cur = (nk, nv)
    return acc.finish()


def _ring_attention_zigzag(q, k, v, causal, scale, group, attend, accumulator):
    import torch
    import torch.distributed as dist
    if scale is None:
        scale = q.shape[-1] ** -0.5
    attend = attend or _cuda_attend
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    n = q.shape[2]
    if n % 2:
        raise ValueError("a zig-zag shard holds two equal chunks")
    c = n // 2
    half = lambda t, i: t[:, :, i * c:(i + 1) * c].contiguous()
    mine = zigzag_chunks(rank, world)
    qs = [half(q, 0), half(q, 1)]
    accs = [(accumulator or _CudaAccumulator)(qs[0]), (accumulator or _CudaAccumulator)(qs[1])]
    to_rank = lambda r: dist.get_global_rank(group, r) if group is not None else r
    nxt, prv = to_rank((rank + 1) % world), to_rank((rank - 1) % world)
    cur = (k.contiguous(), v.contiguous())
    for h in range(world):
        src = (rank - h) % world
        reqs = []
        if h + 1 < world:
            nk, nv = torch.empty_like(cur[0]), torch.empty_like(cur[1])
            ops = [dist.P2POp(dist.isend, cur[0], nxt, group), dist.P2POp(dist.isend, cur[1], nxt, group),
                   dist.P2POp(dist.irecv, nk, prv, group), dist.P2POp(dist.irecv, nv, prv, group)]
            reqs = dist.batch_isend_irecv(ops)
        for j, kc in enumerate(zigzag_chunks(src, world)):
            ks, vs = half(cur[0], j), half(cur[1], j)
            for i, qc in enumerate(mine):
                mode = chunk_mask(qc, kc, causal)
                if mode is not None:
                    o_part, lse_part = attend(qs[i], ks, vs, mode == "causal", scale)
                    accs[i].merge(o_part, lse_part)
        for r in reqs:
            r.wait()
        if h + 1 < world:
            cur = (nk, nv)
    (o0, l0), (o1, l1) = accs[0].finish(), accs[1].finish()
    if isinstance(o0, torch.Tensor):
        return torch.cat([o0, o1], dim=2), torch.cat([l0, l1], dim=2)
    import numpy as np
    return np.concatenate([o0, o1], axis=2), np.concatenate([l0, l1], axis=2)


def ring_attention_emulated(q, k, v, shards: int, causal: bool, scale: float | None = None,
                            layout: str = "contiguous", attend=None, accumulator=None):
    """The ring schedule of `ring_attention` for `shards` virtual ranks in one
    process (no communication): each virtual rank's queries attend to the K/V
    shards in the order that rank would receive them.  Returns the
    full-sequence (o, lse) in sequence order.  For checking the per-hop masks
    and the merge kernels on one GPU; `attend` and `accumulator` default to the
    CUDA kernels (other implementations exercise the schedule on the CPU)."""
    import torch
    B, Hq, N, d = q.shape
    attend = attend or _cuda_attend
    acc_cls = accumulator or _CudaAccumulator
    if scale is None:
        scale = d ** -0.5
    cat = lambda xs, dim: (torch.cat(xs, dim=dim) if isinstance(xs[0], torch.Tensor)
                           else __import__("numpy").concatenate(xs, axis=dim))
    if layout == "contiguous":
        if N % shards:
            raise ValueError("sequence length must divide into the shards")
        n = N // shards
        outs, lses = [], []
        for r in range(shards):
            qr = q[:, :, r * n:(r + 1) * n].contiguous()
            acc = acc_cls(qr)
            for h in range(shards):
                src = (r - h) % shards
                mode = hop_mask(r, src, causal)
                if mode is None:
                    continue
                ks = k[:, :, src * n:(src + 1) * n].contiguous()
                vs = v[:, :, src * n:(src + 1) * n].contiguous()
                o_part, lse_part = attend(qr, ks, vs, mode == "causal", scale)
                acc.merge(o_part, lse_part)
            o, lse = acc.finish()
            outs.append(o)
            lses.append(lse)
        return cat(outs, 2), cat(lses, 2)
    if layout != "zigzag":
        raise ValueError(f"unknown layout {layout!r}")
    if N % (2 * shards):
        raise ValueError("sequence length must divide into 2 * shards chunks")
    c = N // (2 * shards)
    chunk = lambda t, ch: t[:, :, ch * c:(ch + 1) * c].contiguous()
    by_chunk = {}
    for r in range(shards):
        for qc in zigzag_chunks(r, shards):
            qs = chunk(q, qc)
            acc = acc_cls(qs)
            for h in range(shards):
                src = (r - h) % shards
                for kc in zigzag_chunks(src, shards):
                    mode = chunk_mask(qc, kc, causal)
                    if mode is None:
                        continue
                    o_part, lse_part = attend(qs, chunk(k, kc), chunk(v, kc), mode == "causal", scale)
                    acc.merge(o_part, lse_part)
            by_chunk[qc] = acc.finish()
    order = range(2 * shards)
    return cat([by_chunk[i][0] for i in order], 2), cat([by_chunk[i][1] for i in order], 2)
