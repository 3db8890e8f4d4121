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


def ring_attention(q, k, v, causal: bool, scale: float | None = None, group=None, attend=None,
                   accumulator=None):
    """This rank's attention output over the whole (sharded) sequence.

    q [B, Hq, n, d], k/v [B, Hkv, n, d]: this rank's shard (same n on every
    rank).  Returns (o [B, Hq, n, d] bf16, lse [B, Hq, n] fp32).
    """
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


def ring_attention_emulated(q, k, v, shards: int, causal: bool, scale: float | None = None):
    """The ring schedule of `ring_attention` for `shards` virtual ranks in one
    process (no communication): shard r of q attends to the K/V shards in the
    order rank r would receive them.  Returns the full-sequence (o, lse).
    For checking the per-hop masks and the merge kernels on one GPU."""
    import torch
    B, Hq, N, d = q.shape
    if N % shards:
        raise ValueError("sequence length must divide into the shards")
    n = N // shards
    if scale is None:
        scale = d ** -0.5
    outs, lses = [], []
    for r in range(shards):
        qr = q[:, :, r * n:(r + 1) * n].contiguous()
        acc = _CudaAccumulator(qr)
        for h in range(shards):
            src = (r - h) % shards
            mode = hop_mask(r, src, causal)
            if mode is None:
                continue
            ks = k[:, :, src * n:(src + 1) * n].contiguous()
            vs = v[:, :, src * n:(src + 1) * n].contiguous()
            o_part, lse_part = _cuda_attend(qr, ks, vs, mode == "causal", scale)
            acc.merge(o_part, lse_part)
        o, lse = acc.finish()
        outs.append(o)
        lses.append(lse)
    return torch.cat(outs, dim=2), torch.cat(lses, dim=2)
