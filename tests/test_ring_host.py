"""The ring-attention schedule on CPU ranks (gloo, world sizes 2 to 4; contiguous
and zig-zag shard layouts): every
rank's output, assembled hop by hop from the K/V shards that travel around the
ring and merged by log-sum-exp, equals attention over the whole sequence.

The ranks run the library's ring driver with the oracle as the per-hop
attention and an fp64 log-sum-exp accumulator, so this checks the schedule
(which shard arrives at which hop, which hops are masked or skipped, the
send/receive pairing) independently of the CUDA kernels; the kernels are
checked against the oracle on the GPU (single-process emulation of the same
schedule)."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class _Fp64Accumulator:
    def __init__(self, q):
        B, H, n, d = q.shape
        self.o = None
        self.lse = None

    def merge(self, o_part, lse_part):
        o_part = np.asarray(o_part, dtype=np.float64)
        lse_part = np.asarray(lse_part, dtype=np.float64)
        if self.o is None:
            self.o, self.lse = o_part.copy(), lse_part.copy()
            return
        m = np.maximum(self.lse, lse_part)
        safe = np.where(np.isneginf(m), 0.0, m)
        wa = np.where(np.isneginf(self.lse), 0.0, np.exp(self.lse - safe))
        wp = np.where(np.isneginf(lse_part), 0.0, np.exp(lse_part - safe))
        tot = wa + wp
        with np.errstate(invalid="ignore", divide="ignore"):
            self.o = np.where(tot[..., None] > 0, (wa[..., None] * self.o + wp[..., None] * o_part) / tot[..., None],
                              0.0)
            self.lse = np.where(tot > 0, safe + np.log(tot), -np.inf)

    def finish(self):
        return self.o, self.lse


def _oracle_attend(q, k, v, causal, scale):
    import oracle
    bits = lambda t: t.numpy().view(np.uint16)
    return oracle.attn(bits(q), bits(k), bits(v), causal, scale=scale)


def _worker(rank, world, port, causal, q_out, layout="contiguous"):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    sys.path.insert(0, os.path.join(root, "tests"))
    import torch
    import torch.distributed as dist
    from tiled_attention_17_b200 import ring
    from tiled_attention_17_b200.inputs import random_prefill
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        n = 6
        q, k, v = random_prefill(1, 4, 2, n * world, n * world, 3, seed=40 + world)   # the whole sequence
        if layout == "zigzag":
            shard = lambda a: torch.from_numpy(np.ascontiguousarray(ring.zigzag_shard(a, rank, world)).view(np.int16))
        else:
            shard = lambda a: torch.from_numpy(np.ascontiguousarray(a[:, :, rank * n:(rank + 1) * n]).view(np.int16))
        o, lse = ring.ring_attention(shard(q), shard(k), shard(v), causal, scale=0.8,
                                     attend=_oracle_attend, accumulator=_Fp64Accumulator, layout=layout)
        q_out.put((rank, o, lse))
    finally:
        dist.destroy_process_group()


def _run_ring(world, causal, layout):
    ctx = mp.get_context("spawn")
    qo = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, causal, qo, layout)) for r in range(world)]
    for p in procs:
        p.start()
    out = sorted([qo.get(timeout=180) for _ in procs], key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return out


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("causal", [True, False])
def test_ring_schedule_matches_whole_sequence(world, causal):
    import oracle
    from tiled_attention_17_b200.inputs import random_prefill
    out = _run_ring(world, causal, "contiguous")
    n = 6
    q, k, v = random_prefill(1, 4, 2, n * world, n * world, 3, seed=40 + world)
    o_ref, lse_ref = oracle.attn(q, k, v, causal, scale=0.8)
    o = np.concatenate([t[1] for t in out], axis=2)
    lse = np.concatenate([t[2] for t in out], axis=2)
    assert np.allclose(o, o_ref, rtol=0, atol=1e-12)
    assert np.allclose(lse, lse_ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("world", [2, 3, 4])
@pytest.mark.parametrize("causal", [True, False])
def test_zigzag_ring_matches_whole_sequence(world, causal):
    """The zig-zag layout: rank r holds chunks r and 2P-1-r; its output rows,
    put back in sequence order, equal whole-sequence attention."""
    import oracle
    from tiled_attention_17_b200 import ring
    from tiled_attention_17_b200.inputs import random_prefill
    out = _run_ring(world, causal, "zigzag")
    n = 6
    q, k, v = random_prefill(1, 4, 2, n * world, n * world, 3, seed=40 + world)
    o_ref, lse_ref = oracle.attn(q, k, v, causal, scale=0.8)
    for rank, o, lse in out:
        assert np.allclose(o, ring.zigzag_shard(o_ref, rank, world), rtol=0, atol=1e-12)
        assert np.allclose(lse, ring.zigzag_shard(lse_ref, rank, world), rtol=0, atol=1e-12)


def test_zigzag_layout_and_balance():
    from tiled_attention_17_b200 import ring
    x = np.arange(16).reshape(1, 1, 16)
    # 4 ranks, 8 chunks of 2: rank r holds chunks r and 7 - r
    assert ring.zigzag_shard(x, 0, 4).ravel().tolist() == [0, 1, 14, 15]
    assert ring.zigzag_shard(x, 3, 4).ravel().tolist() == [6, 7, 8, 9]
    allrows = sorted(np.concatenate([ring.zigzag_shard(x, r, 4).ravel() for r in range(4)]).tolist())
    assert allrows == list(range(16))
    for world in (2, 3, 4, 8):
        zz = [ring.visible_chunk_pairs(r, world, True, "zigzag") for r in range(world)]
        ct = [ring.visible_chunk_pairs(r, world, True, "contiguous") for r in range(world)]
        total = (2 * world) ** 2 / 2          # all causal (chunk x chunk) blocks, diagonals as halves
        assert sum(zz) == sum(ct) == total
        assert len(set(zz)) == 1              # zig-zag: every rank the same work
        assert ct[-1] == (4 * world - 2) and ct[0] == 2      # contiguous: 2, 6, 10, ...


def test_hop_masks():
    from tiled_attention_17_b200.ring import hop_mask
    assert hop_mask(2, 1, True) == "full" and hop_mask(2, 2, True) == "causal" and hop_mask(2, 3, True) is None
    assert all(hop_mask(r, s, False) == "full" for r in range(3) for s in range(3))


@pytest.mark.parametrize("layout", ["contiguous", "zigzag"])
@pytest.mark.parametrize("shards", [2, 3, 4])
@pytest.mark.parametrize("causal", [True, False])
def test_emulated_ring_schedule(layout, shards, causal):
    """The one-process emulation of the ring (the form the GPU tests run with the
    CUDA kernels), here with the oracle per hop and an fp64 merge: the
    reassembled output equals whole-sequence attention."""
    import torch
    import oracle
    from tiled_attention_17_b200 import ring
    from tiled_attention_17_b200.inputs import random_prefill
    N = 6 * shards
    q, k, v = random_prefill(1, 4, 2, N, N, 3, seed=60 + shards)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16))
    o, lse = ring.ring_attention_emulated(t(q), t(k), t(v), shards, causal, scale=0.8, layout=layout,
                                          attend=_oracle_attend, accumulator=_Fp64Accumulator)
    o_ref, lse_ref = oracle.attn(q, k, v, causal, scale=0.8)
    assert np.allclose(o, o_ref, rtol=0, atol=1e-12)
    assert np.allclose(lse, lse_ref, rtol=0, atol=1e-12)
