"""Multi-rank host logic of bench.py on CPU (gloo, world size 2): max-over-ranks
timing, distinct per-rank inputs, and the reference arm running on rank 0 only."""
import os
import socket

import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    dist = bench.init_dist(world, backend="gloo", timeout_s=60)
    try:
        vals = bench.max_over_ranks([1.0 + rank, 10.0 - rank], dist)
        seed = bench.rank_seed(1702, rank)
        bench.barrier(dist)
        q.put((rank, vals, seed))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_seeds():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    out.sort()
    for rank, vals, _ in out:
        assert vals == [2.0, 10.0]
    assert out[0][2] != out[1][2]


def test_reference_arm_only_rank0_prints(monkeypatch, capsys):
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3", "--gpus", "2"]) == 0
    assert capsys.readouterr().out == ""


def test_sample_rows_cover_all_depths():
    import bench
    rows, flops = bench.prefill_sample_rows(4)
    c = bench.PREFILL
    assert rows.size == c.B * c.Hq * c.Nq // 4
    i = rows % c.Nq
    assert i.min() == 0 and i.max() >= c.Nq - 4
    full_rows, full_flops = bench.prefill_sample_rows(1)
    from tiled_attention_17_b200 import accounting
    assert full_flops == accounting.prefill_flops(c.B, c.Hq, c.Nq, c.Nkv, c.d, True)
