"""Data-parallel host logic on CPU (gloo, world size 2): token shards cover
the batch exactly once, the all-reduced per-rank histograms equal the
histogram of the whole batch, and every rank then takes the same bias step.
The per-rank routing here is the CPU oracle (no GPU in this test)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out_q):
    import oracle
    from expert_load_balancing_tcgen05_b200 import dist as D
    from expert_load_balancing_tcgen05_b200 import workloads as W
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        T, N, K = 1001, 64, 6
        s = W.make_scores(T, N, seed=21).numpy()
        b = W.make_bias(N, seed=22).numpy()
        lo, hi = D.token_range(T, rank, world)
        idx, _ = oracle.select(s[lo:hi], b, K, 4, 2, 2, True, 2.5)
        counts = torch.from_numpy(oracle.histogram(idx, N).astype(np.int32))
        D.allreduce_counts(counts)
        total = D.global_total(hi - lo, K)
        nb = oracle.bias_update(counts.numpy().astype(np.int64), total, b, 0.001, 0)
        gathered = [torch.zeros(N) for _ in range(world)]
        dist.all_gather(gathered, torch.from_numpy(nb))
        out_q.put((rank, lo, hi, counts.numpy().tolist(), total,
                   all(torch.equal(gathered[0], g) for g in gathered)))
    finally:
        dist.destroy_process_group()


def test_token_range_partitions():
    from expert_load_balancing_tcgen05_b200.dist import token_range
    for T in (0, 1, 7, 1001, 16384):
        for world in (1, 2, 3, 8):
            ranges = [token_range(T, r, world) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == T
            assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
            sizes = [h - l for l, h in ranges]
            assert max(sizes) - min(sizes) <= 1


def test_two_rank_counts_allreduce_and_identical_bias_step():
    import oracle
    from expert_load_balancing_tcgen05_b200 import workloads as W
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    T, N, K = 1001, 64, 6
    s = W.make_scores(T, N, seed=21).numpy()
    b = W.make_bias(N, seed=22).numpy()
    idx, _ = oracle.select(s, b, K, 4, 2, 2, True, 2.5)
    full = oracle.histogram(idx, N).tolist()
    assert [r[1:3] for r in res] == [(0, 501), (501, 1001)]
    for r in res:
        assert r[3] == full          # all-reduced per-rank counts == whole-batch histogram
        assert r[4] == T * K         # global assignment total
        assert r[5]                  # identical bias on every rank
