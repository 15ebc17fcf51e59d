"""The multi-GPU path on CPU: two gloo ranks exercise the host logic that
bench.py runs under torchrun (disjoint stream shards, independent inputs per
rank, timing reduced as the maximum over ranks, whole-job throughput).  No
data-path collective exists: decode streams are independent."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        import workloads as W
        shard = bench.shard_streams(3, rank)
        # shards are disjoint and cover 0 .. world*3-1
        ids = torch.tensor(list(shard), dtype=torch.int64)
        gathered = [torch.zeros_like(ids) for _ in range(world)]
        dist.all_gather(gathered, ids)
        all_ids = torch.cat(gathered).tolist()
        # each rank draws its own streams: the data differs between ranks
        w = W.Workload("tiny", 3, 255, 256, "last", n_q_heads=16, n_kv_heads=1)
        inp = W.make_inputs(w, streams=shard)
        digest = torch.tensor([float(inp.idx_k_cache.double().sum()), float(inp.q.double().sum())])
        dg = [torch.zeros_like(digest) for _ in range(world)]
        dist.all_gather(dg, digest)
        # timing: the slowest rank decides
        local_ms = [1.0 + rank, 10.0 - rank]
        mx = bench.max_over_ranks(local_ms)
        q.put((rank, all_ids, [d.tolist() for d in dg], mx,
               bench.job_tokens_per_s(32, world, mx[0])))
    finally:
        dist.destroy_process_group()


def test_two_rank_replicas_gloo():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    for rank, all_ids, digests, mx, tps in res:
        assert sorted(all_ids) == list(range(6))
        assert digests[0] != digests[1]
        assert mx == [2.0, 10.0]
        assert tps == pytest.approx(64 / 2.0e-3)


def test_single_process_reduction_is_identity():
    import bench
    assert bench.max_over_ranks([1.5, 2.5]) == [1.5, 2.5]
    assert list(bench.shard_streams(32, 0)) == list(range(32))
    assert list(bench.shard_streams(32, 3)) == list(range(96, 128))
