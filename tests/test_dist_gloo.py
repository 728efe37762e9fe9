"""The multi-rank host logic of bench.py on two gloo ranks (CPU only): every rank
gets an independent layer (its own seed, same shapes), the job's time is the
slowest rank's, and the whole-job throughput counts every rank's tokens."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, q):
    import datetime

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from workloads import WORKLOADS, generate_head, small_workload

        w = bench.rank_workload(WORKLOADS[2], rank)
        small = bench.rank_workload(small_workload(2, seq_len=256, chunk=256, hq=2, hkv=1), rank)
        head = generate_head(small, "k", 0)
        gathered = [torch.empty_like(head) for _ in range(world)]
        dist.all_gather(gathered, head)
        t_max = bench.max_over_ranks(10.0 * (rank + 1), world, torch.device("cpu"))
        value = bench.job_throughput(w.seq_len, 5, world, t_max)
        q.put((rank, w.seed, w.seq_len, t_max, value, all(not torch.equal(gathered[0], g) for g in gathered[1:])))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_bench_rank_logic_on_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=150)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    seeds = [r[1] for r in res]
    assert seeds == [1, 1001]  # rank 0 keeps the workload's seed
    assert all(r[2] == 32768 for r in res)
    assert all(r[3] == 20.0 for r in res)  # max over ranks, seen by every rank
    assert all(abs(r[4] - 32768 * 5 * 2 / 0.020) < 1e-6 for r in res)
    assert all(r[5] for r in res)  # ranks hold different data


def _shard_main(rank, world, port, q):
    import datetime

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from workloads import generate_head, small_workload, structure

        w = small_workload(2, seq_len=256, chunk=256, hq=8, hkv=4)
        local, q0, k0 = bench.shard_heads(w, rank, world)
        st = structure(local)
        qs = torch.stack([generate_head(local, "q", q0 + h, st=st) for h in range(local.hq)])
        ks = torch.stack([generate_head(local, "k", k0 + h, st=st) for h in range(local.hkv)])
        gq = [torch.empty_like(qs) for _ in range(world)]
        gk = [torch.empty_like(ks) for _ in range(world)]
        dist.all_gather(gq, qs)
        dist.all_gather(gk, ks)
        t_max = bench.max_over_ranks(10.0 * (rank + 1), world, torch.device("cpu"))
        # plain bytes through the queue (tensors would travel as shared memory that
        # disappears with the child process)
        q.put((rank, local.hq, local.hkv, q0, k0, torch.cat(gq).view(torch.int16).numpy().tobytes(),
               torch.cat(gk).view(torch.int16).numpy().tobytes(), t_max, bench.job_throughput(w.seq_len, 5, 1, t_max)))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_kv_group_sharding_on_two_gloo_ranks():
    """KV-group sharding of one layer: the ranks' heads are disjoint, keep each query
    head with its KV head, and together are bit-identical to the unsharded layer;
    the job counts one layer's tokens over the slowest rank's time."""
    from workloads import generate_layer, small_workload

    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=150) for _ in range(world))  # drain before joining: large items
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [(r[1], r[2], r[3], r[4]) for r in res] == [(4, 2, 0, 0), (4, 2, 4, 2)]
    full = generate_layer(small_workload(2, seq_len=256, chunk=256, hq=8, hkv=4), with_v=False)
    for r in res:
        assert r[5] == full["q"].view(torch.int16).numpy().tobytes()
        assert r[6] == full["k"].view(torch.int16).numpy().tobytes()
        assert r[7] == 20.0 and abs(r[8] - 256 * 5 / 0.020) < 1e-6
