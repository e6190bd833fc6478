"""The multi-rank host logic of bench.py on the CPU: two gloo ranks.

bench.py runs one replica per GPU (weak scaling): each rank draws its own batch (seed =
rank), times its own steps, and the job's step time is the slowest rank's (an all-reduce
MAX); the whole-job throughput counts every rank's bytes.  Here two processes on
127.0.0.1 check the reduction, that the replicas' inputs are independent, and the
throughput formula.
"""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    from quantized_paged_kv_02_b200 import inputs
    dist.init_process_group("gloo", rank=rank, world_size=world)
    r, w, local = bench.dist_env()
    got = bench.max_over_ranks([1.0 + r, 10.0 - r, 3.5], w, torch.device("cpu"))
    q = inputs.make("c5", small=True, seed=r).q.float()
    qs = [torch.zeros_like(q) for _ in range(w)]
    dist.all_gather(qs, q)
    out[rank] = {"rank": r, "world": w, "local": local, "max": got,
                 "replicas_differ": not torch.equal(qs[0], qs[1])}
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    for rank in range(world):
        r = res[rank]
        assert (r["rank"], r["world"], r["local"]) == (rank, world, rank)
        assert r["max"] == [2.0, 10.0, 3.5]               # every rank sees the slowest rank's times
        assert r["replicas_differ"]


def test_throughput_is_whole_job():
    import bench
    assert bench.throughput(1e9, 1, 1.0) == pytest.approx(1000.0)
    assert bench.throughput(1e9, 4, 2.0) == pytest.approx(2000.0)   # 4 ranks, each 1 GB in 2 ms
    assert bench.max_over_ranks([1.0, 2.0], 1, None) == [1.0, 2.0]


def test_per_unit_bytes_for_every_workload():
    """The oracle sample's byte count (bench.unit_bytes) works for every bench workload."""
    import bench
    from quantized_paged_kv_02_b200 import inputs
    for name in bench.WORKLOADS:
        w = inputs.make(name, small=True)
        assert bench.unit_bytes(w, 0) > 0


def test_step_launch_count_comes_from_the_library():
    """bench.py counts a step's launches as the write kernel plus what kvq_decode_plan
    reports for the decode call (host only: the cache can live in CPU memory here)."""
    import bench
    from quantized_paged_kv_02_b200 import inputs, kvq
    for name, want in (("c5", 2), ("c4", 3), ("c4-int2", 3)):
        s = inputs._spec(name, False)
        c = kvq.PagedKVCache(s.cache_dtype, s.act_dtype, s.scale_mode, 64, s.block_size,
                             s.num_kv_heads, s.head_dim, device="cpu", max_seqs=s.batch,
                             static_k_scale=None, static_v_scale=None)
        assert c.decode_plan(s.batch, s.num_q_heads, 16384)[1] == want
    assert "decode_plan" in open(bench.__file__).read()


def test_oracle_pool_runs_rounds_on_worker_processes():
    """The CPU baseline's pool: spawned workers (no fork from a CUDA context), each with its
    own unit cache; a round is one step on every worker, timed first start to last end."""
    import bench
    pool = bench.OraclePool("c1", workers=2)
    try:
        assert pool.workers == 2 and pool.cores >= 1
        t = pool.round()
        assert 0.0 < t < 60.0
        assert pool.bytes_per_round() == 2 * pool.case["bytes"] > 0
    finally:
        pool.close()
