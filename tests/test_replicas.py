"""CPU, 2 ranks over gloo: the replica plumbing bench.py uses for N > 1 GPUs
(barrier, max-over-ranks timing, whole-job aggregation).  Decode attention has
no exchange step, so replicas share no data-path collective."""

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    r, lr, ws = bench.dist_env()
    dist = bench.init_dist(ws, lr, backend="gloo")
    try:
        bench.barrier(dist)
        # each replica reports its own elapsed time; the job time is the slowest rank
        t = bench.max_over_ranks(10.0 + rank, dist)
        q.put((r, ws, t))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_over_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    assert got == [(0, 2, 11.0), (1, 2, 11.0)]


def test_whole_job_value_counts_every_rank():
    import bench
    alg, kv = bench.decode_bytes([10, 20], 2, 8, 2, 128, 16, 2)
    assert kv == 2 * 30 * 2 * 128 * 2
    assert alg == kv + 2 * 2 * 8 * 128 * 2 + (1 + 2) * 4 + 4 * 2


def test_oracle_all_cores_rate_runs_in_spawned_workers():
    """The all-cores oracle timing of bench.py (spawned processes, pools in shared memory)
    on the tiny batch: every worker reports, and the rate is positive."""
    import bench
    import workloads
    from oracle import RefAllocator
    w = workloads.tiny()
    alloc = RefAllocator(w.num_blocks, w.block_size, shuffle_seed=w.alloc_seed)
    workloads.run_setup(w, alloc)
    _, _, tables, lens = workloads.run_step_allocation(w, alloc)
    rate, procs, desc = bench.oracle_rate_all_cores(w, tables, lens, 0.2, workers=2)
    assert procs == 2 and rate > 0 and "spawned" in desc
