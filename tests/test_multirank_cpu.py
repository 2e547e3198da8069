"""The benchmark's multi-GPU plumbing on the CPU: two gloo ranks, each with its own batch
(weak scaling: no collective on the data path), combined only by the timing reductions
(max over ranks of the step time, sum of the work)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    from paged_kv_attention_39_b200 import workloads as W
    ws, r, local = bench.dist_setup()
    assert (ws, r) == (world, rank)
    # each rank builds its own batch from seed + rank
    wl = W.c2_bf16_decode(seed=rank, batch=4, lmin=32, lmax=64)
    kv = W.algorithmic_kv_bytes(wl)
    ms = 1.0 + rank  # stand-in per-rank step times
    bench.barrier(ws)
    mx = bench.allreduce_max(ms, ws)
    tot = bench.allreduce_sum(kv, ws)
    q.put((rank, mx, tot, kv, int(wl.sched.seq_lens.sum())))
    dist.destroy_process_group()


def test_two_gloo_ranks_reduce_timing_and_work():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, mx0, tot0, kv0, t0), (r1, mx1, tot1, kv1, t1) = res
    assert mx0 == mx1 == 2.0                 # max over ranks
    assert tot0 == tot1 == kv0 + kv1         # whole-job work
    assert t0 != t1                          # the ranks ran different batches
