"""The multi-GPU bench plumbing on CPU: two gloo ranks, one clip per rank
(weak scaling, no data-path collective), max-over-ranks timing, every rank
taking the same collective steps."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from rope_block_sparse_b200 import synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    r, w, _ = bench.dist_setup(world)
    try:
        t_local = 10.0 * (rank + 1)
        t_max = bench.allreduce_max(t_local, w)
        bench.barrier(w)
        # each rank draws its own clip: seed = rank
        x = synth.draw_tensor("q", 1, 2, (2, 4, 8), "normal", seed=rank)
        q.put((r, w, t_max, float(x.float().sum())))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_timing_and_independent_clips():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [o[0] for o in out] == [0, 1]
    assert all(o[1] == 2 for o in out)
    assert all(o[2] == 20.0 for o in out)          # max over ranks, seen by both
    assert out[0][3] != out[1][3]                  # different clips per rank


def test_flop_counts():
    # dense: 4 * d * heads * N^2
    assert bench.attention_flops(124992, 56, 1) == pytest.approx(336.0e12, rel=1e-3)
    # sparse with every block == dense
    N, nblk = 1000, 8
    import numpy as np

    all_blocks = np.broadcast_to(np.arange(nblk, dtype=np.int32), (1, 2, nblk, nblk))
    assert bench.attention_flops(N, 2, 1, blocks=all_blocks) == pytest.approx(bench.attention_flops(N, 2, 1))
    assert bench.prologue_bytes(124992, 56, 1) == 124992 * 43008


def test_wide_workload_counts():
    """42 heads x 128 carry the same hidden width as 56 x 96, hence the same dense
    FLOPs; the fused prologue's pooled means are 2 x 4 B per (head, block, channel)."""
    w = synth.WORKLOADS["video5s_d128"]
    assert w.heads * w.head_dim == 56 * 96
    assert bench.attention_flops(w.N, w.heads, w.B, d=w.head_dim) == bench.attention_flops(w.N, 56, 1)
    assert bench.pooled_bytes(124992, 56, 1) == 2 * 4 * 56 * 977 * 96
