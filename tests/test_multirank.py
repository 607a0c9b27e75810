"""Host-side logic of the multi-rank bench on CPU: two gloo ranks.

The bench runs one independent replica of the workload per GPU (weak scaling,
no data-path collective).  What the ranks share is the timing: each rank
times its own steps on the device, the job's step time is the slowest rank's
(one MAX all-reduce that every rank takes), and the job's throughput is the
work of all ranks divided by that time.  The oracle arm runs on rank 0 only;
the other ranks exit without work.
"""
import os
import socket

import numpy as np

import pytest
import torch
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, per_rank_ms, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    try:
        dev = torch.device("cpu")
        ms = bench.max_over_ranks(per_rank_ms[rank], world, dev)
        # a second collective in the same order on every rank (the e2e timing)
        ms2 = bench.max_over_ranks(2.0 * per_rank_ms[rank], world, dev)
        out[rank] = (ms, ms2, bench.job_tflops(world, 1e12, ms))
    finally:
        torch.distributed.destroy_process_group()


def test_max_over_ranks_and_job_throughput_gloo():
    world = 2
    per_rank_ms = [12.5, 17.25]
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, per_rank_ms, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
        for p in procs:
            if p.is_alive():          # a rank that never returned: end it (its own process)
                p.kill()
                p.join()
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        res = dict(out)
    assert set(res) == {0, 1}
    for r in range(world):
        ms, ms2, tf = res[r]
        assert ms == max(per_rank_ms)                 # every rank sees the slowest rank's time
        assert ms2 == 2.0 * max(per_rank_ms)
        # 2 replicas x 1 TFLOP each per step, over the slowest rank's step time
        assert tf == pytest.approx(2 * 1.0 / (max(per_rank_ms) * 1e-3))


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.5, 1, torch.device("cpu")) == 3.5
    assert bench.job_tflops(1, 2e12, 1000.0) == pytest.approx(2.0)
    # weak scaling: N replicas at the same step time deliver N times the work
    assert bench.job_tflops(8, 2e12, 1000.0) == pytest.approx(8 * bench.job_tflops(1, 2e12, 1000.0))


def test_reference_arm_runs_on_rank_zero_only():
    class Args:
        workload = "tiny"
        steps = 1
        warmup = 3
    # a non-zero rank returns at once, without touching the oracle or printing a line
    assert bench.run_reference(Args(), rank=1, world=2) is None


def test_head_ranges_partition_the_heads():
    from sparse_attention_diffusion_rt_b200 import shard
    for H in (1, 7, 16, 24, 30):
        for world in (1, 2, 3, 4, 8):
            if world > H:
                continue
            ranges = [shard.head_range(H, world, r) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == H
            assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))      # contiguous, no overlap
            sizes = [h1 - h0 for h0, h1 in ranges]
            assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1
    with pytest.raises(ValueError):
        shard.head_range(4, 2, 2)


def test_shard_mask_slices_per_head_masks_only():
    from sparse_attention_diffusion_rt_b200 import shard
    shared = np.ones((1, 3, 3), np.uint8)
    assert shard.shard_mask(shared, 2, 5) is shared
    per_head = np.arange(6 * 2 * 2).reshape(6, 2, 2).astype(np.uint8)
    np.testing.assert_array_equal(shard.shard_mask(per_head, 2, 5), per_head[2:5])


def _shard_rank_main(rank, world, port, H, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    from sparse_attention_diffusion_rt_b200 import shard
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    try:
        h0, h1 = shard.head_range(H, world, rank)
        counts = torch.zeros(H, dtype=torch.int64)
        counts[h0:h1] = 1
        torch.distributed.all_reduce(counts)                   # every head owned by exactly one rank
        # each rank draws only its own heads' inputs; together they are the whole problem's
        from sparse_attention_diffusion_rt_b200 import inputs
        w = inputs.Workload("t", 2, H, 70, 16, 64, kept=1, n_sparse_steps=1, seed=5)
        mine = inputs.qkv_steps(w, 2, heads=(h0, h1))
        same = True
        for s in range(2):
            for x in range(3):
                full = torch.zeros((w.B, H, w.L, w.d), dtype=torch.float32)
                full[:, h0:h1] = mine[s][x].float()
                torch.distributed.all_reduce(full)             # disjoint head ranges: the sum is the union
                same &= torch.equal(full.to(torch.bfloat16), inputs.qkv_steps(w, 2)[s][x])
        out[rank] = (counts.tolist(), bool(same))
    finally:
        torch.distributed.destroy_process_group()


def test_head_sharding_gloo_every_head_once():
    world, H = 2, 7
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_shard_rank_main, args=(r, world, port, H, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
        for p in procs:
            if p.is_alive():
                p.kill()
                p.join()
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        res = dict(out)
    assert res[0][0] == res[1][0] == [1] * H
    assert res[0][1] and res[1][1]
