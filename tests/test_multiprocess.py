"""Host logic of the multi-rank bench on CPU: two gloo ranks (127.0.0.1).  Each rank runs an
independent copy of the workload, so the only cross-rank steps are the barrier and the
max-over-ranks reduction of the measured time; whole-job throughput divides all ranks' work by
that maximum."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        per_rank_ms = [12.5, 17.25][rank]
        t = bench.max_over_ranks(per_rank_ms, world, torch.device("cpu"))
        dist.barrier()
        out[rank] = t
        # rank 0 alone runs the CPU reference arm; the others return without work
        class A:  # minimal argparse stand-in
            steps, warmup, workload = 1, 0, "tiny"
        if rank != 0:
            assert bench.run_reference(A, rank, world) is None
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    world, port = 2, _free_port()
    out = mp.Manager().dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    assert out[0] == out[1] == 17.25


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.5, 1, torch.device("cpu")) == 3.5


def test_weak_scaling_value_counts_all_ranks():
    import bench
    from spacetime_attention_b200 import synthetic as syn
    w = syn.WORKLOADS["cogvideox_2b"]
    assert bench.step_flops(w) == w.dense_flops()
    # 2100 units on 148 SMs: the last 28 are split 5 ways -> attention + combine kernel + RoPE
    assert bench.attention_launches(w, 148) == 2 and bench.launches_per_step(w, 148) == 3
    assert bench.attention_launches(w, 150) == 1          # 2100 = 14 * 150: no partial wave
    w2 = syn.WORKLOADS["long_video"]
    assert bench.step_flops(w2) == 2 * w2.skiparse_flops()
    # 4608 Skiparse units: 20 left over on 148 SMs, split 7 ways, for each of the two calls
    assert bench.launches_per_step(w2, 148) == 5


def test_cross_launch_count():
    import bench
    from spacetime_attention_b200 import synthetic as syn
    # 113 blocks * 24 heads = 2712 units, 48 left for the last wave, 2 KV tiles: no split
    assert bench.cross_launches(syn.WORKLOADS["open_sora_plan"], 226, 148) == 1
    # 1 block * 2 heads, 8 KV tiles: the two units are split over KV ranges (+ combine kernel)
    assert bench.cross_launches(syn.custom("x", 1, 2, 64, (1, 3, 5), 1000, (16, 24, 24)), 1000, 148) == 2
