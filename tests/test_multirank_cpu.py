"""The multi-rank (replica) logic of bench.py on CPU: two gloo ranks.

Tokens are independent, so N GPUs run N replicas of the layer on their own
token batches with no data-path collective; the only cross-rank steps are the
barrier and the max-over-ranks reduction of the timed region."""
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


def _worker(rank, world, port, q):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [2.0, 3.0][rank]
        bench.barrier(world)
        ms = bench.all_max(local_ms, world)
        value = bench.whole_job_tokens_per_s(32, world, ms)
        env = bench.dist_env()
        q.put((rank, ms, value, env))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_time_and_sum_the_tokens():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get() for _ in range(world))
    for rank, ms, value, env in got:
        assert ms == 3.0                                  # slowest rank
        assert value == pytest.approx(64 / 3e-3)          # both ranks' tokens / max time
        assert env == (world, rank, 0)


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.all_max(1.5, 1) == 1.5
    assert bench.whole_job_tokens_per_s(32, 1, 0.5) == pytest.approx(64000.0)


def test_launch_counts_follow_the_dispatch_in_abi():
    """gpu_launches is a claim: one layer call launches exactly these kernels (abi.cu forward_path)."""
    import bench
    from fine_grained_sparse_fp32_b200.inputs import CONFIGS
    # router logits, top-K, dispatch (one CTA), swap-AB FFN, combine
    assert bench.launches_per_step(CONFIGS["decode"]) == 5
    # E4M3 weights: the x quantiser (two-term, or FP8 activations) before the FP8 tensor-core FFN
    assert bench.launches_per_step(CONFIGS["fp8_decode"]) == 6
    assert bench.launches_per_step(CONFIGS["fp8a8_decode"]) == 6
    # FP32 tiny layer: router logits, top-K, dispatch, streaming FFN up + down, combine
    assert bench.launches_per_step(CONFIGS["tiny"]) == 6
    # split + tensor-core router, top-K (with chunk histograms), scatter with the scan, FFN up + down, combine
    assert bench.launches_per_step(CONFIGS["prefill"]) == 7
    assert bench.launches_per_step(CONFIGS["fp8_prefill"]) == 7
    # more than 64 chunks: scan and scatter are separate launches
    assert bench.launches_per_step(CONFIGS["skew"]) == 8


def test_both_bench_arms_report_the_same_workload():
    import bench
    a, b = bench.decode_config(1), bench.decode_config(1)
    assert a == b and a["tokens_per_gpu"] == 32 and "GB of expert weights" in a["l2"]
