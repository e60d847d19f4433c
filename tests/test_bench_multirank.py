"""bench.py's multi-process plumbing on CPU: two gloo ranks, as torchrun would
start them (one process per GPU on the GPU machine, NCCL there)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    import bench
    import torch.distributed as dist
    w, r, _ = bench.dist_setup()
    try:
        assert (w, r) == (world, rank)
        # each rank's time differs; every rank must see the slowest
        slowest = bench.max_over_ranks(10.0 + 5.0 * rank, w)
        bench.barrier(w)
        value = bench.whole_job_tflops(w, 2.0e12, 4, slowest)
        results[rank] = (slowest, value)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_time_and_whole_job_value():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, results)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        res = dict(results)
    # max over ranks: 15 ms; value = 2 ranks x 2 TFLOP x 4 steps / 15 ms
    for rank in range(world):
        slowest, value = res[rank]
        assert slowest == pytest.approx(15.0)
        assert value == pytest.approx(2 * 2.0 * 4 / 15e-3)


def test_whole_job_value_is_weak_scaling():
    import bench
    one = bench.whole_job_tflops(1, 1e12, 10, 100.0)
    eight = bench.whole_job_tflops(8, 1e12, 10, 100.0)
    assert eight == pytest.approx(8 * one)


def test_reference_arm_under_torchrun_prints_one_line_from_rank_zero():
    """`bench.py --impl reference --gpus 2` launched the way the driver launches it:
    rank 0 times the oracle and prints one JSON line; rank 1 exits 0 without work."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py",
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3", "--config", "tiny"]
    out = subprocess.run(cmd, cwd=root, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    res = json.loads(lines[0])
    assert res["impl"] == "reference" and res["n_gpus"] == 2 and res["value"] > 0
    assert res["config"]["workload"] == "tiny" and res["e2e"]["h2d_bytes_per_step"] == 0


def test_head_shards_cover_the_problem_once():
    """--shard heads: the ranks' shards split the kv heads (with their query
    groups) and together hold exactly the problem's useful FLOPs; head counts
    that do not split are refused."""
    import bench
    import workloads
    for name, world in (("model46k", 8), ("model46k", 4), ("train4k", 4), ("long262k", 2)):
        w = workloads.workload(name)
        shards = [workloads.shard_heads(w, world, r) for r in range(world)]
        assert all(s.heads_kv * world == w.heads_kv and s.heads_q * world == w.heads_q for s in shards)
        assert all(s.heads_q // s.heads_kv == w.heads_q // w.heads_kv for s in shards)   # whole GQA groups
        assert sum(bench.fwd_flops(s) for s in shards) == bench.fwd_flops(w)
        assert len({s.seed for s in shards}) == world
        # the whole-job value counts every shard: world x per-rank FLOPs over the slowest rank
        assert bench.whole_job_tflops(world, bench.fwd_flops(shards[0]), 1, 1.0) == pytest.approx(
            bench.fwd_flops(w) / 1e-3 / 1e12)
    with pytest.raises(ValueError):
        workloads.shard_heads(workloads.workload("train4k"), 8, 0)   # 4 kv heads over 8 ranks


def test_reference_arm_with_head_shards_reports_strong_scaling():
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py",
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3", "--config", "tiny",
           "--shard", "heads"]
    out = subprocess.run(cmd, cwd=root, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    res = json.loads(lines[0])
    assert res["scaling"] == "strong" and res["config"]["workload"] == "tiny"
