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
        assert len({s.seed for s in shards}) == 1           # one problem: the same draws on every rank
        # the whole-job value counts every shard: world x per-rank FLOPs over the slowest rank
        assert bench.whole_job_tflops(world, bench.fwd_flops(shards[0]), 1, 1.0) == pytest.approx(
            bench.fwd_flops(w) / 1e-3 / 1e12)
    with pytest.raises(ValueError):
        workloads.shard_heads(workloads.workload("train4k"), 8, 0)   # 4 kv heads over 8 ranks


def test_reference_arm_with_head_shards_times_the_whole_problem_on_rank_zero():
    """--shard heads applies to the GPU arm; the oracle arm still times a sample
    of the whole problem on rank 0 and says so (weak scaling, no shard)."""
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
    assert res["scaling"] == "weak" and res["config"]["workload"] == "tiny"
    assert "rank 0 only" in res["config"]["parallelism"]


def _shard_rank_main(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    import torch
    import torch.distributed as dist
    import workloads
    from oracle import bca_oracle as orc
    dist.init_process_group("gloo")
    try:
        w = workloads.custom("shard_case", 1, [40, 70, 30], None, 6, 2, 32, seed=9)
        s = workloads.shard_heads(w, world, rank)
        inp = workloads.make_inputs(s, with_grad_out=True)
        res = orc.backward(inp["q"], inp["k"], inp["v"], inp["dout"], s.q_offsets, s.kv_offsets,
                           inp["gamma_q"], inp["gamma_k"])
        parts = {}
        for nm in ("out", "dq", "dk", "dv"):
            t = torch.from_numpy(res[nm]).contiguous()
            got = [torch.empty_like(t) for _ in range(world)]
            dist.all_gather(got, t)
            parts[nm] = torch.cat(got, dim=2).numpy()        # heads are axis 2 of [B, S, H, D]
        lse = torch.from_numpy(res["lse"]).contiguous()
        got = [torch.empty_like(lse) for _ in range(world)]
        dist.all_gather(got, lse)
        parts["lse"] = torch.cat(got, dim=1).numpy()          # [B, H, S]
        results[rank] = parts
    finally:
        dist.destroy_process_group()


def test_head_shards_put_together_are_the_unsharded_result():
    """Two gloo ranks each take their kv heads (with their query groups) of one
    problem and run the oracle on their shard; the gathered outputs and
    gradients equal the unsharded oracle's element by element (dgamma, a sum
    over heads, is the sum of the shards' and is not gathered here)."""
    import numpy as np
    import workloads
    from oracle import bca_oracle as orc
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        procs = [ctx.Process(target=_shard_rank_main, args=(r, world, port, results)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        res = dict(results)
    w = workloads.custom("shard_case", 1, [40, 70, 30], None, 6, 2, 32, seed=9)
    inp = workloads.make_inputs(w, with_grad_out=True)
    full = orc.backward(inp["q"], inp["k"], inp["v"], inp["dout"], w.q_offsets, w.kv_offsets,
                        inp["gamma_q"], inp["gamma_k"])
    for nm in ("out", "lse", "dq", "dk", "dv"):
        np.testing.assert_allclose(res[0][nm], full[nm], rtol=0, atol=1e-12, err_msg=nm)
        np.testing.assert_array_equal(res[0][nm], res[1][nm])
