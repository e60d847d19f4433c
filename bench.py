#!/usr/bin/env python3
"""Benchmark: useful TFLOP/s of block-causal GQA attention with QK-RMSNorm on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--pass fwd|fwdbwd]
                    [--impl ours|reference]

One step is one pass of the hot path over one batch of synthetic input:
the forward (and, for training workloads, the backward) of the workload.
Useful FLOPs count unmasked (query, key) pairs only: forward = 4*D*B*Hq*pairs
(two matmuls over the mask area), backward = 2.5x forward (MAGI-1 App. B.2.1,
the Flash-Attention convention).  Multi-GPU runs are independent replicas
(the path has no exchange step): value = all ranks' FLOPs / max-over-ranks time.

``--impl reference`` times the fp64 CPU oracle (the only reference there is)
on a bounded sample of the same workload, on the host cores, rank 0 only.
"""
import argparse
import hashlib
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

DATASHEET_BF16_TFLOPS = 2250.0   # NVIDIA HGX B200 dense bf16, for context only
HEAD_START_CYCLES = 2_000_000   # GPU spin queued ahead of each timed step (~1 ms at 1.965 GHz)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ------------------------------------------------------------------ work model
def row_visible_keys(w):
    """Visible keys of every query row: query chunk c is kv chunk c' = n_kv - n_q + c
    and sees kv chunks from the first of its sample (packed samples) and from
    c' - R + 1 (KV range R) up to c'; plus the keys of a last global block, and
    every key if c' belongs to that block."""
    qo, ko = w.q_offsets, w.kv_offsets
    nq, nkv = len(qo) - 1, len(ko) - 1
    first_global = nkv - w.n_global
    g0, skv = int(ko[first_global]), int(ko[-1])
    sample_first = np.zeros(nkv, np.int64)
    if w.samples is not None:
        for i in range(len(w.samples) - 1):
            sample_first[w.samples[i]:w.samples[i + 1]] = w.samples[i]
    n = np.empty(w.seqlen_q, np.int64)
    for c in range(nq):
        own = nkv - nq + c
        if own >= first_global:
            n[qo[c]:qo[c + 1]] = skv
            continue
        first = sample_first[own]
        if w.kv_range > 0:
            first = max(first, own - w.kv_range + 1)
        lo, hi = int(ko[first]), int(ko[own + 1])
        n[qo[c]:qo[c + 1]] = (hi - lo) + (skv - g0) - max(0, min(hi, skv) - max(lo, g0))
    return n


def fwd_flops(w):
    return 4.0 * w.head_dim * w.batch * w.heads_q * float(row_visible_keys(w).sum())


def bwd_flops(w):
    return 2.5 * fwd_flops(w)


def fwd_bytes(w):
    """Algorithmic HBM bytes of the forward: read q, k, v once, write out and lse."""
    q = w.batch * w.seqlen_q * w.heads_q * w.head_dim * 2
    kv = 2 * w.batch * w.seqlen_kv * w.heads_kv * w.head_dim * 2
    return q + kv + q + w.batch * w.heads_q * w.seqlen_q * 4


def bwd_main_bytes(w):
    """Algorithmic HBM bytes of the backward's main kernel (bca_bwd_main_kernel):
    it reads the folded query operand Q^ and dO [B,Sq,Hq,D] bf16, the normalised
    keys K^ and V [B,Skv,Hkv,D] bf16 and one 16-byte row of {-lse, -Delta} pieces
    per query row, and adds into the fp32 accumulators of G_q [B,Sq,Hq,D] and of
    dV and G_k [B,Skv,Hkv,D], each read and written once."""
    q = w.batch * w.seqlen_q * w.heads_q * w.head_dim
    kv = w.batch * w.seqlen_kv * w.heads_kv * w.head_dim
    sq_pad = (w.seqlen_q + 127) // 128 * 128
    return 2 * q * 2 + 2 * kv * 2 + w.batch * w.heads_q * sq_pad * 16 + q * 8 + 2 * kv * 8


# ------------------------------------------------------------------ peaks, clocks
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """Samples SM clocks and throttle reasons with nvidia-smi while running."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def _query_once(self):
        try:
            out = subprocess.run(["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                                  "--format=csv,noheader,nounits"], capture_output=True, text=True, timeout=10)
            return [l for l in out.stdout.splitlines() if l.strip()]
        except Exception:
            return []

    def start(self):
        self.lines += self._query_once()
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=10)
                self.lines += [l for l in out.splitlines() if l.strip()]
            except Exception:
                self.proc.kill()
        self.lines += self._query_once()

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in self.lines:
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def kernel_source_sha():
    h = hashlib.sha256()
    for f in ("bca_fwd.cu", "bca_bwd.cu", "bca_bwd_split.cu", "bca_bwd_common.cuh", "sm100.cuh", "bca_norm.cuh",
              "bca_kernels.h", "bca_mask.cuh"):
        p = os.path.join(ROOT, "block_causal_attention_gqa_b200", "csrc", f)
        if os.path.exists(p):
            h.update(open(p, "rb").read())
    return h.hexdigest()[:16]


def ncu_traffic_entry(kernel, workload_name):
    """The committed ncu DRAM-traffic record of (kernel, workload), if it was
    taken on the current kernel sources (else None)."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    try:
        e = json.load(open(p)).get(kernel, {}).get(workload_name)
    except Exception:
        return None
    if e and e.get("kernel_source_sha") == kernel_source_sha():
        return e
    return None


def ncu_traffic(kernel, workload_name):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel sources (else None)."""
    e = ncu_traffic_entry(kernel, workload_name)
    return float(e["dram_bytes_per_launch"]) if e else None


# ------------------------------------------------------------------ distributed
def dist_setup():
    """One process per GPU (torchrun's RANK / LOCAL_RANK / WORLD_SIZE): NCCL on
    GPUs; gloo when no GPU is present (the host-side logic's CPU tests)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], device=dev, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(world, flops_per_step_per_rank, steps, slowest_rank_ms):
    """Throughput of the whole job: every rank runs `steps` steps of its own
    (replica) workload; the job takes as long as its slowest rank."""
    return world * flops_per_step_per_rank * steps / (slowest_rank_ms * 1e-3) / 1e12


# ------------------------------------------------------------------ our arm
def run_ours(args, w, world, rank, local, light=False, pass_=None, steps=None, warmup=None):
    """Times `steps` steps of the workload on this rank's GPU.  light=True (the
    extra workloads measured beside the headline) skips the end-to-end leg and
    returns the device-timed figures only."""
    import block_causal_attention_gqa_b200 as bca
    dev = torch.device("cuda", local)
    pass_ = pass_ or args.pass_
    steps = steps or args.steps
    warmup = warmup or args.warmup
    do_bwd = pass_ == "fwdbwd"
    inp = workloads.make_inputs(w, device=str(dev), with_grad_out=do_bwd)
    q, k, v, gq, gk = inp["q"], inp["k"], inp["v"], inp["gamma_q"], inp["gamma_k"]
    out = torch.empty_like(q)
    lse = torch.empty(w.batch, w.heads_q, w.seqlen_q, device=dev, dtype=torch.float32)
    if do_bwd:
        dout = inp["dout"]
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        dgq = torch.empty(w.head_dim, device=dev)
        dgk = torch.empty(w.head_dim, device=dev)
        dims = bca.make_dims(w.batch, w.seqlen_q, w.seqlen_kv, w.heads_q, w.heads_kv, w.head_dim,
                             len(w.q_chunks), len(w.kv_chunks))
        ws = torch.empty(max(bca.magi_bca_bwd_workspace_size(dims), 1), device=dev, dtype=torch.uint8)
    stream = torch.cuda.current_stream(dev)
    l2_flush = torch.empty(512 * 1024 * 1024 // 4, device=dev, dtype=torch.float32)

    # rotary angle tables (workloads with rope) stay on the device: a training loop
    # computes them there from its learnable frequencies
    rq, rk = inp.get("rope_q"), inp.get("rope_k")

    def fwd_call(q_, k_, v_, out_, lse_):
        if w.rope:
            bca.magi_bca_fwd_rope(q_, k_, v_, w.q_offsets, w.kv_offsets, gq, gk, rq, rk, out=out_, lse=lse_,
                                  stream=stream, **w.mask_kw)
        else:
            bca.magi_bca_fwd(q_, k_, v_, w.q_offsets, w.kv_offsets, gq, gk, out=out_, lse=lse_, stream=stream,
                             **w.mask_kw)

    def bwd_call(q_, k_, v_, out_, do_, lse_, dq_, dk_, dv_):
        if w.rope:
            bca.magi_bca_bwd_rope(q_, k_, v_, out_, do_, lse_, w.q_offsets, w.kv_offsets, gq, gk, rq, rk, dq=dq_,
                                  dk=dk_, dv=dv_, dgamma_q=dgq, dgamma_k=dgk, workspace=ws, stream=stream,
                                  **w.mask_kw, deterministic=w.deterministic)
        else:
            bca.magi_bca_bwd(q_, k_, v_, out_, do_, lse_, w.q_offsets, w.kv_offsets, gq, gk, dq=dq_, dk=dk_,
                             dv=dv_, dgamma_q=dgq, dgamma_k=dgk, workspace=ws, stream=stream, **w.mask_kw,
                             deterministic=w.deterministic)

    def step(ev=None, kev=None):
        # ev: events around the forward and backward calls; kev: a pair the
        # library records around the dominant main kernel (the backward's when
        # there is one, else the forward's) through magi_bca_profile_events
        if ev is not None:
            ev[0].record(stream)
        if kev is not None and not do_bwd:
            bca.magi_bca_profile_events(kev[0], kev[1])
        fwd_call(q, k, v, out, lse)
        if ev is not None:
            ev[1].record(stream)
        if do_bwd:
            if kev is not None:
                bca.magi_bca_profile_events(kev[0], kev[1])
            bwd_call(q, k, v, out, inp["dout"], lse, dq, dk, dv)
            if ev is not None:
                ev[2].record(stream)
        if kev is not None:
            bca.magi_bca_profile_events()

    for _ in range(warmup):
        l2_flush.zero_()
        step()
    torch.cuda.synchronize()
    n_ev = 3 if do_bwd else 2
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(steps)]
    kevs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
    props = torch.cuda.get_device_properties(dev)
    uuid = getattr(props, "uuid", None)
    sampler = ClockSampler(f"GPU-{uuid}" if uuid else local)
    sampler.start()
    barrier(world)
    torch.cuda.synchronize()
    t_wall0 = time.perf_counter()
    host_s = []
    for i in range(steps):
        l2_flush.zero_()           # inputs of small workloads fit in L2: flush between steps
        # a bounded spin (about 1 ms) keeps the GPU busy while the host enqueues
        # the step, so the events time the device work and not the host's
        # argument marshalling (which a training loop overlaps with the previous
        # step); the host time per step is reported beside it
        torch.cuda._sleep(HEAD_START_CYCLES)
        h0 = time.perf_counter()
        step(evs[i], kevs[i])
        host_s.append(time.perf_counter() - h0)
    torch.cuda.synchronize()
    barrier(world)
    t_wall = time.perf_counter() - t_wall0
    sampler.stop()
    fwd_ms = [e[0].elapsed_time(e[1]) for e in evs]
    bwd_ms = [e[1].elapsed_time(e[2]) for e in evs] if do_bwd else [0.0] * len(evs)
    step_ms_total = sum(f + b for f, b in zip(fwd_ms, bwd_ms))
    step_ms_total = max_over_ranks(step_ms_total, world)
    st = bca.magi_bca_last_device_status()
    if st != 0:
        raise RuntimeError(f"device status {st} after the timed region")
    peaks, peak_src = load_peaks()
    burst, sustained = peaks["bf16_tflops"], peaks["bf16_tflops_sustained"]
    flops_step = fwd_flops(w) + (bwd_flops(w) if do_bwd else 0.0)
    value = whole_job_tflops(world, flops_step, steps, step_ms_total)
    kernel_ms = [e[0].elapsed_time(e[1]) for e in kevs]
    dom_ms = float(np.mean(kernel_ms))
    dom_flops = bwd_flops(w) if do_bwd else fwd_flops(w)
    achieved = dom_flops / (dom_ms * 1e-3) / 1e12
    if light:
        clocks = sampler.summary()
        return {"workload": w.name, "pass": pass_, "value": round(value, 2), "unit": "TFLOP/s", "steps": steps,
                "ms_per_step": round(step_ms_total / steps, 4),
                "fwd_ms": round(float(np.mean(fwd_ms)), 4),
                "bwd_ms": round(float(np.mean(bwd_ms)), 4) if do_bwd else None,
                "frac_of_burst": round(value / world / burst, 4),
                "frac_of_sustained": round(value / world / sustained, 4),
                "dominant_kernel": {"kernel": ("bca_bwd_main_kernel" if do_bwd else "bca_fwd_kernel"),
                                    "achieved": round(achieved, 1), "avg_launch_ms": round(dom_ms, 4),
                                    "frac_of_burst": round(achieved / burst, 4),
                                    "frac_of_sustained": round(achieved / sustained, 4)},
                "clocks": {"sm_mhz": clocks["sm_mhz"], "reasons": clocks["reasons"]}}

    # e2e: through the public API with host buffers (pinned), copies in the timed
    # region.  Double-buffered as a training loop would run it: step i's inputs
    # are copied in on one stream and step i-1's results copied out on another
    # while step i computes; the compute stream waits for its inputs, the copies
    # wait for the buffers they overwrite to be free.
    hq = inp["q"].cpu().pin_memory()
    hk = inp["k"].cpu().pin_memory()
    hv = inp["v"].cpu().pin_memory()
    hdo = inp["dout"].cpu().pin_memory() if do_bwd else None
    h_out = torch.empty(q.shape, dtype=q.dtype).pin_memory()
    h_lse = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
    if do_bwd:
        h_dq = torch.empty(q.shape, dtype=q.dtype).pin_memory()
        h_dk = torch.empty(k.shape, dtype=k.dtype).pin_memory()
        h_dv = torch.empty(v.shape, dtype=v.dtype).pin_memory()
    e2e_steps = max(1, min(steps, 20))

    def buffer_set():
        b = {"q": torch.empty_like(q), "k": torch.empty_like(k), "v": torch.empty_like(v),
             "out": torch.empty_like(out), "lse": torch.empty_like(lse)}
        if do_bwd:
            b.update(dout=torch.empty_like(inp["dout"]), dq=torch.empty_like(q), dk=torch.empty_like(k),
                     dv=torch.empty_like(v))
        return b

    sets = [buffer_set(), buffer_set()]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]     # inputs of the set are on the device
    ev_done = [torch.cuda.Event() for _ in range(2)]   # compute on the set finished
    ev_out = [torch.cuda.Event() for _ in range(2)]    # results of the set copied out

    def e2e_step(i):
        b, n = sets[i % 2], i % 2
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(ev_done[n])            # step i-2 no longer reads these inputs
            b["q"].copy_(hq, non_blocking=True)
            b["k"].copy_(hk, non_blocking=True)
            b["v"].copy_(hv, non_blocking=True)
            if do_bwd:
                b["dout"].copy_(hdo, non_blocking=True)
            ev_in[n].record(s_in)
        stream.wait_event(ev_in[n])
        if i >= 2:
            stream.wait_event(ev_out[n])               # step i-2's results are out of this set
        fwd_call(b["q"], b["k"], b["v"], b["out"], b["lse"])
        if do_bwd:
            bwd_call(b["q"], b["k"], b["v"], b["out"], b["dout"], b["lse"], b["dq"], b["dk"], b["dv"])
        ev_done[n].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_done[n])
            if do_bwd:
                h_dq.copy_(b["dq"], non_blocking=True)
                h_dk.copy_(b["dk"], non_blocking=True)
                h_dv.copy_(b["dv"], non_blocking=True)
            else:
                h_out.copy_(b["out"], non_blocking=True)
                h_lse.copy_(b["lse"], non_blocking=True)
            ev_out[n].record(s_out)

    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    e0.record(stream)
    s_in.wait_event(e0)
    s_out.wait_event(e0)
    for i in range(e2e_steps):
        e2e_step(i + 2)
    for n in range(2):
        stream.wait_event(ev_out[n])
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    h2d = (q.numel() + k.numel() + v.numel() + (q.numel() if do_bwd else 0)) * 2
    d2h = (q.numel() + 2 * k.numel()) * 2 if do_bwd else q.numel() * 2 + lse.numel() * 4

    e2e_value = whole_job_tflops(world, flops_step, e2e_steps, e2e_ms)

    # dominant kernel (the backward main kernel when there is a backward, else
    # the forward kernel), timed alone by the events the library recorded
    # around its launch in every timed step
    fwd_avg = float(np.mean(fwd_ms))
    bwd_avg = float(np.mean(bwd_ms)) if do_bwd else 0.0
    if do_bwd:
        # deterministic backward: the events bracket the dq pass and the dK/dV pass
        dom = "bca_bwd_dq_kernel+bca_bwd_dkdv_kernel" if w.deterministic else "bca_bwd_main_kernel"
        alg_bytes = None if w.deterministic else bwd_main_bytes(w)
    else:
        dom, alg_bytes = "bca_fwd_kernel", fwd_bytes(w)
    clocks = sampler.summary()
    # Both measured peaks, always: the burst figure (a GEMM timed alone at full
    # clock) is the target's denominator; the sustained one (a seconds-long GEMM
    # loop under the 1 kW cap) is printed beside it.
    peak = burst
    peak_note = (f"{peak_src} bf16_tflops (burst), the target's denominator; frac_of_sustained divides by "
                 f"{peak_src} bf16_tflops_sustained (seconds-long GEMM loop under the power cap)")
    roofline = {"bound": "tensor", "kernel": dom, "achieved": round(achieved, 1), "peak": peak,
                "peak_source": peak_note, "unit": "TFLOP/s",
                "frac": round(achieved / peak, 4), "peak_sustained": sustained,
                "frac_of_sustained": round(achieved / sustained, 4),
                "frac_of_datasheet_2250": round(achieved / DATASHEET_BF16_TFLOPS, 4),
                "traffic": ncu_traffic(dom, w.name),
                "traffic_source": (ncu_traffic_entry(dom, w.name) or {}).get(
                    "source", "no ncu record at the current kernel sources"),
                "avg_launch_ms": round(dom_ms, 4),
                "algorithmic_bytes_per_launch": alg_bytes}
    # HBM rate of the dominant kernel: ncu's DRAM bytes per launch (and, for the
    # forward, the algorithmic bytes) over the live launch time
    if roofline["traffic"] is not None and dom_ms > 0:
        roofline["dram_gbs"] = round(roofline["traffic"] / (dom_ms * 1e-3) / 1e9, 1)
        roofline["dram_frac_of_hbm_peak"] = round(roofline["dram_gbs"] / peaks["hbm_gbs"], 4)
    if roofline["algorithmic_bytes_per_launch"] is not None and dom_ms > 0:
        roofline["algorithmic_gbs"] = round(roofline["algorithmic_bytes_per_launch"] / (dom_ms * 1e-3) / 1e9, 1)
    launches_per_step = bca_fwd_launches() + (bca_bwd_launches(w) if do_bwd else 0)
    res = {
        "metric": "block-causal attention useful TFLOP/s on 1 B200 and % of dense BF16 peak",
        "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": steps,
        "warmup": warmup, "ms_per_step": round(step_ms_total / steps, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16 q/k/v, gamma 1+N(0,0.1))",
        "config": {"workload": w.name, "pass": pass_, "batch": w.batch, "seqlen_q": w.seqlen_q,
                   "seqlen_kv": w.seqlen_kv, "q_chunks": f"{len(w.q_chunks)}x{w.q_chunks[0]}",
                   "kv_chunks": f"{len(w.kv_chunks)}x{w.kv_chunks[0]}", "heads_q": w.heads_q,
                   "heads_kv": w.heads_kv, "head_dim": w.head_dim, "kv_range": w.kv_range, "rope": w.rope,
                   "deterministic": w.deterministic,
                   "parallelism": f"replicas x{world}",
                   "l2": "flushed (512 MB write) between timed steps, outside the step events",
                   "head_start": "~1 ms GPU spin queued before each step's first event",
                   "fwd_ms": round(fwd_avg, 4), "bwd_ms": round(bwd_avg, 4) if do_bwd else None,
                   "host_enqueue_ms_per_step": round(1e3 * float(np.median(host_s)), 4),
                   "useful_tflop_per_step": round(flops_step / 1e12, 4)},
        "pct_of_measured_peak": round(100 * value / world / burst, 2),
        "pct_of_measured_sustained_peak": round(100 * value / world / sustained, 2),
        "pct_of_datasheet_peak": round(100 * value / world / DATASHEET_BF16_TFLOPS, 2),
        "e2e": {"value": round(e2e_value, 2), "unit": "TFLOP/s", "h2d_bytes_per_step": int(h2d),
                "d2h_bytes_per_step": int(d2h), "steps": e2e_steps},
        "gpu_launches": int(launches_per_step * steps),
        "roofline": roofline,
        "clocks": clocks,
        "wall_s_timed_region": round(t_wall, 3),
    }
    return res


def also_steps(w, pass_):
    """Steps for a workload timed beside the headline: about two seconds of
    device time (from the useful FLOPs at ~1 PFLOP/s), between 10 and 400."""
    f = fwd_flops(w) + (bwd_flops(w) if pass_ == "fwdbwd" else 0.0)
    return int(min(400, max(10, 2.0 / (f / 1e15))))


def bca_fwd_launches():
    return 2   # key pre-pass, forward kernel


def bca_bwd_launches(w):
    # prep (query and key rows), main, finalize (plus a memset of the padded lse rows
    # when Sq % 128 != 0); deterministic: also the dq pass and the dgamma reduction
    return 5 if w.deterministic else 3


# ------------------------------------------------------------------ oracle (CPU)
def oracle_sample(w, inp, rows, do_bwd):
    """Runs the oracle on the given query rows (all heads, batch 0)."""
    from oracle import bca_oracle as orc
    rq, rk = inp.get("rope_q"), inp.get("rope_k")
    orc.forward_rows(inp["q"], inp["k"], inp["v"], w.q_offsets, w.kv_offsets, inp["gamma_q"],
                     inp["gamma_k"], rows, batches=[0], **w.mask_kw, rope_q=rq, rope_k=rk)
    if do_bwd:
        orc.backward_rows(inp["q"], inp["k"], inp["v"], inp["dout"], w.q_offsets, w.kv_offsets,
                          inp["gamma_q"], inp["gamma_k"], q_rows=rows, batches=[0], **w.mask_kw,
                          rope_q=rq, rope_k=rk)


def sample_flops(w, rows, do_bwd):
    keys = row_visible_keys(w)[rows]
    f = 4.0 * w.head_dim * w.heads_q * float(keys.sum())
    return f * (1 + (2.5 if do_bwd else 0.0))


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count()


def time_oracle(w, do_bwd, budget_s):
    """Times the oracle on growing blocks of rows (evenly spread over the
    query sequence) until ~budget_s of CPU work; returns (TFLOP/s, rows, s)."""
    inp = workloads.make_inputs(w, with_grad_out=do_bwd)
    rng = np.random.default_rng(0)
    n = 16
    done_rows, done_t, done_f = 0, 0.0, 0.0
    while done_t < budget_s:
        rows = np.sort(rng.choice(w.seqlen_q, size=min(n, w.seqlen_q), replace=False))
        t0 = time.perf_counter()
        oracle_sample(w, inp, rows, do_bwd)
        dt = time.perf_counter() - t0
        done_rows += len(rows)
        done_t += dt
        done_f += sample_flops(w, rows, do_bwd)
        if dt < budget_s / 8:
            n *= 2
    return done_f / done_t / 1e12, done_rows, done_t


def run_reference(args, w, world, rank):
    if rank != 0:
        return None
    do_bwd = args.pass_ == "fwdbwd"
    per_step = max(0.05, 90.0 / max(1, args.steps + args.warmup))
    inp = workloads.make_inputs(w, with_grad_out=do_bwd)
    rows_per_step = 8
    # calibrate the sample size to the per-step budget
    t0 = time.perf_counter()
    oracle_sample(w, inp, np.arange(rows_per_step), do_bwd)
    dt = time.perf_counter() - t0
    rows_per_step = int(max(1, min(w.seqlen_q, rows_per_step * per_step / max(dt, 1e-6))))
    rng = np.random.default_rng(1)
    for _ in range(args.warmup):
        oracle_sample(w, inp, np.sort(rng.choice(w.seqlen_q, rows_per_step, replace=False)), do_bwd)
    tot_t, tot_f = 0.0, 0.0
    for _ in range(args.steps):
        rows = np.sort(rng.choice(w.seqlen_q, rows_per_step, replace=False))
        t0 = time.perf_counter()
        oracle_sample(w, inp, rows, do_bwd)
        tot_t += time.perf_counter() - t0
        tot_f += sample_flops(w, rows, do_bwd)
    value = tot_f / tot_t / 1e12
    sample = (f"{rows_per_step} random query rows x all {w.heads_q} heads of batch 0 per step "
              f"({'fwd+bwd' if do_bwd else 'fwd'}), fp64 NumPy")
    return {
        "impl": "reference",
        "metric": "block-causal attention useful TFLOP/s on 1 B200 and % of dense BF16 peak",
        "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * tot_t / args.steps, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "pass": args.pass_, "batch": w.batch, "seqlen_q": w.seqlen_q,
                   "seqlen_kv": w.seqlen_kv, "q_chunks": f"{len(w.q_chunks)}x{w.q_chunks[0]}",
                   "kv_chunks": f"{len(w.kv_chunks)}x{w.kv_chunks[0]}", "heads_q": w.heads_q,
                   "heads_kv": w.heads_kv, "head_dim": w.head_dim, "kv_range": w.kv_range, "rope": w.rope,
                   "deterministic": w.deterministic},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cpu_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ------------------------------------------------------------------ main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="long262k",
                    help="workload name (see workloads.WORKLOADS); the default is the largest single-GPU "
                         "training workload")
    ap.add_argument("--also", default="train4k,model46k,stream4of16",
                    help="comma-separated workloads timed in the same process after the headline one "
                         "(device-timed only, each in its own default pass), reported under 'also'; "
                         "'none' to skip.  Single GPU without --shard only.")
    ap.add_argument("--pass", dest="pass_", default=None, choices=["fwd", "fwdbwd"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--shard", default="replicas", choices=["replicas", "heads"],
                    help="replicas: every rank runs the whole workload (weak scaling); heads: the "
                         "kv heads (with their query-head groups) are split over the ranks, one "
                         "problem in all (strong scaling, no collective on the data path)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    w = workloads.workload(args.config)
    if args.pass_ is None:
        args.pass_ = "fwdbwd" if w.backward else "fwd"
    world, rank, local = dist_setup()
    try:
        if args.impl == "reference":
            # the oracle arm always times a sample of the whole problem on rank 0
            # (--shard does not apply to it): weak scaling, one process at work
            res = run_reference(args, w, world, rank)
            if res is not None and args.shard == "heads":
                res["config"]["parallelism"] = ("oracle on rank 0 only (a sample of the whole problem); "
                                                "--shard heads applies to the GPU arm")
        elif args.shard == "heads":
            res = run_ours(args, workloads.shard_heads(w, world, rank), world, rank, local)
            # the line describes the whole problem: value and e2e already count
            # every rank's share (world x the per-rank FLOPs over the slowest rank);
            # the per-pass times and the roofline are rank 0's shard
            res["scaling"] = "strong"
            res["config"].update({"workload": w.name, "heads_q": w.heads_q, "heads_kv": w.heads_kv,
                                  "parallelism": f"kv heads split over {world} ranks",
                                  "per_rank_figures": "fwd_ms, bwd_ms and roofline are rank 0's shard "
                                                      f"({w.heads_q // world} query / {w.heads_kv // world} kv heads)",
                                  "useful_tflop_per_step": round(fwd_flops(w) / 1e12 + (
                                      bwd_flops(w) / 1e12 if args.pass_ == "fwdbwd" else 0.0), 4)})
            res["roofline"]["scope"] = "per rank (rank 0 shard)"
            if res["roofline"].get("traffic") is None:
                res["roofline"]["traffic_note"] = "no ncu capture of the sharded launch"
        else:
            res = run_ours(args, w, world, rank, local)
            if rank == 0 and world == 1 and not args.no_cpu_baseline:
                tf, nrows, secs = time_oracle(w, args.pass_ == "fwdbwd", budget_s=12.0)
                res["cpu_baseline"] = {"value": tf, "unit": "TFLOP/s", "cores": cpu_threads(), "kind": "oracle",
                                       "sample": f"{nrows} random query rows x all {w.heads_q} heads of batch 0 "
                                                 f"({args.pass_}), fp64 NumPy, {secs:.1f} s"}
            also = [a for a in args.also.split(",") if a and a != "none" and a != w.name]
            if world == 1 and also:
                torch.cuda.empty_cache()
                res["also"] = {}
                for name in also:
                    wa = workloads.workload(name)
                    pa = "fwdbwd" if wa.backward else "fwd"
                    res["also"][name] = run_ours(args, wa, world, rank, local, light=True, pass_=pa,
                                                 steps=also_steps(wa, pa), warmup=max(args.warmup, 3))
                    torch.cuda.empty_cache()
        if rank == 0 and res is not None:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
