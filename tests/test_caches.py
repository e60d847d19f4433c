"""The library's own device memory stays bounded (GPU).

A streaming loop grows the key/value cache every chunk, so each forward call
has a new key length.  The library keeps one normalised-key buffer per stream
(grown to the largest length) and at most 64 schedules per device (least
recently used evicted), so after 80 forwards at different lengths on one
stream its footprint is the largest call's key buffer plus a bounded number of
small schedules; results stay exact against the oracle throughout, and
magi_bca_release_caches() returns everything."""
import numpy as np
import pytest
import torch

import block_causal_attention_gqa_b200 as bca
import workloads
from oracle import bca_oracle as orc
from tests._helpers import assert_close, assert_lse_close, to_np

pytestmark = pytest.mark.gpu


def test_streaming_kv_growth_keeps_the_library_footprint_bounded():
    bca.magi_bca_release_caches()
    assert bca.magi_bca_cache_bytes() == 0
    dev = "cuda"
    Hq, Hkv, D, L = 4, 2, 128, 128          # one active chunk of 128 tokens
    n_calls = 80
    gen = torch.Generator(device="cpu").manual_seed(5)
    gq = (1 + 0.1 * torch.randn(D, generator=gen)).to(dev)
    gk = (1 + 0.1 * torch.randn(D, generator=gen)).to(dev)
    q = torch.randn(1, L, Hq, D, generator=gen).to(torch.bfloat16).to(dev)
    kmax = torch.randn(1, L * n_calls, Hkv, D, generator=gen).to(torch.bfloat16)
    vmax = torch.randn(1, L * n_calls, Hkv, D, generator=gen).to(torch.bfloat16)
    kd, vd = kmax.to(dev), vmax.to(dev)
    stream = torch.cuda.current_stream()
    peak = 0
    for n in range(1, n_calls + 1):
        k, v = kd[:, :n * L].contiguous(), vd[:, :n * L].contiguous()
        out, lse = bca.magi_bca_fwd(q, k, v, [0, L], [i * L for i in range(n + 1)], gq, gk, stream=stream)
        if n in (1, 37, n_calls):
            torch.cuda.synchronize()
            o_ref, l_ref = orc.forward(q.cpu(), kmax[:, :n * L], vmax[:, :n * L], [0, L],
                                       [i * L for i in range(n + 1)], gq.cpu(), gk.cpu())
            assert_close(f"out at {n} chunks", to_np(out), o_ref)
            assert_lse_close(f"lse at {n} chunks", to_np(lse), l_ref)
        peak = max(peak, bca.magi_bca_cache_bytes())
    torch.cuda.synchronize()
    assert bca.magi_bca_last_device_status() == 0
    key_buffer = L * n_calls * Hkv * D * 2          # the largest call's normalised keys
    schedule_cap = 64 * 4096                         # 64 schedules of a few KB at most
    held = bca.magi_bca_cache_bytes()
    print(f"cache bytes after {n_calls} key lengths: {held} (peak {peak}); key buffer {key_buffer}")
    assert key_buffer <= held <= key_buffer + schedule_cap
    assert peak <= key_buffer + schedule_cap
    bca.magi_bca_release_caches()
    assert bca.magi_bca_cache_bytes() == 0
    out, _ = bca.magi_bca_fwd(q, kd[:, :L].contiguous(), vd[:, :L].contiguous(), [0, L], [0, L], gq, gk)
    torch.cuda.synchronize()
    o_ref, _ = orc.forward(q.cpu(), kmax[:, :L], vmax[:, :L], [0, L], [0, L], gq.cpu(), gk.cpu())
    assert_close("out after release", to_np(out), o_ref)


def test_a_new_shape_under_capture_is_refused_cleanly():
    """Memory for a shape is allocated on its first call; on a capturing stream
    that call is refused (status -2) without breaking the capture."""
    dev = "cuda"
    w = workloads.custom("capture_new_shape", 1, [192, 64], None, 4, 2, 128, seed=61)
    inp = workloads.make_inputs(w, with_grad_out=False)
    q, k, v = inp["q"].to(dev), inp["k"].to(dev), inp["v"].to(dev)
    gq, gk = inp["gamma_q"].to(dev), inp["gamma_k"].to(dev)
    out = torch.empty_like(q)
    lse = torch.empty(1, 4, w.seqlen_q, device=dev)
    bca.magi_bca_release_caches()
    side = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    status = None
    with torch.cuda.stream(side):
        g.capture_begin()
        try:
            bca.magi_bca_fwd(q, k, v, w.q_offsets, w.kv_offsets, gq, gk, out=out, lse=lse, stream=side)
        except bca.MagiBcaError as e:
            status = e.status
        finally:
            g.capture_end()
    assert status == -2
    del g
    bca.magi_bca_fwd(q, k, v, w.q_offsets, w.kv_offsets, gq, gk, out=out, lse=lse)
    torch.cuda.synchronize()
    o_ref, _ = orc.forward(inp["q"], inp["k"], inp["v"], w.q_offsets, w.kv_offsets, inp["gamma_q"], inp["gamma_k"])
    assert_close("out after a refused capture", to_np(out), o_ref)
