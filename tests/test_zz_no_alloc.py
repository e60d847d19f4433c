"""The allocation-free backward (magi_bca_bwd_noalloc) against the regular one
and against the fp64 oracle.

magi_bca_bwd_noalloc serves callers that cannot allocate device memory or pass
a workspace: its workspace and schedule live in a device array the library
holds from load until exit.  This file is collected last on purpose, so a run
that stops at the first failure has run every other test before it.  The test
calls both entry points through the C ABI on the same inputs, twice in a row
(the array keeps the previous call's contents, which must not leak into the
next result), and compares with the tolerance the parity tests use, both with
the workspace entry point and with the oracle."""
import pytest
import torch

import block_causal_attention_gqa_b200 as bca
import workloads
from oracle import bca_oracle as orc
from tests._helpers import assert_close, grad_bound, rel_l2, to_np

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["train4k", "ragged", "packed_global"])
def test_noalloc_backward_matches_regular_backward_twice(name):
    if name == "train4k":
        w = workloads.workload("train4k")
    elif name == "ragged":
        w = workloads.custom("ragged_d128", 2, [100, 333, 1000, 67], None, 4, 2, 128, seed=11)
    else:
        w = workloads.custom("packed_global_ragged", 2, [100, 333, 250, 67, 400, 190], None, 4, 2, 128, seed=52,
                             samples=[0, 2, 3, 6], n_global=1)
    inp = workloads.make_inputs(w, with_grad_out=True)
    dev = "cuda"
    q, k, v = inp["q"].to(dev), inp["k"].to(dev), inp["v"].to(dev)
    gq, gk = inp["gamma_q"].to(dev), inp["gamma_k"].to(dev)
    dout = inp["dout"].to(dev)
    out, lse = bca.magi_bca_fwd(q, k, v, w.q_offsets, w.kv_offsets, gq, gk, **w.mask_kw)
    ref = bca.magi_bca_bwd(q, k, v, out, dout, lse, w.q_offsets, w.kv_offsets, gq, gk, **w.mask_kw)
    torch.cuda.synchronize()
    want = orc.backward(inp["q"], inp["k"], inp["v"], inp["dout"], w.q_offsets, w.kv_offsets,
                        inp["gamma_q"], inp["gamma_k"], **w.mask_kw)
    for call in range(2):
        got = (torch.full_like(q, 3.0), torch.full_like(k, 3.0), torch.full_like(v, 3.0),
               torch.full((w.head_dim,), 3.0, device=dev), torch.full((w.head_dim,), 3.0, device=dev))
        bca.magi_bca_bwd_noalloc(q, k, v, out, dout, lse, w.q_offsets, w.kv_offsets, gq, gk, *got, **w.mask_kw)
        torch.cuda.synchronize()
        assert bca.magi_bca_last_device_status() == 0
        for nm, a, b in zip(("dq", "dk", "dv"), got[:3], ref[:3]):
            assert_close(f"call {call} {nm}", to_np(a), to_np(b))
        for nm, a, b in zip(("dgamma_q", "dgamma_k"), got[3:], ref[3:]):
            r = rel_l2(to_np(a), to_np(b))
            assert r <= 5e-3, f"call {call} {nm}: rel L2 {r:.3e}"
        for nm, a in zip(("dq", "dk", "dv"), got[:3]):
            assert_close(f"call {call} {nm} vs oracle", to_np(a), want[nm], max_abs=grad_bound(w.name))
        for nm, a in zip(("dgamma_q", "dgamma_k"), got[3:]):
            r = rel_l2(to_np(a), want[nm])
            assert r <= 5e-3, f"call {call} {nm} vs oracle: rel L2 {r:.3e}"


def test_noalloc_rejects_problems_beyond_its_array():
    w = workloads.custom("big", 1, [8192] * 4, None, 32, 8, 128, seed=3)   # workspace ~ 0.8 GB
    dev = "cuda"
    B, S, Hq, Hkv, D = 1, w.seqlen_q, 32, 8, 128
    q = torch.zeros(B, S, Hq, D, device=dev, dtype=torch.bfloat16)
    k = torch.zeros(B, S, Hkv, D, device=dev, dtype=torch.bfloat16)
    lse = torch.zeros(B, Hq, S, device=dev)
    g = torch.ones(D, device=dev)
    with pytest.raises(bca.MagiBcaError) as ei:
        bca.magi_bca_bwd_noalloc(q, k, k, q, q, lse, w.q_offsets, w.kv_offsets, g, g, torch.empty_like(q),
                                 torch.empty_like(k), torch.empty_like(k))
    assert ei.value.status == -4


def test_noalloc_refuses_a_capturing_stream():
    """Each call copies its schedule from host memory, so on a stream that is
    being captured it returns MAGI_BCA_UNSUPPORTED and enqueues nothing (the
    capture then ends with an empty graph); afterwards it runs normally."""
    w = workloads.custom("ragged_d128", 1, [100, 333, 67], None, 4, 2, 128, seed=11)
    inp = workloads.make_inputs(w, with_grad_out=True)
    dev = "cuda"
    q, k, v = inp["q"].to(dev), inp["k"].to(dev), inp["v"].to(dev)
    gq, gk = inp["gamma_q"].to(dev), inp["gamma_k"].to(dev)
    dout = inp["dout"].to(dev)
    out, lse = bca.magi_bca_fwd(q, k, v, w.q_offsets, w.kv_offsets, gq, gk)
    grads = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v))
    bca.magi_bca_bwd_noalloc(q, k, v, out, dout, lse, w.q_offsets, w.kv_offsets, gq, gk, *grads)
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    status = None
    with torch.cuda.stream(side):
        g.capture_begin()
        try:
            bca.magi_bca_bwd_noalloc(q, k, v, out, dout, lse, w.q_offsets, w.kv_offsets, gq, gk, *grads,
                                     stream=side)
        except bca.MagiBcaError as e:
            status = e.status
        finally:
            g.capture_end()
    assert status == -2
    del g
    bca.magi_bca_bwd_noalloc(q, k, v, out, dout, lse, w.q_offsets, w.kv_offsets, gq, gk, *grads)
    torch.cuda.synchronize()
    assert bca.magi_bca_last_device_status() == 0
    want = orc.backward(inp["q"], inp["k"], inp["v"], inp["dout"], w.q_offsets, w.kv_offsets,
                        inp["gamma_q"], inp["gamma_k"])
    for nm, a in zip(("dq", "dk", "dv"), grads):
        assert_close(f"after refusal {nm}", to_np(a), want[nm], max_abs=grad_bound(w.name))
