"""GPU parity of the rotary-embedding entry points (magi_bca_fwd_rope /
magi_bca_bwd_rope) against the fp64 oracle: q and k rotated before the norm
(MAGI-1 §2.2.2, learnable 3D RoPE), angles from workloads.rope_angles."""
import numpy as np
import pytest
import torch

import block_causal_attention_gqa_b200 as bca
import workloads
from oracle import bca_oracle as orc
from tests._helpers import assert_close, assert_lse_close, grad_bound, rel_l2, to_np

pytestmark = pytest.mark.gpu

CASES = {
    "rope_ragged_d128": (workloads.custom("rope_ragged_d128", 2, [100, 333, 1000, 67], None, 4, 2, 128, seed=31,
                                          rope=True), "qk"),
    "rope_stream_d64": (workloads.custom("rope_stream_d64", 2, [150, 250], [300, 200, 150, 250], 8, 2, 64, seed=32,
                                         rope=True), "qk"),
    "rope_q_only": (workloads.custom("rope_q_only", 1, [256, 384, 128], None, 6, 2, 128, seed=33, rope=True), "q"),
    "rope_window_r2": (workloads.custom("rope_window_r2", 1, [300, 200, 150, 250], None, 8, 2, 128, seed=34,
                                        rope=True, kv_range=2), "qk"),
    "rope_train4k": (workloads.custom("rope_train4k", 1, [1024] * 4, None, 16, 4, 128, seed=35, rope=True), "qk"),
    "rope_packed_global": (workloads.custom("rope_packed_global", 1, [300, 200, 150, 250], None, 8, 2, 128, seed=37,
                                            rope=True, samples=[0, 2, 4], n_global=1), "qk"),
}


def tables(inp, which):
    rq = inp["rope_q"] if "q" in which else None
    rk = inp["rope_k"] if "k" in which else None
    return rq, rk


@pytest.mark.parametrize("name", list(CASES))
def test_rope_forward_and_backward_all_rows(name):
    w, which = CASES[name]
    inp = workloads.make_inputs(w, with_grad_out=True)
    rq, rk = tables(inp, which)
    dev = "cuda"
    q, k, v, do = (inp[x].to(dev) for x in ("q", "k", "v", "dout"))
    gq, gk = inp["gamma_q"].to(dev), inp["gamma_k"].to(dev)
    rqd = rq.to(dev) if rq is not None else None
    rkd = rk.to(dev) if rk is not None else None
    out, lse = bca.magi_bca_fwd_rope(q, k, v, w.q_offsets, w.kv_offsets, gq, gk, rqd, rkd, **w.mask_kw)
    dq, dk, dv, dgq, dgk, drq, drk = bca.magi_bca_bwd_rope(q, k, v, out, do, lse, w.q_offsets, w.kv_offsets, gq, gk,
                                                           rqd, rkd, **w.mask_kw)
    torch.cuda.synchronize()
    assert bca.magi_bca_last_device_status() == 0
    ref = orc.backward(inp["q"], inp["k"], inp["v"], inp["dout"], w.q_offsets, w.kv_offsets, inp["gamma_q"],
                       inp["gamma_k"], **w.mask_kw, rope_q=rq, rope_k=rk)
    assert_close(f"{name} out", to_np(out), ref["out"])
    assert_lse_close(f"{name} lse", to_np(lse), ref["lse"])
    for nm, got in (("dq", dq), ("dk", dk), ("dv", dv)):
        e, r = assert_close(f"{name} {nm}", to_np(got), ref[nm], max_abs=grad_bound(name))
        print(f"{name} {nm}: max abs {e:.2e} rel L2 {r:.2e}")
    # sums over batch, tokens and heads (dgamma) or batch and heads (angles): relative L2 only
    for nm, got in (("dgamma_q", dgq), ("dgamma_k", dgk), ("drope_q", drq), ("drope_k", drk)):
        if nm in ref:
            r = rel_l2(to_np(got), ref[nm])
            print(f"{name} {nm}: rel L2 {r:.2e}")
            assert r <= 5e-3, f"{name} {nm}: rel L2 {r:.2e}"
        else:
            assert got is None


def test_rope_with_zero_angles_matches_the_plain_entry_points():
    w = workloads.custom("rope_zero", 1, [200, 300], None, 4, 2, 128, seed=36)
    inp = workloads.make_inputs(w, with_grad_out=True)
    dev = "cuda"
    q, k, v, do = (inp[x].to(dev) for x in ("q", "k", "v", "dout"))
    gq, gk = inp["gamma_q"].to(dev), inp["gamma_k"].to(dev)
    zq = torch.zeros(w.seqlen_q, w.head_dim // 2, device=dev)
    zk = torch.zeros(w.seqlen_kv, w.head_dim // 2, device=dev)
    o0, l0 = bca.magi_bca_fwd(q, k, v, w.q_offsets, w.kv_offsets, gq, gk)
    o1, l1 = bca.magi_bca_fwd_rope(q, k, v, w.q_offsets, w.kv_offsets, gq, gk, zq, zk)
    g0 = bca.magi_bca_bwd(q, k, v, o0, do, l0, w.q_offsets, w.kv_offsets, gq, gk)
    g1 = bca.magi_bca_bwd_rope(q, k, v, o1, do, l1, w.q_offsets, w.kv_offsets, gq, gk, zq, zk)
    torch.cuda.synchronize()
    assert torch.equal(o0, o1) and torch.equal(l0, l1)   # the forward is deterministic: same bits
    # dq, dk, dv, dgamma: pieces of a kv tile and of a query tile are summed by
    # bulk reduce-adds and atomics in no fixed order, so two runs agree to
    # rounding only; a tolerance well inside the oracle's bar.
    for a, b in zip(g0[:5], g1[:5]):
        a, b = a.double(), b.double()
        assert (a - b).norm() <= 1e-3 * b.norm()
        assert (a - b).abs().max() <= 2e-3


def test_rope_full_size_sampled_rows():
    w = workloads.workload("model46k_rope")
    inp = workloads.make_inputs(w, with_grad_out=True)
    dev = "cuda"
    q, k, v, do = (inp[x].to(dev) for x in ("q", "k", "v", "dout"))
    gq, gk = inp["gamma_q"].to(dev), inp["gamma_k"].to(dev)
    rq, rk = inp["rope_q"].to(dev), inp["rope_k"].to(dev)
    out, lse = bca.magi_bca_fwd_rope(q, k, v, w.q_offsets, w.kv_offsets, gq, gk, rq, rk)
    dq, _, _, _, _, _, _ = bca.magi_bca_bwd_rope(q, k, v, out, do, lse, w.q_offsets, w.kv_offsets, gq, gk, rq, rk)
    torch.cuda.synchronize()
    rows = workloads.sample_rows(w.seqlen_q, w.q_offsets, 1024, seed=300)
    idx = torch.as_tensor(rows)
    o_ref, l_ref = orc.forward_rows(inp["q"], inp["k"], inp["v"], w.q_offsets, w.kv_offsets, inp["gamma_q"],
                                    inp["gamma_k"], rows, rope_q=inp["rope_q"], rope_k=inp["rope_k"])
    assert_close("model46k_rope out rows", to_np(out.cpu()[:, idx]), o_ref)
    assert_lse_close("model46k_rope lse rows", to_np(lse.cpu()[:, :, idx]), l_ref)
    ref = orc.backward_rows(inp["q"], inp["k"], inp["v"], inp["dout"], w.q_offsets, w.kv_offsets, inp["gamma_q"],
                            inp["gamma_k"], q_rows=rows[:512], rope_q=inp["rope_q"], rope_k=inp["rope_k"])
    assert_close("model46k_rope dq rows", to_np(dq.cpu()[:, torch.as_tensor(rows[:512])]), ref["dq"])
