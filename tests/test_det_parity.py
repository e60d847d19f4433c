"""GPU tests of the deterministic backward (dims.deterministic = 1): parity
with the fp64 oracle on every row of small workloads and on sampled rows at
full size, and bit-identical results from repeated calls (different workspace
contents, other work in between, the allocation-free entry point).  The
deterministic path takes dq from a query-major pass with no reductions across
CTAs, gives each kv tile one CTA, and reduces dgamma and the angle gradients
in a fixed order, so equal inputs must give equal bits."""
import numpy as np
import pytest
import torch

import block_causal_attention_gqa_b200 as bca
import workloads
from oracle import bca_oracle as orc
from tests._helpers import assert_close, dgamma_bound, grad_bound, rel_l2, to_np
from tests.test_fwd_parity import SMALL

pytestmark = pytest.mark.gpu

DET_SMALL = ["train4k", "tiny", "ragged_d128", "ragged_d64_gqa3", "stream_small", "token_causal", "many_chunks",
             "gqa8_long_rows", "window_r2_ragged", "window_stream_r3_d64", "xattn_video_text", "xattn_chunkwise",
             "packed_global_ragged", "packed_global_r2_d64", "packed_stream_global"]


def to_dev(inp):
    dev = "cuda"
    t = {x: inp[x].to(dev) for x in ("q", "k", "v", "dout", "gamma_q", "gamma_k")}
    for x in ("rope_q", "rope_k"):
        if x in inp:
            t[x] = inp[x].to(dev)
    return t


def det_bwd(w, t, out, lse, rope=False, workspace=None):
    if rope:
        return bca.magi_bca_bwd_rope(t["q"], t["k"], t["v"], out, t["dout"], lse, w.q_offsets, w.kv_offsets,
                                     t["gamma_q"], t["gamma_k"], t["rope_q"], t["rope_k"], **w.mask_kw,
                                     workspace=workspace, deterministic=True)
    return bca.magi_bca_bwd(t["q"], t["k"], t["v"], out, t["dout"], lse, w.q_offsets, w.kv_offsets, t["gamma_q"],
                            t["gamma_k"], **w.mask_kw, workspace=workspace, deterministic=True)


def fwd(w, t, rope=False):
    if rope:
        return bca.magi_bca_fwd_rope(t["q"], t["k"], t["v"], w.q_offsets, w.kv_offsets, t["gamma_q"], t["gamma_k"],
                                     t["rope_q"], t["rope_k"], **w.mask_kw)
    return bca.magi_bca_fwd(t["q"], t["k"], t["v"], w.q_offsets, w.kv_offsets, t["gamma_q"], t["gamma_k"],
                            **w.mask_kw)


def workspace_filled(w, byte):
    dims = bca.make_dims(w.batch, w.seqlen_q, w.seqlen_kv, w.heads_q, w.heads_kv, w.head_dim,
                         len(w.q_chunks), len(w.kv_chunks), **w.mask_kw, deterministic=True)
    return torch.full((bca.magi_bca_bwd_workspace_size(dims),), byte, device="cuda", dtype=torch.uint8)


@pytest.mark.parametrize("name", DET_SMALL)
def test_deterministic_backward_all_rows(name):
    w = SMALL[name]
    inp = workloads.make_inputs(w, with_grad_out=True)
    t = to_dev(inp)
    out, lse = fwd(w, t)
    dq, dk, dv, dgq, dgk = det_bwd(w, t, out, lse)
    torch.cuda.synchronize()
    assert bca.magi_bca_last_device_status() == 0
    ref = orc.backward(inp["q"], inp["k"], inp["v"], inp["dout"], w.q_offsets, w.kv_offsets,
                       inp["gamma_q"], inp["gamma_k"], **w.mask_kw)
    bound = grad_bound(name)
    for nm, got in (("dq", dq), ("dk", dk), ("dv", dv)):
        e, r = assert_close(f"{name} {nm}", to_np(got), ref[nm], max_abs=bound)
        print(f"{name} {nm}: max abs {e:.2e} rel L2 {r:.2e}")
    for nm, got in (("dgamma_q", dgq), ("dgamma_k", dgk)):
        r = rel_l2(to_np(got), ref[nm])
        print(f"{name} {nm}: rel L2 {r:.2e}")
        assert r <= dgamma_bound(name), f"{name} {nm}: rel L2 {r:.3e}"


@pytest.mark.parametrize("name", ["train4k", "ragged_d64_gqa3", "window_r2_ragged", "xattn_chunkwise",
                                  "packed_global_ragged"])
def test_deterministic_backward_is_bitwise_reproducible(name):
    w = SMALL[name]
    t = to_dev(workloads.make_inputs(w, with_grad_out=True))
    out, lse = fwd(w, t)
    first = det_bwd(w, t, out, lse, workspace=workspace_filled(w, 0x00))
    # other work between the calls (a large write moves L2 contents and timing)
    junk = torch.empty(256 * 1024 * 1024 // 4, device="cuda")
    junk.fill_(3.0)
    second = det_bwd(w, t, out, lse, workspace=workspace_filled(w, 0xAB))
    torch.cuda.synchronize()
    assert bca.magi_bca_last_device_status() == 0
    for nm, a, b in zip(("dq", "dk", "dv", "dgamma_q", "dgamma_k"), first, second):
        assert torch.equal(a, b), f"{name} {nm}: two deterministic calls differ"


def test_deterministic_and_default_backward_agree():
    # the two paths compute the same quantities with different summation orders
    w = SMALL["ragged_d128"]
    t = to_dev(workloads.make_inputs(w, with_grad_out=True))
    out, lse = fwd(w, t)
    det = det_bwd(w, t, out, lse)
    dflt = bca.magi_bca_bwd(t["q"], t["k"], t["v"], out, t["dout"], lse, w.q_offsets, w.kv_offsets,
                            t["gamma_q"], t["gamma_k"])
    torch.cuda.synchronize()
    for nm, a, b in zip(("dq", "dk", "dv", "dgamma_q", "dgamma_k"), det, dflt):
        r = rel_l2(to_np(a), to_np(b))
        assert r <= 2e-3, f"{nm}: deterministic vs default rel L2 {r:.2e}"


def test_deterministic_noalloc_matches_the_workspace_entry_bitwise():
    w = SMALL["ragged_d64_gqa3"]
    t = to_dev(workloads.make_inputs(w, with_grad_out=True))
    out, lse = fwd(w, t)
    a = det_bwd(w, t, out, lse)
    dq, dk, dv = torch.empty_like(t["q"]), torch.empty_like(t["k"]), torch.empty_like(t["v"])
    dgq = torch.empty(w.head_dim, device="cuda")
    dgk = torch.empty(w.head_dim, device="cuda")
    b = bca.magi_bca_bwd_noalloc(t["q"], t["k"], t["v"], out, t["dout"], lse, w.q_offsets, w.kv_offsets,
                                 t["gamma_q"], t["gamma_k"], dq, dk, dv, dgq, dgk, **w.mask_kw,
                                 deterministic=True)
    torch.cuda.synchronize()
    assert bca.magi_bca_last_device_status() == 0
    for nm, x, y in zip(("dq", "dk", "dv", "dgamma_q", "dgamma_k"), a, b):
        assert torch.equal(x, y), f"{nm}: allocation-free and workspace entries differ"


ROPE_CASES = {
    "rope_ragged_d128": workloads.custom("det_rope_ragged_d128", 2, [100, 333, 1000, 67], None, 4, 2, 128,
                                         seed=41, rope=True),
    "rope_window_d64": workloads.custom("det_rope_window_d64", 1, [300, 200, 150, 250], None, 8, 2, 64, seed=42,
                                        rope=True, kv_range=2),
}


@pytest.mark.parametrize("name", list(ROPE_CASES))
def test_deterministic_rope_backward(name):
    w = ROPE_CASES[name]
    inp = workloads.make_inputs(w, with_grad_out=True)
    t = to_dev(inp)
    out, lse = fwd(w, t, rope=True)
    g1 = det_bwd(w, t, out, lse, rope=True, workspace=workspace_filled(w, 0x00))
    g2 = det_bwd(w, t, out, lse, rope=True, workspace=workspace_filled(w, 0x5A))
    torch.cuda.synchronize()
    assert bca.magi_bca_last_device_status() == 0
    names = ("dq", "dk", "dv", "dgamma_q", "dgamma_k", "drope_q", "drope_k")
    for nm, a, b in zip(names, g1, g2):
        assert torch.equal(a, b), f"{name} {nm}: two deterministic calls differ"
    ref = orc.backward(inp["q"], inp["k"], inp["v"], inp["dout"], w.q_offsets, w.kv_offsets, inp["gamma_q"],
                       inp["gamma_k"], **w.mask_kw, rope_q=inp["rope_q"], rope_k=inp["rope_k"])
    for nm, got in zip(names[:3], g1[:3]):
        e, r = assert_close(f"{name} {nm}", to_np(got), ref[nm], max_abs=grad_bound(w.name))
        print(f"{name} {nm}: max abs {e:.2e} rel L2 {r:.2e}")
    for nm, got in zip(names[3:], g1[3:]):
        r = rel_l2(to_np(got), ref[nm])
        print(f"{name} {nm}: rel L2 {r:.2e}")
        assert r <= 5e-3, f"{name} {nm}: rel L2 {r:.3e}"


def test_deterministic_full_size_sampled_and_reproducible():
    w = workloads.workload("model46k")
    inp = workloads.make_inputs(w, with_grad_out=True)
    t = to_dev(inp)
    out, lse = fwd(w, t)
    dq, dk, dv, dgq, dgk = det_bwd(w, t, out, lse)
    again = det_bwd(w, t, out, lse)
    torch.cuda.synchronize()
    assert bca.magi_bca_last_device_status() == 0
    for nm, a, b in zip(("dq", "dk", "dv", "dgamma_q", "dgamma_k"), (dq, dk, dv, dgq, dgk), again):
        assert torch.equal(a, b), f"model46k {nm}: two deterministic calls differ"
    del again
    dq, dk, dv = dq.cpu(), dk.cpu(), dv.cpu()
    torch.cuda.empty_cache()
    rows = workloads.sample_rows(w.seqlen_q, w.q_offsets, 1024, seed=400)
    ref = orc.backward_rows(inp["q"], inp["k"], inp["v"], inp["dout"], w.q_offsets, w.kv_offsets,
                            inp["gamma_q"], inp["gamma_k"], q_rows=rows)
    e, r = assert_close("model46k det dq rows", to_np(dq[:, torch.as_tensor(rows)]), ref["dq"])
    print(f"model46k det dq rows: max abs {e:.2e} rel L2 {r:.2e}")
    last = int(w.kv_offsets[-2])
    kr = np.sort(np.random.default_rng(401).choice(np.arange(last, w.seqlen_kv), 128, replace=False))
    ref = orc.backward_rows(inp["q"], inp["k"], inp["v"], inp["dout"], w.q_offsets, w.kv_offsets,
                            inp["gamma_q"], inp["gamma_k"], kv_rows=kr, kv_heads=[3])
    kidx = torch.as_tensor(kr)
    for nm, got in (("dk", dk), ("dv", dv)):
        e, r = assert_close(f"model46k det {nm} rows", to_np(got[:, kidx][:, :, [3]]), ref[nm])
        print(f"model46k det {nm} rows: max abs {e:.2e} rel L2 {r:.2e}")
