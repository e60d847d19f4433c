"""GPU parity of the backward against the fp64 oracle (through the C ABI).

Small workloads: dq, dk, dv, dgamma_q, dgamma_k on every row.  Full-size
training workloads: dq on 4096 stratified query rows per head, dk/dv on
sampled keys of the last chunk (exact and cheap: only last-chunk queries see
them) where the oracle finishes in seconds, and everywhere the identities
that hold at any size: sum_j dV_j = sum over the group of sum_i dO_i (rows of
P sum to 1) and dq.q = dk.k = 0 up to eps (RMSNorm is scale invariant).
The backward consumes the GPU forward's out and lse, as a training step does;
the oracle recomputes everything from q, k, v, dO."""
import numpy as np
import pytest
import torch

import block_causal_attention_gqa_b200 as bca
import workloads
from oracle import bca_oracle as orc
from tests._helpers import assert_close, dgamma_bound, grad_bound, rel_l2, to_np
from tests.test_fwd_parity import SMALL

pytestmark = pytest.mark.gpu

BWD_SMALL = ["train4k", "ragged_d128", "ragged_d64_gqa3", "stream_small", "single_chunk_mha", "token_causal",
             "many_chunks", "gqa8_long_rows", "tiny", "window_r1_ragged", "window_r2_ragged",
             "window_stream_r3_d64", "window_token_r5", "window_aligned_r3", "xattn_video_text",
             "xattn_short_q_d64", "xattn_chunkwise", "packed_ragged", "packed_global_ragged", "packed_global_r2_d64",
             "packed_stream_global", "packed_global_gqa8"]
# Every case uses the stated bound (max abs 1e-2, rel L2 5e-3) unless
# tests/_helpers.GRAD_MAX_ABS names it with the figure that justifies more.


def gpu_fwd_bwd(inp, w):
    dev = "cuda"
    q, k, v = inp["q"].to(dev), inp["k"].to(dev), inp["v"].to(dev)
    gq, gk = inp["gamma_q"].to(dev), inp["gamma_k"].to(dev)
    dout = inp["dout"].to(dev)
    out, lse = bca.magi_bca_fwd(q, k, v, w.q_offsets, w.kv_offsets, gq, gk, **w.mask_kw)
    dq, dk, dv, dgq, dgk = bca.magi_bca_bwd(q, k, v, out, dout, lse, w.q_offsets, w.kv_offsets, gq, gk,
                                            **w.mask_kw)
    torch.cuda.synchronize()
    assert bca.magi_bca_last_device_status() == 0
    return dq, dk, dv, dgq, dgk


@pytest.mark.parametrize("name", BWD_SMALL)
def test_backward_all_rows(name):
    w = SMALL[name]
    inp = workloads.make_inputs(w, with_grad_out=True)
    dq, dk, dv, dgq, dgk = gpu_fwd_bwd(inp, w)
    ref = orc.backward(inp["q"], inp["k"], inp["v"], inp["dout"], w.q_offsets, w.kv_offsets,
                       inp["gamma_q"], inp["gamma_k"], **w.mask_kw)
    bound = grad_bound(name)
    for nm, got in (("dq", dq), ("dk", dk), ("dv", dv)):
        e, r = assert_close(f"{name} {nm}", to_np(got), ref[nm], max_abs=bound)
        print(f"{name} {nm}: max abs {e:.2e} rel L2 {r:.2e}")
    # dgamma sums B*S*H terms; its scale grows with S, so only the relative L2 applies
    for nm, got in (("dgamma_q", dgq), ("dgamma_k", dgk)):
        r = rel_l2(to_np(got), ref[nm])
        print(f"{name} {nm}: rel L2 {r:.2e}")
        assert r <= dgamma_bound(name), f"{name} {nm}: rel L2 {r:.3e}"


def test_backward_workspace_and_no_dgamma():
    w = SMALL["ragged_d128"]
    inp = workloads.make_inputs(w, with_grad_out=True)
    dev = "cuda"
    q, k, v = inp["q"].to(dev), inp["k"].to(dev), inp["v"].to(dev)
    gq, gk = inp["gamma_q"].to(dev), inp["gamma_k"].to(dev)
    dout = inp["dout"].to(dev)
    out, lse = bca.magi_bca_fwd(q, k, v, w.q_offsets, w.kv_offsets, gq, gk)
    dims = bca.make_dims(w.batch, w.seqlen_q, w.seqlen_kv, w.heads_q, w.heads_kv, w.head_dim,
                         len(w.q_chunks), len(w.kv_chunks))
    need = bca.magi_bca_bwd_workspace_size(dims)
    small = torch.empty(need - 256, device=dev, dtype=torch.uint8)
    with pytest.raises(bca.MagiBcaError) as ei:
        bca.magi_bca_bwd(q, k, v, out, dout, lse, w.q_offsets, w.kv_offsets, gq, gk, workspace=small)
    assert ei.value.status == -4
    ws = torch.full((need,), 0xAB, device=dev, dtype=torch.uint8)   # stale contents must not matter
    dq, dk, dv, a, b = bca.magi_bca_bwd(q, k, v, out, dout, lse, w.q_offsets, w.kv_offsets, gq, gk,
                                        workspace=ws, want_dgamma=False)
    torch.cuda.synchronize()
    assert a is None and b is None
    ref = orc.backward(inp["q"], inp["k"], inp["v"], inp["dout"], w.q_offsets, w.kv_offsets,
                       inp["gamma_q"], inp["gamma_k"])
    for nm, got in (("dq", dq), ("dk", dk), ("dv", dv)):
        assert_close(nm, to_np(got), ref[nm])


def identities(name, w, inp, dq, dk, dv):
    """Checks that hold at any size, on all rows."""
    g = w.heads_q // w.heads_kv
    do = inp["dout"].double()
    sum_dv = dv.double().cpu().sum(1)                                       # [B, Hkv, D]
    want = do.reshape(w.batch, w.seqlen_q, w.heads_kv, g, w.head_dim).sum((1, 3))
    r = rel_l2(sum_dv.numpy(), want.numpy())
    assert r <= 5e-3, f"{name}: sum_j dV != sum_i dO (rel {r:.2e})"
    for nm, grad, x in (("dq", dq, inp["q"]), ("dk", dk, inp["k"])):
        gx = grad.double().cpu()
        xx = x.double()
        cos = (gx * xx).sum(-1).abs() / (gx.norm(dim=-1) * xx.norm(dim=-1)).clamp_min(1e-30)
        assert float(cos.max()) <= 2e-2, f"{name}: {nm}.x not ~0 (max cos {float(cos.max()):.2e})"


def gamma_identity(name, inp, dgq, dgk):
    """gamma_q . dgamma_q = gamma_k . dgamma_k at any size: both equal
    sum_ij dS_ij S_ij, because scaling either gain by (1 + e) scales every
    logit by (1 + e).  Holds for the raw-gain gradients of the whole problem."""
    gq, gk = inp["gamma_q"].double(), inp["gamma_k"].double()
    a = float((gq * dgq.double().cpu()).sum())
    b = float((gk * dgk.double().cpu()).sum())
    scale = float(gq.norm() * dgq.double().cpu().norm() + gk.norm() * dgk.double().cpu().norm())
    assert abs(a - b) <= 2e-3 * scale, f"{name}: gamma_q.dgamma_q {a:.6e} vs gamma_k.dgamma_k {b:.6e}"
    print(f"{name}: gamma.dgamma identity {a:.4e} vs {b:.4e} (|diff| / scale {abs(a - b) / scale:.1e})")


# Full size: dq on 4096 sampled query rows; dk/dv exact on sampled keys of the
# last chunk (only the last chunk's queries see them, so the oracle needs one
# chunk of full rows) for the listed kv heads; the any-size identities; and
# dgamma through the gamma identity (an exact dgamma needs the full fp64
# backward: 37 TFLOP on model46k, 726 on long262k).
# packed46k: keys of chunk 6, the last chunk of its sample (the last chunk is the
# global block, whose keys every query sees)
@pytest.mark.parametrize("name,kv_heads,n_keys,key_chunk", [("model46k", [0, 5], 256, -1), ("long262k", [0], 64, -1),
                                                            ("window262k", [0, 1], 256, -1),
                                                            ("xattn46k", [0, 7], 256, -1),
                                                            ("packed46k", [2], 128, 6)])
def test_backward_full_size_sampled(name, kv_heads, n_keys, key_chunk):
    w = workloads.workload(name)
    inp = workloads.make_inputs(w, with_grad_out=True)
    dq, dk, dv, dgq, dgk = gpu_fwd_bwd(inp, w)
    dq, dk, dv = dq.cpu(), dk.cpu(), dv.cpu()
    torch.cuda.empty_cache()
    identities(name, w, inp, dq, dk, dv)
    gamma_identity(name, inp, dgq, dgk)
    rows = workloads.sample_rows(w.seqlen_q, w.q_offsets, 4096, seed=200)
    ref = orc.backward_rows(inp["q"], inp["k"], inp["v"], inp["dout"], w.q_offsets, w.kv_offsets,
                            inp["gamma_q"], inp["gamma_k"], q_rows=rows, **w.mask_kw)
    idx = torch.as_tensor(rows)
    e, r = assert_close(f"{name} dq rows", to_np(dq[:, idx]), ref["dq"])
    print(f"{name} dq rows: max abs {e:.2e} rel L2 {r:.2e}")
    if kv_heads:
        kc = key_chunk % len(w.kv_chunks)
        k_lo, k_hi = int(w.kv_offsets[kc]), int(w.kv_offsets[kc + 1])
        kr = np.sort(np.random.default_rng(201).choice(np.arange(k_lo, k_hi), n_keys, replace=False))
        ref = orc.backward_rows(inp["q"], inp["k"], inp["v"], inp["dout"], w.q_offsets, w.kv_offsets,
                                inp["gamma_q"], inp["gamma_k"], kv_rows=kr, kv_heads=kv_heads, **w.mask_kw)
        kidx = torch.as_tensor(kr)
        for nm, got in (("dk", dk), ("dv", dv)):
            e, r = assert_close(f"{name} {nm} rows", to_np(got[:, kidx][:, :, kv_heads]), ref[nm])
            print(f"{name} {nm} rows: max abs {e:.2e} rel L2 {r:.2e}")


def test_backward_canaries_and_finite_outputs():
    """Every output of the backward inside a larger buffer filled with a canary:
    nothing is written past (or before) the gradients, and every gradient is
    finite, for the default and the deterministic path."""
    w = SMALL["ragged_d64_gqa3"]
    inp = workloads.make_inputs(w, with_grad_out=True)
    dev = "cuda"
    q, k, v = inp["q"].to(dev), inp["k"].to(dev), inp["v"].to(dev)
    gq, gk = inp["gamma_q"].to(dev), inp["gamma_k"].to(dev)
    dout = inp["dout"].to(dev)
    out, lse = bca.magi_bca_fwd(q, k, v, w.q_offsets, w.kv_offsets, gq, gk)
    pad = 4096

    def padded(like, value):
        big = torch.full((pad + like.numel() + pad,), value, device=dev, dtype=like.dtype)
        return big, big[pad:pad + like.numel()].view(like.shape)

    ref = orc.backward(inp["q"], inp["k"], inp["v"], inp["dout"], w.q_offsets, w.kv_offsets,
                       inp["gamma_q"], inp["gamma_k"])
    for det in (False, True):
        bq, dq = padded(q, 7.0)
        bk, dk = padded(k, 7.0)
        bv, dv = padded(v, 7.0)
        bgq, dgq = padded(gq, 7.0)
        bgk, dgk = padded(gk, 7.0)
        bca.magi_bca_bwd(q, k, v, out, dout, lse, w.q_offsets, w.kv_offsets, gq, gk, dq=dq, dk=dk, dv=dv,
                         dgamma_q=dgq, dgamma_k=dgk, deterministic=det)
        torch.cuda.synchronize()
        assert bca.magi_bca_last_device_status() == 0
        for nm, big, t in (("dq", bq, dq), ("dk", bk, dk), ("dv", bv, dv), ("dgamma_q", bgq, dgq),
                           ("dgamma_k", bgk, dgk)):
            assert (big[:pad] == 7.0).all() and (big[pad + t.numel():] == 7.0).all(), f"{nm}: canary overwritten"
            assert torch.isfinite(t).all(), f"{nm}: non-finite values (deterministic={det})"
        for nm, got in (("dq", dq), ("dk", dk), ("dv", dv)):
            assert_close(f"canary {nm} det={det}", to_np(got), ref[nm], max_abs=grad_bound("ragged_d64_gqa3"))
