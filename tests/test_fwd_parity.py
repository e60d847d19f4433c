"""GPU parity of the forward against the fp64 oracle (through the C ABI).

Small workloads are compared on every row; the model-scale, streaming and
long-context workloads at full size (the launch bench.py times) on 4096
stratified query rows per head.  Tolerance: max abs 1e-2 and relative L2
5e-3 for bf16 inputs with fp32 accumulation."""
import numpy as np
import pytest
import torch

import block_causal_attention_gqa_b200 as bca
import workloads
from oracle import bca_oracle as orc
from tests._helpers import assert_close, assert_lse_close, grad_bound, to_np, rel_l2

pytestmark = pytest.mark.gpu


def run_gpu(inp, w, lse=True):
    dev = "cuda"
    q, k, v = inp["q"].to(dev), inp["k"].to(dev), inp["v"].to(dev)
    out, l = bca.magi_bca_fwd(q, k, v, w.q_offsets, w.kv_offsets, inp["gamma_q"].to(dev),
                              inp["gamma_k"].to(dev), want_lse=lse, **w.mask_kw)
    torch.cuda.synchronize()
    assert bca.magi_bca_last_device_status() == 0
    return out, l


SMALL = {
    "tiny": workloads.workload("tiny"),
    "train4k": workloads.workload("train4k"),
    "ragged_d128": workloads.custom("ragged_d128", 2, [100, 333, 1000, 67], None, 4, 2, 128, seed=11),
    "ragged_d64_gqa3": workloads.custom("ragged_d64_gqa3", 1, [70, 130, 200], None, 6, 2, 64, seed=12),
    "stream_small": workloads.custom("stream_small", 2, [150, 250], [300, 200, 150, 250], 8, 2, 128, seed=13),
    "single_chunk_mha": workloads.custom("single_chunk_mha", 1, [777], None, 2, 2, 128, seed=14),
    "token_causal": workloads.custom("token_causal", 1, [1] * 37, None, 2, 1, 64, seed=15),
    "many_chunks": workloads.custom("many_chunks", 1, [50] * 20, None, 4, 1, 128, seed=16),
    "gqa8_long_rows": workloads.custom("gqa8_long_rows", 1, [640] * 3, None, 16, 2, 128, seed=17,
                                       token_scale=True),
    # KV range (MAGI-1 §2.4.4, Fig. 12): each chunk sees itself and the R - 1 chunks before it
    "window_r1_ragged": workloads.custom("window_r1_ragged", 2, [100, 333, 200, 67], None, 4, 2, 128, seed=21,
                                         kv_range=1),
    "window_r2_ragged": workloads.custom("window_r2_ragged", 1, [300, 200, 150, 250, 100], None, 8, 2, 128,
                                         seed=22, kv_range=2),
    "window_stream_r3_d64": workloads.custom("window_stream_r3_d64", 2, [150, 250], [300, 200, 150, 250], 8, 2, 64,
                                             seed=23, kv_range=3),
    "window_token_r5": workloads.custom("window_token_r5", 1, [1] * 37, None, 2, 1, 64, seed=24, kv_range=5),
    "window_aligned_r3": workloads.custom("window_aligned_r3", 1, [256] * 8, None, 4, 1, 128, seed=25,
                                          kv_range=3),
    # cross-attention (MAGI-1 §2.2.2 text K/V; §7 chunk-wise text conditioning)
    "xattn_video_text": workloads.custom("xattn_video_text", 2, [1000], [333], 8, 2, 128, seed=26),
    "xattn_short_q_d64": workloads.custom("xattn_short_q_d64", 1, [77], [1000], 4, 2, 64, seed=27),
    "xattn_chunkwise": workloads.custom("xattn_chunkwise", 1, [300, 200, 250], [77, 120, 64], 8, 2, 128,
                                        seed=28, kv_range=1),
    # packed samples (MAGI-1 §4.1.2, Figure 15 (f)) and a last global block (Figure 15 (g))
    "packed_ragged": workloads.custom("packed_ragged", 2, [100, 333, 250, 67, 400, 190], None, 4, 2, 128, seed=51,
                                      samples=[0, 2, 3, 6]),
    "packed_global_ragged": workloads.custom("packed_global_ragged", 2, [100, 333, 250, 67, 400, 190], None, 4, 2,
                                             128, seed=52, samples=[0, 2, 3, 6], n_global=1),
    "packed_global_r2_d64": workloads.custom("packed_global_r2_d64", 1, [256, 256, 256, 130, 126, 256, 256], None,
                                             8, 2, 64, seed=53, samples=[0, 3, 5, 7], n_global=1, kv_range=2),
    "packed_stream_global": workloads.custom("packed_stream_global", 2, [150, 250], [300, 200, 150, 250], 8, 2, 128,
                                             seed=54, samples=[0, 1, 4], n_global=1),
    "packed_global_gqa8": workloads.custom("packed_global_gqa8", 1, [640, 320, 640], None, 16, 2, 128, seed=55,
                                           samples=[0, 1, 3], n_global=1),
}


@pytest.mark.parametrize("name", list(SMALL))
def test_forward_all_rows(name):
    w = SMALL[name]
    inp = workloads.make_inputs(w, with_grad_out=False)
    out, lse = run_gpu(inp, w)
    o_ref, l_ref = orc.forward(inp["q"], inp["k"], inp["v"], w.q_offsets, w.kv_offsets,
                               inp["gamma_q"], inp["gamma_k"], **w.mask_kw)
    e, r = assert_close(f"{name} out", to_np(out), o_ref)
    el, rl = assert_lse_close(f"{name} lse", to_np(lse), l_ref)
    print(f"{name}: out max abs {e:.2e} rel L2 {r:.2e}; lse max abs {el:.2e} rel L2 {rl:.2e}")
    if "q_f32" in inp:
        # information only: error against the unrounded fp32 inputs
        o32, _ = orc.forward(inp["q_f32"], inp["k_f32"], inp["v_f32"], w.q_offsets, w.kv_offsets,
                             inp["gamma_q"], inp["gamma_k"], **w.mask_kw)
        print(f"{name}: rel L2 vs unrounded fp32 inputs {rel_l2(to_np(out), o32):.3e}")


def test_forward_without_lse_and_canary():
    w = SMALL["ragged_d128"]
    inp = workloads.make_inputs(w, with_grad_out=False)
    dev = "cuda"
    q, k, v = inp["q"].to(dev), inp["k"].to(dev), inp["v"].to(dev)
    n = q.numel()
    big = torch.full((n + 4096,), 7.0, device=dev, dtype=torch.bfloat16)
    out = big[:n].view(q.shape)
    bca.magi_bca_fwd(q, k, v, w.q_offsets, w.kv_offsets, inp["gamma_q"].to(dev), inp["gamma_k"].to(dev),
                     out=out, want_lse=False)
    torch.cuda.synchronize()
    assert (big[n:] == 7.0).all(), "write past the end of out"
    o_ref, _ = orc.forward(inp["q"], inp["k"], inp["v"], w.q_offsets, w.kv_offsets,
                           inp["gamma_q"], inp["gamma_k"])
    assert_close("no-lse out", to_np(out), o_ref)


def test_forward_is_deterministic():
    w = SMALL["train4k"]
    inp = workloads.make_inputs(w, with_grad_out=False)
    o1, l1 = run_gpu(inp, w)
    o2, l2 = run_gpu(inp, w)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


LARGE = ["model46k", "stream4of16", "long262k", "window262k", "xattn46k", "packed46k"]


@pytest.mark.parametrize("name", LARGE)
def test_forward_full_size_sampled_rows(name):
    w = workloads.workload(name)
    inp = workloads.make_inputs(w, with_grad_out=False)
    out, lse = run_gpu(inp, w)
    out_c, lse_c = out.cpu(), lse.cpu()
    del out, lse
    torch.cuda.empty_cache()
    # 4096 rows per head, spread over the batch elements
    per_batch = 4096 // w.batch
    for b in range(w.batch):
        rows = workloads.sample_rows(w.seqlen_q, w.q_offsets, per_batch, seed=100 + b)
        o_ref, l_ref = orc.forward_rows(inp["q"], inp["k"], inp["v"], w.q_offsets, w.kv_offsets,
                                        inp["gamma_q"], inp["gamma_k"], rows, batches=[b], **w.mask_kw)
        idx = torch.as_tensor(rows)
        e, r = assert_close(f"{name} out b{b}", to_np(out_c[b:b + 1, idx]), o_ref)
        el, rl = assert_lse_close(f"{name} lse b{b}", to_np(lse_c[b:b + 1][:, :, idx]), l_ref)
        print(f"{name} b{b}: out max abs {e:.2e} rel L2 {r:.2e}; lse max abs {el:.2e} rel L2 {rl:.2e}")
