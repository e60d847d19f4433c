"""The diagnostic timing hook records its events around the main kernels."""
import pytest
import torch

import block_causal_attention_gqa_b200 as bca
import workloads


@pytest.mark.gpu
def test_profile_events_time_the_main_kernels():
    w = workloads.workload("tiny")
    inp = workloads.make_inputs(w, device="cuda", with_grad_out=True)
    b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    bca.magi_bca_profile_events(b0, b1)
    try:
        out, lse = bca.magi_bca_fwd(inp["q"], inp["k"], inp["v"], w.q_offsets, w.kv_offsets,
                                    inp["gamma_q"], inp["gamma_k"])
        bca.magi_bca_profile_events(c0, c1)
        bca.magi_bca_bwd(inp["q"], inp["k"], inp["v"], out, inp["dout"], lse, w.q_offsets, w.kv_offsets,
                         inp["gamma_q"], inp["gamma_k"])
    finally:
        bca.magi_bca_profile_events()
    torch.cuda.synchronize()
    fwd_ms, bwd_ms = b0.elapsed_time(b1), c0.elapsed_time(c1)
    assert 0.0 < fwd_ms < 1000.0 and 0.0 < bwd_ms < 1000.0
    # cleared: a further call records nothing new
    t = b1.elapsed_time(c0)
    bca.magi_bca_fwd(inp["q"], inp["k"], inp["v"], w.q_offsets, w.kv_offsets, inp["gamma_q"], inp["gamma_k"])
    torch.cuda.synchronize()
    assert b1.elapsed_time(c0) == t
