"""The device-timeout path without a fault: a bounded wait on an mbarrier
that nothing arrives at gives up after its poll limit, records a status code
that the host reads as MAGI_BCA_DEVICE_TIMEOUT, and leaves the CUDA context
usable (the next forward runs and matches the oracle)."""
import pytest
import torch

import block_causal_attention_gqa_b200 as bca
import workloads
from oracle import bca_oracle as orc
from tests._helpers import assert_close, to_np
from tests.test_fwd_parity import SMALL

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_a_timeout_and_the_context_survives():
    assert bca.magi_bca_last_device_status() == 0          # (reading clears any earlier word)
    bca.magi_bca_selftest_wait_timeout()
    torch.cuda.synchronize()
    assert bca.magi_bca_last_device_status() == -6          # MAGI_BCA_DEVICE_TIMEOUT
    assert bca.magi_bca_last_device_status() == 0          # read once, then cleared
    w = SMALL["tiny"]
    inp = workloads.make_inputs(w, with_grad_out=False)
    dev = "cuda"
    out, lse = bca.magi_bca_fwd(inp["q"].to(dev), inp["k"].to(dev), inp["v"].to(dev), w.q_offsets, w.kv_offsets,
                                inp["gamma_q"].to(dev), inp["gamma_k"].to(dev))
    torch.cuda.synchronize()
    assert bca.magi_bca_last_device_status() == 0
    o_ref, _ = orc.forward(inp["q"], inp["k"], inp["v"], w.q_offsets, w.kv_offsets, inp["gamma_q"], inp["gamma_k"])
    assert_close("forward after the timeout", to_np(out), o_ref)
