"""bench.py's FLOP and byte accounting, which every reported TFLOP/s divides
into: useful forward FLOPs = 4 D B Hq x (visible query-key pairs), the
backward 2.5 times that (MAGI-1 App. B.2.1), checked against a brute-force
count of the oracle's token mask and against closed forms of the named
workloads."""
import numpy as np
import pytest

import bench
import workloads
from oracle import bca_oracle as orc


def pairs_from_mask(w):
    return int(orc.block_causal_mask(w.q_offsets, w.kv_offsets, **w.mask_kw).sum())


@pytest.mark.parametrize("w", [
    workloads.workload("tiny"),
    workloads.workload("train4k"),
    workloads.custom("ragged", 2, [100, 333, 1000, 67], None, 4, 2, 128, seed=0),
    workloads.custom("stream", 2, [150, 250], [300, 200, 150, 250], 8, 2, 64, seed=0),
    workloads.custom("window", 1, [300, 200, 150, 250, 100], None, 8, 2, 128, seed=0, kv_range=2),
    workloads.custom("xattn", 1, [777], [64], 4, 1, 128, seed=0),
    workloads.custom("chunkwise_text", 1, [300, 200, 250], [77, 120, 64], 4, 2, 64, seed=0, kv_range=1),
    workloads.custom("packed", 1, [100, 333, 250, 67, 400, 190], None, 4, 2, 128, seed=0, samples=[0, 2, 3, 6]),
    workloads.custom("packed_global_r2", 1, [100, 333, 250, 67, 400, 190], None, 4, 2, 128, seed=0,
                     samples=[0, 2, 3, 6], n_global=1, kv_range=2),
    workloads.custom("packed_stream_global", 2, [150, 250], [300, 200, 150, 250], 8, 2, 64, seed=0,
                     samples=[0, 1, 4], n_global=1),
], ids=lambda w: w.name)
def test_forward_flops_count_the_visible_pairs(w):
    want = 4.0 * w.head_dim * w.batch * w.heads_q * pairs_from_mask(w)
    assert bench.fwd_flops(w) == want
    assert bench.bwd_flops(w) == 2.5 * want


def equal_chunks_pairs(L, n_q, n_kv):
    """Pairs seen by n_q equal query chunks of L tokens that are the last n_q of
    n_kv equal kv chunks: chunk c (from 0) sees n_kv - n_q + c + 1 chunks."""
    return L * L * sum(n_kv - n_q + c + 1 for c in range(n_q))


@pytest.mark.parametrize("name,L,n_q,n_kv,tflop", [
    ("tiny", 64, 2, 2, 6.29e-6),
    ("train4k", 1024, 4, 4, 0.0859),
    ("model46k", 5760, 8, 8, 14.68),
    ("stream4of16", 5760, 4, 16, 47.29),
    ("long262k", 8192, 32, 32, 290.3),
])
def test_forward_flops_of_the_named_workloads(name, L, n_q, n_kv, tflop):
    w = workloads.workload(name)
    closed = 4.0 * w.head_dim * w.batch * w.heads_q * equal_chunks_pairs(L, n_q, n_kv)
    assert bench.fwd_flops(w) == closed
    assert abs(closed / 1e12 - tflop) <= 5e-4 * tflop + 1e-9


def test_kv_range_on_equal_chunks():
    """window262k: 32 chunks of 8192, each sees itself and up to 7 chunks before."""
    w = workloads.workload("window262k")
    chunks = sum(min(c + 1, 8) for c in range(32))
    assert bench.fwd_flops(w) == 4.0 * 128 * 1 * 16 * 8192 * 8192 * chunks


def test_forward_bytes():
    w = workloads.workload("model46k")
    q = 46080 * 24 * 128 * 2
    kv = 2 * 46080 * 8 * 128 * 2
    assert bench.fwd_bytes(w) == q + kv + q + 24 * 46080 * 4
    assert abs(bench.fwd_bytes(w) / 1e9 - 0.759) < 1e-3


def test_backward_main_bytes():
    """The backward main kernel's algorithmic bytes: Q^, dO and the 16-byte
    {-lse, -Delta} rows read once, K^ and V read once, and the fp32 dq, dV and
    G_k accumulators read and written once."""
    w = workloads.workload("model46k")
    rows_q, rows_k, D = 46080 * 24, 46080 * 8, 128
    pad = -(-46080 // 128) * 128
    want = (2 * rows_q * D * 2 + 24 * pad * 16 + 2 * rows_k * D * 2
            + 2 * (rows_q * D * 4) + 2 * 2 * (rows_k * D * 4))
    assert bench.bwd_main_bytes(w) == want


def test_traffic_records_are_complete():
    """Every DRAM-traffic record that bench.py may quote names its kernel
    sources, the ncu command and where the figure comes from; a figure scaled
    from a smaller capture says so."""
    import json
    import os
    d = json.load(open(os.path.join(os.path.dirname(bench.__file__), "profiles", "ncu_traffic.json")))
    assert d
    for kernel, per_w in d.items():
        assert kernel in ("bca_fwd_kernel", "bca_bwd_main_kernel")
        for name, e in per_w.items():
            assert name in workloads.WORKLOADS, name
            assert e["dram_bytes_per_launch"] == e["dram_bytes_read"] + e["dram_bytes_write"]
            assert len(e["kernel_source_sha"]) == 16 and e["command"].startswith("ncu ")
            assert "--clock-control none" in e["command"]
            assert e["source"]
            if "long65k" in e["command"] and name != "long65k":
                assert "scaled" in e["source"]
