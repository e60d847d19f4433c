"""The entry points inside CUDA graph capture: a forward + backward step
captured once (after a warm-up call that builds the schedules and the
forward's key buffer) and replayed gives the same results as the eager calls,
for the default and the deterministic backward.  Replaying a captured step
removes the per-call host work (argument checks, schedule lookup, launch
setup) from a training loop."""
import pytest
import torch

import block_causal_attention_gqa_b200 as bca
import workloads
from tests.test_fwd_parity import SMALL

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("det", [False, True])
def test_captured_step_replays_the_eager_results(det):
    w = SMALL["train4k"]
    inp = workloads.make_inputs(w, with_grad_out=True)
    dev = "cuda"
    q, k, v = inp["q"].to(dev), inp["k"].to(dev), inp["v"].to(dev)
    gq, gk = inp["gamma_q"].to(dev), inp["gamma_k"].to(dev)
    dout = inp["dout"].to(dev)
    dims = bca.make_dims(w.batch, w.seqlen_q, w.seqlen_kv, w.heads_q, w.heads_kv, w.head_dim,
                         len(w.q_chunks), len(w.kv_chunks), deterministic=det)
    ws = torch.empty(bca.magi_bca_bwd_workspace_size(dims), device=dev, dtype=torch.uint8)
    out, lse = torch.empty_like(q), torch.empty(w.batch, w.heads_q, w.seqlen_q, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dgq, dgk = torch.empty(w.head_dim, device=dev), torch.empty(w.head_dim, device=dev)
    stream = torch.cuda.Stream()

    def step():
        bca.magi_bca_fwd(q, k, v, w.q_offsets, w.kv_offsets, gq, gk, out=out, lse=lse, stream=stream)
        bca.magi_bca_bwd(q, k, v, out, dout, lse, w.q_offsets, w.kv_offsets, gq, gk, dq=dq, dk=dk, dv=dv,
                         dgamma_q=dgq, dgamma_k=dgk, workspace=ws, stream=stream, deterministic=det)

    with torch.cuda.stream(stream):
        step()                        # eager: builds and caches the schedules and the key buffer
    torch.cuda.synchronize()
    assert bca.magi_bca_last_device_status() == 0
    eager = [t.clone() for t in (out, lse, dq, dk, dv, dgq, dgk)]
    for t in (out, lse, dq, dk, dv, dgq, dgk):
        t.zero_()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        step()
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    assert bca.magi_bca_last_device_status() == 0
    names = ("out", "lse", "dq", "dk", "dv", "dgamma_q", "dgamma_k")
    for nm, a, b in zip(names, eager, (out, lse, dq, dk, dv, dgq, dgk)):
        if det or nm in ("out", "lse"):
            assert torch.equal(a, b), f"{nm}: replay differs from the eager call"
        else:   # the default backward's fp32 reductions run in a timing-dependent order
            r = float((a.double() - b.double()).norm() / b.double().norm().clamp_min(1e-30))
            assert r <= 1e-3, f"{nm}: replay vs eager rel L2 {r:.2e}"
    del graph
