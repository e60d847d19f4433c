"""CPU model of the kernels' rounding points (test infrastructure).

Reproduces, in float64 arithmetic with explicit bf16 roundings, what the CUDA
forward and backward round and where:

forward   q^ = bf16(q r_q gamma_q gamma_k scale log2 e); k^ = bf16(k r_k); logits
          x = q^ . k^ (log2 units); P = exp2(x - m); O = sum bf16(P) v / sum P
          -> bf16; lse = m + log2(sum P).
backward  P = exp2(x - lse) from the same operands; Delta = rowsum(dO * bf16(O));
          dS = P (dP - Delta); dV = bf16(P)^T dO; gamma_k dk~ and dq~ from bf16(dS)
          with the folded query operand and k^; RMSNorm Jacobians in float64;
          outputs rounded to bf16.

It is used to tell bf16-operand error from defects: when the GPU result equals
this model's to two digits, a tolerance miss is a property of bf16 operands.
(Accumulation inside the tensor cores is modelled as exact.)"""
import numpy as np
import torch

from oracle import bca_oracle as orc


def _bf(x):
    return x.to(torch.bfloat16).to(torch.float64)


def _rot(x, t):
    """Rotary pairs (i, i + D/2) by the per-token angles t [S, D/2] (exact)."""
    if t is None:
        return x
    h = x.shape[-1] // 2
    c, s = torch.cos(t)[None, :, None, :], torch.sin(t)[None, :, None, :]
    a, b = x[..., :h], x[..., h:]
    return torch.cat([a * c - b * s, b * c + a * s], dim=-1)


def model_fwd_bwd(inp, q_offsets, kv_offsets, eps=1e-6, kv_range=0, rope_q=None, rope_k=None, samples=None,
                  n_global=0):
    q = inp["q"].double()
    k = inp["k"].double()
    v = inp["v"].double()
    do = inp["dout"].double()
    gq = inp["gamma_q"].double()
    gk = inp["gamma_k"].double()
    B, Sq, Hq, D = q.shape
    Hkv = k.shape[2]
    g = Hq // Hkv
    sc = 1.0 / np.sqrt(D)
    l2e = 1.0 / np.log(2.0)
    rq = torch.rsqrt((q * q).mean(-1, keepdim=True) + eps)
    rk = torch.rsqrt((k * k).mean(-1, keepdim=True) + eps)
    tq = None if rope_q is None else torch.as_tensor(rope_q).double()
    tk = None if rope_k is None else torch.as_tensor(rope_k).double()
    q_raw, k_raw = q, k
    q, k = _rot(q, tq), _rot(k, tk)          # a rotation keeps the RMS of the raw row
    mask = torch.tensor(orc.block_causal_mask(q_offsets, kv_offsets, kv_range=kv_range, samples=samples,
                                              n_global=n_global))
    kr, vr = k.repeat_interleave(g, 2), v.repeat_interleave(g, 2)
    kh = _bf(kr * rk.repeat_interleave(g, 2))
    qh = _bf(q * rq * (gq * gk * sc * l2e))
    x = torch.einsum("bihd,bjhd->bhij", qh, kh)
    x = x.masked_fill(~mask, -np.inf)
    m = x.amax(-1, keepdim=True)
    p = torch.exp2(x - m)
    l = p.sum(-1, keepdim=True)
    out = torch.einsum("bhij,bjhd->bihd", _bf(p), vr) / l.permute(0, 2, 1, 3)
    lse2 = m + torch.log2(l)
    out_bf = _bf(out)
    pb = torch.exp2(x - lse2)
    dp = torch.einsum("bihd,bjhd->bhij", do, vr)
    delta = (do * out_bf).sum(-1).permute(0, 2, 1)[..., None]
    ds = _bf(pb * (dp - delta))
    dv = torch.einsum("bhij,bihd->bjhd", _bf(pb), do).view(B, -1, Hkv, g, D).sum(3)
    q_op = qh / (gk * sc * l2e)                      # what the folded operand represents
    dkt = sc * torch.einsum("bhij,bihd->bjhd", ds, q_op).view(B, -1, Hkv, g, D).sum(3)
    dqt = sc * torch.einsum("bhij,bjhd->bihd", ds, kh * gk)
    dq, dgq = orc.rms_norm_backward(q.numpy(), gq.numpy(), dqt.numpy(), eps)
    dk, dgk = orc.rms_norm_backward(k.numpy(), gk.numpy(), dkt.numpy(), eps)
    dq, _ = orc.rope_backward(q_raw.numpy(), rope_q, dq)
    dk, _ = orc.rope_backward(k_raw.numpy(), rope_k, dk)
    return dict(out=out_bf.numpy(), lse=(lse2 / l2e).squeeze(-1).numpy(), dq=_bf(torch.tensor(dq)).numpy(),
                dk=_bf(torch.tensor(dk)).numpy(), dv=_bf(dv).numpy(), dgamma_q=dgq, dgamma_k=dgk)
