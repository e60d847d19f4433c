"""fp64 CPU oracle for block-causal grouped-query attention with QK-RMSNorm.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import
this module.  It shares no code with the CUDA path and imports nothing from
it.

It is the plain definition of the operation, written out step by step in
float64 with an explicit per-token mask (no tiling, no online softmax, no
folding of scales):

1. QK-normalisation (MAGI-1 §2.2.2, "QK normalization"; MAGI-1 notes §3.2.2,
   "QK-Norm + GQA").  The norm is per-head RMSNorm with a learnable gain:
   ``rmsnorm(x) = x / sqrt(mean_d x^2 + eps) * gamma``.  The notes' DiT block
   sketch writes ``l2_normalize``; this oracle takes the RMS reading (the two
   differ by sqrt(D) in the logit scale), and ``eps`` is a parameter with
   default 1e-6.
2. Grouped-query attention (MAGI-1 §2.2.2; notes §3.2.2 model table,
   "128 heads (8 groups)"): query head ``h`` reads key/value head
   ``h // (Hq // Hkv)`` (contiguous groups).
3. Block-causal mask (MAGI-1 §2, Fig. 1; notes §2 and Fig. 1: full attention
   inside a chunk, causal attention between chunks).  Query token i of
   query chunk c may see key token j iff j's kv chunk index is at most
   ``n_kv - n_q + c``: the query chunks are the last ``n_q`` chunks of the
   key/value sequence (streaming layout: active chunks after the cached clean
   chunks, MAGI-1 §2 and §2.4.4; identity when n_q == n_kv).
   Optional KV range R (MAGI-1 §2.4.4 and §2.6, Fig. 12: "restricting the KV
   range to preceding content"; KV range 1 means no access to earlier video
   content): with R > 0 the kv chunk index must also be at least
   ``n_kv - n_q + c - R + 1``, so a chunk sees itself and the R - 1 chunks
   before it; R = 0 means no limit.
4. Softmax attention with scale ``1/sqrt(D)`` (a reading: the pages give no
   scale), ``O = softmax(scale * q~ k~^T + mask) v``; the log-sum-exp
   ``lse = ln sum_j exp(scale * q~_i . k~_j)`` over unmasked j, natural log, in
   units of the scaled logits.
5. Backward (training layout; FLOP convention of MAGI-1 App. B.2.1: the
   backward recomputes the forward), analytic in float64: dV = P^T dO,
   dP = dO V^T, Delta = rowsum(dO * O), dS = P * (dP - Delta),
   dq~ = scale dS k~, dk~ = scale dS^T q~, summed over each query-head group
   for k and v, then the RMSNorm Jacobian back to the raw q and k, and the
   gain gradients dgamma = sum over (batch, token, head) of dx~ * x_hat.
6. Optional packed samples and a last global block (MAGI-1 §4.1.2 and
   Figure 15 (f), (g); App. B.1, Figure 23): several samples packed into one sequence
   attend only within themselves, and the last kv chunks may form a global
   block that every query sees and whose queries see every key (see
   ``block_causal_mask``).
7. Optional rotary position embedding before the norm (MAGI-1 §2.2.2 and the
   notes' DiT-block sketch: learnable 3D RoPE applied to q and k, then
   QK-norm).  The pages give no formula; the reading here: per token an angle
   for each of the D/2 feature pairs (i, i + D/2), shared by all heads and
   batch elements (the 3D split and the learnable frequencies produce these
   angles outside the attention), ``y_i = x_i cos t - x_{i+D/2} sin t``,
   ``y_{i+D/2} = x_{i+D/2} cos t + x_i sin t``.  The backward returns the
   angle gradients as well, summed over batch and heads.

Every function below is pinned by ``tests/test_oracle_pins.py`` against
brute force, a library routine or an invariant; none is "parity unpinned".
"""
from __future__ import annotations

import numpy as np

__all__ = ["rms_norm", "rms_norm_backward", "chunk_of", "matched_kv_chunk",
           "block_causal_mask", "forward", "forward_rows", "backward", "backward_rows",
           "rope", "rope_backward", "DEFAULT_EPS"]

DEFAULT_EPS = 1e-6


def _f64(x):
    """Any array-like (numpy or torch, any float dtype) -> float64 ndarray."""
    if hasattr(x, "detach"):
        x = x.detach().cpu()
        if str(x.dtype) == "torch.bfloat16":
            x = x.float()
        x = x.numpy()
    return np.asarray(x, dtype=np.float64)


def rope(x, angles):
    """Rotary embedding over the last axis of x [..., S, H, D]: feature pair
    (i, i + D/2) of token s rotates by angles[s, i] (angles [S, D/2])."""
    x = _f64(x)
    if angles is None:
        return x
    t = _f64(angles)
    h = x.shape[-1] // 2
    c, s = np.cos(t)[:, None, :], np.sin(t)[:, None, :]
    a, b = x[..., :h], x[..., h:]
    return np.concatenate([a * c - b * s, b * c + a * s], axis=-1)


def rope_backward(x, angles, dy):
    """Gradients of y = rope(x, angles) given dy: (dx, dangles), dangles [S, D/2]
    summed over every leading axis and the heads."""
    x = _f64(x)
    dy = _f64(dy)
    if angles is None:
        return dy, None
    t = _f64(angles)
    h = x.shape[-1] // 2
    c, s = np.cos(t)[:, None, :], np.sin(t)[:, None, :]
    y = rope(x, angles)
    ga, gb = dy[..., :h], dy[..., h:]
    dx = np.concatenate([ga * c + gb * s, gb * c - ga * s], axis=-1)
    # dy_a/dt = -y_b, dy_b/dt = y_a
    dt = -ga * y[..., h:] + gb * y[..., :h]
    dt = dt.reshape((-1,) + dt.shape[-3:]).sum(axis=(0, 2))
    return dx, dt


def rms_norm(x, gamma, eps=DEFAULT_EPS):
    """RMSNorm over the last axis: x / sqrt(mean(x^2) + eps) * gamma."""
    x = _f64(x)
    g = _f64(gamma)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * g


def rms_norm_backward(x, gamma, dy, eps=DEFAULT_EPS):
    """Gradients of y = rms_norm(x, gamma) given dy.

    With r = 1/sqrt(mean(x^2) + eps), x_hat = x r and g = gamma * dy:
    dx = r * (g - x_hat * mean(g * x_hat)), dgamma = sum over leading axes
    of dy * x_hat.  Returns (dx, dgamma)."""
    x = _f64(x)
    gm = _f64(gamma)
    dy = _f64(dy)
    d = x.shape[-1]
    r = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    xh = x * r
    g = gm * dy
    dx = r * (g - xh * np.sum(g * xh, axis=-1, keepdims=True) / d)
    dgamma = np.sum((dy * xh).reshape(-1, d), axis=0)
    return dx, dgamma


def chunk_of(offsets, n_tokens):
    """Chunk index of every token, from cumulative offsets [0, ..., n]."""
    offs = np.asarray(offsets, dtype=np.int64)
    idx = np.empty(n_tokens, dtype=np.int64)
    for c in range(len(offs) - 1):
        idx[offs[c]:offs[c + 1]] = c
    return idx


def matched_kv_chunk(q_chunk, n_q_chunks, n_kv_chunks):
    """The kv chunk that holds query chunk ``q_chunk`` (tail-aligned)."""
    return n_kv_chunks - n_q_chunks + np.asarray(q_chunk)


def block_causal_mask(q_offsets, kv_offsets, rows=None, kv_range=0, samples=None, n_global=0):
    """Boolean mask M[i, j]: query token i may attend key token j.

    Built token by token from chunk ids, not from tile arithmetic.  With
    ``kv_range`` R > 0, key chunks more than R - 1 chunks before the query's
    own kv chunk are masked as well.

    Packed samples (MAGI-1 §4.1.2, Figure 15 (f), "varlen block-causal"):
    ``samples`` = cumulative kv-chunk counts [0, ..., n_kv] of the samples
    packed one after another into the sequence; a query token sees only keys
    of its own sample (the sample of its matched kv chunk).  None = one sample.

    Global block (Figure 15 (g), a varlen block-causal mask with a global
    block; App. B.1, Figure 23, a last global block): the last ``n_global`` kv
    chunks.  Every query token sees
    its keys, and the query tokens matched to it see every key.  Both rules
    hold whatever the sample or the KV range."""
    q_offsets = np.asarray(q_offsets)
    kv_offsets = np.asarray(kv_offsets)
    nq, nkv = len(q_offsets) - 1, len(kv_offsets) - 1
    cq = chunk_of(q_offsets, int(q_offsets[-1]))
    ck = chunk_of(kv_offsets, int(kv_offsets[-1]))
    if rows is not None:
        cq = cq[np.asarray(rows)]
    own = matched_kv_chunk(cq, nq, nkv)[:, None]
    m = ck[None, :] <= own
    if kv_range and kv_range > 0:
        m &= ck[None, :] >= own - (int(kv_range) - 1)
    if samples is not None:
        sid = chunk_of(np.asarray(samples), nkv)          # sample of every kv chunk
        m &= sid[ck][None, :] == sid[own]
    if n_global and n_global > 0:
        first = nkv - int(n_global)
        m |= ck[None, :] >= first                          # everyone sees the global keys
        m |= own >= first                                  # global queries see every key
    return m


def torch_index(rows):
    import torch
    return torch.as_tensor(np.asarray(rows, dtype=np.int64))


def _check(q, k, v, q_offsets, kv_offsets):
    B, Sq, Hq, D = q.shape
    Bk, Skv, Hkv, Dk = k.shape
    assert v.shape == k.shape and Bk == B and Dk == D
    assert Hq % Hkv == 0
    assert q_offsets[0] == 0 and q_offsets[-1] == Sq
    assert kv_offsets[0] == 0 and kv_offsets[-1] == Skv
    assert len(q_offsets) <= len(kv_offsets)
    return B, Sq, Hq, D, Skv, Hkv


def _attend_rows(qn_rows, kn, vv, mask_rows, scale):
    """Softmax attention of a block of normalised query rows [R, D] against
    all normalised keys [S, D]; returns (O [R, D], lse [R], P [R, S])."""
    s = qn_rows @ kn.T
    s *= scale
    s[~mask_rows] = -np.inf
    m = np.max(s, axis=1, keepdims=True)
    s -= m
    p = np.exp(s, out=s)
    l = np.sum(p, axis=1, keepdims=True)
    p /= l
    return p @ vv, (m + np.log(l))[:, 0], p


def forward_rows(q, k, v, q_offsets, kv_offsets, gamma_q, gamma_k, rows, heads=None,
                 batches=None, scale=None, eps=DEFAULT_EPS, block=None, kv_range=0, rope_q=None,
                 rope_k=None, samples=None, n_global=0):
    """Forward on a subset of query rows.

    ``rows`` is an int array of query-token indices; ``heads`` / ``batches``
    restrict the query heads and batch elements (default all).  Returns
    (out [nb, R, nh, D], lse [nb, nh, R]) in float64 for those rows only."""
    rows = np.asarray(rows, dtype=np.int64)
    k = _f64(k)
    v = _f64(v)
    q_offsets = np.asarray(q_offsets)
    kv_offsets = np.asarray(kv_offsets)
    B, Sq, Hq, D, Skv, Hkv = _check(q, k, v, q_offsets, kv_offsets)
    # only the requested query rows are converted (row i of qsel is rows[i])
    qsel = _f64(q[:, rows]) if not hasattr(q, "detach") else _f64(q[:, torch_index(rows)])
    qsel = rope(qsel, None if rope_q is None else _f64(rope_q)[rows])
    k = rope(k, rope_k)
    scale = 1.0 / np.sqrt(D) if not scale else float(scale)
    heads = list(range(Hq)) if heads is None else list(heads)
    batches = list(range(B)) if batches is None else list(batches)
    group = Hq // Hkv
    if block is None:   # rows per step, so one logit block stays near 512 MB
        block = int(max(16, min(512, (1 << 26) // Skv)))
    out = np.zeros((len(batches), len(rows), len(heads), D))
    lse = np.zeros((len(batches), len(heads), len(rows)))
    for bi, b in enumerate(batches):
        kn_all = rms_norm(k[b], gamma_k, eps)            # [Skv, Hkv, D]
        for hi, h in enumerate(heads):
            hk = h // group
            kn = kn_all[:, hk, :]
            vv = v[b, :, hk, :]
            for r0 in range(0, len(rows), block):
                rr = rows[r0:r0 + block]
                qn = rms_norm(qsel[b, r0:r0 + block, h, :], gamma_q, eps)
                mask = block_causal_mask(q_offsets, kv_offsets, rows=rr, kv_range=kv_range, samples=samples,
                                         n_global=n_global)
                o, ls, _ = _attend_rows(qn, kn, vv, mask, scale)
                out[bi, r0:r0 + len(rr), hi, :] = o
                lse[bi, hi, r0:r0 + len(rr)] = ls
    return out, lse


def forward(q, k, v, q_offsets, kv_offsets, gamma_q, gamma_k, scale=None, eps=DEFAULT_EPS, kv_range=0,
            rope_q=None, rope_k=None, samples=None, n_global=0):
    """Full forward.  Returns (out [B, Sq, Hq, D], lse [B, Hq, Sq]), float64."""
    Sq = q.shape[1]
    return forward_rows(q, k, v, q_offsets, kv_offsets, gamma_q, gamma_k,
                        rows=np.arange(Sq), scale=scale, eps=eps, kv_range=kv_range, rope_q=rope_q,
                        rope_k=rope_k, samples=samples, n_global=n_global)


def backward(q, k, v, dout, q_offsets, kv_offsets, gamma_q, gamma_k, scale=None,
             eps=DEFAULT_EPS, kv_range=0, rope_q=None, rope_k=None, samples=None, n_global=0):
    """Full analytic backward in float64.

    Returns dict(dq, dk, dv, dgamma_q, dgamma_k, out, lse) and, with rotary
    angles, drope_q, drope_k; dq/dk are the gradients with respect to the raw
    (pre-rotation, pre-norm) q and k."""
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    do = _f64(dout)
    gq = _f64(gamma_q)
    gk = _f64(gamma_k)
    q_offsets = np.asarray(q_offsets)
    kv_offsets = np.asarray(kv_offsets)
    B, Sq, Hq, D, Skv, Hkv = _check(q, k, v, q_offsets, kv_offsets)
    scale = 1.0 / np.sqrt(D) if not scale else float(scale)
    group = Hq // Hkv
    mask = block_causal_mask(q_offsets, kv_offsets, kv_range=kv_range, samples=samples, n_global=n_global)
    dqn = np.zeros_like(q)
    dkn = np.zeros_like(k)
    dv = np.zeros_like(v)
    out = np.zeros_like(q)
    lse = np.zeros((B, Hq, Sq))
    q_raw, k_raw = q, k
    q, k = rope(q_raw, rope_q), rope(k_raw, rope_k)
    qn_all = rms_norm(q, gq, eps)
    kn_all = rms_norm(k, gk, eps)
    for b in range(B):
        for h in range(Hq):
            hk = h // group
            qn = qn_all[b, :, h, :]
            kn = kn_all[b, :, hk, :]
            vv = v[b, :, hk, :]
            o, ls, p = _attend_rows(qn, kn, vv, mask, scale)
            out[b, :, h, :] = o
            lse[b, h, :] = ls
            g = do[b, :, h, :]
            dv[b, :, hk, :] += p.T @ g
            dp = g @ vv.T
            delta = np.sum(g * o, axis=1, keepdims=True)
            ds = p * (dp - delta)
            dqn[b, :, h, :] = scale * (ds @ kn)
            dkn[b, :, hk, :] += scale * (ds.T @ qn)
    dq, dgq = rms_norm_backward(q, gq, dqn, eps)
    dk, dgk = rms_norm_backward(k, gk, dkn, eps)
    dq, drq = rope_backward(q_raw, rope_q, dq)
    dk, drk = rope_backward(k_raw, rope_k, dk)
    res = dict(dq=dq, dk=dk, dv=dv, dgamma_q=dgq, dgamma_k=dgk, out=out, lse=lse)
    if rope_q is not None:
        res["drope_q"] = drq
    if rope_k is not None:
        res["drope_k"] = drk
    return res


def backward_rows(q, k, v, dout, q_offsets, kv_offsets, gamma_q, gamma_k, q_rows=None,
                  kv_rows=None, kv_heads=None, batches=None, scale=None, eps=DEFAULT_EPS,
                  block=None, kv_range=0, rope_q=None, rope_k=None, samples=None, n_global=0):
    """Exact backward on chosen rows, without a full backward.

    * dq of query rows ``q_rows`` (all heads): needs only those rows' P, dP
      and Delta.
    * dk, dv of key rows ``kv_rows`` for kv heads ``kv_heads``: needs every
      query row that sees those keys (rows are located from the mask) and
      each such row's full softmax; cheap when the keys sit in the last chunk.

    Only the query rows needed are converted to float64.  Returns
    dict(dq [nb, R, Hq, D], dk [nb, Rk, nkh, D], dv [nb, Rk, nkh, D]), keys
    present only for the parts requested."""
    k = _f64(k)
    v = _f64(v)
    gq = _f64(gamma_q)
    gk = _f64(gamma_k)
    q_offsets = np.asarray(q_offsets)
    kv_offsets = np.asarray(kv_offsets)
    B, Sq, Hq, D, Skv, Hkv = _check(q, k, v, q_offsets, kv_offsets)
    scale = 1.0 / np.sqrt(D) if not scale else float(scale)
    group = Hq // Hkv
    if block is None:
        block = int(max(16, min(256, (1 << 25) // Skv)))
    batches = list(range(B)) if batches is None else list(batches)

    def take(x, rows):
        return _f64(x[:, torch_index(rows)] if hasattr(x, "detach") else x[:, rows])

    res = {}
    rk = None if rope_k is None else _f64(rope_k)
    if q_rows is not None:
        q_rows = np.asarray(q_rows, dtype=np.int64)
        qraw, dsel = take(q, q_rows), take(dout, q_rows)
        rq = None if rope_q is None else _f64(rope_q)[q_rows]
        qsel = rope(qraw, rq)
        dq = np.zeros((len(batches), len(q_rows), Hq, D))
        for bi, b in enumerate(batches):
            kn_all = rms_norm(rope(k[b], rk), gk, eps)
            for r0 in range(0, len(q_rows), block):
                rr = q_rows[r0:r0 + block]
                mask = block_causal_mask(q_offsets, kv_offsets, rows=rr, kv_range=kv_range, samples=samples,
                                         n_global=n_global)
                dqn = np.zeros((len(rr), Hq, D))
                for h in range(Hq):
                    hk = h // group
                    qn = rms_norm(qsel[b, r0:r0 + block, h, :], gq, eps)
                    o, _, p = _attend_rows(qn, kn_all[:, hk, :], v[b, :, hk, :], mask, scale)
                    g = dsel[b, r0:r0 + block, h, :]
                    dp = g @ v[b, :, hk, :].T
                    delta = np.sum(g * o, axis=1, keepdims=True)
                    dp -= delta
                    dp *= p
                    dqn[:, h, :] = scale * (dp @ kn_all[:, hk, :])
                dqr, _ = rms_norm_backward(qsel[b, r0:r0 + block], gq, dqn, eps)
                dq[bi, r0:r0 + len(rr)], _ = rope_backward(qraw[b, r0:r0 + block],
                                                           None if rq is None else rq[r0:r0 + block], dqr)
        res["dq"] = dq
    if kv_rows is not None:
        kv_rows = np.asarray(kv_rows, dtype=np.int64)
        kv_heads = list(range(Hkv)) if kv_heads is None else list(kv_heads)
        dk = np.zeros((len(batches), len(kv_rows), len(kv_heads), D))
        dv = np.zeros((len(batches), len(kv_rows), len(kv_heads), D))
        # every query row that sees at least one of the requested keys
        full_mask = block_causal_mask(q_offsets, kv_offsets, kv_range=kv_range, samples=samples, n_global=n_global)
        seeing = np.nonzero(full_mask[:, kv_rows].any(axis=1))[0]
        del full_mask
        qsel, dsel = take(q, seeing), take(dout, seeing)
        qsel = rope(qsel, None if rope_q is None else _f64(rope_q)[seeing])
        for bi, b in enumerate(batches):
            kr_all = rope(k[b], rk)
            kn_all = rms_norm(kr_all, gk, eps)
            for khi, hk in enumerate(kv_heads):
                kn = kn_all[:, hk, :]
                vv = v[b, :, hk, :]
                dkn = np.zeros((len(kv_rows), D))
                for h in range(hk * group, (hk + 1) * group):
                    for r0 in range(0, len(seeing), block):
                        rr = seeing[r0:r0 + block]
                        qn = rms_norm(qsel[b, r0:r0 + block, h, :], gq, eps)
                        mask = block_causal_mask(q_offsets, kv_offsets, rows=rr, kv_range=kv_range,
                                                 samples=samples, n_global=n_global)
                        o, _, p = _attend_rows(qn, kn, vv, mask, scale)
                        g = dsel[b, r0:r0 + block, h, :]
                        delta = np.sum(g * o, axis=1, keepdims=True)
                        pc = p[:, kv_rows]
                        dpc = g @ vv[kv_rows].T
                        dsc = pc * (dpc - delta)
                        dv[bi, :, khi, :] += pc.T @ g
                        dkn += scale * (dsc.T @ qn)
                dkr, _ = rms_norm_backward(kr_all[kv_rows, hk, :], gk, dkn, eps)
                if rk is None:
                    dk[bi, :, khi, :] = dkr
                else:
                    dkx, _ = rope_backward(k[b, kv_rows, hk, :][:, None, :], rk[kv_rows], dkr[:, None, :])
                    dk[bi, :, khi, :] = dkx[:, 0, :]
        res["dk"] = dk
        res["dv"] = dv
    return res
