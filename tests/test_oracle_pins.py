"""Pins for the fp64 oracle: each test checks it against something other than
itself (a hand-written fixture, brute force, a library routine, a closed
form or an invariant that the method fixes), so that a dropped term, a wrong
sign or index, or a transposed operand fails at least one of them."""
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import bca_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def offs(lens):
    return np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)


def rand_case(rng, B, q_lens, kv_lens, Hq, Hkv, D, gamma=True):
    Sq, Skv = sum(q_lens), sum(kv_lens)
    q = rng.standard_normal((B, Sq, Hq, D))
    k = rng.standard_normal((B, Skv, Hkv, D))
    v = rng.standard_normal((B, Skv, Hkv, D))
    gq = 1 + 0.1 * rng.standard_normal(D) if gamma else np.ones(D)
    gk = 1 + 0.1 * rng.standard_normal(D) if gamma else np.ones(D)
    return q, k, v, gq, gk, offs(q_lens), offs(kv_lens)


def read_mask_fixture(name):
    rows, meta = [], {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if line[0].isalpha():
                key, *vals = line.split()
                meta[key] = [int(x) for x in vals]
            else:
                rows.append([c == "1" for c in line])
    return meta, np.array(rows)


# ---------------------------------------------------------------- the mask

@pytest.mark.parametrize("name", ["mask_train_2_1_3.txt", "mask_stream_2of3.txt",
                                  "mask_kvrange2_train_2_1_2_1.txt", "mask_kvrange3_stream_2of4.txt",
                                  "mask_packed_train_2_1_2_1_2.txt", "mask_packed_global_train_2_1_2_1_2.txt",
                                  "mask_packed_stream_2of4.txt", "mask_packed_kvrange2_global_1x5.txt"])
def test_mask_matches_hand_written_fixture(name):
    meta, want = read_mask_fixture(name)
    got = orc.block_causal_mask(offs(meta["q_chunks"]), offs(meta["kv_chunks"]),
                                kv_range=meta.get("kv_range", [0])[0], samples=meta.get("samples"),
                                n_global=meta.get("n_global", [0])[0])
    assert got.shape == want.shape
    assert np.array_equal(got, want)


# ------------------------------------------------------- brute force (loops)

def brute_force(q, k, v, qo, ko, gq, gk, eps=1e-6):
    """Pure-Python loops straight from the definition (tiny inputs only)."""
    B, Sq, Hq, D = q.shape
    Skv, Hkv = k.shape[1], k.shape[2]
    nq, nkv = len(qo) - 1, len(ko) - 1
    scale = 1.0 / math.sqrt(D)

    def chunk(o, t):
        for c in range(len(o) - 1):
            if o[c] <= t < o[c + 1]:
                return c
        raise AssertionError

    def norm(x, g):
        ms = sum(xx * xx for xx in x) / len(x)
        r = 1.0 / math.sqrt(ms + eps)
        return [xx * r * gg for xx, gg in zip(x, g)]

    out = np.zeros((B, Sq, Hq, D))
    lse = np.zeros((B, Hq, Sq))
    for b in range(B):
        for h in range(Hq):
            hk = h // (Hq // Hkv)
            for i in range(Sq):
                qi = norm(list(q[b, i, h]), list(gq))
                ci = chunk(qo, i) + (nkv - nq)
                logits = []
                for j in range(Skv):
                    if chunk(ko, j) <= ci:
                        kj = norm(list(k[b, j, hk]), list(gk))
                        logits.append((j, scale * sum(a * c for a, c in zip(qi, kj))))
                mx = max(s for _, s in logits)
                den = sum(math.exp(s - mx) for _, s in logits)
                lse[b, h, i] = mx + math.log(den)
                for d in range(D):
                    out[b, i, h, d] = sum(math.exp(s - mx) / den * v[b, j, hk, d] for j, s in logits)
    return out, lse


@pytest.mark.parametrize("q_lens,kv_lens", [([2, 3, 1], [2, 3, 1]), ([3, 2], [2, 3, 2]),
                                            ([1, 1, 1, 1], [1, 1, 1, 1])])
def test_forward_matches_brute_force(q_lens, kv_lens):
    rng = np.random.default_rng(11)
    q, k, v, gq, gk, qo, ko = rand_case(rng, 2, q_lens, kv_lens, 4, 2, 4)
    o, l = orc.forward(q, k, v, qo, ko, gq, gk)
    ob, lb = brute_force(q, k, v, qo, ko, gq, gk)
    np.testing.assert_allclose(o, ob, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l, lb, rtol=0, atol=1e-12)


# ----------------------------------------------------- library special cases

def torch_reference(q, k, v, qo, ko, gq, gk, eps=1e-6, mask=None):
    """fp64 torch: F.rms_norm + repeat_interleave (GQA) + SDPA with a boolean
    mask built here from per-token chunk ids."""
    Q = torch.tensor(q)
    K = torch.tensor(k)
    V = torch.tensor(v)
    D = Q.shape[-1]
    Qn = F.rms_norm(Q, (D,), weight=torch.tensor(gq), eps=eps)
    Kn = F.rms_norm(K, (D,), weight=torch.tensor(gk), eps=eps)
    g = Q.shape[2] // K.shape[2]
    Kn = Kn.repeat_interleave(g, dim=2)
    Vr = V.repeat_interleave(g, dim=2)
    if mask is None:
        cq = torch.bucketize(torch.arange(Q.shape[1]), torch.tensor(qo[1:]), right=True)
        ck = torch.bucketize(torch.arange(K.shape[1]), torch.tensor(ko[1:]), right=True)
        shift = (len(ko) - 1) - (len(qo) - 1)
        mask = ck[None, :] <= (cq[:, None] + shift)
    o = F.scaled_dot_product_attention(Qn.transpose(1, 2), Kn.transpose(1, 2), Vr.transpose(1, 2),
                                       attn_mask=mask)
    return o.transpose(1, 2).numpy()


@pytest.mark.parametrize("q_lens,kv_lens,Hq,Hkv,D", [
    ([7, 13, 5, 9], [7, 13, 5, 9], 6, 2, 16),
    ([11, 4], [3, 8, 11, 4], 4, 4, 8),
    ([33], [33], 3, 1, 32),
])
def test_forward_matches_torch_sdpa_fp64(q_lens, kv_lens, Hq, Hkv, D):
    rng = np.random.default_rng(5)
    q, k, v, gq, gk, qo, ko = rand_case(rng, 2, q_lens, kv_lens, Hq, Hkv, D)
    o, _ = orc.forward(q, k, v, qo, ko, gq, gk)
    np.testing.assert_allclose(o, torch_reference(q, k, v, qo, ko, gq, gk), rtol=0, atol=1e-12)


def test_single_chunk_is_full_bidirectional_attention():
    rng = np.random.default_rng(6)
    q, k, v, gq, gk, qo, ko = rand_case(rng, 1, [40], [40], 4, 2, 16)
    o, _ = orc.forward(q, k, v, qo, ko, gq, gk)
    full = torch_reference(q, k, v, qo, ko, gq, gk, mask=torch.ones(40, 40, dtype=torch.bool))
    np.testing.assert_allclose(o, full, rtol=0, atol=1e-12)


def test_unit_chunks_are_token_causal_attention():
    rng = np.random.default_rng(7)
    n = 17
    q, k, v, gq, gk, qo, ko = rand_case(rng, 1, [1] * n, [1] * n, 2, 1, 8)
    o, _ = orc.forward(q, k, v, qo, ko, gq, gk)
    causal = torch_reference(q, k, v, qo, ko, gq, gk,
                             mask=torch.ones(n, n, dtype=torch.bool).tril())
    np.testing.assert_allclose(o, causal, rtol=0, atol=1e-12)


def test_lse_is_log_sum_exp_of_scaled_logits():
    rng = np.random.default_rng(8)
    q, k, v, gq, gk, qo, ko = rand_case(rng, 1, [3, 5], [4, 3, 5], 2, 1, 8)
    _, l = orc.forward(q, k, v, qo, ko, gq, gk)
    Qn = F.rms_norm(torch.tensor(q), (8,), weight=torch.tensor(gq), eps=1e-6)[0]
    Kn = F.rms_norm(torch.tensor(k), (8,), weight=torch.tensor(gk), eps=1e-6)[0, :, 0]
    mask = torch.tensor(read_mask_like(qo, ko))
    for h in range(2):
        s = (Qn[:, h] @ Kn.T) / math.sqrt(8)
        s = s.masked_fill(~mask, -math.inf)
        np.testing.assert_allclose(l[0, h], torch.logsumexp(s, dim=1).numpy(), rtol=0, atol=1e-12)


def read_mask_like(qo, ko):
    # q chunk c sees kv chunks <= c + (n_kv - n_q), built from token loops
    nq, nkv = len(qo) - 1, len(ko) - 1
    m = np.zeros((qo[-1], ko[-1]), dtype=bool)
    for c in range(nq):
        m[qo[c]:qo[c + 1], :ko[c + nkv - nq + 1]] = True
    return m


# ------------------------------------------------------------- invariants

def test_later_chunk_kv_does_not_change_earlier_outputs():
    rng = np.random.default_rng(9)
    q, k, v, gq, gk, qo, ko = rand_case(rng, 1, [5, 6, 7], [5, 6, 7], 4, 2, 8)
    o1, l1 = orc.forward(q, k, v, qo, ko, gq, gk)
    k2, v2 = k.copy(), v.copy()
    k2[:, 11:] = rng.standard_normal(k2[:, 11:].shape) * 5
    v2[:, 11:] = rng.standard_normal(v2[:, 11:].shape) * 5
    o2, l2 = orc.forward(q, k2, v2, qo, ko, gq, gk)
    assert np.array_equal(o1[:, :11], o2[:, :11])
    assert np.array_equal(l1[:, :, :11], l2[:, :, :11])
    assert not np.allclose(o1[:, 11:], o2[:, 11:])


def test_constant_v_gives_v():
    rng = np.random.default_rng(10)
    q, k, v, gq, gk, qo, ko = rand_case(rng, 2, [4, 4, 4], [4, 4, 4], 4, 2, 8)
    c = rng.standard_normal((1, 1, 2, 8))
    v = np.broadcast_to(c, v.shape).copy()
    o, _ = orc.forward(q, k, v, qo, ko, gq, gk)
    want = np.broadcast_to(np.repeat(c, 2, axis=2), o.shape)
    np.testing.assert_allclose(o, want, rtol=0, atol=1e-13)


def test_softmax_rows_sum_to_one_and_vanish_outside_the_mask():
    # with v_j = e_j (one-hot, Skv <= D) the output row IS the softmax row
    rng = np.random.default_rng(12)
    lens = [3, 2, 4]
    S = sum(lens)
    q, k, _, gq, gk, qo, ko = rand_case(rng, 1, lens, lens, 2, 1, 16)
    v = np.zeros((1, S, 1, 16))
    v[0, np.arange(S), 0, np.arange(S)] = 1.0
    o, _ = orc.forward(q, k, v, qo, ko, gq, gk)
    p = o[0, :, :, :S]                      # [Sq, Hq, Skv]
    np.testing.assert_allclose(p.sum(-1), 1.0, rtol=0, atol=1e-14)
    assert (p >= 0).all()
    mask = read_mask_like(qo, ko)
    assert (p[~np.broadcast_to(mask[:, None, :], p.shape)] == 0).all()
    assert (p[np.broadcast_to(mask[:, None, :], p.shape)] > 0).all()


def test_permutation_within_a_chunk_permutes_outputs():
    rng = np.random.default_rng(13)
    lens = [4, 6, 5]
    q, k, v, gq, gk, qo, ko = rand_case(rng, 1, lens, lens, 2, 2, 8)
    perm = np.arange(15)
    perm[4:10] = rng.permutation(np.arange(4, 10))
    o1, _ = orc.forward(q, k, v, qo, ko, gq, gk)
    o2, _ = orc.forward(q[:, perm], k[:, perm], v[:, perm], qo, ko, gq, gk)
    np.testing.assert_allclose(o2, o1[:, perm], rtol=0, atol=1e-13)


def test_gqa_equals_mha_with_repeated_kv():
    rng = np.random.default_rng(14)
    q, k, v, gq, gk, qo, ko = rand_case(rng, 2, [3, 5], [3, 5], 6, 2, 8)
    o1, l1 = orc.forward(q, k, v, qo, ko, gq, gk)
    o2, l2 = orc.forward(q, np.repeat(k, 3, axis=2), np.repeat(v, 3, axis=2), qo, ko, gq, gk)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-14)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-14)


def test_rms_norm_closed_forms_and_library():
    rng = np.random.default_rng(15)
    x = rng.standard_normal((7, 32)) * rng.uniform(0.01, 10, (7, 1))
    y = orc.rms_norm(x, np.ones(32), eps=1e-6)
    ms = np.mean(x * x, axis=1)
    np.testing.assert_allclose(np.mean(y * y, axis=1), ms / (ms + 1e-6), rtol=1e-13)
    g = rng.standard_normal(32)
    want = F.rms_norm(torch.tensor(x), (32,), weight=torch.tensor(g), eps=1e-6).numpy()
    np.testing.assert_allclose(orc.rms_norm(x, g, 1e-6), want, rtol=0, atol=1e-13)


def test_positive_token_rescaling_of_q_and_k_leaves_output_unchanged():
    rng = np.random.default_rng(16)
    q, k, v, gq, gk, qo, ko = rand_case(rng, 1, [6, 6], [6, 6], 2, 1, 8)
    sq = np.exp(rng.standard_normal((1, 12, 1, 1)))
    sk = np.exp(rng.standard_normal((1, 12, 1, 1)))
    o1, _ = orc.forward(q, k, v, qo, ko, gq, gk, eps=0.0)
    o2, _ = orc.forward(q * sq, k * sk, v, qo, ko, gq, gk, eps=0.0)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-13)
    o3, _ = orc.forward(q * sq, k * sk, v, qo, ko, gq, gk, eps=1e-6)
    np.testing.assert_allclose(o1, o3, rtol=0, atol=1e-4)


def test_forward_rows_subset_matches_full():
    rng = np.random.default_rng(17)
    q, k, v, gq, gk, qo, ko = rand_case(rng, 2, [5, 4], [6, 5, 4], 4, 2, 8)
    o, l = orc.forward(q, k, v, qo, ko, gq, gk)
    rows = np.array([0, 3, 5, 8])
    o2, l2 = orc.forward_rows(q, k, v, qo, ko, gq, gk, rows, heads=[1, 3], batches=[1])
    np.testing.assert_array_equal(o2, o[1:2][:, rows][:, :, [1, 3]])
    np.testing.assert_array_equal(l2, l[1:2][:, [1, 3]][:, :, rows])


# -------------------------------------------------------------- backward

def oracle_loss(params, dout, qo, ko):
    q, k, v, gq, gk = params
    o, _ = orc.forward(q, k, v, qo, ko, gq, gk)
    return float(np.sum(o * dout))


def test_backward_matches_central_finite_differences():
    rng = np.random.default_rng(18)
    q, k, v, gq, gk, qo, ko = rand_case(rng, 1, [2, 3], [2, 3], 4, 2, 4)
    do = rng.standard_normal(q.shape)
    g = orc.backward(q, k, v, do, qo, ko, gq, gk)
    params = [q, k, v, gq, gk]
    names = ["dq", "dk", "dv", "dgamma_q", "dgamma_k"]
    h = 1e-6
    for pi, name in enumerate(names):
        base = params[pi]
        num = np.zeros_like(base)
        it = np.nditer(base, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            pp = [p.copy() for p in params]
            pp[pi][idx] += h
            lp = oracle_loss(pp, do, qo, ko)
            pp[pi][idx] -= 2 * h
            lm = oracle_loss(pp, do, qo, ko)
            num[idx] = (lp - lm) / (2 * h)
        np.testing.assert_allclose(g[name], num, rtol=1e-6, atol=1e-7, err_msg=name)


def test_backward_matches_torch_autograd_fp64():
    rng = np.random.default_rng(19)
    q, k, v, gq, gk, qo, ko = rand_case(rng, 2, [5, 7, 4], [5, 7, 4], 6, 2, 16)
    do = rng.standard_normal(q.shape)
    g = orc.backward(q, k, v, do, qo, ko, gq, gk)
    T = [torch.tensor(x, requires_grad=True) for x in (q, k, v, gq, gk)]
    D = 16
    Qn = F.rms_norm(T[0], (D,), weight=T[3], eps=1e-6)
    Kn = F.rms_norm(T[1], (D,), weight=T[4], eps=1e-6).repeat_interleave(3, dim=2)
    Vr = T[2].repeat_interleave(3, dim=2)
    mask = torch.tensor(read_mask_like(qo, ko))
    o = F.scaled_dot_product_attention(Qn.transpose(1, 2), Kn.transpose(1, 2), Vr.transpose(1, 2),
                                       attn_mask=mask).transpose(1, 2)
    (o * torch.tensor(do)).sum().backward()
    for t, name in zip(T, ["dq", "dk", "dv", "dgamma_q", "dgamma_k"]):
        np.testing.assert_allclose(g[name], t.grad.numpy(), rtol=0, atol=1e-11, err_msg=name)
    np.testing.assert_allclose(g["out"], o.detach().numpy(), rtol=0, atol=1e-12)


def test_backward_rows_match_full_backward():
    rng = np.random.default_rng(20)
    q, k, v, gq, gk, qo, ko = rand_case(rng, 2, [4, 5, 6], [3, 4, 5, 6], 4, 2, 8)
    do = rng.standard_normal(q.shape)
    full = orc.backward(q, k, v, do, qo, ko, gq, gk)
    qr = np.array([0, 4, 9, 14])
    kr = np.array([12, 13, 17])           # last chunk keys
    part = orc.backward_rows(q, k, v, do, qo, ko, gq, gk, q_rows=qr, kv_rows=kr, kv_heads=[1])
    np.testing.assert_allclose(part["dq"], full["dq"][:, qr], rtol=0, atol=1e-12)
    np.testing.assert_allclose(part["dk"], full["dk"][:, kr][:, :, [1]], rtol=0, atol=1e-12)
    np.testing.assert_allclose(part["dv"], full["dv"][:, kr][:, :, [1]], rtol=0, atol=1e-12)


def test_backward_structure_and_identities():
    rng = np.random.default_rng(21)
    q, k, v, gq, gk, qo, ko = rand_case(rng, 1, [4, 5, 6], [4, 5, 6], 4, 2, 8)
    do = rng.standard_normal(q.shape)
    g = orc.backward(q, k, v, do, qo, ko, gq, gk, eps=0.0)
    # dV summed over keys = dO summed over queries of the group (rows of P sum to 1)
    for hk in range(2):
        np.testing.assert_allclose(g["dv"][0, :, hk].sum(0), do[0, :, 2 * hk:2 * hk + 2].sum((0, 1)),
                                   rtol=0, atol=1e-12)
    # RMSNorm (eps = 0) is scale invariant, so raw gradients are orthogonal to the input
    np.testing.assert_allclose(np.sum(g["dq"] * q, -1), 0, atol=1e-12)
    np.testing.assert_allclose(np.sum(g["dk"] * k, -1), 0, atol=1e-12)
    # keys of chunk c receive no gradient from queries of earlier chunks:
    # changing q and dO of chunk 0 leaves dk, dv of chunks 1-2 unchanged
    q2, do2 = q.copy(), do.copy()
    q2[:, :4] = rng.standard_normal(q2[:, :4].shape)
    do2[:, :4] = rng.standard_normal(do2[:, :4].shape)
    g2 = orc.backward(q2, k, v, do2, qo, ko, gq, gk, eps=0.0)
    np.testing.assert_allclose(g2["dk"][:, 4:], g["dk"][:, 4:], rtol=0, atol=1e-13)
    np.testing.assert_allclose(g2["dv"][:, 4:], g["dv"][:, 4:], rtol=0, atol=1e-13)
    assert not np.allclose(g2["dk"][:, :4], g["dk"][:, :4])


# ---------------------------------------------------------------- KV range

def test_kv_range_one_is_full_attention_inside_each_chunk():
    """KV range 1 (no access to earlier chunks) = independent bidirectional
    attention per chunk, computed by torch SDPA without a mask."""
    rng = np.random.default_rng(31)
    lens = [5, 9, 3, 7]
    q, k, v, gq, gk, qo, ko = rand_case(rng, 2, lens, lens, 4, 2, 16)
    o, _ = orc.forward(q, k, v, qo, ko, gq, gk, kv_range=1)
    for c in range(len(lens)):
        sl = slice(qo[c], qo[c + 1])
        n = lens[c]
        want = torch_reference(q[:, sl], k[:, sl], v[:, sl], offs([n]), offs([n]), gq, gk,
                               mask=torch.ones(n, n, dtype=torch.bool))
        np.testing.assert_allclose(o[:, sl], want, rtol=0, atol=1e-12)


@pytest.mark.parametrize("R", [1, 2, 5])
def test_kv_range_on_unit_chunks_is_sliding_window_causal_attention(R):
    """One-token chunks with KV range R: token i sees tokens i-R+1 .. i, the
    textbook sliding-window causal mask (built here with torch band ops)."""
    rng = np.random.default_rng(32 + R)
    n = 19
    q, k, v, gq, gk, qo, ko = rand_case(rng, 1, [1] * n, [1] * n, 2, 1, 8)
    o, _ = orc.forward(q, k, v, qo, ko, gq, gk, kv_range=R)
    ones = torch.ones(n, n, dtype=torch.bool)
    band = ones.tril() & ones.triu(-(R - 1))
    np.testing.assert_allclose(o, torch_reference(q, k, v, qo, ko, gq, gk, mask=band), rtol=0, atol=1e-12)


def test_kv_range_covering_every_chunk_changes_nothing():
    rng = np.random.default_rng(33)
    q, k, v, gq, gk, qo, ko = rand_case(rng, 1, [4, 6], [3, 5, 4, 6], 4, 2, 8)
    o0, l0 = orc.forward(q, k, v, qo, ko, gq, gk)
    for R in (4, 5, 100):
        o, l = orc.forward(q, k, v, qo, ko, gq, gk, kv_range=R)
        assert np.array_equal(o, o0) and np.array_equal(l, l0)
    o3, _ = orc.forward(q, k, v, qo, ko, gq, gk, kv_range=3)
    assert not np.allclose(o3, o0)   # the first active chunk loses kv chunk 0


def test_kv_outside_every_window_does_not_change_outputs():
    rng = np.random.default_rng(34)
    lens = [4, 5, 6, 3]
    q, k, v, gq, gk, qo, ko = rand_case(rng, 1, lens, lens, 4, 2, 8)
    o1, l1 = orc.forward(q, k, v, qo, ko, gq, gk, kv_range=2)
    k2, v2 = k.copy(), v.copy()
    k2[:, :4] += rng.standard_normal(k2[:, :4].shape)   # chunk 0: outside the windows of chunks 2 and 3
    v2[:, :4] += 1.0
    o2, l2 = orc.forward(q, k2, v2, qo, ko, gq, gk, kv_range=2)
    late = slice(qo[2], qo[4])
    assert np.array_equal(o1[:, late], o2[:, late]) and np.array_equal(l1[..., late], l2[..., late])
    assert not np.allclose(o1[:, :qo[2]], o2[:, :qo[2]])


def test_kv_range_backward_matches_central_finite_differences():
    rng = np.random.default_rng(35)
    q, k, v, gq, gk, qo, ko = rand_case(rng, 1, [2, 1, 2], [2, 1, 2], 2, 1, 4)
    do = rng.standard_normal(q.shape)
    g = orc.backward(q, k, v, do, qo, ko, gq, gk, kv_range=2)
    params = [q, k, v, gq, gk]
    h = 1e-6
    for pi, name in enumerate(["dq", "dk", "dv", "dgamma_q", "dgamma_k"]):
        base = params[pi]
        num = np.zeros_like(base)
        it = np.nditer(base, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            pp = [p.copy() for p in params]
            pp[pi][idx] += h
            lp = float(np.sum(orc.forward(*pp[:3], qo, ko, *pp[3:], kv_range=2)[0] * do))
            pp[pi][idx] -= 2 * h
            lm = float(np.sum(orc.forward(*pp[:3], qo, ko, *pp[3:], kv_range=2)[0] * do))
            num[idx] = (lp - lm) / (2 * h)
        np.testing.assert_allclose(g[name], num, rtol=1e-6, atol=1e-7, err_msg=name)


def test_kv_range_backward_rows_match_full_backward():
    rng = np.random.default_rng(36)
    lens = [5, 4, 6, 3]
    q, k, v, gq, gk, qo, ko = rand_case(rng, 1, lens, lens, 4, 2, 8)
    do = rng.standard_normal(q.shape)
    full = orc.backward(q, k, v, do, qo, ko, gq, gk, kv_range=2)
    rows = np.array([0, 4, 9, 12, 17])
    kv_rows = np.array([1, 6, 10, 16])
    part = orc.backward_rows(q, k, v, do, qo, ko, gq, gk, q_rows=rows, kv_rows=kv_rows, kv_range=2)
    np.testing.assert_allclose(part["dq"][0], full["dq"][0, rows], rtol=0, atol=1e-12)
    np.testing.assert_allclose(part["dk"][0], full["dk"][0, kv_rows], rtol=0, atol=1e-12)
    np.testing.assert_allclose(part["dv"][0], full["dv"][0, kv_rows], rtol=0, atol=1e-12)


# ------------------------------------------------------- cross-attention

def test_one_chunk_pair_of_different_lengths_is_full_cross_attention():
    """One query chunk against one key/value chunk of another length (text K/V,
    MAGI-1 §2.2.2): every query sees every key, as torch SDPA without a mask."""
    rng = np.random.default_rng(41)
    for Sq, Skv in ((23, 9), (7, 31)):
        q, k, v, gq, gk, qo, ko = rand_case(rng, 2, [Sq], [Skv], 6, 2, 16)
        o, _ = orc.forward(q, k, v, qo, ko, gq, gk)
        want = torch_reference(q, k, v, qo, ko, gq, gk, mask=torch.ones(Sq, Skv, dtype=torch.bool))
        np.testing.assert_allclose(o, want, rtol=0, atol=1e-12)


def test_chunkwise_text_conditioning_is_cross_attention_per_chunk():
    """KV range 1 with text chunks of their own lengths (MAGI-1 §7, chunk-wise text
    conditioning): query chunk c attends exactly to text chunk c."""
    rng = np.random.default_rng(42)
    q_lens, t_lens = [6, 9, 4], [3, 5, 7]
    q, k, v, gq, gk, qo, ko = rand_case(rng, 1, q_lens, t_lens, 4, 2, 8)
    o, _ = orc.forward(q, k, v, qo, ko, gq, gk, kv_range=1)
    for c in range(3):
        qs, ks = slice(qo[c], qo[c + 1]), slice(ko[c], ko[c + 1])
        want = torch_reference(q[:, qs], k[:, ks], v[:, ks], offs([q_lens[c]]), offs([t_lens[c]]), gq, gk,
                               mask=torch.ones(q_lens[c], t_lens[c], dtype=torch.bool))
        np.testing.assert_allclose(o[:, qs], want, rtol=0, atol=1e-12)


# ------------------------------------------------------- rotary embedding

def test_rope_with_zero_angles_changes_nothing():
    rng = np.random.default_rng(51)
    q, k, v, gq, gk, qo, ko = rand_case(rng, 1, [5, 7], [5, 7], 4, 2, 8)
    z = np.zeros((12, 4))
    o0, l0 = orc.forward(q, k, v, qo, ko, gq, gk)
    o1, l1 = orc.forward(q, k, v, qo, ko, gq, gk, rope_q=z, rope_k=z)
    assert np.array_equal(o0, o1) and np.array_equal(l0, l1)


def test_rope_with_one_angle_table_row_for_every_token_changes_nothing():
    """The same rotation of every q and k leaves all dot products unchanged (unit
    gains: the norm's per-feature gain would not commute with the rotation)."""
    rng = np.random.default_rng(52)
    q, k, v, gq, gk, qo, ko = rand_case(rng, 2, [4, 6, 3], [4, 6, 3], 4, 2, 16, gamma=False)
    t = np.tile(rng.uniform(-3, 3, (1, 8)), (13, 1))
    o0, _ = orc.forward(q, k, v, qo, ko, gq, gk)
    o1, _ = orc.forward(q, k, v, qo, ko, gq, gk, rope_q=t, rope_k=t)
    np.testing.assert_allclose(o1, o0, rtol=0, atol=1e-12)
    t2 = rng.uniform(-3, 3, (13, 8))
    o2, _ = orc.forward(q, k, v, qo, ko, gq, gk, rope_q=t2, rope_k=t2)
    assert not np.allclose(o2, o0)


def test_rope_on_positions_depends_only_on_relative_position():
    """Angles s * w_i (one axis): shifting every position by the same amount
    leaves the attention unchanged (unit gains)."""
    rng = np.random.default_rng(53)
    q, k, v, gq, gk, qo, ko = rand_case(rng, 1, [5, 4, 6], [5, 4, 6], 4, 1, 16, gamma=False)
    w = 1.0 / (100.0 ** (np.arange(8) / 8))
    pos = np.arange(15)[:, None]
    o0, l0 = orc.forward(q, k, v, qo, ko, gq, gk, rope_q=pos * w, rope_k=pos * w)
    o1, l1 = orc.forward(q, k, v, qo, ko, gq, gk, rope_q=(pos + 37) * w, rope_k=(pos + 37) * w)
    np.testing.assert_allclose(o1, o0, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l1, l0, rtol=0, atol=1e-12)


def test_rope_backward_matches_central_finite_differences():
    rng = np.random.default_rng(54)
    q, k, v, gq, gk, qo, ko = rand_case(rng, 1, [2, 3], [1, 2, 3], 2, 1, 4)
    tq = rng.uniform(-2, 2, (5, 2))
    tk = rng.uniform(-2, 2, (6, 2))
    do = rng.standard_normal(q.shape)
    g = orc.backward(q, k, v, do, qo, ko, gq, gk, rope_q=tq, rope_k=tk)
    params = [q, k, v, gq, gk, tq, tk]

    def loss(pp):
        o, _ = orc.forward(pp[0], pp[1], pp[2], qo, ko, pp[3], pp[4], rope_q=pp[5], rope_k=pp[6])
        return float(np.sum(o * do))

    h = 1e-6
    for pi, name in enumerate(["dq", "dk", "dv", "dgamma_q", "dgamma_k", "drope_q", "drope_k"]):
        num = np.zeros_like(params[pi])
        it = np.nditer(params[pi], flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            pp = [p.copy() for p in params]
            pp[pi][idx] += h
            lp = loss(pp)
            pp[pi][idx] -= 2 * h
            num[idx] = (lp - loss(pp)) / (2 * h)
        np.testing.assert_allclose(g[name], num, rtol=1e-6, atol=1e-7, err_msg=name)


def test_rope_backward_rows_match_full_backward():
    rng = np.random.default_rng(55)
    q, k, v, gq, gk, qo, ko = rand_case(rng, 1, [5, 4, 6], [5, 4, 6], 4, 2, 8)
    tq = rng.uniform(-3, 3, (15, 4))
    tk = rng.uniform(-3, 3, (15, 4))
    do = rng.standard_normal(q.shape)
    full = orc.backward(q, k, v, do, qo, ko, gq, gk, rope_q=tq, rope_k=tk)
    rows, kv_rows = np.array([0, 6, 9, 14]), np.array([2, 7, 12])
    part = orc.backward_rows(q, k, v, do, qo, ko, gq, gk, q_rows=rows, kv_rows=kv_rows, rope_q=tq, rope_k=tk)
    np.testing.assert_allclose(part["dq"][0], full["dq"][0, rows], rtol=0, atol=1e-12)
    np.testing.assert_allclose(part["dk"][0], full["dk"][0, kv_rows], rtol=0, atol=1e-12)
    np.testing.assert_allclose(part["dv"][0], full["dv"][0, kv_rows], rtol=0, atol=1e-12)


def read_rope_fixture(name):
    cases, cur = [], {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            cur[key] = np.array([float(x) for x in vals])
            if key == "y":
                cases.append(cur)
                cur = {}
    return cases


def test_rope_matches_hand_written_quarter_turns():
    """Direction and pairing: a quarter turn of pair 0 sends e0 to e4 and e4 to
    -e0 (pairs are (i, i + D/2), turning counter-clockwise).  Rotating by -t
    or pairing (2i, 2i + 1) fails here."""
    cases = read_rope_fixture("rope_quarter_turn_d8.txt")
    assert len(cases) == 7
    for c in cases:
        x = c["x"].reshape(1, 1, 1, 8)          # [B, S, H, D]
        y = orc.rope(x, (np.pi * c["angles"]).reshape(1, 4))
        np.testing.assert_allclose(y.reshape(8), c["y"], rtol=0, atol=1e-14)


def torch_rope_reference(q, k, v, qo, ko, gq, gk, tq, tk, eps=1e-6, order="rope_then_norm"):
    """fp64 torch composition, independent of the oracle's rotation code: the
    pairs (x_i, x_{i+D/2}) as complex numbers multiplied by exp(i t)
    (torch.polar), then F.rms_norm with the gains, then SDPA with a boolean
    block-causal mask.  order="norm_then_rope" swaps the first two steps."""
    def rot(x, t):
        D = x.shape[-1]
        z = torch.complex(x[..., :D // 2], x[..., D // 2:])
        w = torch.polar(torch.ones_like(t), t)[None, :, None, :]   # [1, S, 1, D/2]
        r = z * w
        return torch.cat([r.real, r.imag], dim=-1)

    Q, K, V = (x if torch.is_tensor(x) else torch.tensor(x) for x in (q, k, v))
    D = Q.shape[-1]
    Gq, Gk = (x if torch.is_tensor(x) else torch.tensor(x) for x in (gq, gk))
    Tq, Tk = (x if torch.is_tensor(x) else torch.tensor(x) for x in (tq, tk))
    if order == "rope_then_norm":
        Qn = F.rms_norm(rot(Q, Tq), (D,), weight=Gq, eps=eps)
        Kn = F.rms_norm(rot(K, Tk), (D,), weight=Gk, eps=eps)
    else:
        Qn = rot(F.rms_norm(Q, (D,), weight=Gq, eps=eps), Tq)
        Kn = rot(F.rms_norm(K, (D,), weight=Gk, eps=eps), Tk)
    g = Q.shape[2] // K.shape[2]
    mask = torch.tensor(read_mask_like(qo, ko))
    o = F.scaled_dot_product_attention(Qn.transpose(1, 2), Kn.repeat_interleave(g, dim=2).transpose(1, 2),
                                       V.repeat_interleave(g, dim=2).transpose(1, 2), attn_mask=mask)
    return o.transpose(1, 2)


def test_rope_comes_before_the_norm_with_non_unit_gains():
    """Order against the norm (notes page, DiT-block sketch: RoPE on q and k,
    then QK-norm), with gains far from 1 so the two orders differ: the oracle
    equals rotate-then-RMSNorm and differs from RMSNorm-then-rotate."""
    rng = np.random.default_rng(56)
    q, k, v, gq, gk, qo, ko = rand_case(rng, 2, [5, 4, 6], [5, 4, 6], 4, 2, 16)
    gq = rng.uniform(0.2, 2.0, 16)
    gk = rng.uniform(0.2, 2.0, 16)
    tq = rng.uniform(-3, 3, (15, 8))
    tk = rng.uniform(-3, 3, (15, 8))
    o, _ = orc.forward(q, k, v, qo, ko, gq, gk, rope_q=tq, rope_k=tk)
    want = torch_rope_reference(q, k, v, qo, ko, gq, gk, tq, tk).numpy()
    np.testing.assert_allclose(o, want, rtol=0, atol=1e-12)
    other = torch_rope_reference(q, k, v, qo, ko, gq, gk, tq, tk, order="norm_then_rope").numpy()
    assert np.abs(other - want).max() > 1e-2


def test_rope_backward_matches_torch_autograd_fp64():
    """Every gradient, the angle gradients included, against torch autograd
    through the independent composition (complex rotation, F.rms_norm, SDPA)."""
    rng = np.random.default_rng(57)
    q, k, v, gq, gk, qo, ko = rand_case(rng, 2, [3, 5, 4], [3, 5, 4], 6, 2, 16)
    tq = rng.uniform(-3, 3, (12, 8))
    tk = rng.uniform(-3, 3, (12, 8))
    do = rng.standard_normal(q.shape)
    g = orc.backward(q, k, v, do, qo, ko, gq, gk, rope_q=tq, rope_k=tk)
    T = [torch.tensor(x, requires_grad=True) for x in (q, k, v, gq, gk, tq, tk)]
    o = torch_rope_reference(T[0], T[1], T[2], qo, ko, T[3], T[4], T[5], T[6])
    (o * torch.tensor(do)).sum().backward()
    for t, name in zip(T, ["dq", "dk", "dv", "dgamma_q", "dgamma_k", "drope_q", "drope_k"]):
        np.testing.assert_allclose(g[name], t.grad.numpy(), rtol=0, atol=1e-11, err_msg=name)
    np.testing.assert_allclose(g["out"], o.detach().numpy(), rtol=0, atol=1e-12)



# ------------------------------------------- packed samples and the global block

def loop_mask(q_lens, kv_lens, samples, n_global, kv_range=0):
    """Token-by-token mask from the rules as stated (independent of the
    oracle's vectorised construction): same sample and not a later chunk (and
    within the KV range), or a global key, or a global query."""
    nq, nkv = len(q_lens), len(kv_lens)
    kv_chunk = [c for c, n in enumerate(kv_lens) for _ in range(n)]
    q_own = [nkv - nq + c for c, n in enumerate(q_lens) for _ in range(n)]
    sample_of_chunk = {}
    for sidx in range(len(samples) - 1):
        for c in range(samples[sidx], samples[sidx + 1]):
            sample_of_chunk[c] = sidx
    first_global = nkv - n_global
    m = np.zeros((len(q_own), len(kv_chunk)), dtype=bool)
    for i, own in enumerate(q_own):
        for j, ck in enumerate(kv_chunk):
            same = sample_of_chunk[ck] == sample_of_chunk[own]
            in_range = ck <= own and (kv_range <= 0 or ck >= own - kv_range + 1)
            m[i, j] = (same and in_range) or ck >= first_global or own >= first_global
    return m


def test_packed_samples_equal_each_sample_alone():
    """Samples packed into one sequence give, row for row, what each sample
    gives on its own (forward and backward), with ragged chunks and GQA."""
    rng = np.random.default_rng(71)
    sample_chunks = [[5, 3], [4], [2, 6, 3]]
    lens = [n for sc in sample_chunks for n in sc]
    q, k, v, gq, gk, qo, ko = rand_case(rng, 2, lens, lens, 4, 2, 8)
    do = rng.standard_normal(q.shape)
    samples = offs([len(sc) for sc in sample_chunks])
    packed = orc.backward(q, k, v, do, qo, ko, gq, gk, samples=samples)
    t0 = 0
    dg = {"dgamma_q": 0.0, "dgamma_k": 0.0}
    for sc in sample_chunks:
        sl = slice(t0, t0 + sum(sc))
        o = offs(sc)
        alone = orc.backward(q[:, sl], k[:, sl], v[:, sl], do[:, sl], o, o, gq, gk)
        for nm in ("out", "dq", "dk", "dv"):
            np.testing.assert_allclose(packed[nm][:, sl], alone[nm], rtol=0, atol=1e-12, err_msg=nm)
        np.testing.assert_allclose(packed["lse"][:, :, sl], alone["lse"], rtol=0, atol=1e-12)
        for nm in dg:
            dg[nm] = dg[nm] + alone[nm]
        t0 += sum(sc)
    for nm in dg:
        np.testing.assert_allclose(packed[nm], dg[nm], rtol=0, atol=1e-11, err_msg=nm)


@pytest.mark.parametrize("kv_range", [0, 2])
def test_packed_global_block_matches_torch_sdpa_with_a_loop_mask(kv_range):
    rng = np.random.default_rng(72)
    lens = [3, 5, 2, 4, 6, 3]
    samples = [0, 2, 3, 6]            # chunks 0-1 | 2 | 3-5; chunk 5 is the global block
    q, k, v, gq, gk, qo, ko = rand_case(rng, 2, lens, lens, 6, 2, 16)
    o, _ = orc.forward(q, k, v, qo, ko, gq, gk, kv_range=kv_range, samples=samples, n_global=1)
    mask = torch.tensor(loop_mask(lens, lens, samples, 1, kv_range))
    np.testing.assert_allclose(o, torch_reference(q, k, v, qo, ko, gq, gk, mask=mask), rtol=0, atol=1e-12)


def test_packed_streaming_layout_matches_torch_sdpa_with_a_loop_mask():
    rng = np.random.default_rng(73)
    kv_lens, q_lens = [4, 3, 5, 2, 6], [2, 6]          # the query chunks are kv chunks 3 and 4
    samples = [0, 2, 5]                                 # kv chunks 0-1 | 2-4
    for n_global in (0, 1):
        q, k, v, gq, gk, qo, ko = rand_case(rng, 1, q_lens, kv_lens, 4, 1, 8)
        o, _ = orc.forward(q, k, v, qo, ko, gq, gk, samples=samples, n_global=n_global)
        mask = torch.tensor(loop_mask(q_lens, kv_lens, samples, n_global))
        np.testing.assert_allclose(o, torch_reference(q, k, v, qo, ko, gq, gk, mask=mask), rtol=0, atol=1e-12)


def test_other_samples_kv_does_not_change_a_sample_and_the_global_block_does():
    rng = np.random.default_rng(74)
    lens = [4, 4, 3, 5, 2]
    samples = [0, 2, 5]                                 # chunks 0-1 | 2-4
    q, k, v, gq, gk, qo, ko = rand_case(rng, 1, lens, lens, 2, 1, 8)
    o0, _ = orc.forward(q, k, v, qo, ko, gq, gk, samples=samples)
    k2, v2 = k.copy(), v.copy()
    k2[:, :8] = rng.standard_normal(k2[:, :8].shape)      # sample 0's keys and values
    v2[:, :8] = rng.standard_normal(v2[:, :8].shape)
    o1, _ = orc.forward(q, k2, v2, qo, ko, gq, gk, samples=samples)
    assert np.array_equal(o0[:, 8:], o1[:, 8:])            # sample 1 untouched
    assert not np.allclose(o0[:, :8], o1[:, :8])
    # with the last chunk global, changing its values changes every row
    g0, _ = orc.forward(q, k, v, qo, ko, gq, gk, samples=samples, n_global=1)
    v3 = v.copy()
    v3[:, 16:] += 1.0
    g1, _ = orc.forward(q, k, v3, qo, ko, gq, gk, samples=samples, n_global=1)
    assert np.all(np.abs(g1 - g0).max(axis=(0, 2, 3)) > 1e-6)


def test_one_sample_and_no_global_block_is_the_plain_mask():
    rng = np.random.default_rng(75)
    q, k, v, gq, gk, qo, ko = rand_case(rng, 1, [3, 5, 4], [3, 5, 4], 2, 1, 8)
    a, la = orc.forward(q, k, v, qo, ko, gq, gk)
    b, lb = orc.forward(q, k, v, qo, ko, gq, gk, samples=[0, 3], n_global=0)
    assert np.array_equal(a, b) and np.array_equal(la, lb)


def test_packed_global_backward_matches_central_finite_differences():
    rng = np.random.default_rng(76)
    lens = [2, 1, 2, 2]
    samples = [0, 1, 4]
    q, k, v, gq, gk, qo, ko = rand_case(rng, 1, lens, lens, 2, 1, 4)
    do = rng.standard_normal(q.shape)
    kw = dict(samples=samples, n_global=1, kv_range=2)
    g = orc.backward(q, k, v, do, qo, ko, gq, gk, **kw)
    params = [q, k, v, gq, gk]

    def loss(pp):
        o, _ = orc.forward(pp[0], pp[1], pp[2], qo, ko, pp[3], pp[4], **kw)
        return float(np.sum(o * do))

    h = 1e-6
    for pi, name in enumerate(["dq", "dk", "dv", "dgamma_q", "dgamma_k"]):
        num = np.zeros_like(params[pi])
        it = np.nditer(params[pi], flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            pp = [p.copy() for p in params]
            pp[pi][idx] += h
            lp = loss(pp)
            pp[pi][idx] -= 2 * h
            num[idx] = (lp - loss(pp)) / (2 * h)
        np.testing.assert_allclose(g[name], num, rtol=1e-6, atol=1e-7, err_msg=name)


def test_packed_global_backward_rows_match_full_backward():
    rng = np.random.default_rng(77)
    lens = [5, 4, 6, 3, 4]
    kw = dict(samples=[0, 2, 4, 5], n_global=1)
    q, k, v, gq, gk, qo, ko = rand_case(rng, 1, lens, lens, 4, 2, 8)
    do = rng.standard_normal(q.shape)
    full = orc.backward(q, k, v, do, qo, ko, gq, gk, **kw)
    rows, kv_rows = np.array([0, 6, 9, 15, 20]), np.array([2, 7, 12, 19, 21])
    part = orc.backward_rows(q, k, v, do, qo, ko, gq, gk, q_rows=rows, kv_rows=kv_rows, **kw)
    np.testing.assert_allclose(part["dq"][0], full["dq"][0, rows], rtol=0, atol=1e-12)
    np.testing.assert_allclose(part["dk"][0], full["dk"][0, kv_rows], rtol=0, atol=1e-12)
    np.testing.assert_allclose(part["dv"][0], full["dv"][0, kv_rows], rtol=0, atol=1e-12)
    fo, fl = orc.forward(q, k, v, qo, ko, gq, gk, **kw)
    po, pl = orc.forward_rows(q, k, v, qo, ko, gq, gk, rows, **kw)
    np.testing.assert_allclose(po, fo[:, rows], rtol=0, atol=1e-12)
