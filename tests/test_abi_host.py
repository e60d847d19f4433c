"""Host-only checks of the C ABI: the library loads without a GPU, exports
every symbol the header declares, rejects bad arguments before touching the
device, and its tile schedule covers exactly the unmasked (query, key) pairs."""
import ctypes
import os
import re

import numpy as np
import pytest

import block_causal_attention_gqa_b200 as bca
import workloads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "magi_bca.h")

OK, INVALID_ARG, UNSUPPORTED, BAD_OFFSETS, WS_SMALL, CUDA_ERROR, TIMEOUT, CHECK = 0, -1, -2, -3, -4, -5, -6, -7


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(magi_bca_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    lib = bca.library()
    names = declared_functions()
    assert set(names) == set(bca.EXPORTED_SYMBOLS)
    for n in names:
        assert hasattr(lib, n), n
    assert lib.magi_bca_version().startswith(b"magi_bca")


def test_status_strings():
    for code in (OK, INVALID_ARG, UNSUPPORTED, BAD_OFFSETS, WS_SMALL, CUDA_ERROR, TIMEOUT, CHECK):
        assert bca.magi_bca_status_string(code) != "unknown status"
    assert bca.magi_bca_status_string(12345) == "unknown status"


def _offs(lens):
    return np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)


def call_fwd(dims, qo, ko, ptr=256, null=None):
    """Calls magi_bca_fwd with fake (never dereferenced) pointers."""
    lib = bca.library()
    p = [ptr] * 7
    if null is not None:
        p[null] = None
    qo = np.ascontiguousarray(qo, dtype=np.int32)
    ko = np.ascontiguousarray(ko, dtype=np.int32)
    return lib.magi_bca_fwd(p[0], p[1], p[2], bca._i32p(qo), bca._i32p(ko), p[3], p[4], p[5], p[6],
                            ctypes.byref(dims), None)


def dims_for(qo, ko, B=1, Hq=4, Hkv=2, D=128, eps=1e-6, scale=0.0):
    return bca.make_dims(B, int(qo[-1]), int(ko[-1]), Hq, Hkv, D, len(qo) - 1, len(ko) - 1, scale, eps)


@pytest.mark.parametrize("case,expect", [
    ("null_q", INVALID_ARG), ("null_out", INVALID_ARG), ("misaligned", INVALID_ARG),
    ("batch0", INVALID_ARG), ("neg_eps", INVALID_ARG), ("nan_scale", INVALID_ARG),
    ("head_dim_96", UNSUPPORTED), ("gqa_indivisible", UNSUPPORTED),
    ("first_not_zero", BAD_OFFSETS), ("last_not_seqlen", BAD_OFFSETS), ("empty_chunk", BAD_OFFSETS),
    ("decreasing", BAD_OFFSETS), ("more_q_than_kv_chunks", BAD_OFFSETS), ("negative_kv_range", INVALID_ARG),
    ("deterministic_2", INVALID_ARG),
])
def test_invalid_arguments_are_rejected_on_the_host(case, expect):
    qo, ko = _offs([10, 20]), _offs([10, 20])
    d = dims_for(qo, ko)
    kw = {}
    if case == "null_q":
        kw["null"] = 0
    elif case == "null_out":
        kw["null"] = 5
    elif case == "misaligned":
        kw["ptr"] = 258
    elif case == "batch0":
        d.batch = 0
    elif case == "neg_eps":
        d.rms_eps = -1.0
    elif case == "nan_scale":
        d.softmax_scale = float("nan")
    elif case == "head_dim_96":
        d.head_dim = 96
    elif case == "gqa_indivisible":
        d.heads_q, d.heads_kv = 6, 4
    elif case == "first_not_zero":
        qo = np.array([1, 10, 30], np.int32)
    elif case == "last_not_seqlen":
        d.seqlen_q = 31
    elif case == "empty_chunk":
        qo, ko = _offs([10, 0, 20]), _offs([10, 0, 20])
        d = dims_for(qo, ko)
    elif case == "decreasing":
        qo = np.array([0, 20, 10, 30], np.int32)
        ko = qo.copy()
        d = dims_for(_offs([10, 10, 10]), _offs([10, 10, 10]))
    elif case == "more_q_than_kv_chunks":
        qo, ko = _offs([10, 10, 10]), _offs([15, 15])
        d = dims_for(qo, ko)
    elif case == "negative_kv_range":
        d.kv_range = -1
    elif case == "deterministic_2":
        d.deterministic = 2
    assert call_fwd(d, qo, ko, **kw) == expect


def test_matched_chunks_of_different_lengths_are_accepted():
    """Cross-attention: query chunks may differ in length from their kv chunks."""
    for q_lens, kv_lens in (([1000], [333]), ([300, 200, 250], [77, 120, 64]), ([10, 20], [5, 15, 10])):
        qo, ko = _offs(q_lens), _offs(kv_lens)
        assert call_fwd(dims_for(qo, ko), qo, ko) not in (INVALID_ARG, BAD_OFFSETS)


def test_valid_arguments_reach_the_device_check():
    """With valid arguments and no usable sm_100 device the call fails with
    a CUDA or unsupported status (never OK, never a host-side argument code)."""
    qo, ko = _offs([10, 20]), _offs([10, 20])
    st = call_fwd(dims_for(qo, ko), qo, ko)
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:
        has_gpu = False
    if not has_gpu:
        assert st in (CUDA_ERROR, UNSUPPORTED)


def test_bwd_workspace_size_rejects_bad_dims():
    d = dims_for(_offs([10]), _offs([10]))
    d.head_dim = 0
    assert bca.magi_bca_bwd_workspace_size(d) == 0


# ------------------------------------------------------------ the schedule

def row_ends(qo, ko, Sq):
    nq, nkv = len(qo) - 1, len(ko) - 1
    ends = np.empty(Sq, np.int64)
    for c in range(nq):
        ends[qo[c]:qo[c + 1]] = ko[nkv - nq + c + 1]
    return ends


def row_intervals(qo, ko, kv_range=0, samples=None, n_global=0):
    """Per query row the visible keys [begin, end) by the block-causal rule: its
    matched kv chunk's end, and the start of the chunk R - 1 before it (KV
    range R) or of its sample, whichever is later; rows of the global block's
    query chunks see [0, Skv).  Also returns the first global key g0 (every row
    sees [g0, Skv)).  Checked against the oracle's token-level mask below."""
    nq, nkv = len(qo) - 1, len(ko) - 1
    Sq = int(qo[-1])
    first_global = nkv - n_global
    sample_first = np.zeros(nkv, np.int64)
    if samples is not None:
        for i in range(len(samples) - 1):
            sample_first[samples[i]:samples[i + 1]] = samples[i]
    begin = np.zeros(Sq, np.int64)
    end = np.empty(Sq, np.int64)
    for c in range(nq):
        own = nkv - nq + c
        if own >= first_global:
            begin[qo[c]:qo[c + 1]] = 0
            end[qo[c]:qo[c + 1]] = ko[-1]
            continue
        first = sample_first[own]
        if kv_range > 0:
            first = max(first, own - kv_range + 1)
        end[qo[c]:qo[c + 1]] = ko[own + 1]
        begin[qo[c]:qo[c + 1]] = ko[first]
    return begin, end, int(ko[first_global])


class TileMask:
    """any()/all() of the visibility of a (query rows, keys) block: a row sees
    [begin, end) and the global keys [g0, Skv)."""

    def __init__(self, qo, ko, kv_range=0, samples=None, n_global=0):
        self.begin, self.end, self.g0 = row_intervals(qo, ko, kv_range, samples, n_global)
        self.Sq, self.Skv = int(qo[-1]), int(ko[-1])

    def _any(self, b, e, k0, k1):
        return ((b < k1) & (e > k0)) | (self.g0 < k1)

    def _all(self, b, e, k0, k1):
        # [k0, k1) inside [b, e) | [g0, Skv) (k1 <= Skv)
        return ((b <= k0) & (e >= k1)) | (self.g0 <= k0) | ((b <= k0) & (e >= self.g0))

    def any(self, r0, r1, k0, k1):
        b, e = self.begin[r0:min(r1, self.Sq)], self.end[r0:min(r1, self.Sq)]
        return bool(self._any(b, e, k0, min(k1, self.Skv)).any())

    def all(self, r0, r1, k0, k1):
        b, e = self.begin[r0:min(r1, self.Sq)], self.end[r0:min(r1, self.Sq)]
        return bool(self._all(b, e, k0, min(k1, self.Skv)).all())

    def any_tiles(self, r0, r1, n_tiles):
        """any() for key tiles 0..n_tiles-1 at once (128-key tiles)."""
        b, e = self.begin[r0:min(r1, self.Sq)], self.end[r0:min(r1, self.Sq)]
        k0 = np.arange(n_tiles) * 128
        k1 = np.minimum(k0 + 128, self.Skv)
        return self._any(b[:, None], e[:, None], k0[None, :], k1[None, :]).any(axis=0)

    def any_row_tiles(self, n_qt, k0, k1):
        """any() for query tiles 0..n_qt-1 at once against keys [k0, k1)."""
        hit = self._any(self.begin, self.end, k0, min(k1, self.Skv))
        pad = np.zeros(n_qt * 128, bool)
        pad[:self.Sq] = hit
        return pad.reshape(n_qt, 128).any(axis=1)

    def all_row_tiles(self, n_qt, k0, k1):
        """all() for query tiles 0..n_qt-1 at once against keys [k0, k1) (rows past Sq ignored)."""
        ok = self._all(self.begin, self.end, k0, min(k1, self.Skv))
        pad = np.ones(n_qt * 128, bool)
        pad[:self.Sq] = ok
        return pad.reshape(n_qt, 128).all(axis=1)


def interval_mask(qo, ko, kv_range=0, samples=None, n_global=0):
    b, e, g0 = row_intervals(qo, ko, kv_range, samples, n_global)
    keys = np.arange(int(ko[-1]))
    return ((keys[None, :] >= b[:, None]) & (keys[None, :] < e[:, None])) | (keys[None, :] >= g0)


@pytest.mark.parametrize("q_lens,kv_lens,R", [([2, 3, 1], [2, 3, 1], 0), ([2, 3, 1], [2, 3, 1], 2),
                                              ([3, 2], [1, 2, 3, 2], 2), ([1] * 9, [1] * 9, 3)])
def test_row_intervals_match_the_oracle_mask(q_lens, kv_lens, R):
    from oracle import bca_oracle as orc
    qo, ko = _offs(q_lens), _offs(kv_lens)
    assert np.array_equal(orc.block_causal_mask(qo, ko, kv_range=R), interval_mask(qo, ko, R))


@pytest.mark.parametrize("q_lens,kv_lens,R,samples,G", [
    ([2, 1, 2, 1, 2], [2, 1, 2, 1, 2], 0, [0, 2, 3, 5], 0),
    ([2, 1, 2, 1, 2], [2, 1, 2, 1, 2], 0, [0, 2, 3, 5], 1),
    ([2, 1], [2, 1, 2, 1], 0, [0, 2, 4], 0),
    ([1] * 5, [1] * 5, 2, [0, 3, 5], 1),
    ([3, 4, 2, 5], [3, 4, 2, 5], 0, None, 2),
    ([2, 3], [4, 2, 3], 0, [0, 1, 3], 2),
])
def test_row_intervals_with_samples_and_global_block_match_the_oracle_mask(q_lens, kv_lens, R, samples, G):
    from oracle import bca_oracle as orc
    qo, ko = _offs(q_lens), _offs(kv_lens)
    want = orc.block_causal_mask(qo, ko, kv_range=R, samples=samples, n_global=G)
    assert np.array_equal(want, interval_mask(qo, ko, R, samples, G))


def check_schedule(q_lens, kv_lens, B, Hq, Hkv, D=128, kv_range=0, samples=None, n_global=0):
    qo, ko = _offs(q_lens), _offs(kv_lens)
    Sq, Skv = int(qo[-1]), int(ko[-1])
    units = bca.magi_bca_fwd_schedule(qo, ko, B, Hq, Hkv, D, kv_range=kv_range, samples=samples,
                                      n_global=n_global)
    assert units.shape[1] == 12
    M = TileMask(qo, ko, kv_range, samples, n_global)
    n_kt = -(-Skv // 128)
    g = Hq // Hkv
    seen = np.zeros((B, Hq, (Sq + 127) // 128), np.int64)
    costs = []
    checked = set()   # visibility depends only on the query tile, not on batch or head
    for b, hk, h0, m00, h1, m01, n_full, n_tiles, t_begin, t_full_begin, g_begin, g_end in units:
        assert 0 <= g_begin <= g_end <= n_kt and (g_begin == g_end == 0 or g_begin >= n_tiles)
        subs = [(h0, m00)] + ([(h1, m01)] if h1 >= 0 else [])
        for h, m0 in subs:
            assert h // g == hk and m0 % 128 == 0
            seen[b, h, m0 // 128] += 1
            key = (m0, n_full, n_tiles, t_begin, t_full_begin, g_begin, g_end)
            if key in checked:
                continue
            checked.add(key)
            tiles_seen = list(np.nonzero(M.any_tiles(m0, m0 + 128, n_kt))[0])
            # exactly the tiles with some visible (row, key) pair are visited
            visited = list(range(t_begin, n_tiles)) + list(range(g_begin, g_end))
            assert tiles_seen == visited, (tiles_seen, t_begin, n_tiles, g_begin, g_end)
            # tiles the kernel leaves unmasked are fully visible to every row
            for t in range(max(t_begin, t_full_begin), min(n_full, n_tiles)):
                assert M.all(m0, m0 + 128, t * 128, t * 128 + 128), t
            g0 = M.g0
            for t in range(g_begin, g_end):
                if not (t * 128 < g0 or t * 128 + 128 > Skv):
                    assert M.all(m0, m0 + 128, t * 128, t * 128 + 128), t
        costs.append((n_tiles - t_begin + g_end - g_begin) * len(subs))
    # every (batch, head, query tile) exactly once
    assert (seen == 1).all()
    # longest first
    assert all(a >= b for a, b in zip(costs, costs[1:]))
    return units


@pytest.mark.parametrize("q_lens,kv_lens,B,Hq,Hkv", [
    ([64, 64], [64, 64], 1, 2, 1),
    ([1024] * 4, [1024] * 4, 1, 16, 4),
    ([5760] * 8, [5760] * 8, 1, 24, 8),
    ([5760] * 4, [5760] * 16, 2, 24, 8),
    ([100, 333, 1000, 67], [100, 333, 1000, 67], 2, 4, 2),
    ([150, 250], [300, 200, 150, 250], 2, 8, 2),
    ([1] * 37, [1] * 37, 1, 2, 1),
    ([777], [777], 1, 3, 1),
])
def test_fwd_schedule_covers_each_query_tile_once_with_correct_extents(q_lens, kv_lens, B, Hq, Hkv):
    check_schedule(q_lens, kv_lens, B, Hq, Hkv)


@pytest.mark.parametrize("q_lens,kv_lens,R", [
    ([64, 64, 64], [64, 64, 64], 1),
    ([300, 200, 150, 250, 100], [300, 200, 150, 250, 100], 2),
    ([150, 250], [300, 200, 150, 250], 2),
    ([1024] * 8, [1024] * 8, 3),
    ([1] * 37, [1] * 37, 5),
    ([5760] * 4, [5760] * 16, 8),
    ([1000], [333], 0),                    # cross-attention against a text sequence
    ([77], [1000], 0),
    ([300, 200, 250], [77, 120, 64], 1),   # chunk-wise text conditioning
])
def test_fwd_schedule_with_kv_range(q_lens, kv_lens, R):
    check_schedule(q_lens, kv_lens, 2, 8, 2, kv_range=R)


def test_aligned_chunks_need_no_mask():
    # chunk lengths that are multiples of 128 never straddle a tile
    units = check_schedule([1024] * 4, [1024] * 4, 1, 16, 4)
    assert (units[:, 6] == units[:, 7]).all()
    units = check_schedule([5760] * 4, [5760] * 16, 2, 24, 8)
    assert (units[:, 6] == units[:, 7]).all()


def test_paired_sub_tiles_share_extent_and_kv_head():
    units = check_schedule([5760] * 8, [5760] * 8, 1, 24, 8)
    paired = units[units[:, 4] >= 0]
    assert len(paired) >= 0.95 * len(units)
    assert (paired[:, 2] // 3 == paired[:, 1]).all() and (paired[:, 4] // 3 == paired[:, 1]).all()


def test_workload_shapes():
    w = workloads.workload("model46k")
    assert (w.seqlen_q, w.heads_q, w.heads_kv, w.head_dim) == (46080, 24, 8, 128)
    w = workloads.workload("stream4of16")
    assert (w.batch, w.seqlen_q, w.seqlen_kv) == (2, 23040, 92160)


def check_bwd_schedule(q_lens, kv_lens, B, Hq, Hkv, num_sms=148, kv_range=0, deterministic=False, samples=None,
                       n_global=0):
    qo, ko = _offs(q_lens), _offs(kv_lens)
    Sq, Skv = int(qo[-1]), int(ko[-1])
    G = Hq // Hkv
    units = bca.magi_bca_bwd_schedule(qo, ko, B, Hq, Hkv, 128, num_sms, kv_range=kv_range,
                                      deterministic=deterministic, samples=samples, n_global=n_global)
    assert units.shape[1] == 12
    M = TileMask(qo, ko, kv_range, samples, n_global)
    n_qt, n_kt = -(-Sq // 128), -(-Skv // 128)
    cover = np.zeros((B, Hkv, n_kt, n_qt, G), np.int64)
    lengths = []
    tile_any, tile_all = {}, {}
    for b, hk, n0, s0, s1, diag_end, diag_hi_begin, split, jump, diag_global, z0, z1 in units:
        assert z0 == 0 and z1 == 0 and jump >= 0
        assert n0 % 128 == 0 and s0 < s1
        if n0 not in tile_any:
            tile_any[n0] = M.any_row_tiles(n_qt, n0, n0 + 128)
            tile_all[n0] = M.all_row_tiles(n_qt, n0, n0 + 128)
        v = np.arange(s0, s1, dtype=np.int64)
        first = v < split
        steps = np.where(first, v, v + jump)
        assert (steps >= 0).all() and (steps < n_qt * G).all()
        t, g = steps // G, steps % G
        np.add.at(cover, (b, hk, n0 // 128, t, g), 1)
        assert tile_any[n0][t].all()                         # some row of each tile sees some key
        masked = np.where(first, (t < diag_end) | (t >= diag_hi_begin), t == diag_global)
        assert tile_all[n0][t[~masked]].all(), (n0, diag_end, diag_hi_begin, diag_global)   # unmasked: all visible
        lengths.append(s1 - s0)
    # every (kv tile, query tile, head) with a visible pair: exactly once
    for kt in range(n_kt):
        want = M.any_row_tiles(n_qt, kt * 128, kt * 128 + 128).astype(np.int64)
        assert (cover[:, :, kt, :, :] == want[None, None, :, None]).all(), kt
    assert all(a >= b for a, b in zip(lengths, lengths[1:]))
    return units


@pytest.mark.parametrize("q_lens,kv_lens,B,Hq,Hkv", [
    ([64, 64], [64, 64], 1, 2, 1),
    ([1024] * 4, [1024] * 4, 1, 16, 4),
    ([100, 333, 1000, 67], [100, 333, 1000, 67], 2, 4, 2),
    ([150, 250], [300, 200, 150, 250], 2, 8, 2),
    ([1] * 37, [1] * 37, 1, 2, 1),
    ([5760] * 4, [5760] * 16, 2, 24, 8),
])
def test_bwd_schedule_covers_each_visible_step_once(q_lens, kv_lens, B, Hq, Hkv):
    check_bwd_schedule(q_lens, kv_lens, B, Hq, Hkv)


@pytest.mark.parametrize("q_lens,kv_lens,R", [
    ([64, 64, 64], [64, 64, 64], 1),
    ([300, 200, 150, 250, 100], [300, 200, 150, 250, 100], 2),
    ([150, 250], [300, 200, 150, 250], 2),
    ([1024] * 8, [1024] * 8, 3),
    ([1] * 37, [1] * 37, 5),
    ([5760] * 4, [5760] * 16, 8),
    ([1000], [333], 0),
    ([77], [1000], 0),
    ([300, 200, 250], [77, 120, 64], 1),
])
def test_bwd_schedule_with_kv_range(q_lens, kv_lens, R):
    check_bwd_schedule(q_lens, kv_lens, 2, 8, 2, kv_range=R)


@pytest.mark.parametrize("q_lens,kv_lens,B,Hq,Hkv,R", [
    ([1024] * 4, [1024] * 4, 1, 16, 4, 0),
    ([100, 333, 1000, 67], [100, 333, 1000, 67], 2, 4, 2, 0),
    ([150, 250], [300, 200, 150, 250], 2, 8, 2, 0),
    ([300, 200, 150, 250, 100], [300, 200, 150, 250, 100], 1, 8, 2, 2),
    ([1] * 37, [1] * 37, 1, 2, 1, 5),
])
def test_deterministic_bwd_schedule_has_one_unit_per_kv_tile(q_lens, kv_lens, B, Hq, Hkv, R):
    """The deterministic backward writes each kv tile's dV and G_k from exactly
    one CTA: every (batch, kv head, kv tile) is one unit holding all its steps."""
    units = check_bwd_schedule(q_lens, kv_lens, B, Hq, Hkv, kv_range=R, deterministic=True)
    keys = [tuple(u[:3]) for u in units]
    assert len(keys) == len(set(keys))
    pieces = check_bwd_schedule(q_lens, kv_lens, B, Hq, Hkv, num_sms=148, kv_range=R)
    for key in set(keys):
        mine = [u for u in pieces if tuple(u[:3]) == key]
        whole = [u for u in units if tuple(u[:3]) == key][0]
        assert min(u[3] for u in mine) == whole[3] and max(u[4] for u in mine) == whole[4]


def test_dims_struct_layout():
    """magi_bca_dims: ten 4-byte fields, then kv_range, deterministic, n_samples,
    n_global_chunks, and the host pointer to the sample offsets."""
    assert ctypes.sizeof(bca.Dims) == 64
    assert bca.Dims.kv_range.offset == 40 and bca.Dims.deterministic.offset == 44
    assert bca.Dims.n_samples.offset == 48 and bca.Dims.n_global_chunks.offset == 52
    assert bca.Dims.sample_chunk_offsets.offset == 56
    assert bca.make_dims(1, 8, 8, 2, 1, 64, 1, 1, deterministic=True).deterministic == 1


def lpt_span(costs, machines):
    import heapq
    load = [0.0] * machines
    for c in sorted(costs, reverse=True):
        heapq.heapreplace(load, load[0] + c)
    return max(load)


def test_bwd_schedule_balances_the_sms():
    """train4k: 128 kv tiles with 32, 24, 16 or 8 visible query tiles x 4 heads.
    Whole tiles (or the earlier 8-query-tile pieces: 320 units, three waves)
    leave SMs idle; the step-granular pieces must come within 15% of perfect
    balance, counting two steps of overhead per piece."""
    units = check_bwd_schedule([1024] * 4, [1024] * 4, 1, 16, 4)
    steps = units[:, 4] - units[:, 3]
    assert steps.sum() == 4 * 8 * (32 + 24 + 16 + 8) * 4
    span = lpt_span(list(steps + 2.0), 148)
    ideal = (steps.sum() + 2.0 * len(steps)) / 148
    assert span <= 1.15 * ideal, (span, ideal, len(steps))
    old = lpt_span([32 + 2.0] * 320, 148)
    assert span < 0.85 * old
    # a problem with far more work than SMs is left in whole kv tiles
    big = check_bwd_schedule([5760] * 8, [5760] * 8, 1, 24, 8)
    assert len(big) == 8 * 360


def test_profile_events_argument_check():
    lib = bca.library()
    assert lib.magi_bca_profile_events(256, None) == INVALID_ARG
    assert lib.magi_bca_profile_events(None, 256) == INVALID_ARG
    assert lib.magi_bca_profile_events(None, None) == OK


@pytest.mark.parametrize("entry", ["fwd", "fwd_rope", "bwd", "bwd_rope", "bwd_noalloc"])
def test_no_cpu_fallback_host_tensors_are_refused(entry):
    """The product path has no CPU or PyTorch fallback: every entry point
    refuses host tensors before anything is computed."""
    import torch
    B, S, H, D = 1, 128, 2, 64
    q = torch.zeros(B, S, H, D, dtype=torch.bfloat16)
    k = torch.zeros(B, S, 1, D, dtype=torch.bfloat16)
    v = torch.zeros_like(k)
    g = torch.ones(D)
    lse = torch.zeros(B, H, S)
    ang = torch.zeros(S, D // 2)
    offs = [0, 64, 128]
    calls = {
        "fwd": lambda: bca.magi_bca_fwd(q, k, v, offs, offs, g, g),
        "fwd_rope": lambda: bca.magi_bca_fwd_rope(q, k, v, offs, offs, g, g, ang, ang),
        "bwd": lambda: bca.magi_bca_bwd(q, k, v, q, q, lse, offs, offs, g, g),
        "bwd_rope": lambda: bca.magi_bca_bwd_rope(q, k, v, q, q, lse, offs, offs, g, g, ang, ang),
        "bwd_noalloc": lambda: bca.magi_bca_bwd_noalloc(q, k, v, q, q, lse, offs, offs, g, g, q, k, v),
    }
    with pytest.raises(TypeError, match="CUDA tensor"):
        calls[entry]()


def test_tensors_on_another_device_are_refused():
    """A call runs on q's device; a tensor elsewhere (another GPU, the host)
    is refused before any pointer reaches a kernel."""
    import torch
    here = torch.device("cuda", 0)
    t0 = torch.zeros(4)
    with pytest.raises(ValueError, match="gamma_k is on cpu"):
        bca._check_same_device(here, (("gamma_k", t0),))
    bca._check_same_device(torch.device("cpu"), (("k", t0), ("lse", None)))


def random_layouts(seed, n):
    """Seeded random chunk layouts: 1-6 kv chunks of 1-700 tokens (rarely tile
    aligned), the query side the last 1..n_kv of them (training layout when all)
    or, one time in four, chunks of other lengths (cross-attention), a KV range
    of 0-3, batch 1-2 and a GQA ratio of 1-4."""
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(n):
        n_kv = int(rng.integers(1, 7))
        kv = [int(x) for x in rng.integers(1, 701, n_kv)]
        n_q = int(rng.integers(1, n_kv + 1))
        if rng.random() < 0.25:
            q = [int(x) for x in rng.integers(1, 701, n_q)]
        else:
            q = kv[n_kv - n_q:]
        hkv = int(rng.integers(1, 3))
        out.append((q, kv, int(rng.integers(1, 3)), hkv * int(rng.integers(1, 5)), hkv, int(rng.integers(0, 4))))
    return out


@pytest.mark.parametrize("q_lens,kv_lens,B,Hq,Hkv,R", random_layouts(2024, 24))
def test_schedules_on_random_layouts(q_lens, kv_lens, B, Hq, Hkv, R):
    """Both schedules against the oracle's token mask (through the row
    intervals) on random layouts: the forward visits exactly the kv tiles with
    a visible pair and masks every tile it does not see whole; the backward
    covers each visible (kv tile, query tile, head) once, pieced and whole."""
    from oracle import bca_oracle as orc
    qo, ko = _offs(q_lens), _offs(kv_lens)
    assert np.array_equal(orc.block_causal_mask(qo, ko, kv_range=R), interval_mask(qo, ko, R))
    check_schedule(q_lens, kv_lens, B, Hq, Hkv, kv_range=R)
    check_bwd_schedule(q_lens, kv_lens, B, Hq, Hkv, kv_range=R)
    check_bwd_schedule(q_lens, kv_lens, B, Hq, Hkv, kv_range=R, deterministic=True)
    check_bwd_schedule(q_lens, kv_lens, B, Hq, Hkv, num_sms=7, kv_range=R)


def test_maximum_sizes():
    """The kernels index rows with 32-bit TMA coordinates and flattened 32-bit
    row numbers: a problem with 2^31 or more query (or key) rows is refused on
    the host; one just below the limit passes the checks."""
    lib = bca.library()
    # 2^31 query rows: batch 1, 2^27 tokens, 16 heads
    S = 1 << 27
    qo = np.array([0, S], np.int32)
    d = bca.make_dims(1, S, S, 16, 2, 128, 1, 1)
    assert lib.magi_bca_fwd_schedule(bca._i32p(qo), bca._i32p(qo), ctypes.byref(d), None, 0) == UNSUPPORTED
    assert bca.magi_bca_bwd_workspace_size(d) == 0
    # just below: 2^31 - 16 query rows pass the same checks (the workspace query
    # runs them without building the 8-million-unit schedule)
    S2 = (1 << 27) - 1
    d2 = bca.make_dims(1, S2, S2, 16, 2, 128, 1, 1)
    ws = bca.magi_bca_bwd_workspace_size(d2)
    assert ws >= S2 * 16 * 128 * (2 + 4)   # at least Q^ (bf16) and the fp32 dq accumulator


def random_packed_layouts(seed, n):
    """Seeded random packed layouts: 1-4 samples of 1-4 chunks of 1-600 tokens,
    the training layout or (one time in three) the streaming one (the query
    side the last 1..n_kv chunks), a KV range of 0-3, a global block of 0-2
    trailing kv chunks, batch 1-2 and a GQA ratio of 1-4."""
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(n):
        sample_chunks = [int(rng.integers(1, 5)) for _ in range(int(rng.integers(1, 5)))]
        n_kv = sum(sample_chunks)
        kv = [int(x) for x in rng.integers(1, 601, n_kv)]
        n_q = n_kv if rng.random() < 2 / 3 else int(rng.integers(1, n_kv + 1))
        samples = [int(x) for x in np.concatenate([[0], np.cumsum(sample_chunks)])]
        hkv = int(rng.integers(1, 3))
        out.append((kv[n_kv - n_q:], kv, int(rng.integers(1, 3)), hkv * int(rng.integers(1, 5)), hkv,
                    int(rng.integers(0, 4)), samples, int(rng.integers(0, min(2, n_kv) + 1))))
    return out


@pytest.mark.parametrize("q_lens,kv_lens,B,Hq,Hkv,R,samples,G", random_packed_layouts(2025, 24))
def test_schedules_on_random_packed_layouts_with_global_blocks(q_lens, kv_lens, B, Hq, Hkv, R, samples, G):
    """Packed samples and a last global block (MAGI-1 §4.1.2, Figure 15 (f), (g)):
    the interval form of the mask equals the oracle's token mask, the forward
    visits exactly the kv tiles with a visible pair (both ranges) and masks every
    tile it does not see whole, and the backward covers each visible (kv tile,
    query tile, head) once, pieced and whole."""
    from oracle import bca_oracle as orc
    qo, ko = _offs(q_lens), _offs(kv_lens)
    assert np.array_equal(orc.block_causal_mask(qo, ko, kv_range=R, samples=samples, n_global=G),
                          interval_mask(qo, ko, R, samples, G))
    kw = dict(kv_range=R, samples=samples, n_global=G)
    check_schedule(q_lens, kv_lens, B, Hq, Hkv, **kw)
    check_bwd_schedule(q_lens, kv_lens, B, Hq, Hkv, **kw)
    check_bwd_schedule(q_lens, kv_lens, B, Hq, Hkv, deterministic=True, **kw)
    check_bwd_schedule(q_lens, kv_lens, B, Hq, Hkv, num_sms=7, **kw)


@pytest.mark.parametrize("case,expect", [("samples_not_covering", BAD_OFFSETS), ("samples_empty", BAD_OFFSETS),
                                         ("samples_null", INVALID_ARG), ("global_too_many", BAD_OFFSETS),
                                         ("global_negative", INVALID_ARG), ("samples_negative", INVALID_ARG)])
def test_bad_samples_and_global_blocks_are_rejected_on_the_host(case, expect):
    qo = ko = _offs([10, 20, 5])
    kw = {}
    if case == "samples_not_covering":
        kw = dict(samples=[0, 1, 2])
    elif case == "samples_empty":
        kw = dict(samples=[0, 1, 1, 3])
    elif case == "global_too_many":
        kw = dict(n_global=4)
    elif case == "global_negative":
        kw = dict(n_global=-1)
    d = bca.make_dims(1, 35, 35, 4, 2, 128, 3, 3, **kw)
    if case == "samples_null":
        d.n_samples = 2
        d.sample_chunk_offsets = None
    elif case == "samples_negative":
        d.n_samples = -1
    assert call_fwd(d, qo, ko) == expect
