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

OK, INVALID_ARG, UNSUPPORTED, BAD_OFFSETS, WS_SMALL, CUDA_ERROR, TIMEOUT = 0, -1, -2, -3, -4, -5, -6


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
    for code in (OK, INVALID_ARG, UNSUPPORTED, BAD_OFFSETS, WS_SMALL, CUDA_ERROR, TIMEOUT):
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
    ("decreasing", BAD_OFFSETS), ("more_q_than_kv_chunks", BAD_OFFSETS), ("unmatched_lengths", BAD_OFFSETS),
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
    elif case == "unmatched_lengths":
        qo, ko = _offs([10, 20]), _offs([5, 15, 10])
        d = dims_for(qo, ko)
    assert call_fwd(d, qo, ko, **kw) == expect


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


def check_schedule(q_lens, kv_lens, B, Hq, Hkv, D=128):
    qo, ko = _offs(q_lens), _offs(kv_lens)
    Sq, Skv = int(qo[-1]), int(ko[-1])
    units = bca.magi_bca_fwd_schedule(qo, ko, B, Hq, Hkv, D)
    ends = row_ends(qo, ko, Sq)
    g = Hq // Hkv
    seen = np.zeros((B, Hq, (Sq + 127) // 128), np.int64)
    costs = []
    for b, hk, h0, m00, h1, m01, n_full, n_tiles in units:
        subs = [(h0, m00)] + ([(h1, m01)] if h1 >= 0 else [])
        for h, m0 in subs:
            assert h // g == hk and m0 % 128 == 0
            seen[b, h, m0 // 128] += 1
            rows = ends[m0:min(m0 + 128, Sq)]
            # tiles [0, n_full) fully visible to every row; tile n_full.. needs the mask
            assert n_full == rows.min() // 128
            assert n_tiles == -(-rows.max() // 128)
            assert n_tiles * 128 >= rows.max() and (n_tiles - 1) * 128 < rows.max()
            # no visited tile is fully masked for every row
            assert (n_tiles - 1) * 128 < rows.max()
        costs.append(n_tiles * len(subs))
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


def check_bwd_schedule(q_lens, kv_lens, B, Hq, Hkv, num_sms=148):
    qo, ko = _offs(q_lens), _offs(kv_lens)
    Sq, Skv = int(qo[-1]), int(ko[-1])
    G = Hq // Hkv
    units = bca.magi_bca_bwd_schedule(qo, ko, B, Hq, Hkv, 128, num_sms)
    ends = row_ends(qo, ko, Sq)
    n_qt, n_kt = -(-Sq // 128), -(-Skv // 128)
    cover = np.zeros((B, Hkv, n_kt, n_qt, G), np.int64)
    lengths = []
    for b, hk, n0, s0, s1, diag_end, _, _ in units:
        assert n0 % 128 == 0 and 0 <= s0 < s1 <= n_qt * G
        n_end = min(n0 + 128, Skv)
        for s in range(s0, s1):
            t, g = divmod(s, G)
            cover[b, hk, n0 // 128, t, g] += 1
            rows = ends[t * 128:min(t * 128 + 128, Sq)]
            assert (rows > n0).any()                  # some row of the tile sees some key
            assert (rows.min() < n_end) == (t < diag_end), (t, diag_end)
        lengths.append(s1 - s0)
    # every (kv tile, query tile, head) where some query sees some key: exactly once
    for kt in range(n_kt):
        for t in range(n_qt):
            want = int((ends[t * 128:min(t * 128 + 128, Sq)] > kt * 128).any())
            assert (cover[:, :, kt, t, :] == want).all(), (kt, t)
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
