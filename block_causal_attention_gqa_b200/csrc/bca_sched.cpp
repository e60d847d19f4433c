// Host-side argument checks and the chunk-aware tile scheduler (see bca_sched.h).
#include "bca_sched.h"

#include "bca_kernels.h"

#include <algorithm>
#include <cmath>
#include <functional>
#include <queue>
#include <tuple>

namespace magi {

int validate_dims(const magi_bca_dims* dims) {
  if (dims == nullptr) return MAGI_BCA_INVALID_ARG;
  const magi_bca_dims& d = *dims;
  if (d.batch <= 0 || d.seqlen_q <= 0 || d.seqlen_kv <= 0 || d.heads_q <= 0 || d.heads_kv <= 0 ||
      d.head_dim <= 0 || d.n_q_chunks <= 0 || d.n_kv_chunks <= 0)
    return MAGI_BCA_INVALID_ARG;
  if (!(d.rms_eps >= 0.f) || !std::isfinite(d.rms_eps)) return MAGI_BCA_INVALID_ARG;
  if (!(d.softmax_scale >= 0.f) || !std::isfinite(d.softmax_scale)) return MAGI_BCA_INVALID_ARG;
  if (d.kv_range < 0) return MAGI_BCA_INVALID_ARG;
  if (d.deterministic != 0 && d.deterministic != 1) return MAGI_BCA_INVALID_ARG;
  if (d.head_dim != 64 && d.head_dim != 128) return MAGI_BCA_UNSUPPORTED;
  if (d.heads_q % d.heads_kv != 0) return MAGI_BCA_UNSUPPORTED;
  if (d.n_q_chunks > d.n_kv_chunks) return MAGI_BCA_BAD_OFFSETS;
  // TMA coordinates and the flattened index arithmetic are 32-bit.
  const int64_t rows_q = (int64_t)d.batch * d.seqlen_q * d.heads_q;
  const int64_t rows_kv = (int64_t)d.batch * d.seqlen_kv * d.heads_kv;
  if (rows_q >= (int64_t(1) << 31) || rows_kv >= (int64_t(1) << 31)) return MAGI_BCA_UNSUPPORTED;
  return MAGI_BCA_OK;
}

int validate_offsets(const int32_t* qo, const int32_t* ko, const magi_bca_dims& d) {
  if (qo == nullptr || ko == nullptr) return MAGI_BCA_INVALID_ARG;
  if (qo[0] != 0 || ko[0] != 0) return MAGI_BCA_BAD_OFFSETS;
  if (qo[d.n_q_chunks] != d.seqlen_q || ko[d.n_kv_chunks] != d.seqlen_kv) return MAGI_BCA_BAD_OFFSETS;
  for (int c = 0; c < d.n_q_chunks; ++c)
    if (qo[c + 1] <= qo[c]) return MAGI_BCA_BAD_OFFSETS;
  for (int c = 0; c < d.n_kv_chunks; ++c)
    if (ko[c + 1] <= ko[c]) return MAGI_BCA_BAD_OFFSETS;
  // Matched chunks may differ in length (cross-attention against text K/V).
  if (d.n_samples < 0 || d.n_global_chunks < 0) return MAGI_BCA_INVALID_ARG;
  if (d.n_global_chunks > d.n_kv_chunks) return MAGI_BCA_BAD_OFFSETS;
  if (d.n_samples > 1) {
    const int32_t* so = d.sample_chunk_offsets;
    if (so == nullptr) return MAGI_BCA_INVALID_ARG;
    if (so[0] != 0 || so[d.n_samples] != d.n_kv_chunks) return MAGI_BCA_BAD_OFFSETS;
    for (int i = 0; i < d.n_samples; ++i)
      if (so[i + 1] <= so[i]) return MAGI_BCA_BAD_OFFSETS;
  }
  return MAGI_BCA_OK;
}

MaskSpec build_mask_spec(const int32_t* qo, const int32_t* ko, const magi_bca_dims& d) {
  MaskSpec m;
  const int nq = d.n_q_chunks, nkv = d.n_kv_chunks;
  const int first_global = nkv - d.n_global_chunks;   // kv chunks [first_global, nkv) are global
  // first kv chunk of the sample that holds kv chunk c
  std::vector<int> sample_first(nkv, 0);
  if (d.n_samples > 1)
    for (int i = 0; i < d.n_samples; ++i)
      for (int c = d.sample_chunk_offsets[i]; c < d.sample_chunk_offsets[i + 1]; ++c) sample_first[c] = d.sample_chunk_offsets[i];
  m.lo.resize(nq);
  m.hi.resize(nq);
  m.n_normal_q = nq;
  for (int c = 0; c < nq; ++c) {
    const int own = nkv - nq + c;
    if (own >= first_global) {   // a global query chunk sees every key
      m.lo[c] = 0;
      m.hi[c] = d.seqlen_kv;
      m.n_normal_q = std::min(m.n_normal_q, c);
      continue;
    }
    int first = sample_first[own];
    if (d.kv_range > 0) first = std::max(first, own - d.kv_range + 1);
    m.lo[c] = ko[first];
    m.hi[c] = ko[own + 1];
  }
  m.global_q_row = qo[m.n_normal_q];
  m.global_key = ko[first_global];
  return m;
}

void append_mask_blob(std::vector<int32_t>& blob, const int32_t* qo, const MaskSpec& m, int n_q_chunks) {
  blob.insert(blob.end(), qo, qo + n_q_chunks + 1);
  blob.insert(blob.end(), m.lo.begin(), m.lo.end());
  blob.insert(blob.end(), m.hi.begin(), m.hi.end());
}

MaskArgs mask_args_at(const int32_t* dev, const MaskSpec& m, int n_q_chunks) {
  MaskArgs a;
  a.q_offsets = dev;
  a.q_lo = dev + n_q_chunks + 1;
  a.q_hi = a.q_lo + n_q_chunks;
  a.n_q_chunks = n_q_chunks;
  a.n_normal_q = m.n_normal_q;
  a.global_q_row = m.global_q_row;
  a.global_key = m.global_key;
  return a;
}

namespace {

int chunk_of_row(const int32_t* qo, int n_q_chunks, int row) {
  const int32_t* it = std::upper_bound(qo, qo + n_q_chunks + 1, row);
  return static_cast<int>(it - qo) - 1;
}

}  // namespace

QTileExtent qtile_extent(const int32_t* qo, const MaskSpec& m, const magi_bca_dims& d, int m0) {
  const int last = std::min(m0 + kBlockM, d.seqlen_q) - 1;
  const int c0 = chunk_of_row(qo, d.n_q_chunks, m0), c1 = chunk_of_row(qo, d.n_q_chunks, last);
  // extremes of the visible ranges over the tile's chunks (global chunks have
  // lo = 0, so lo is not monotone over all rows)
  int lo_min = d.seqlen_kv, lo_max = 0, hi_min = d.seqlen_kv, hi_max = 0;
  for (int c = c0; c <= c1; ++c) {
    lo_min = std::min(lo_min, m.lo[c]);
    lo_max = std::max(lo_max, m.lo[c]);
    hi_min = std::min(hi_min, m.hi[c]);
    hi_max = std::max(hi_max, m.hi[c]);
  }
  QTileExtent e;
  e.n_full = hi_min / kBlockN;
  e.n_tiles = (hi_max + kBlockN - 1) / kBlockN;
  e.t_begin = lo_min / kBlockN;
  e.t_full_begin = (lo_max + kBlockN - 1) / kBlockN;
  e.g_begin = e.g_end = 0;
  const bool global_rows = last >= m.global_q_row;   // these see every key through the first range
  if (m.global_key < d.seqlen_kv && !global_rows) {
    const int gb = std::max(m.global_key / kBlockN, e.n_tiles);
    const int ge = (d.seqlen_kv + kBlockN - 1) / kBlockN;
    if (gb < ge) {
      e.g_begin = gb;
      e.g_end = ge;
    }
  }
  return e;
}

std::vector<int32_t> build_fwd_schedule(const int32_t* qo, const int32_t* ko, const magi_bca_dims& d) {
  const int n_qt = (d.seqlen_q + kBlockM - 1) / kBlockM;
  const int group = d.heads_q / d.heads_kv;
  const MaskSpec ms = build_mask_spec(qo, ko, d);
  std::vector<QTileExtent> ext(n_qt);
  for (int t = 0; t < n_qt; ++t) ext[t] = qtile_extent(qo, ms, d, t * kBlockM);

  struct Unit {
    int b, hk, h0, m00, h1, m01, first_tile;
    QTileExtent e;
    int cost() const { return ((e.n_tiles - e.t_begin) + (e.g_end - e.g_begin)) * (h1 >= 0 ? 2 : 1); }
  };
  auto same = [](const QTileExtent& x, const QTileExtent& y) {
    return x.n_full == y.n_full && x.n_tiles == y.n_tiles && x.t_begin == y.t_begin &&
           x.t_full_begin == y.t_full_begin && x.g_begin == y.g_begin && x.g_end == y.g_end;
  };
  std::vector<Unit> units;
  units.reserve((size_t)d.batch * d.heads_kv * n_qt * ((group + 1) / 2));
  for (int b = 0; b < d.batch; ++b) {
    for (int hk = 0; hk < d.heads_kv; ++hk) {
      // Walk the (tile, head) sub-tiles of this kv head in tile-major order
      // and pair neighbours that share an extent.
      int pend_h = -1, pend_t = -1;
      for (int t = 0; t < n_qt; ++t) {
        for (int h = hk * group; h < (hk + 1) * group; ++h) {
          if (pend_h >= 0 && same(ext[pend_t], ext[t])) {
            units.push_back({b, hk, pend_h, pend_t * kBlockM, h, t * kBlockM, pend_t, ext[t]});
            pend_h = -1;
            pend_t = -1;
          } else {
            if (pend_h >= 0) units.push_back({b, hk, pend_h, pend_t * kBlockM, -1, 0, pend_t, ext[pend_t]});
            pend_h = h;
            pend_t = t;
          }
        }
      }
      if (pend_h >= 0) units.push_back({b, hk, pend_h, pend_t * kBlockM, -1, 0, pend_t, ext[pend_t]});
    }
  }
  // Longest first (list scheduling in launch order approximates LPT); among
  // equal costs keep one (batch, kv head) together so the CTAs that run at
  // the same time stream the same K/V through L2.
  std::stable_sort(units.begin(), units.end(), [](const Unit& a, const Unit& b) {
    const int ca = a.cost(), cb = b.cost();
    if (ca != cb) return ca > cb;
    return std::tie(a.b, a.hk, a.first_tile, a.h0) < std::tie(b.b, b.hk, b.first_tile, b.h0);
  });
  std::vector<int32_t> out;
  out.reserve(units.size() * kFwdUnitInts);
  for (const Unit& u : units) {
    const int32_t v[kFwdUnitInts] = {u.b,       u.hk,       u.h0,      u.m00,          u.h1,      u.m01,
                                     u.e.n_full, u.e.n_tiles, u.e.t_begin, u.e.t_full_begin, u.e.g_begin, u.e.g_end};
    out.insert(out.end(), v, v + kFwdUnitInts);
  }
  return out;
}

namespace {

// Longest-processing-time list scheduling of `costs` (sorted, largest first)
// on `machines` identical machines: the CTA scheduler starts the next CTA in
// launch order on whichever SM frees first.  Returns the makespan.
double lpt_makespan(const std::vector<double>& costs, int machines) {
  std::priority_queue<double, std::vector<double>, std::greater<double>> load;
  for (int m = 0; m < machines; ++m) load.push(0.0);
  double span = 0.0;
  for (double c : costs) {
    const double t = load.top() + c;
    load.pop();
    load.push(t);
    span = std::max(span, t);
  }
  return span;
}

}  // namespace

std::vector<int32_t> build_bwd_schedule(const int32_t* qo, const int32_t* ko, const magi_bca_dims& d, int num_sms) {
  const int n_qt = (d.seqlen_q + kBlockM - 1) / kBlockM;
  const int n_kt = (d.seqlen_kv + kBlockN - 1) / kBlockN;
  const int group = d.heads_q / d.heads_kv;
  const MaskSpec ms = build_mask_spec(qo, ko, d);
  const int gq_row = ms.global_q_row;   // rows [gq_row, seqlen_q) see every key
  auto lo_of = [&](int r) { return ms.lo[chunk_of_row(qo, d.n_q_chunks, r)]; };
  auto hi_of = [&](int r) { return ms.hi[chunk_of_row(qo, d.n_q_chunks, r)]; };
  // Over each query tile's non-global rows: the smallest visible end and the
  // largest first visible key (monotone in the row over those rows).  A tile
  // of global rows only never needs the mask.
  std::vector<int> tile_lo(n_qt), tile_bhi(n_qt);
  for (int t = 0; t < n_qt; ++t) {
    const int r0 = t * kBlockM, r1 = std::min(r0 + kBlockM, gq_row);
    if (r0 >= r1) {
      tile_lo[t] = INT32_MAX;
      tile_bhi[t] = -1;
    } else {
      tile_lo[t] = hi_of(r0);
      tile_bhi[t] = lo_of(r1 - 1);
    }
  }
  // first non-global row in [0, gq_row] for which pred(row) holds (pred is monotone there)
  auto first_row = [&](auto pred) {
    int lo = 0, hi = gq_row;
    while (lo < hi) {
      const int mid = (lo + hi) / 2;
      if (pred(mid)) hi = mid; else lo = mid + 1;
    }
    return lo;
  };
  // One step = (query tile qt, head g of the kv head's group), numbered qt * group + g.
  // A sequence is a kv tile's steps: query tiles [qa0, qa1), then [qb0, qb1).
  struct Seq {
    int b, hk, n0, qa0, qa1, qb0, qb1, diag_end, diag_hi_begin, diag_global;
    int n() const { return (qa1 - qa0) + (qb1 - qb0); }   // query tiles
  };
  std::vector<Seq> seqs;
  for (int kt = 0; kt < n_kt; ++kt) {
    const int n0 = kt * kBlockN;
    const int n_end = std::min(n0 + kBlockN, d.seqlen_kv);
    int qa0 = 0, qa1 = 0, qb0 = 0, qb1 = 0, diag_end = 0, diag_hi_begin = n_qt, diag_global = -1;
    if (n_end > ms.global_key) {
      // the tile holds global keys: every row sees some key of it; the mask is
      // needed everywhere unless the whole tile is global
      qa0 = 0;
      qa1 = n_qt;
      diag_end = n0 >= ms.global_key ? 0 : n_qt;
    } else {
      // non-global rows [row_lo, row_hi) see some key: visible end past n0,
      // first visible key before n_end
      const int row_lo = first_row([&](int r) { return hi_of(r) > n0; });
      const int row_hi = first_row([&](int r) { return lo_of(r) >= n_end; });
      if (row_lo < row_hi) {
        qa0 = row_lo / kBlockM;
        qa1 = (row_hi + kBlockM - 1) / kBlockM;
        diag_end = qa0;
        while (diag_end < qa1 && tile_lo[diag_end] < n_end) ++diag_end;
        diag_hi_begin = qa0;
        while (diag_hi_begin < qa1 && tile_bhi[diag_hi_begin] <= n0) ++diag_hi_begin;
      }
      if (gq_row < d.seqlen_q) {   // the global query rows not already covered
        qb0 = std::max(gq_row / kBlockM, qa1);
        qb1 = n_qt;
        if (qb0 < qb1 && qb0 * kBlockM < gq_row) diag_global = qb0;   // it also holds non-global rows
        if (qa0 == qa1) {           // no block-causal run: the global rows are the only one
          qa0 = qb0;
          qa1 = qb1;
          diag_end = diag_global >= 0 ? qb0 + 1 : qb0;
          diag_hi_begin = n_qt;
          qb0 = qb1 = 0;
          diag_global = -1;
        }
      }
      if (qa0 == qa1) continue;    // nobody sees this kv tile
    }
    for (int b = 0; b < d.batch; ++b)
      for (int hk = 0; hk < d.heads_kv; ++hk)
        seqs.push_back({b, hk, n0, qa0, qa1, qb0, qb1, diag_end, diag_hi_begin, diag_global});
  }
  // Cut every sequence into k near-equal pieces of at most `len` steps; pick
  // `len` by simulating the CTA scheduler, charging each piece a fixed
  // overhead (its K/V load and pipeline fill, and the dV/dK reduction at the
  // end) of about two steps.
  constexpr double kPieceOverhead = 2.0;
  const int sms = std::max(num_sms, 1);
  int max_len = 1;
  int64_t total = 0;
  for (const Seq& q : seqs) {
    max_len = std::max(max_len, q.n() * group);
    total += q.n() * group;
  }
  // pieces shorter than an eighth of an SM's share only add overhead
  const double min_len = std::max(4.0, (double)total / (8.0 * sms));
  std::vector<int> candidates;
  if (d.deterministic == 0)
    for (double c = max_len; c >= min_len; c /= 1.08) candidates.push_back((int)std::lround(c));
  if (candidates.empty()) candidates.push_back(max_len);
  int best_len = max_len;
  double best_span = 0.0;
  std::vector<double> costs;
  for (int len : candidates) {
    if (len <= 0) continue;
    costs.clear();
    for (const Seq& q : seqs) {
      const int n = q.n() * group;
      const int k = (n + len - 1) / len;
      for (int i = 0; i < k; ++i) costs.push_back((double)(n * (i + 1) / k - n * i / k) + kPieceOverhead);
    }
    std::sort(costs.begin(), costs.end(), std::greater<double>());
    const double span = lpt_makespan(costs, sms);
    if (best_span == 0.0 || span < best_span - 1e-9) {
      best_span = span;
      best_len = len;
    }
  }
  struct Piece {
    int b, hk, n0, v0, v1, diag_end, diag_hi_begin, split, jump, diag_global;
  };
  std::vector<Piece> pieces;
  for (const Seq& q : seqs) {
    const int n = q.n() * group;
    const int k = (n + best_len - 1) / best_len;
    // virtual steps: [qa0 * G, qa1 * G) are absolute; the second run follows at qa1 * G
    const int v_begin = q.qa0 * group;
    const bool two = q.qb1 > q.qb0;
    const int split = two ? q.qa1 * group : INT32_MAX;
    const int jump = two ? (q.qb0 - q.qa1) * group : 0;
    for (int i = 0; i < k; ++i)
      pieces.push_back({q.b, q.hk, q.n0, v_begin + n * i / k, v_begin + n * (i + 1) / k, q.diag_end,
                        q.diag_hi_begin, split, jump, two ? q.diag_global : -1});
  }
  std::stable_sort(pieces.begin(), pieces.end(), [](const Piece& a, const Piece& b) {
    const int ca = a.v1 - a.v0, cb = b.v1 - b.v0;
    if (ca != cb) return ca > cb;
    return std::tie(a.b, a.hk, a.v0, a.n0) < std::tie(b.b, b.hk, b.v0, b.n0);
  });
  std::vector<int32_t> out;
  out.reserve(pieces.size() * kUnitInts);
  for (const Piece& u : pieces) {
    const int32_t v[kUnitInts] = {u.b,     u.hk,    u.n0,          u.v0, u.v1, u.diag_end, u.diag_hi_begin,
                                  u.split, u.jump, u.diag_global, 0,    0};
    out.insert(out.end(), v, v + kUnitInts);
  }
  return out;
}

}  // namespace magi
