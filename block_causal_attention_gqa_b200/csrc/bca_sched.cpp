// Host-side argument checks and the chunk-aware tile scheduler (see bca_sched.h).
#include "bca_sched.h"

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
  return MAGI_BCA_OK;
}

int row_kv_end(const int32_t* qo, const int32_t* ko, const magi_bca_dims& d, int row) {
  // chunk c with qo[c] <= row < qo[c+1]
  const int32_t* it = std::upper_bound(qo, qo + d.n_q_chunks + 1, row);
  const int c = static_cast<int>(it - qo) - 1;
  return ko[d.n_kv_chunks - d.n_q_chunks + c + 1];
}

int row_kv_begin(const int32_t* qo, const int32_t* ko, const magi_bca_dims& d, int row) {
  if (d.kv_range <= 0) return 0;
  const int32_t* it = std::upper_bound(qo, qo + d.n_q_chunks + 1, row);
  const int c = static_cast<int>(it - qo) - 1;
  const int first = d.n_kv_chunks - d.n_q_chunks + c - d.kv_range + 1;
  return ko[std::max(first, 0)];
}

QTileExtent qtile_extent(const int32_t* qo, const int32_t* ko, const magi_bca_dims& d, int m0) {
  const int last = std::min(m0 + kBlockM, d.seqlen_q) - 1;
  // visible ends and beginnings are non-decreasing in the row index
  const int lo = row_kv_end(qo, ko, d, m0);
  const int hi = row_kv_end(qo, ko, d, last);
  const int blo = row_kv_begin(qo, ko, d, m0);
  const int bhi = row_kv_begin(qo, ko, d, last);
  QTileExtent e;
  e.n_full = lo / kBlockN;
  e.n_tiles = (hi + kBlockN - 1) / kBlockN;
  e.t_begin = blo / kBlockN;
  e.t_full_begin = (bhi + kBlockN - 1) / kBlockN;
  return e;
}

std::vector<int32_t> build_fwd_schedule(const int32_t* qo, const int32_t* ko, const magi_bca_dims& d) {
  const int n_qt = (d.seqlen_q + kBlockM - 1) / kBlockM;
  const int group = d.heads_q / d.heads_kv;
  std::vector<QTileExtent> ext(n_qt);
  for (int t = 0; t < n_qt; ++t) ext[t] = qtile_extent(qo, ko, d, t * kBlockM);

  struct Unit {
    int b, hk, h0, m00, h1, m01, n_full, n_tiles, t_begin, t_full_begin, first_tile;
  };
  auto same = [](const QTileExtent& x, const QTileExtent& y) {
    return x.n_full == y.n_full && x.n_tiles == y.n_tiles && x.t_begin == y.t_begin &&
           x.t_full_begin == y.t_full_begin;
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
            units.push_back({b, hk, pend_h, pend_t * kBlockM, h, t * kBlockM, ext[t].n_full, ext[t].n_tiles,
                             ext[t].t_begin, ext[t].t_full_begin, pend_t});
            pend_h = -1;
            pend_t = -1;
          } else {
            if (pend_h >= 0)
              units.push_back({b, hk, pend_h, pend_t * kBlockM, -1, 0, ext[pend_t].n_full, ext[pend_t].n_tiles,
                               ext[pend_t].t_begin, ext[pend_t].t_full_begin, pend_t});
            pend_h = h;
            pend_t = t;
          }
        }
      }
      if (pend_h >= 0)
        units.push_back({b, hk, pend_h, pend_t * kBlockM, -1, 0, ext[pend_t].n_full, ext[pend_t].n_tiles,
                         ext[pend_t].t_begin, ext[pend_t].t_full_begin, pend_t});
    }
  }
  // Longest first (list scheduling in launch order approximates LPT); among
  // equal costs keep one (batch, kv head) together so the CTAs that run at
  // the same time stream the same K/V through L2.
  std::stable_sort(units.begin(), units.end(), [](const Unit& a, const Unit& b) {
    const int ca = (a.n_tiles - a.t_begin) * (a.h1 >= 0 ? 2 : 1), cb = (b.n_tiles - b.t_begin) * (b.h1 >= 0 ? 2 : 1);
    if (ca != cb) return ca > cb;
    return std::tie(a.b, a.hk, a.first_tile, a.h0) < std::tie(b.b, b.hk, b.first_tile, b.h0);
  });
  std::vector<int32_t> out;
  out.reserve(units.size() * kFwdUnitInts);
  for (const Unit& u : units) {
    const int32_t v[kFwdUnitInts] = {u.b, u.hk, u.h0, u.m00, u.h1, u.m01, u.n_full, u.n_tiles,
                                     u.t_begin, u.t_full_begin, 0, 0};
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
  // deterministic backward: one unit per kv tile, so each tile's dV and G_k
  // are written by exactly one CTA
  const int n_qt = (d.seqlen_q + kBlockM - 1) / kBlockM;
  const int n_kt = (d.seqlen_kv + kBlockN - 1) / kBlockN;
  const int group = d.heads_q / d.heads_kv;
  std::vector<int> tile_lo(n_qt);   // smallest visible end among the tile's rows
  std::vector<int> tile_bhi(n_qt);  // largest first visible key among the tile's rows
  for (int t = 0; t < n_qt; ++t) {
    tile_lo[t] = row_kv_end(qo, ko, d, t * kBlockM);
    tile_bhi[t] = row_kv_begin(qo, ko, d, std::min(t * kBlockM + kBlockM, d.seqlen_q) - 1);
  }
  // first row in [0, seqlen_q] for which pred(row) holds (pred is monotone in the row)
  auto first_row = [&](auto pred) {
    int lo = 0, hi = d.seqlen_q;
    while (lo < hi) {
      const int mid = (lo + hi) / 2;
      if (pred(mid)) hi = mid; else lo = mid + 1;
    }
    return lo;
  };
  // One step = (query tile qt, head g of the kv head's group), numbered qt * group + g.
  struct Seq {
    int b, hk, n0, s_begin, s_end, diag_end, diag_hi_begin;
  };
  std::vector<Seq> seqs;
  for (int kt = 0; kt < n_kt; ++kt) {
    const int n0 = kt * kBlockN;
    const int n_end = std::min(n0 + kBlockN, d.seqlen_kv);
    // rows [row_lo, row_hi) see some key of the tile: visible end past n0, first key before n_end
    const int row_lo = first_row([&](int r) { return row_kv_end(qo, ko, d, r) > n0; });
    const int row_hi = first_row([&](int r) { return row_kv_begin(qo, ko, d, r) >= n_end; });
    if (row_lo >= row_hi) continue;  // nobody sees this kv tile
    const int qb = row_lo / kBlockM, qe = (row_hi + kBlockM - 1) / kBlockM;
    int diag_end = qb;
    while (diag_end < qe && tile_lo[diag_end] < n_end) ++diag_end;
    int diag_hi_begin = qb;
    while (diag_hi_begin < qe && tile_bhi[diag_hi_begin] <= n0) ++diag_hi_begin;
    for (int b = 0; b < d.batch; ++b)
      for (int hk = 0; hk < d.heads_kv; ++hk)
        seqs.push_back({b, hk, n0, qb * group, qe * group, diag_end, diag_hi_begin});
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
    max_len = std::max(max_len, q.s_end - q.s_begin);
    total += q.s_end - q.s_begin;
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
      const int n = q.s_end - q.s_begin;
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
  std::vector<Seq> pieces;
  for (const Seq& q : seqs) {
    const int n = q.s_end - q.s_begin;
    const int k = (n + best_len - 1) / best_len;
    for (int i = 0; i < k; ++i)
      pieces.push_back({q.b, q.hk, q.n0, q.s_begin + n * i / k, q.s_begin + n * (i + 1) / k, q.diag_end,
                        q.diag_hi_begin});
  }
  std::stable_sort(pieces.begin(), pieces.end(), [](const Seq& a, const Seq& b) {
    const int ca = a.s_end - a.s_begin, cb = b.s_end - b.s_begin;
    if (ca != cb) return ca > cb;
    return std::tie(a.b, a.hk, a.s_begin, a.n0) < std::tie(b.b, b.hk, b.s_begin, b.n0);
  });
  std::vector<int32_t> out;
  out.reserve(pieces.size() * kUnitInts);
  for (const Seq& u : pieces) {
    const int32_t v[kUnitInts] = {u.b, u.hk, u.n0, u.s_begin, u.s_end, u.diag_end, u.diag_hi_begin, 0};
    out.insert(out.end(), v, v + kUnitInts);
  }
  return out;
}

}  // namespace magi
