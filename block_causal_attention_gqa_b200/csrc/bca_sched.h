// Host-side argument checks and the chunk-aware tile scheduler.
//
// Block-causal attention (MAGI-1 §2, Figure 1) lets query chunk c see every
// key of kv chunks 0 .. n_kv - n_q + c.  Over 128 x 128 tiles this means:
//   * a query tile whose rows all sit in chunks whose visible range ends at
//     or after column tile j's end needs tile j with no mask ("full" tile);
//   * tiles between the smallest and the largest visible end of the tile's
//     rows straddle a chunk boundary and need the per-row mask ("diagonal");
//   * tiles past the largest end are never visited.
// Without a KV range the visible range always starts at key 0, so the full
// tiles of a query tile are the prefix [0, n_full) and the diagonal ones
// [n_full, n_tiles).  A KV range R (MAGI-1 §2.4.4, Fig. 12) also gives each
// row a first visible key, the start of kv chunk c - R + 1; tiles entirely
// below the smallest first key of a tile's rows are skipped (t_begin) and
// tiles below the largest one need the mask as well (t_full_begin).
#pragma once
#include <cstdint>
#include <vector>

#include "../../include/magi_bca.h"

namespace magi {

constexpr int kBlockM = 128;  // query rows per sub-tile (one TMEM lane per row)
constexpr int kBlockN = 128;  // kv rows per tile
constexpr int kUnitInts = 8;      // int32 values per backward work unit
constexpr int kFwdUnitInts = 12;  // int32 values per forward work unit

// Checks dims and offsets.  Returns MAGI_BCA_OK or a negative status.
int validate_dims(const magi_bca_dims* dims);
int validate_offsets(const int32_t* q_offsets, const int32_t* kv_offsets, const magi_bca_dims& d);

struct QTileExtent {
  int t_begin;       // kv tiles [t_begin, n_tiles) are visited
  int t_full_begin;  // tiles below it straddle some row's first visible key (KV range)
  int n_full;        // tiles at or above it straddle some row's visible end
  int n_tiles;
};

// Visible-key end for query row `row` (row < seqlen_q).
int row_kv_end(const int32_t* q_offsets, const int32_t* kv_offsets, const magi_bca_dims& d, int row);
// First visible key of query row `row`: 0, or with a KV range R the start of
// kv chunk c - R + 1 (c = the row's matched kv chunk).
int row_kv_begin(const int32_t* q_offsets, const int32_t* kv_offsets, const magi_bca_dims& d, int row);

// Extent of the query tile starting at row m0.
QTileExtent qtile_extent(const int32_t* q_offsets, const int32_t* kv_offsets, const magi_bca_dims& d,
                         int m0);

// Forward schedule: units of up to two sub-tiles with the same (batch,
// kv head, extent), sorted longest first and, among equals, grouped by
// (batch, kv head) so concurrently running units share K/V in L2.  Emits per
// unit {batch, kv_head, head_0, m0_0, head_1, m0_1, n_full, n_tiles,
// t_begin, t_full_begin, 0, 0}.
std::vector<int32_t> build_fwd_schedule(const int32_t* q_offsets, const int32_t* kv_offsets,
                                        const magi_bca_dims& d);

// Backward schedule, kv-tile major: for kv tile t (rows [t*128, t*128+128))
// the query tiles that see any of its keys are the q tiles [q_begin, q_end):
// visible ends and (under a KV range) visible beginnings are non-decreasing
// in the row, so the rows that see some key of it form one contiguous range.
// A step is one (query tile qt, head g of the kv head's group), numbered
// qt * group + g; each kv tile's steps are cut into near-equal pieces whose
// length is chosen by simulating list scheduling of the pieces on `num_sms`
// SMs.  Emits per unit {batch, kv_head, n0, step_begin, step_end, diag_end,
// diag_hi_begin, 0}: query tiles below diag_end straddle the first row that
// sees the kv tile, and query tiles at or above diag_hi_begin straddle the
// first row (under a KV range) that no longer sees all of it, so both need
// the mask; units are sorted longest first.  With d.deterministic every kv
// tile is one unit (no pieces), so one CTA writes each tile's dV and G_k.
std::vector<int32_t> build_bwd_schedule(const int32_t* q_offsets, const int32_t* kv_offsets,
                                        const magi_bca_dims& d, int num_sms);

}  // namespace magi
