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
// [n_full, n_tiles).  A KV range R (MAGI-1 §2.4.4, Fig. 12) or packed samples
// (MAGI-1 §4.1.2, Figure 15 (f)) also give each row a first visible key, the
// start of kv chunk c - R + 1 or of its sample; tiles entirely below the
// smallest first key of a tile's rows are skipped (t_begin) and tiles below the
// largest one need the mask as well (t_full_begin).  A last global block
// (Figure 15 (g)) adds a second range of kv tiles, its keys, to every query
// tile that does not already see every key.
#pragma once
#include <cstdint>
#include <vector>

#include "../../include/magi_bca.h"

namespace magi {

constexpr int kBlockM = 128;  // query rows per sub-tile (one TMEM lane per row)
constexpr int kBlockN = 128;  // kv rows per tile
constexpr int kUnitInts = 12;     // int32 values per backward work unit
constexpr int kFwdUnitInts = 12;  // int32 values per forward work unit

// Checks dims and offsets (chunk and sample offsets).  Returns MAGI_BCA_OK or
// a negative status.
int validate_dims(const magi_bca_dims* dims);
int validate_offsets(const int32_t* q_offsets, const int32_t* kv_offsets, const magi_bca_dims& d);

// The keys every query chunk sees.  By the block-causal rule query chunk c
// (matched to kv chunk m = n_kv - n_q + c) sees kv chunks up to m, from the
// first chunk of m's sample and (KV range R) from m - R + 1 on: the keys
// [lo[c], hi[c]).  A global block (the last n_global kv chunks) adds its keys
// [global_key, seqlen_kv) to every query's set, and the query chunks matched to
// it (c >= n_normal_q) see every key: lo = 0, hi = seqlen_kv.  lo and hi are
// non-decreasing over the chunks [0, n_normal_q); the global query chunks are
// the last ones.  The kernels receive lo and hi as device arrays.
struct MaskSpec {
  std::vector<int32_t> lo, hi;  // per query chunk
  int n_normal_q = 0;           // query chunks [0, n_normal_q) are not global
  int global_q_row = 0;         // first row of a global query chunk (seqlen_q if none)
  int global_key = 0;           // first global key (seqlen_kv if none)
};
MaskSpec build_mask_spec(const int32_t* q_offsets, const int32_t* kv_offsets, const magi_bca_dims& d);

struct QTileExtent {
  int t_begin;       // kv tiles [t_begin, n_tiles) are visited
  int t_full_begin;  // tiles below it straddle some row's first visible key
  int n_full;        // tiles at or above it straddle some row's visible end
  int n_tiles;
  int g_begin, g_end;  // then the global block's tiles [g_begin, g_end) (empty: 0, 0)
};

// Extent of the query tile starting at row m0.
QTileExtent qtile_extent(const int32_t* q_offsets, const MaskSpec& m, const magi_bca_dims& d, int m0);

// Forward schedule: units of up to two sub-tiles with the same (batch,
// kv head, extent), sorted longest first and, among equals, grouped by
// (batch, kv head) so concurrently running units share K/V in L2.  Emits per
// unit {batch, kv_head, head_0, m0_0, head_1, m0_1, n_full, n_tiles,
// t_begin, t_full_begin, g_begin, g_end}.
std::vector<int32_t> build_fwd_schedule(const int32_t* q_offsets, const int32_t* kv_offsets,
                                        const magi_bca_dims& d);

// Backward schedule, kv-tile major: for kv tile t (keys [t*128, t*128+128))
// the query rows that see any of its keys are, by the block-causal rule, one
// contiguous range (lo and hi are non-decreasing over the non-global rows),
// plus every global query row, plus every row at all when the tile holds
// global keys.  A step is one (query tile qt, head g of the kv head's group),
// numbered qt * group + g.  A kv tile's steps are the query tiles of the
// block-causal range and then those of the global rows not yet in it; each
// tile's steps are cut into near-equal pieces whose length is chosen by
// simulating list scheduling of the pieces on `num_sms` SMs.  Emits per unit
// {batch, kv_head, n0, step_begin, step_end, diag_end, diag_hi_begin, split,
// jump, diag_global, 0, 0}: unit steps v in [step_begin, step_end) are the
// absolute step v below split and v + jump from split on; query tiles of the
// first run below diag_end or at or above diag_hi_begin need the mask, and in
// the second run only tile diag_global (-1: none).  Units are sorted longest
// first.  With d.deterministic every kv tile is one unit (no pieces), so one CTA
// writes each tile's dV and G_k.
std::vector<int32_t> build_bwd_schedule(const int32_t* q_offsets, const int32_t* kv_offsets,
                                        const magi_bca_dims& d, int num_sms);

}  // namespace magi
