// Device side of the mask and the schedule: which keys a query row sees, which
// query rows see a key, and the decoding of the work units (bca_sched.h).
//
// A query row of chunk c sees the keys [q_lo[c], q_hi[c]) by the block-causal
// rule (its own and earlier chunks of its sample, within the KV range) and the
// global block's keys [global_key, seqlen_kv); rows from global_q_row on (the
// global block's queries) see every key.  Over the non-global chunks q_lo and
// q_hi are non-decreasing, so the non-global rows that see a key form one
// range, found by binary search.
#pragma once
#include <cstdint>

#include "bca_kernels.h"
#include "bca_sched.h"

namespace magi {

__device__ __forceinline__ int find_chunk(const int32_t* offs, int n, int row) {
  int lo = 0, hi = n;  // offs[lo] <= row < offs[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(offs + mid) <= row) lo = mid; else hi = mid;
  }
  return lo;
}

// Visible keys [lo, hi) of query row `row` by the block-causal rule (global
// rows: the whole sequence); the global keys come on top.
__device__ __forceinline__ void row_keys(const MaskArgs& m, int row, int& lo, int& hi) {
  const int c = find_chunk(m.q_offsets, m.n_q_chunks, row);
  lo = __ldg(m.q_lo + c);
  hi = __ldg(m.q_hi + c);
}

// The non-global query rows that see `key` by the block-causal rule:
// [row_min, row_max) (empty when row_min >= row_max).  Rows from
// m.global_q_row on see every key, and every row sees a key at or above
// m.global_key (below seqlen_kv).
__device__ __forceinline__ void key_rows(const MaskArgs& m, int key, int& row_min, int& row_max) {
  // first non-global chunk whose visible end passes the key: its rows see it
  // (the key then lies in its matched chunk, at or after its first visible key)
  int lo = 0, hi = m.n_normal_q;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(m.q_hi + mid) > key) hi = mid; else lo = mid + 1;
  }
  row_min = __ldg(m.q_offsets + lo);
  // first non-global chunk whose first visible key is past the key
  lo = 0;
  hi = m.n_normal_q;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(m.q_lo + mid) > key) hi = mid; else lo = mid + 1;
  }
  row_max = __ldg(m.q_offsets + lo);
}

// A forward (query-major) unit visits kv tiles [t_begin, n_tiles) and then the
// global block's tiles [g_begin, g_end); visited tile j counts from 0.
struct FwdTiles {
  int t_begin, n_tiles, t_full_begin, n_full, g_begin, g_end;
  __device__ __forceinline__ int count() const { return (n_tiles - t_begin) + (g_end - g_begin); }
  __device__ __forceinline__ int tile(int j) const {
    const int na = n_tiles - t_begin;
    return j < na ? t_begin + j : g_begin + (j - na);
  }
  // Whether visited tile j needs the per-row mask: in the first range unless
  // every row sees it whole; in the global range where it straddles the
  // block's first key or the end of the sequence.
  __device__ __forceinline__ bool masked(int j, int global_key, int seqlen_kv) const {
    const int t = tile(j);
    if (j < n_tiles - t_begin) return t < t_full_begin || t >= n_full;
    return t * 128 < global_key || t * 128 + 128 > seqlen_kv;
  }
};

__device__ __forceinline__ FwdTiles fwd_tiles(const int32_t* u) {
  FwdTiles f;
  f.n_full = __ldg(u + 6);
  f.n_tiles = __ldg(u + 7);
  f.t_begin = __ldg(u + 8);
  f.t_full_begin = __ldg(u + 9);
  f.g_begin = __ldg(u + 10);
  f.g_end = __ldg(u + 11);
  return f;
}

// A backward (kv-major) unit runs steps v in [v_begin, v_end): absolute step
// (query tile * group + head) v below `split`, v + jump from there on.
struct BwdSteps {
  int v_begin, v_end, diag_end, diag_hi_begin, split, jump, diag_global;
  __device__ __forceinline__ int count() const { return v_end - v_begin; }
  __device__ __forceinline__ int abs_step(int t) const {
    const int v = v_begin + t;
    return v < split ? v : v + jump;
  }
  // Whether step t (query tile qt) needs the per-key mask.
  __device__ __forceinline__ bool diag(int t, int qt) const {
    return v_begin + t < split ? (qt < diag_end || qt >= diag_hi_begin) : qt == diag_global;
  }
};

__device__ __forceinline__ BwdSteps bwd_steps(const int32_t* u) {
  BwdSteps s;
  s.v_begin = __ldg(u + 3);
  s.v_end = __ldg(u + 4);
  s.diag_end = __ldg(u + 5);
  s.diag_hi_begin = __ldg(u + 6);
  s.split = __ldg(u + 7);
  s.jump = __ldg(u + 8);
  s.diag_global = __ldg(u + 9);
  return s;
}

// ------------------------------------------------------------ debug build
// Built with -DMAGI_BCA_DEBUG (build.py --debug), every attention kernel first
// checks its work unit against the problem's sizes; a unit out of range (a
// scheduler defect) records kErrDbgUnit in the device status word and the CTA
// returns before any memory access, barrier or TMEM allocation.  The host reads
// the code as MAGI_BCA_DEVICE_CHECK.  The product build compiles the checks out.
#ifdef MAGI_BCA_DEBUG
constexpr bool kDebugChecks = true;
#else
constexpr bool kDebugChecks = false;
#endif
constexpr int kErrDbgUnit = 3001;

__device__ __forceinline__ bool debug_fail(int* status) {
  atomicCAS(status, 0, kErrDbgUnit);
  return false;
}

// A forward (query-major) unit: batch, kv head, its query heads and rows, and
// both kv tile ranges inside the problem.
__device__ __forceinline__ bool fwd_unit_in_range(const int32_t* u, int batch, int heads_q, int heads_kv,
                                                  int seqlen_q, int seqlen_kv, int* status) {
  const int group = heads_q / heads_kv;
  const int n_kt = (seqlen_kv + 127) / 128;
  const int b = __ldg(u + 0), hk = __ldg(u + 1), h0 = __ldg(u + 2), m0 = __ldg(u + 3), h1 = __ldg(u + 4),
            m1 = __ldg(u + 5);
  const FwdTiles f = fwd_tiles(u);
  bool ok = b >= 0 && b < batch && hk >= 0 && hk < heads_kv;
  ok = ok && h0 >= hk * group && h0 < (hk + 1) * group && m0 >= 0 && m0 < seqlen_q && m0 % 128 == 0;
  ok = ok && (h1 == -1 || (h1 >= hk * group && h1 < (hk + 1) * group && m1 >= 0 && m1 < seqlen_q && m1 % 128 == 0));
  ok = ok && f.t_begin >= 0 && f.t_begin <= f.n_tiles && f.n_tiles <= n_kt;
  ok = ok && ((f.g_begin == 0 && f.g_end == 0) || (f.n_tiles <= f.g_begin && f.g_begin <= f.g_end && f.g_end <= n_kt));
  return ok || debug_fail(status);
}

// A backward (kv-major) unit: batch, kv head, kv tile and every step it runs.
__device__ __forceinline__ bool bwd_unit_in_range(const int32_t* u, int batch, int heads_q, int heads_kv,
                                                  int seqlen_q, int seqlen_kv, int* status) {
  const int group = heads_q / heads_kv;
  const int n_steps_all = (seqlen_q + 127) / 128 * group;
  const int b = __ldg(u + 0), hk = __ldg(u + 1), n0 = __ldg(u + 2);
  const BwdSteps bs = bwd_steps(u);
  bool ok = b >= 0 && b < batch && hk >= 0 && hk < heads_kv && n0 >= 0 && n0 < seqlen_kv && n0 % 128 == 0;
  ok = ok && bs.v_begin < bs.v_end && bs.jump >= 0;
  ok = ok && bs.abs_step(0) >= 0 && bs.abs_step(bs.count() - 1) < n_steps_all;
  return ok || debug_fail(status);
}

}  // namespace magi
