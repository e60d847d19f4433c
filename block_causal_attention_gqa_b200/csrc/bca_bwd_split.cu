// The deterministic backward's two passes, sm_100a (see bca_bwd.cu for the
// fused default path).  With dims.deterministic no sum may depend on timing:
//   bca_bwd_dq_kernel    query-major: one CTA per 128-row query sub-tile owns its
//                        rows' G_q and sums it over the visible kv tiles in tile
//                        order (S, dP, dS' and G_q in TMEM), no reductions across CTAs
//   bca_bwd_dkdv_kernel  kv-major: the fused kernel's work without G_q, one unit
//                        per kv tile, so each tile's dV and G_k are added once onto zero
// The dq pass recomputes S and dP, 7/5 of the fused path's tensor work.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "bca_bwd_common.cuh"
#include "bca_kernels.h"
#include "bca_mask.cuh"
#include "bca_norm.cuh"
#include "sm100.cuh"

namespace magi {
namespace {

using namespace sm100;

// ------------------------------------------------------------------ dK/dV pass
// The kv-major half of the split backward (with bca_bwd_dq_kernel): the main
// kernel's work without G_q.  Per step (query tile, head) of its kv tile:
//   S'^T  = K^ Q^^T - lse2,  dP'^T = V dO^T - Delta   (TMEM, in two 64-query halves)
//   P^T   = exp2(S'^T),  dS'^T = P^T dP'^T            (bf16, back into the S^T columns)
//   dV   += P^T dO,  G_k += dS'^T Q^                  (both A operands from TMEM)
// Without G_q nothing needs dS'^T in shared memory (G_q read it transposed),
// so it stays in TMEM: P^T of queries [16k, 16k + 16) goes to S^T columns
// [16k, 16k + 8) and dS'^T to [16k + 8, 16k + 16).  That frees the shared
// memory for a {-lse, -Delta} block per Q^/dO stage, loaded with the stage.
// Each 64-query half of step t+1's S'^T and dP'^T is issued as soon as the
// softmax has finished the same half of step t (and dK~/dV of that half are
// queued), so the tensor pipe computes step t+1's first half while the
// softmax works on step t's second half.  TMEM: S^T [0, 128), dP^T [128, 256),
// dV [256, 256 + D), G_k [384, 384 + D).
template <int D>
struct DkdvLayout {
  static constexpr int kTile = 128 * D * 2;      // [128][D] bf16
  static constexpr int kK = 0;
  static constexpr int kV = kK + kTile;
  static constexpr int kQn = kV + kTile;         // 2 stages
  static constexpr int kDo = kQn + 2 * kTile;    // 2 stages
  // per stage: 128 query rows x 8 bf16 {-lse2, -Delta pieces}, then a zeroed
  // 128-byte tail: the extra K-step of the second 64-query half reads one core
  // matrix (8 rows) past the block, which A's zero core matrix multiplies, so it
  // must hold finite values even before the other stage's first load
  static constexpr int kLdStride = 2048 + 128;
  static constexpr int kLd = kDo + 2 * kTile;
  static constexpr int kOnes = kLd + 2 * kLdStride;   // constant A rows of the extra K-step (3 x 128 B)
  static constexpr int kBars = kOnes + 384;
  static constexpr int kTmemSlot = kBars + 16 * 8;
  static constexpr int kTotal = kTmemSlot + 16;
};

struct DkdvBars {
  uint64_t kv_full, s_lo, s_hi, ds_half, ds_ready, acc_full;
  uint64_t q_full[2], q_empty[2];
};
static_assert(sizeof(DkdvBars) <= 16 * 8, "dK/dV barriers exceed their slot");

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
bca_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_qn, const __grid_constant__ CUtensorMap tm_do,
                    const __grid_constant__ CUtensorMap tm_dv, const __grid_constant__ CUtensorMap tm_dk,
                    const BwdParams p, const int smem_alloc) {
  using L = DkdvLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  const uintptr_t base = (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023);
  uint8_t* smem = reinterpret_cast<uint8_t*>(base);
  if (base - reinterpret_cast<uintptr_t>(smem_raw) + L::kTotal > (uintptr_t)smem_alloc) {
    if (threadIdx.x == 0) atomicCAS(p.status, 0, kErrSmem);
    return;
  }
  DkdvBars* bars = reinterpret_cast<DkdvBars*>(smem + L::kBars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kTmemSlot);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int32_t* u = p.units + (size_t)blockIdx.x * kUnitInts;
  if constexpr (kDebugChecks) {
    if (!bwd_unit_in_range(u, p.batch, p.heads_q, p.heads_kv, p.seqlen_q, p.seqlen_kv, p.status)) return;
  }
  const int b = __ldg(u + 0), hk = __ldg(u + 1), n0 = __ldg(u + 2);
  const BwdSteps bs = bwd_steps(u);   // steps t -> absolute steps, and which need the mask
  const int group = p.heads_q / p.heads_kv;
  const int n_steps = bs.count();

  if (threadIdx.x == 0) {
    mbar_init(&bars->kv_full, 1);
    mbar_init(&bars->s_lo, 1);
    mbar_init(&bars->s_hi, 1);
    mbar_init(&bars->ds_half, kComputeWarpgroups);
    mbar_init(&bars->ds_ready, kComputeWarpgroups);
    mbar_init(&bars->acc_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->q_full[s], 1);
      mbar_init(&bars->q_empty[s], 1);   // committed by the MMA thread once dK~ and dV have read the stage
    }
    fence_mbar_init();
  }
  // A rows of the extra K-step, as in the main kernel: ones at k = 0..2 (picks
  // -lse2), ones at k = 3..5 (picks -Delta), a zero core matrix for k = 8..15.
  if (threadIdx.x < 96) {
    const int blk = threadIdx.x >> 5, w = threadIdx.x & 31;
    const int k0 = (w & 3) * 2;
    auto one_at = [&](int k) { return blk < 2 && k >= 3 * blk && k < 3 * blk + 3; };
    const uint32_t lo = one_at(k0) ? 0x3F80u : 0u, hi = one_at(k0 + 1) ? 0x3F80u : 0u;
    reinterpret_cast<uint32_t*>(smem + L::kOnes)[threadIdx.x] = lo | (hi << 16);
  } else if (threadIdx.x < 96 + 64) {   // the two 128-byte tails of the piece blocks
    const int i = threadIdx.x - 96;
    reinterpret_cast<uint32_t*>(smem + L::kLd + (i >> 5) * L::kLdStride + 2048)[i & 31] = 0u;
  }
  fence_proxy_async_smem();
  if (warp == kTmaWarp && lane == 0) {
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_qn);
    tma_prefetch_desc(&tm_do);
    tma_prefetch_desc(&tm_dv);
    tma_prefetch_desc(&tm_dk);
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  constexpr uint32_t T_S = 0, T_DP = 128, T_DV = 256, T_DK = 384;

  if (warp == kTmaWarp) {
    // ------------------------------------------------------------ TMA producer
    if (elect_one()) {
      mbar_arrive_expect_tx(&bars->kv_full, 2 * L::kTile);
      for (int box = 0; box < D / 64; ++box) {
        tma_load_4d(smem + L::kK + box * 16384, &tm_k, &bars->kv_full, box * 64, hk, n0, b);
        tma_load_4d(smem + L::kV + box * 16384, &tm_v, &bars->kv_full, box * 64, hk, n0, b);
      }
      for (int t = 0; t < n_steps; ++t) {
        const int st = t & 1;
        if (!mbar_wait(&bars->q_empty[st], ((t >> 1) & 1) ^ 1, p.status, kErrQEmpty)) break;
        const int sa = bs.abs_step(t);
        const int qt = sa / group, h = hk * group + sa % group;
        mbar_arrive_expect_tx(&bars->q_full[st], 2 * L::kTile + 2048);
        for (int box = 0; box < D / 64; ++box) {
          tma_load_4d(smem + L::kQn + st * L::kTile + box * 16384, &tm_qn, &bars->q_full[st], box * 64, h,
                      qt * 128, b);
          tma_load_4d(smem + L::kDo + st * L::kTile + box * 16384, &tm_do, &bars->q_full[st], box * 64, h,
                      qt * 128, b);
        }
        const float* ld_src = p.ld + (((size_t)b * p.heads_q + h) * p.seqlen_q_pad + (size_t)qt * 128) * 4;
        bulk_load(smem + L::kLd + st * L::kLdStride, ld_src, 2048, &bars->q_full[st]);
        if (t + 1 < n_steps) {
          const int sa1 = bs.abs_step(t + 1);
          const int qt1 = sa1 / group, h1 = hk * group + sa1 % group;
          for (int box = 0; box < D / 64; ++box) {
            tma_prefetch_l2_4d(&tm_qn, box * 64, h1, qt1 * 128, b);
            tma_prefetch_l2_4d(&tm_do, box * 64, h1, qt1 * 128, b);
          }
          bulk_prefetch_l2(p.ld + (((size_t)b * p.heads_q + h1) * p.seqlen_q_pad + (size_t)qt1 * 128) * 4, 2048);
        }
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (elect_one()) {
      constexpr uint32_t id_half = make_idesc_bf16(128, 64, false, false);  // S^T, dP^T: 64 query columns
      constexpr uint32_t id_ts = make_idesc_bf16(128, D, false, true);      // dV, dK~: A from TMEM
      const uint32_t kn_a = smem_u32(smem + L::kK), v_a = smem_u32(smem + L::kV);
      const uint32_t qn_a = smem_u32(smem + L::kQn), do_a = smem_u32(smem + L::kDo);
      const uint32_t ld_a = smem_u32(smem + L::kLd), ones_a = smem_u32(smem + L::kOnes);
      const uint64_t ext_lse = make_noswz_desc(ones_a, 256, 0), ext_delta = make_noswz_desc(ones_a + 128, 128, 0);
      // Columns [64 hf, 64 hf + 64) of C = A[128 x D] B^T with B = query rows
      // [64 hf, 64 hf + 64) of the stage (8 KB into each swizzled box), then
      // the extra K-step adding -lse2 (S^T) or -Delta (dP^T) of those queries
      // (their 16-byte piece rows start 1 KB into the stage's block).
      auto half_kmajor = [&](uint32_t d, uint32_t a, uint32_t bb, uint64_t ext_a, uint32_t ld_s, int hf) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_bf16_ss(tmem + d + 64 * hf, make_sw128_desc(a + off, 16, 1024),
                      make_sw128_desc(bb + hf * 8192 + off, 16, 1024), id_half, kk > 0);
        }
        mma_bf16_ss(tmem + d + 64 * hf, ext_a, make_noswz_desc(ld_s + hf * 1024, 128, 128), id_half, true);
      };
      auto issue_half = [&](int st, int hf) {
        const uint32_t ld_s = ld_a + st * L::kLdStride;
        half_kmajor(T_DP, v_a, do_a + st * L::kTile, ext_delta, ld_s, hf);
        half_kmajor(T_S, kn_a, qn_a + st * L::kTile, ext_lse, ld_s, hf);
      };
      bool ok = mbar_wait(&bars->kv_full, 0, p.status, kErrKv);
      if (ok && n_steps > 0) {
        ok = mbar_wait(&bars->q_full[0], 0, p.status, kErrQFull);
        if (ok) {
          tc_fence_after();
          issue_half(0, 0);
          mma_commit(&bars->s_lo);
          issue_half(0, 1);
          mma_commit(&bars->s_hi);
        }
      }
      for (int t = 0; t < n_steps && ok; ++t) {
        const int st = t & 1, st1 = st ^ 1;
        const uint32_t qn_s = qn_a + st * L::kTile, do_s = do_a + st * L::kTile;
        // G_k += dS'^T Q^ and dV += P^T dO over the queries of K-steps [k_begin, k_begin + 4)
        auto dkdv = [&](int k_begin) {
#pragma unroll
          for (int kk = k_begin; kk < k_begin + 4; ++kk) {
            mma_bf16_ts(tmem + T_DK, tmem + T_S + kk * 16 + 8, make_sw128_desc(qn_s + kk * 2048, 16384, 1024),
                        id_ts, t > 0 || kk > 0);
            mma_bf16_ts(tmem + T_DV, tmem + T_S + kk * 16, make_sw128_desc(do_s + kk * 2048, 16384, 1024), id_ts,
                        t > 0 || kk > 0);
          }
        };
        const bool next = t + 1 < n_steps;
        if (!(ok = mbar_wait(&bars->ds_half, t & 1, p.status, kErrDsReady))) break;
        tc_fence_after();
        dkdv(0);
        if (next) {
          // queries 0..63 of step t+1: their S^T / dP^T columns have been read and
          // P^T / dS'^T of step t there are consumed by the products just issued
          if (!(ok = mbar_wait(&bars->q_full[st1], ((t + 1) >> 1) & 1, p.status, kErrQFull))) break;
          tc_fence_after();
          issue_half(st1, 0);
          mma_commit(&bars->s_lo);
        }
        if (!(ok = mbar_wait(&bars->ds_ready, t & 1, p.status, kErrDsReady))) break;
        tc_fence_after();
        dkdv(4);
        mma_commit(&bars->q_empty[st]);   // step t's stage (Q^, dO, pieces) has been read
        if (next) {
          issue_half(st1, 1);
          mma_commit(&bars->s_hi);
        }
      }
      if (ok) mma_commit(&bars->acc_full);
    }
  } else {
    // ------------------------------------------------------------ compute warpgroups
    const int wg = warp >> 2;               // query columns [16 wg, +16) of each 64-column half
    const int j = threadIdx.x & 127;        // key row within the tile == TMEM lane
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const int bar_id = 1 + wg;
    // query rows that see key n0 + j: the non-global rows [row_min, row_max),
    // every row from global_q_row on, and every row if the key is global
    int row_min, row_max;
    key_rows(p.mask, n0 + j, row_min, row_max);
    const bool key_global = n0 + j >= p.mask.global_key && n0 + j < p.seqlen_kv;
    const bool drains = wg * 32 < D;
    bool ok = true;
    for (int t = 0; t < n_steps; ++t) {
      const int qt = bs.abs_step(t) / group;
      const int q0 = qt * 128;
      const bool diag = bs.diag(t, qt);
#pragma unroll
      for (int grp = 0; grp < 2; ++grp) {
        ok = warp_wait(grp ? &bars->s_hi : &bars->s_lo, t & 1, ok, p.status, kErrSFull);
        if (ok) {
          tc_fence_after();
          const int col0 = grp * 64 + wg * 16;
          uint32_t sr[16], dpr[16];
          tmem_ld16(tmem + lane_base + T_S + col0, sr);
          tmem_ld16(tmem + lane_base + T_DP + col0, dpr);
          tmem_wait_ld();
          uint32_t pk[8], dk[8];
          if (!diag) {
#pragma unroll
            for (int c = 0; c < 16; c += 2) {
              float p0, p1;
              if (((c >> 1) & 3) == 3) {   // one pair in four on the FMA pipe
                exp2_poly_pair(f2_pack(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])), p0, p1);
              } else {
                p0 = fast_exp2(__uint_as_float(sr[c]));
                p1 = fast_exp2(__uint_as_float(sr[c + 1]));
              }
              float d0, d1;
              f2_unpack(f2_mul(f2_pack(__uint_as_float(dpr[c]), __uint_as_float(dpr[c + 1])), f2_pack(p0, p1)), d0, d1);
              pk[c >> 1] = pack_bf16x2(p0, p1);
              dk[c >> 1] = pack_bf16x2(d0, d1);
            }
          } else {
            // columns [lim, hl) see key j, and so do global rows (c >= glim) or all if the key is global
            const int lim = row_min - (q0 + col0), hl = row_max - (q0 + col0);
            const int glim = key_global ? -128 : p.mask.global_q_row - (q0 + col0);
#pragma unroll
            for (int c = 0; c < 16; c += 2) {
              const bool v0 = (c >= lim && c < hl) || c >= glim, v1 = (c + 1 >= lim && c + 1 < hl) || c + 1 >= glim;
              const float p0 = v0 ? fast_exp2(__uint_as_float(sr[c])) : 0.f;
              const float p1 = v1 ? fast_exp2(__uint_as_float(sr[c + 1])) : 0.f;
              pk[c >> 1] = pack_bf16x2(p0, p1);
              dk[c >> 1] = pack_bf16x2(p0 * __uint_as_float(dpr[c]), p1 * __uint_as_float(dpr[c + 1]));
            }
          }
          // P^T and dS'^T of these 16 queries over the S^T columns just read
          tmem_st8(tmem + lane_base + T_S + col0, pk);
          tmem_st8(tmem + lane_base + T_S + col0 + 8, dk);
          tmem_wait_st();
          tc_fence_before();
        }
        named_bar_sync(bar_id, 128);
        if (j == 0 && ok) mbar_arrive(grp ? &bars->ds_ready : &bars->ds_half);
      }
    }

    // ---------------------------------------------------------- epilogue
    // dV and G_k of this unit (fp32 in TMEM) into the fp32 accumulators, as in
    // the main kernel: staged in the idle Q^ / dO stage buffers, then two bulk
    // reduce-adds per warpgroup.
    ok = warp_wait(&bars->acc_full, 0, ok && n_steps > 0, p.status, kErrAcc);
    if (ok && drains) {
      tc_fence_after();
      uint32_t rv[32], rk32[32];
      tmem_ld32(tmem + lane_base + T_DV + wg * 32, rv);
      tmem_ld32(tmem + lane_base + T_DK + wg * 32, rk32);
      tmem_wait_ld();
      uint8_t* sv = smem + L::kQn + wg * 16384 + j * 128;
      uint8_t* sk = smem + L::kDo + wg * 16384 + j * 128;
#pragma unroll
      for (int piece = 0; piece < 8; ++piece) {
        const uint32_t off = ((piece ^ (j & 7)) & 7) << 4;
        *reinterpret_cast<uint4*>(sv + off) = make_uint4(rv[4 * piece], rv[4 * piece + 1], rv[4 * piece + 2], rv[4 * piece + 3]);
        *reinterpret_cast<uint4*>(sk + off) =
            make_uint4(rk32[4 * piece], rk32[4 * piece + 1], rk32[4 * piece + 2], rk32[4 * piece + 3]);
      }
      fence_proxy_async_smem();
    }
    named_bar_sync(bar_id, 128);
    if (j == 0 && ok && drains) {
      tma_reduce_add_4d(&tm_dv, smem + L::kQn + wg * 16384, wg * 32, hk, n0, b);
      tma_reduce_add_4d(&tm_dk, smem + L::kDo + wg * 16384, wg * 32, hk, n0, b);
      tma_store_commit();
      tma_store_wait_read();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ dq pass
// Deterministic backward only.  Query-major: one CTA per 128-row query
// sub-tile of the forward schedule (block 2u + s runs sub-tile s of unit u),
// so each query row's G_q is summed over its visible kv tiles in tile order
// inside one CTA, with no reductions across CTAs.  Q^ and dO of the sub-tile
// stay in shared memory; K^ streams through a 3-stage ring and V through a
// 2-stage one (K^ is read twice per tile, by S and by G_q, so it stays
// longer).  Per kv tile j, in TMEM:
//   S    = Q^ K^_j^T                    -> S_buf[j % 2]  (log2 units)
//   dP   = dO V_j^T                     -> DP
//   dS'  = exp2(S - lse2) (dP - Delta)  -> bf16 pairs over the first half of
//                                          each warpgroup's S_buf columns
//   G_q += dS' K^_j                     -> GQ  (A from TMEM, K^ MN-major)
// and at the end G_q goes to the fp32 dq buffer for the finalize kernel.
// Roles: warpgroups 0 and 1 own key columns [0, 64) and [64, 128) of every
// row (thread = query row = TMEM lane), warp 8 issues MMAs, warp 9 runs TMA.
// Per tile j the MMA thread issues dP(j+1) as soon as both warpgroups have
// read dP(j), G_q(j) once dS'(j) is written, then S(j+2): the tensor pipe
// holds the next tile's products while the softmax runs.
constexpr int kDqThreads = 320;
constexpr int kDqKStages = 3, kDqVStages = 2;

template <int D>
struct DqLayout {
  static constexpr int kTile = 128 * D * 2;  // [128][D] bf16
  static constexpr int kQn = 0;
  static constexpr int kDo = kQn + kTile;
  static constexpr int kK = kDo + kTile;                // kDqKStages
  static constexpr int kV = kK + kDqKStages * kTile;    // kDqVStages
  static constexpr int kBars = kV + kDqVStages * kTile;
  static constexpr int kTmemSlot = kBars + 16 * 8;
  static constexpr int kTotal = kTmemSlot + 16;
};

struct DqBars {
  uint64_t q_full, dp_free, ds_ready, gq_full;
  uint64_t s_full[2];
  uint64_t k_full[kDqKStages], k_empty[kDqKStages], v_full[kDqVStages], v_empty[kDqVStages];
};
static_assert(sizeof(DqBars) <= 16 * 8, "dq barriers exceed their slot");

template <int D>
__global__ void __launch_bounds__(kDqThreads, 1)
bca_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_qn, const __grid_constant__ CUtensorMap tm_do,
                  const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                  const BwdParams p, const int smem_alloc) {
  using L = DqLayout<D>;
  const int32_t* u = p.dq_units + (size_t)(blockIdx.x >> 1) * kFwdUnitInts;
  if constexpr (kDebugChecks) {
    if (!fwd_unit_in_range(u, p.batch, p.heads_q, p.heads_kv, p.seqlen_q, p.seqlen_kv, p.status)) return;
  }
  const int sub = blockIdx.x & 1;
  const int h = __ldg(u + (sub ? 4 : 2));
  if (h < 0) return;  // the unit has one sub-tile: this CTA has no work
  extern __shared__ uint8_t smem_raw[];
  const uintptr_t base = (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023);
  uint8_t* smem = reinterpret_cast<uint8_t*>(base);
  if (base - reinterpret_cast<uintptr_t>(smem_raw) + L::kTotal > (uintptr_t)smem_alloc) {
    if (threadIdx.x == 0) atomicCAS(p.status, 0, kErrSmem);
    return;
  }
  DqBars* bars = reinterpret_cast<DqBars*>(smem + L::kBars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kTmemSlot);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = __ldg(u + 0), hk = __ldg(u + 1);
  const int m0 = __ldg(u + (sub ? 5 : 3));
  const FwdTiles ft = fwd_tiles(u);   // the kv tiles this query tile visits (bca_mask.cuh)
  const int n_vis = ft.count();

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->dp_free, 2);   // one arrival per warpgroup
    mbar_init(&bars->ds_ready, 2);
    mbar_init(&bars->gq_full, 1);
    for (int i = 0; i < 2; ++i) mbar_init(&bars->s_full[i], 1);
    for (int i = 0; i < kDqKStages; ++i) {
      mbar_init(&bars->k_full[i], 1);
      mbar_init(&bars->k_empty[i], 1);
    }
    for (int i = 0; i < kDqVStages; ++i) {
      mbar_init(&bars->v_full[i], 1);
      mbar_init(&bars->v_empty[i], 1);
    }
    fence_mbar_init();
  }
  if (warp == 9 && lane == 0) {
    tma_prefetch_desc(&tm_qn);
    tma_prefetch_desc(&tm_do);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 8) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  constexpr uint32_t T_S = 0, T_DP = 256, T_GQ = 384;  // S_buf[i] at columns [128 i, 128 i + 128)

  if (warp == 9) {
    // ------------------------------------------------------------ TMA producer
    if (elect_one()) {
      mbar_arrive_expect_tx(&bars->q_full, 2 * L::kTile);
      for (int box = 0; box < D / 64; ++box) {
        tma_load_4d(smem + L::kQn + box * 16384, &tm_qn, &bars->q_full, box * 64, h, m0, b);
        tma_load_4d(smem + L::kDo + box * 16384, &tm_do, &bars->q_full, box * 64, h, m0, b);
      }
      for (int j = 0; j < n_vis; ++j) {
        const int n0 = ft.tile(j) * 128;
        const int ks = j % kDqKStages, vs = j % kDqVStages;
        if (!mbar_wait(&bars->k_empty[ks], ((j / kDqKStages) & 1) ^ 1, p.status, kErrDqKEmpty)) break;
        mbar_arrive_expect_tx(&bars->k_full[ks], L::kTile);
        for (int box = 0; box < D / 64; ++box)
          tma_load_4d(smem + L::kK + ks * L::kTile + box * 16384, &tm_k, &bars->k_full[ks], box * 64, hk, n0, b);
        if (!mbar_wait(&bars->v_empty[vs], ((j / kDqVStages) & 1) ^ 1, p.status, kErrDqVEmpty)) break;
        mbar_arrive_expect_tx(&bars->v_full[vs], L::kTile);
        for (int box = 0; box < D / 64; ++box)
          tma_load_4d(smem + L::kV + vs * L::kTile + box * 16384, &tm_v, &bars->v_full[vs], box * 64, hk, n0, b);
      }
    }
  } else if (warp == 8) {
    // ------------------------------------------------------------ MMA issuer
    if (elect_one()) {
      constexpr uint32_t id_s = make_idesc_bf16(128, 128, false, false);  // S, dP: both operands K-major
      constexpr uint32_t id_g = make_idesc_bf16(128, D, false, true);     // G_q: A from TMEM, B MN-major
      const uint32_t qn_a = smem_u32(smem + L::kQn), do_a = smem_u32(smem + L::kDo);
      const uint32_t k_a = smem_u32(smem + L::kK), v_a = smem_u32(smem + L::kV);
      // C[128 x 128] = A[128 x D] B[128 x D]^T, both K-major in 64-feature boxes
      auto mma_kk = [&](uint32_t d, uint32_t a, uint32_t bb) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_bf16_ss(tmem + d, make_sw128_desc(a + off, 16, 1024), make_sw128_desc(bb + off, 16, 1024), id_s,
                      kk > 0);
        }
      };
      auto issue_s = [&](int j) { mma_kk(T_S + 128 * (j & 1), qn_a, k_a + (j % kDqKStages) * L::kTile); };
      auto issue_dp = [&](int j) {
        mma_kk(T_DP, do_a, v_a + (j % kDqVStages) * L::kTile);
        mma_commit(&bars->v_empty[j % kDqVStages]);   // V_j is read only by dP(j)
      };
      bool ok = n_vis > 0 && mbar_wait(&bars->q_full, 0, p.status, kErrDqQ);
      ok = ok && mbar_wait(&bars->k_full[0], 0, p.status, kErrDqK);
      ok = ok && mbar_wait(&bars->v_full[0], 0, p.status, kErrDqV);
      if (ok) {
        tc_fence_after();
        issue_s(0);
        issue_dp(0);
        mma_commit(&bars->s_full[0]);
      }
      if (ok && n_vis > 1) {
        ok = mbar_wait(&bars->k_full[1 % kDqKStages], 0, p.status, kErrDqK);
        if (ok) {
          tc_fence_after();
          issue_s(1);
        }
      }
      for (int j = 0; j < n_vis && ok; ++j) {
        if (j + 1 < n_vis) {
          // dP(j+1) overwrites DP once both warpgroups hold dP(j) in registers
          if (!(ok = mbar_wait(&bars->dp_free, j & 1, p.status, kErrDqDpFree))) break;
          const int j1 = j + 1;
          if (!(ok = mbar_wait(&bars->v_full[j1 % kDqVStages], (j1 / kDqVStages) & 1, p.status, kErrDqV))) break;
          tc_fence_after();
          issue_dp(j1);
          mma_commit(&bars->s_full[j1 & 1]);   // S(j+1) was issued earlier
        }
        if (!(ok = mbar_wait(&bars->ds_ready, j & 1, p.status, kErrDqDsReady))) break;
        tc_fence_after();
        // G_q += dS'(j) K^_j: K-step kk covers keys [16 kk, 16 kk + 16); warpgroup
        // w wrote the packed pairs of keys [64 w, 64 w + 64) at S_buf + 64 w
        const uint32_t ks = k_a + (j % kDqKStages) * L::kTile;
        const uint32_t sb = T_S + 128 * (j & 1);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ts(tmem + T_GQ, tmem + sb + (kk >> 2) * 64 + (kk & 3) * 8,
                      make_sw128_desc(ks + kk * 2048, 16384, 1024), id_g, j > 0 || kk > 0);
        mma_commit(&bars->k_empty[j % kDqKStages]);
        if (j + 2 < n_vis) {
          // S(j+2) overwrites S_buf[j % 2] after G_q(j) (issued before it) has read dS'(j)
          const int j2 = j + 2;
          if (!(ok = mbar_wait(&bars->k_full[j2 % kDqKStages], (j2 / kDqKStages) & 1, p.status, kErrDqK))) break;
          tc_fence_after();
          issue_s(j2);
        }
      }
      mma_commit(&bars->gq_full);
    }
  } else {
    // ------------------------------------------------------------ softmax warpgroups
    const int wg = warp >> 2;             // key columns [64 wg, 64 wg + 64)
    const int r = threadIdx.x & 127;      // query row within the tile == TMEM lane
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const int bar_id = 1 + wg;
    const int row = m0 + r;
    // -lse log2(e) and -Delta of the row, rebuilt from the prep kernel's three
    // bf16 pieces each (padding rows past seqlen_q hold zeros)
    float nl, nd;
    {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(
          p.ld + (((size_t)b * p.heads_q + h) * p.seqlen_q_pad + row) * 4));
      nl = (bf16_lo(v.x) + bf16_hi(v.x)) + bf16_lo(v.y);
      nd = (bf16_hi(v.y) + bf16_lo(v.z)) + bf16_hi(v.z);
    }
    // visible keys of the row: [kv_first, limit) and the global block's
    int limit = p.seqlen_kv, kv_first = 0;
    if (row < p.seqlen_q) row_keys(p.mask, row, kv_first, limit);
    const uint64_t nl2 = f2_pack(nl, nl), nd2 = f2_pack(nd, nd);
    bool ok = true;
    // Every thread runs all n_vis iterations and reaches every named barrier
    // even after a failed wait; only the work is skipped.
    for (int j = 0; j < n_vis; ++j) {
      ok = warp_wait(&bars->s_full[j & 1], (j >> 1) & 1, ok, p.status, kErrDqSFull);
      const uint32_t t_s = tmem + lane_base + T_S + 128 * (j & 1) + 64 * wg;
      uint32_t sa[32], sb[32], da[32], db[32];
      if (ok) {
        tc_fence_after();
        tmem_ld32(t_s, sa);
        tmem_ld32(t_s + 32, sb);
        tmem_ld32(tmem + lane_base + T_DP + 64 * wg, da);
        tmem_ld32(tmem + lane_base + T_DP + 64 * wg + 32, db);
        tmem_wait_ld();
        tc_fence_before();
      }
      named_bar_sync(bar_id, 128);
      if (r == 0 && ok) mbar_arrive(&bars->dp_free);
      if (ok) {
        const int tile = ft.tile(j);
        const bool masked = ft.masked(j, p.mask.global_key, p.seqlen_kv);
        uint32_t pk[32];
        auto sval = [&](int c) { return __uint_as_float(c < 32 ? sa[c] : sb[c - 32]); };
        auto dval = [&](int c) { return __uint_as_float(c < 32 ? da[c] : db[c - 32]); };
        if (masked) {
          const int c0 = tile * 128 + 64 * wg;
          // columns [lo, lim) and the global block's [glo, ghi) are visible
          const int lim = limit - c0, lo = kv_first - c0;
          const int glo = p.mask.global_key - c0, ghi = p.seqlen_kv - c0;
#pragma unroll
          for (int c = 0; c < 64; c += 2) {
            const bool v0 = (c >= lo && c < lim) || (c >= glo && c < ghi);
            const bool v1 = (c + 1 >= lo && c + 1 < lim) || (c + 1 >= glo && c + 1 < ghi);
            const float p0 = v0 ? fast_exp2(sval(c) + nl) : 0.f;
            const float p1 = v1 ? fast_exp2(sval(c + 1) + nl) : 0.f;
            pk[c >> 1] = pack_bf16x2(p0 * (dval(c) + nd), p1 * (dval(c + 1) + nd));
          }
        } else {
#pragma unroll
          for (int c = 0; c < 64; c += 2) {
            const uint64_t a2 = f2_add(f2_pack(sval(c), sval(c + 1)), nl2);
            float p0, p1;
            if (((c >> 1) & 3) == 3) {   // one pair in four on the FMA pipe
              exp2_poly_pair(a2, p0, p1);
            } else {
              float a0, a1;
              f2_unpack(a2, a0, a1);
              p0 = fast_exp2(a0);
              p1 = fast_exp2(a1);
            }
            const uint64_t d2 = f2_mul(f2_add(f2_pack(dval(c), dval(c + 1)), nd2), f2_pack(p0, p1));
            float d0, d1;
            f2_unpack(d2, d0, d1);
            pk[c >> 1] = pack_bf16x2(d0, d1);
          }
        }
        tmem_st32(t_s, pk);   // dS' pairs over columns [64 wg, 64 wg + 32) of S_buf
        tmem_wait_st();
        tc_fence_before();
      }
      named_bar_sync(bar_id, 128);
      if (r == 0 && ok) mbar_arrive(&bars->ds_ready);
    }

    // Epilogue: G_q (fp32) of the row, warpgroup w storing columns [w D/2, w D/2 + D/2).
    ok = warp_wait(&bars->gq_full, 0, ok, p.status, kErrDqGq);
    if (ok) {
      tc_fence_after();
      constexpr int kCols = D / 2;
      float* dst = p.dqacc + (((size_t)b * p.seqlen_q + row) * p.heads_q + h) * D + wg * kCols;
#pragma unroll 1
      for (int c = 0; c < kCols / 32; ++c) {
        uint32_t g[32];
        tmem_ld32(tmem + lane_base + T_GQ + wg * kCols + c * 32, g);
        tmem_wait_ld();
        if (n_vis == 0) {   // (chunks are never empty, so every row sees some key)
#pragma unroll
          for (int i = 0; i < 32; ++i) g[i] = 0u;
        }
        if (row < p.seqlen_q) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
          for (int i = 0; i < 8; ++i) d4[i] = make_uint4(g[4 * i], g[4 * i + 1], g[4 * i + 2], g[4 * i + 3]);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int D>
cudaError_t launch_split_d(const CUtensorMap& t_k, const CUtensorMap& t_v, const CUtensorMap& t_qn,
                           const CUtensorMap& t_do, const CUtensorMap& t_dv, const CUtensorMap& t_dk,
                           const BwdParams& p, int n_units, int n_dq_units, cudaStream_t stream) {
  using LK = DkdvLayout<D>;
  using LQ = DqLayout<D>;
  static uint64_t configured_kv = 0, configured_dq = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  int max_optin = 0;
  e = cudaDeviceGetAttribute(&max_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e != cudaSuccess) return e;
  const int alloc_kv = LK::kTotal + 1024 <= max_optin ? LK::kTotal + 1024 : max_optin;
  const int alloc_dq = LQ::kTotal + 1024 <= max_optin ? LQ::kTotal + 1024 : max_optin;
  if (alloc_kv < LK::kTotal || alloc_dq < LQ::kTotal) return cudaErrorInvalidConfiguration;
  e = set_smem_once(configured_kv, dev, bca_bwd_dkdv_kernel<D>, alloc_kv);
  if (e != cudaSuccess) return e;
  e = set_smem_once(configured_dq, dev, bca_bwd_dq_kernel<D>, alloc_dq);
  if (e != cudaSuccess) return e;
  if (n_dq_units > 0) {
    bca_bwd_dq_kernel<D><<<2 * n_dq_units, kDqThreads, alloc_dq, stream>>>(t_qn, t_do, t_k, t_v, p, alloc_dq);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (n_units > 0) {
    bca_bwd_dkdv_kernel<D><<<n_units, kThreads, alloc_kv, stream>>>(t_k, t_v, t_qn, t_do, t_dv, t_dk, p, alloc_kv);
    e = cudaGetLastError();
  }
  return e;
}

}  // namespace

cudaError_t launch_bwd_split(const CUtensorMap& t_k, const CUtensorMap& t_v, const CUtensorMap& t_qn,
                             const CUtensorMap& t_do, const CUtensorMap& t_dv, const CUtensorMap& t_dk,
                             const BwdParams& p, int head_dim, int n_units, int n_dq_units, cudaStream_t stream) {
  if (head_dim == 128) return launch_split_d<128>(t_k, t_v, t_qn, t_do, t_dv, t_dk, p, n_units, n_dq_units, stream);
  return launch_split_d<64>(t_k, t_v, t_qn, t_do, t_dv, t_dk, p, n_units, n_dq_units, stream);
}

}  // namespace magi
