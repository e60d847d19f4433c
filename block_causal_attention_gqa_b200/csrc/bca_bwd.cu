// Backward of block-causal GQA attention with QK-RMSNorm, sm_100a.
//
// The backward recomputes the forward's logits from the forward's own
// operands: the folded query Q^ = bf16(q r_q gamma_q gamma_k scale log2(e))
// and the normalised keys K^ = bf16(k r_k) from the same bca_knorm_kernel, so
// the recomputed P matches the forward's log-sum-exp up to fp32 accumulation
// order (the helpers in bca_norm.cuh fix the rounding points for both passes).
//
// Three launches on the caller's stream:
//   1. prep      one warp per row.  Query rows: Q^ into the workspace; Delta =
//                rowsum(dO * O); -lse*log2(e) and -Delta, each split into three
//                bf16 pieces, in a 16-byte row per query (128-padded layout);
//                zero the row's fp32 dq accumulator (not needed when
//                deterministic: the dq pass stores every row).  Key rows: K^ into the
//                workspace (knorm_row, as the forward's key pre-pass) and zero
//                the row's fp32 dV / G_k accumulators.  Also zeroes dgamma.
//   2. main      one CTA per (batch, kv head, 128-key tile, query-tile range).
//                It keeps K^ and V of its tile in shared memory and walks every
//                (query tile, group head) of its range (backward schedule,
//                bca_sched.h):
//                  S'^T  = K^ Q^^T - lse log2e    dP'^T = V dO^T - Delta    (TMEM)
//                  P^T   = exp2(S'^T)   (masked on diagonal steps)
//                  dS'^T = P^T dP'^T    (bf16 in shared memory)
//                  dV  += P^T dO        (P^T from TMEM)
//                  G_k += dS'^T Q^      -> gamma_k * dk~ = G_k / (r_k log2 e)
//                  G_q  = dS' K^        -> dq~ = scale gamma_k * G_q, drained
//                                          through shared memory with TMA bulk
//                                          reduce-adds into the fp32 accumulator
//                The -lse and -Delta terms come out of the tensor core: one extra
//                K-step of 16 multiplies constant rows (1 at the pieces' k) by the
//                pieces, so the softmax only computes exp2 (one pair in four by
//                a cubic on the FMA pipe, off MUFU) and one product.
//                At the end the CTA adds dV and G_k into fp32 accumulators (long
//                query ranges are split into pieces, so several CTAs may add to
//                one kv tile).
//   3. finalize  one warp per row: dq, dk through the RMSNorm Jacobian, dv, and
//                dgamma_q, dgamma_k.
// Deterministic backward (dims.deterministic): no sum depends on timing.  In
// place of the main kernel, bca_bwd_split.cu runs a query-major dq pass (one
// CTA per query tile owns its rows' G_q) and a kv-major dK/dV pass without
// G_q, with every kv tile one unit, so dV and G_k are added once onto zero;
// the finalize takes whole tokens (angle gradients summed in registers) and
// writes per-block dgamma partials that one small kernel adds in block order.
// The dq pass recomputes S and dP, so the tensor work is 7/5 of the default
// path's.
// These are the five matrix products of the Flash-Attention backward (2.5x the
// forward's FLOPs, MAGI-1 App. B.2.1).  Because gamma_k is folded into the
// query operand, dgamma_k[d] is undefined (NaN/inf) where gamma_k[d] == 0.
//
// Main-kernel roles: warpgroups 0-3 (warps 0-15) each own query columns
// [16w, 16w+16) and [64+16w, 64+16w+16) of S^T and dP^T (thread i of a
// warpgroup owns key row i = TMEM lane i) and 32 columns of G_q to drain;
// warp 16 issues tcgen05 MMAs; warp 17 runs TMA.  All warpgroups finish the
// first 64 query columns before the second, so the dK~/dV products of the
// first half run while the second half is computed.  TMEM: S^T [0,128) (P^T
// of K-step k, 16 queries, overwrites columns [16k, 16k+8) once read), dP^T
// [128,256) (G_q overwrites it), dV [256,256+D), G_k [384,384+D).
//
// Per step the MMA warp issues, in order: dK~/dV for queries 0..63 (after the
// first half of the softmax), dK~/dV for 64..127 and G_q (after the second
// half), then S^T of the next step (its P^T has been read) and, once G_q has
// been drained to registers, dP^T of the next step.  A Q^/dO stage is used by
// S^T, dP^T, dK~, dV, then holds the dq staging until its bulk reduction has
// read it; L2 prefetches of the next step's tiles hide part of the reload.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "bca_bwd_common.cuh"
#include "bca_kernels.h"
#include "bca_mask.cuh"
#include "bca_norm.cuh"
#include "sm100.cuh"

namespace magi {
namespace {

using namespace sm100;

// ------------------------------------------------------------------ prep
// Lane l holds elements [l*E, l*E+E) of a D = 32*E row.
template <int D>
struct RowIO {
  static constexpr int E = D / 32;
  __device__ static void load_bf16(const uint16_t* row, int lane, float (&x)[E]) {
    if constexpr (E == 4) {
      const uint2 w = *reinterpret_cast<const uint2*>(row + lane * 4);
      x[0] = bf16_lo(w.x); x[1] = bf16_hi(w.x); x[2] = bf16_lo(w.y); x[3] = bf16_hi(w.y);
    } else {
      const uint32_t w = *reinterpret_cast<const uint32_t*>(row + lane * 2);
      x[0] = bf16_lo(w); x[1] = bf16_hi(w);
    }
  }
  __device__ static void store_bf16(uint16_t* row, int lane, const float (&x)[E]) {
    if constexpr (E == 4) {
      uint2 w;
      w.x = pack_bf16x2(x[0], x[1]);
      w.y = pack_bf16x2(x[2], x[3]);
      *reinterpret_cast<uint2*>(row + lane * 4) = w;
    } else {
      *reinterpret_cast<uint32_t*>(row + lane * 2) = pack_bf16x2(x[0], x[1]);
    }
  }
  __device__ static void load_f32(const float* row, int lane, float (&x)[E]) {
    if constexpr (E == 4) {
      const float4 v = *reinterpret_cast<const float4*>(row + lane * 4);
      x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
    } else {
      const float2 v = *reinterpret_cast<const float2*>(row + lane * 2);
      x[0] = v.x; x[1] = v.y;
    }
  }
  __device__ static void store_zero_f32(float* row, int lane) {
    if constexpr (E == 4) {
      *reinterpret_cast<float4*>(row + lane * 4) = make_float4(0.f, 0.f, 0.f, 0.f);
    } else {
      *reinterpret_cast<float2*>(row + lane * 2) = make_float2(0.f, 0.f);
    }
  }
};

// x = hi + mid + lo with bf16 pieces (about 24 significant bits in all).
__device__ __forceinline__ void split3(float x, uint16_t& hi, uint16_t& mid, uint16_t& lo) {
  const __nv_bfloat16 h = __float2bfloat16_rn(x);
  const float r1 = x - __bfloat162float(h);
  const __nv_bfloat16 m = __float2bfloat16_rn(r1);
  const float r2 = r1 - __bfloat162float(m);
  const __nv_bfloat16 l = __float2bfloat16_rn(r2);
  hi = __bfloat16_as_ushort(h);
  mid = __bfloat16_as_ushort(m);
  lo = __bfloat16_as_ushort(l);
}
// Packs the pieces of a (k = 0, 1, 2) and b (k = 3, 4, 5) into the first
// three words of a 16-byte row: returns word 0, writes words 1 and 2.
__device__ __forceinline__ uint32_t split3_lo2(float a, uint32_t& w1, float b, uint32_t& w2) {
  uint16_t ah, am, al, bh, bm, bl;
  split3(a, ah, am, al);
  split3(b, bh, bm, bl);
  w1 = (uint32_t)al | ((uint32_t)bh << 16);
  w2 = (uint32_t)bm | ((uint32_t)bl << 16);
  return (uint32_t)ah | ((uint32_t)am << 16);
}

template <int D>
__global__ void __launch_bounds__(256) bca_bwd_prep_kernel(const BwdParams p) {
  using IO = RowIO<D>;
  constexpr int E = IO::E;
  __shared__ float qscale[D];
  for (int d = threadIdx.x; d < D; d += blockDim.x) qscale[d] = qscale_of(p.gamma_q, p.gamma_k, p.scale_log2, d);
  if (blockIdx.x == 0 && threadIdx.x < D) {
    if (p.dgamma_q) p.dgamma_q[threadIdx.x] = 0.f;
    if (p.dgamma_k) p.dgamma_k[threadIdx.x] = 0.f;
  }
  // rotary angle gradients are sums over batch and heads: zero them here
  {
    const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x, nth = (int64_t)gridDim.x * blockDim.x;
    if (p.drope_q)
      for (int64_t i = tid; i < (int64_t)p.seqlen_q * (D / 2); i += nth) p.drope_q[i] = 0.f;
    if (p.drope_k)
      for (int64_t i = tid; i < (int64_t)p.seqlen_kv * (D / 2); i += nth) p.drope_k[i] = 0.f;
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t n_q = (int64_t)p.batch * p.seqlen_q * p.heads_q;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x / 32);
  const int64_t n_k = (int64_t)p.batch * p.seqlen_kv * p.heads_kv;
  // One warp per row: query rows [0, n_q), then key rows.  For a query row the
  // sum of squares uses the order that the forward's prologue reproduces, so
  // Q^ is bit-identical to the forward's.  For a key row, K^ = bf16(k r_k)
  // exactly as the forward's key pre-pass computes it, and the row's fp32
  // dV / G_k accumulators are zeroed.
  for (int64_t rr = (int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5); rr < n_q + n_k; rr += warps) {
    if (rr >= n_q) {
      const int64_t r = rr - n_q;
      const float* ang = p.rope_k ? p.rope_k + ((r / p.heads_kv) % p.seqlen_kv) * (D / 2) : nullptr;
      knorm_row<D>(p.k + r * D, p.kn + r * D, lane, p.eps, ang);
      IO::store_zero_f32(p.dvacc + r * D, lane);
      IO::store_zero_f32(p.dkacc + r * D, lane);
      continue;
    }
    const int64_t r = rr;
    float x[E], o[E], g[E];
    IO::load_bf16(p.q + r * D, lane, x);
    IO::load_bf16(p.out + r * D, lane, o);
    IO::load_bf16(p.dout + r * D, lane, g);
    const float rq = rms_inv<D>(warp_sumsq_row<E>(x), p.eps);
    if (p.rope_q) {   // rotate after the RMS of the raw row, as the forward's prologue does
      float y[E];
      rope_warp<D>(x, p.rope_q + ((r / p.heads_q) % p.seqlen_q) * (D / 2), lane, y);
#pragma unroll
      for (int e = 0; e < E; ++e) x[e] = y[e];
    }
    float qh[E];
#pragma unroll
    for (int e = 0; e < E; ++e) qh[e] = x[e] * rq * qscale[lane * E + e];
    IO::store_bf16(p.qn + r * D, lane, qh);
    float dot = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) dot = fmaf(o[e], g[e], dot);
    dot = warp_sum(dot);
    if (!p.deterministic) IO::store_zero_f32(p.dqacc + r * D, lane);   // (the dq pass stores every row)
    if (lane == 0) {
      const int h = (int)(r % p.heads_q);
      const int64_t bs = r / p.heads_q;
      const int s = (int)(bs % p.seqlen_q);
      const int b = (int)(bs / p.seqlen_q);
      const int64_t bh = (int64_t)b * p.heads_q + h;
      // -lse (log2 units) and -Delta, each as hi + mid + lo bf16 pieces: the
      // main kernel adds them to S^T and dP^T with one extra MMA K-step
      const float nl = -(__ldg(p.lse + bh * p.seqlen_q + s) * kLog2e), nd = -dot;
      uint4 v;
      v.x = split3_lo2(nl, v.y, nd, v.z);
      v.w = 0u;
      *reinterpret_cast<uint4*>(p.ld + (bh * p.seqlen_q_pad + s) * 4) = v;
    }
  }
}

// ------------------------------------------------------------------ main
template <int D>
struct BwdLayout {
  static constexpr int kTile = 128 * D * 2;      // [128][D] bf16
  static constexpr int kK = 0;                   // raw K tile
  static constexpr int kV = kK + kTile;
  static constexpr int kQn = kV + kTile;         // 2 stages
  static constexpr int kDo = kQn + 2 * kTile;    // 2 stages
  static constexpr int kDs = kDo + 2 * kTile;    // dS^T [128 keys][128 queries] bf16, two 64-wide boxes
  static constexpr int kLd = kDs + 32768;        // 128 query rows x 8 bf16 {-lse2, -Delta pieces}
  static constexpr int kOnes = kLd + 2048;       // constant A rows of the extra K-step (3 x 128 B)
  static constexpr int kBars = kOnes + 384;
  static constexpr int kTmemSlot = kBars + 16 * 8;
  static constexpr int kTotal = kTmemSlot + 16;
};

struct BwdBars {
  uint64_t kv_full, s_full, ld_empty, ds_half, ds_ready, dq_full, dq_drained, acc_full;
  uint64_t q_full[2], q_empty[2];
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
bca_bwd_main_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_qn, const __grid_constant__ CUtensorMap tm_do,
                    const __grid_constant__ CUtensorMap tm_dq, const __grid_constant__ CUtensorMap tm_dv,
                    const __grid_constant__ CUtensorMap tm_dk, const BwdParams p, const int smem_alloc) {
  using L = BwdLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  const uintptr_t base = (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023);
  uint8_t* smem = reinterpret_cast<uint8_t*>(base);
  // The layout needs 1024-byte alignment for the swizzled tiles; refuse to run
  // (status, no access) if the allocation cannot hold it at this alignment.
  if (base - reinterpret_cast<uintptr_t>(smem_raw) + L::kTotal > (uintptr_t)smem_alloc) {
    if (threadIdx.x == 0) atomicCAS(p.status, 0, kErrSmem);
    return;
  }
  BwdBars* bars = reinterpret_cast<BwdBars*>(smem + L::kBars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kTmemSlot);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int32_t* u = p.units + (size_t)blockIdx.x * kUnitInts;
  if constexpr (kDebugChecks) {
    if (!bwd_unit_in_range(u, p.batch, p.heads_q, p.heads_kv, p.seqlen_q, p.seqlen_kv, p.status)) return;
  }
  const int b = __ldg(u + 0), hk = __ldg(u + 1), n0 = __ldg(u + 2);
  // this kv tile's steps t = 0 .. n_steps-1; absolute step s = bs.abs_step(t)
  // is (query tile s / group, head s % group of the kv head's group), and
  // bs.diag(t, qt) says whether the step needs the mask (bca_mask.cuh)
  const BwdSteps bs = bwd_steps(u);
  const int group = p.heads_q / p.heads_kv;
  const int n_steps = bs.count();
  // Within each query tile the group's heads are visited from head rot on:
  // neighbouring kv tiles (which walk the same query tiles at the same time)
  // then add their G_q into different heads' dq rows, not all into the same
  // rows at once.  rot depends on the kv tile only, so all pieces of a tile
  // agree on which step is which head.
  const int rot = (n0 >> 7) % group;

  if (threadIdx.x == 0) {
    mbar_init(&bars->kv_full, 1);
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->ds_half, kComputeWarpgroups);
    mbar_init(&bars->ld_empty, 1);
    mbar_init(&bars->ds_ready, kComputeWarpgroups);
    mbar_init(&bars->dq_full, 1);
    mbar_init(&bars->dq_drained, kComputeWarpgroups);
    mbar_init(&bars->acc_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->q_full[s], 1);
      mbar_init(&bars->q_empty[s], kComputeWarpgroups);   // each warpgroup, once its dq staging is read
    }
    fence_mbar_init();
  }
  // A rows of the extra K-step, read with a zero row-group stride: ones at
  // k = 0..2 (picks -lse2 for S^T), ones at k = 3..5 (picks -Delta for dP^T),
  // and a zero core matrix for k = 8..15.
  if (threadIdx.x < 96) {
    const int blk = threadIdx.x >> 5, w = threadIdx.x & 31;   // 32 words per 128-byte block
    const int k0 = (w & 3) * 2;                                 // k of the word's low half
    auto one_at = [&](int k) { return blk < 2 && k >= 3 * blk && k < 3 * blk + 3; };
    const uint32_t lo = one_at(k0) ? 0x3F80u : 0u, hi = one_at(k0 + 1) ? 0x3F80u : 0u;
    reinterpret_cast<uint32_t*>(smem + L::kOnes)[threadIdx.x] = lo | (hi << 16);
  }
  fence_proxy_async_smem();
  if (warp == kTmaWarp && lane == 0) {
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_qn);
    tma_prefetch_desc(&tm_do);
    tma_prefetch_desc(&tm_dq);
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
        const int qt = sa / group, h = hk * group + (sa % group + rot) % group;
        // the single {-lse, -Delta} buffer: the previous step's S^T/dP^T have read it
        if (t > 0 && !mbar_wait(&bars->ld_empty, (t - 1) & 1, p.status, kErrLdEmpty)) break;
        mbar_arrive_expect_tx(&bars->q_full[st], 2 * L::kTile + 2048);
        for (int box = 0; box < D / 64; ++box) {
          tma_load_4d(smem + L::kQn + st * L::kTile + box * 16384, &tm_qn, &bars->q_full[st], box * 64, h,
                      qt * 128, b);
          tma_load_4d(smem + L::kDo + st * L::kTile + box * 16384, &tm_do, &bars->q_full[st], box * 64, h,
                      qt * 128, b);
        }
        const float* ld_src = p.ld + (((size_t)b * p.heads_q + h) * p.seqlen_q_pad + (size_t)qt * 128) * 4;
        bulk_load(smem + L::kLd, ld_src, 2048, &bars->q_full[st]);
        // warm L2 with the next step's tiles: their loads are issued only once
        // a stage frees, and then wait on memory otherwise
        if (t + 1 < n_steps) {
          const int sa1 = bs.abs_step(t + 1);
          const int qt1 = sa1 / group, h1 = hk * group + (sa1 % group + rot) % group;
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
      constexpr uint32_t id_kk = make_idesc_bf16(128, 128, false, false);  // S^T, dP^T
      constexpr uint32_t id_ts = make_idesc_bf16(128, D, false, true);     // dV (A from TMEM)
      constexpr uint32_t id_km = make_idesc_bf16(128, D, false, true);     // dK~: A K-major, B MN-major
      constexpr uint32_t id_mm = make_idesc_bf16(128, D, true, true);      // dQ~: A MN-major, B MN-major
      const uint32_t kn_a = smem_u32(smem + L::kK), v_a = smem_u32(smem + L::kV);
      const uint32_t qn_a = smem_u32(smem + L::kQn), do_a = smem_u32(smem + L::kDo);
      const uint32_t ds_a = smem_u32(smem + L::kDs);
      // C[128 x 128] = A[128 x D] B[128 x D]^T with both operands K-major, then
      // one K-step more: C += ones(k in pick) x pieces^T, which adds -lse2 (S^T)
      // or -Delta (dP^T) of each query column.  The pieces sit in 16-byte rows
      // (no swizzle: 8-row core matrices of 128 B); the constant A rows are read
      // with a zero row-group stride.  The B core matrix at k = 8..15 is the
      // next row group's (finite) data, multiplied by A's zero core matrix.
      const uint32_t ld_a = smem_u32(smem + L::kLd), ones_a = smem_u32(smem + L::kOnes);
      const uint64_t ext_b = make_noswz_desc(ld_a, 128, 128);
      const uint64_t ext_lse = make_noswz_desc(ones_a, 256, 0), ext_delta = make_noswz_desc(ones_a + 128, 128, 0);
      auto mma_kmajor = [&](uint32_t d, uint32_t a, uint32_t bb, uint64_t ext_a) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_bf16_ss(tmem + d, make_sw128_desc(a + off, 16, 1024), make_sw128_desc(bb + off, 16, 1024), id_kk,
                      kk > 0);
        }
        mma_bf16_ss(tmem + d, ext_a, ext_b, id_kk, true);
      };
      bool ok = mbar_wait(&bars->kv_full, 0, p.status, kErrKv);
      // Issue order per step t: dK~/dV (queries 0..63) | dK~/dV (64..127), G_q |
      // S^T(t+1) | dP^T(t+1), so the next step's products queue right behind
      // this step's without waiting for the issuing thread.
      if (ok && n_steps > 0) {
        ok = mbar_wait(&bars->q_full[0], 0, p.status, kErrQFull);
        if (ok) {
          tc_fence_after();
          mma_kmajor(T_DP, v_a, do_a, ext_delta);
          mma_kmajor(T_S, kn_a, qn_a, ext_lse);
          mma_commit(&bars->s_full);
          mma_commit(&bars->ld_empty);
        }
      }
      for (int t = 0; t < n_steps && ok; ++t) {
        const int st = t & 1;
        const uint32_t qn_s = qn_a + st * L::kTile, do_s = do_a + st * L::kTile;
        // G_k += dS'^T Q^ : A = dS'^T [keys][queries] (K-major), B = Q^ [queries][D] (MN-major);
        // dV += P^T dO : A = P^T (TMEM, K = queries), B = dO [queries][D] (MN-major).
        // K-steps 0..3 (queries 0..63) as soon as that half of dS' and P^T is in place.
        auto dkdv = [&](int k_begin) {
#pragma unroll
          for (int kk = k_begin; kk < k_begin + 4; ++kk) {
            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
            mma_bf16_ss(tmem + T_DK, make_sw128_desc(ds_a + off, 16, 1024),
                        make_sw128_desc(qn_s + kk * 2048, 16384, 1024), id_km, t > 0 || kk > 0);
          }
#pragma unroll
          for (int kk = k_begin; kk < k_begin + 4; ++kk)
            mma_bf16_ts(tmem + T_DV, tmem + T_S + kk * 16, make_sw128_desc(do_s + kk * 2048, 16384, 1024), id_ts,
                        t > 0 || kk > 0);
        };
        if (!(ok = mbar_wait(&bars->ds_half, t & 1, p.status, kErrDsReady))) break;
        tc_fence_after();
        dkdv(0);
        if (!(ok = mbar_wait(&bars->ds_ready, t & 1, p.status, kErrDsReady))) break;
        tc_fence_after();
        dkdv(4);
        // G_q = dS' K : A = dS'^T buffer read MN-major (M = queries, K = keys), B = K [keys][D] (MN-major)
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ss(tmem + T_DP, make_sw128_desc(ds_a + kk * 2048, 16384, 1024),
                      make_sw128_desc(kn_a + kk * 2048, 16384, 1024), id_mm, kk > 0);
        mma_commit(&bars->dq_full);   // G_q ready; this step's Q^ / dO stage and dS^T are no longer read
        if (t + 1 < n_steps) {
          const int st1 = (t + 1) & 1;
          // S^T(t+1) only needs P^T(t) read (dV was issued before); dP^T(t+1)
          // overwrites G_q and waits for the drain.
          if (!(ok = mbar_wait(&bars->q_full[st1], ((t + 1) >> 1) & 1, p.status, kErrQFull))) break;
          tc_fence_after();
          mma_kmajor(T_S, kn_a, qn_a + st1 * L::kTile, ext_lse);
          if (!(ok = mbar_wait(&bars->dq_drained, t & 1, p.status, kErrDqDrained))) break;
          tc_fence_after();
          mma_kmajor(T_DP, v_a, do_a + st1 * L::kTile, ext_delta);
          mma_commit(&bars->s_full);
          mma_commit(&bars->ld_empty);
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
    // Query rows that see key n0 + j: the non-global rows [row_min, row_max),
    // every row from global_q_row on, and every row if the key is global.
    int row_min, row_max;
    key_rows(p.mask, n0 + j, row_min, row_max);
    const bool key_global = n0 + j >= p.mask.global_key && n0 + j < p.seqlen_kv;
    // G_q drain: warpgroup w owns G_q columns [32 w, 32 w + 32); with D = 64 only
    // warpgroups 0 and 1 have columns.  Staging chunks are [128 rows][32 floats]
    // with the 128-byte swizzle (16 KB) in this step's Q^ and dO stage buffers.
    const bool drains = wg * 32 < D;
    bool ok = true;
    for (int t = 0; t < n_steps; ++t) {
      const int st = t & 1;
      const int sa = bs.abs_step(t);
      const int qt = sa / group, h = hk * group + (sa % group + rot) % group;
      const int q0 = qt * 128;
      const bool diag = bs.diag(t, qt);
      ok = warp_wait(&bars->s_full, t & 1, ok, p.status, kErrSFull);
      // Warpgroup w owns query columns [16w, 16w+16) of each 64-column half:
      // the first half's dK~/dV products run while the second half is computed.
      if (ok) tc_fence_after();
#pragma unroll
      for (int grp = 0; grp < 2; ++grp) {
        if (ok) {
          const int col0 = grp * 64 + wg * 16;
          uint32_t sr[16], dpr[16];
          tmem_ld16(tmem + lane_base + T_S + col0, sr);
          tmem_ld16(tmem + lane_base + T_DP + col0, dpr);
          tmem_wait_ld();
          uint32_t pk[8], dk[8];
          if (!diag) {
#pragma unroll
            for (int c = 0; c < 16; c += 2) {
              // one pair in four on the FMA pipe (cubic), the rest on MUFU
              float p0, p1;
              if (((c >> 1) & 3) == 3) {
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
            // columns c < lim and c >= hi_lim cannot see key j, unless they are
            // global rows (c >= glim) or the key is global
            const int lim = row_min - (q0 + col0), hl = row_max - (q0 + col0);
            const int glim = key_global ? -128 : p.mask.global_q_row - (q0 + col0);
#pragma unroll
            for (int c = 0; c < 16; c += 2) {
              const bool v0 = (c >= lim && c < hl) || c >= glim, v1 = (c + 1 >= lim && c + 1 < hl) || c + 1 >= glim;
              const float p0 = v0 ? fast_exp2(__uint_as_float(sr[c])) : 0.f;
              const float p1 = v1 ? fast_exp2(__uint_as_float(sr[c + 1])) : 0.f;
              const float d0 = p0 * __uint_as_float(dpr[c]);
              const float d1 = p1 * __uint_as_float(dpr[c + 1]);
              pk[c >> 1] = pack_bf16x2(p0, p1);
              dk[c >> 1] = pack_bf16x2(d0, d1);
            }
          }
          // P^T of these 16 queries (8 packed columns) goes into the first half
          // of the S^T columns just read: K-step kk = col0/16 of dV reads it there.
          tmem_st8(tmem + lane_base + T_S + col0, pk);
          uint8_t* ds_box = smem + L::kDs + grp * 16384;
#pragma unroll
          for (int c8 = 0; c8 < 2; ++c8)
            *reinterpret_cast<uint4*>(ds_box + sw128_offset(j, wg * 16 + c8 * 8)) =
                make_uint4(dk[4 * c8], dk[4 * c8 + 1], dk[4 * c8 + 2], dk[4 * c8 + 3]);
          tmem_wait_st();
          tc_fence_before();
          fence_proxy_async_smem();
        }
        if (grp == 0) {
          named_bar_sync(bar_id, 128);
          if (j == 0 && ok) mbar_arrive(&bars->ds_half);
        }
      }
      named_bar_sync(bar_id, 128);
      if (j == 0 && ok) {
        mbar_arrive(&bars->ds_ready);
        if (t > 0) {
          // The previous step's dq reduction has had this step's MMAs and
          // softmax to read its staging; once it has, that Q^/dO stage goes back
          // to the producer (the next load still has this step's products to land).
          tma_store_wait_read();
          mbar_arrive(&bars->q_empty[st ^ 1]);
        }
      }

      // Drain G_q (TMEM lane = query row of this step) into the fp32 accumulator:
      // TMEM -> registers (then the dP^T/G_q columns are free again), registers ->
      // this step's Q^/dO stage (dq_full also means dK~ and dV have read it), then a TMA bulk
      // reduce-add.  The stage goes back to the producer at the next step.
      ok = warp_wait(&bars->dq_full, t & 1, ok, p.status, kErrDqFull);
      uint32_t gq[32];
      if (ok && drains) {
        tc_fence_after();
        tmem_ld32(tmem + lane_base + T_DP + wg * 32, gq);
        tmem_wait_ld();
        tc_fence_before();
      }
      named_bar_sync(bar_id, 128);
      if (j == 0 && ok) mbar_arrive(&bars->dq_drained);
      // chunk wg: the first D/64 chunks fill this step's Q^ stage, the rest its dO stage
      constexpr int kChunksPerBuffer = D / 64;
      uint8_t* chunk = wg < kChunksPerBuffer ? smem + L::kQn + st * L::kTile + wg * 16384
                                             : smem + L::kDo + st * L::kTile + (wg - kChunksPerBuffer) * 16384;
      if (ok && drains) {
        uint8_t* row = chunk + j * 128;
#pragma unroll
        for (int piece = 0; piece < 8; ++piece)
          *reinterpret_cast<uint4*>(row + (((piece ^ (j & 7)) & 7) << 4)) =
              make_uint4(gq[4 * piece], gq[4 * piece + 1], gq[4 * piece + 2], gq[4 * piece + 3]);
        fence_proxy_async_smem();
      }
      named_bar_sync(bar_id, 128);
      if (j == 0 && ok) {
        if (drains) tma_reduce_add_4d(&tm_dq, chunk, wg * 32, h, q0, b);
        tma_store_commit();   // (an empty group when nothing was issued); released next step
      }
    }
    // every bulk reduction has read its staging (and the last stage is
    // released) before the stage buffers are reused below
    if (j == 0) {
      tma_store_wait_read();
      if (ok && n_steps > 0) mbar_arrive(&bars->q_empty[(n_steps - 1) & 1]);
    }
    named_bar_sync(5, 128 * kComputeWarpgroups);

    // ---------------------------------------------------------- epilogue
    // dV and G_k of this piece (fp32 in TMEM) are added into the fp32
    // accumulators: warpgroup w stages columns [32w, 32w+32) of each into the
    // idle stage buffers (dV -> Q^ stages, G_k -> dO stages) and issues two
    // bulk reduce-adds.  bca_bwd_finalize_kernel turns the sums into dv and dk.
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
      // the reductions only need to have read shared memory before the CTA
      // exits; their global writes complete before the kernel does
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

// ------------------------------------------------------------------ finalize
// One warp per row.  Query rows: dq~ = scale gamma_k G_q, dq through the
// RMSNorm Jacobian, dgamma_q += dq~ q^.  Key rows: dv = bf16(dV), gamma_k dk~ =
// G_k / log2(e), dk through the Jacobian, dgamma_k += dk~ k^.  With r = rsqrt
// (mean x^2 + eps), x^ = x r and g = gamma dx~:  dx = r (g - x^ mean(g x^)).
// kDet (deterministic backward): each warp takes whole tokens, i.e. all rows
// (batch, head) of one query or key token in a fixed order, so a token's angle
// gradient is summed in registers and written once; the block's dgamma sums
// go to per-block slots that bca_bwd_dgamma_reduce_kernel adds in block order.
template <int D, bool kRope, bool kDet>
__global__ void __launch_bounds__(256) bca_bwd_finalize_kernel(const BwdParams p) {
  using IO = RowIO<D>;
  constexpr int E = IO::E;
  __shared__ float red[2][8][D];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int64_t n_q = (int64_t)p.batch * p.seqlen_q * p.heads_q;
  const int64_t n_k = (int64_t)p.batch * p.seqlen_kv * p.heads_kv;
  const int64_t warps = (int64_t)gridDim.x * 8;
  float gacc_q[E], gacc_k[E], gm[E], gk[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    gacc_q[e] = 0.f;
    gacc_k[e] = 0.f;
    gm[e] = __ldg(p.gamma_q + lane * E + e);
    gk[e] = __ldg(p.gamma_k + lane * E + e);
  }
  // Two rows per warp and iteration, all loads issued before the arithmetic,
  // so each warp keeps two rows' reads in flight.
  auto finish_row = [&](int64_t rr, float (&x)[E], float (&g)[E], const float (&dvv)[E], float (&dr)[E]) {
    const bool is_q = rr < n_q;
    const int64_t r = is_q ? rr : rr - n_q;
    // with rotary angles the normalised vector is rope(x): the Jacobian below
    // acts on it, and its result goes back through the transposed rotation
    const float* rope = kRope ? (is_q ? p.rope_q : p.rope_k) : nullptr;
    float* drope = kRope ? (is_q ? p.drope_q : p.drope_k) : nullptr;
    const int64_t tok = (r / (is_q ? p.heads_q : p.heads_kv)) % (is_q ? p.seqlen_q : p.seqlen_kv);
    float dqt[E];
    // g = gamma * dx~   (for query rows dq~ = scale gamma_k G_q is kept for dgamma_q)
#pragma unroll
    for (int e = 0; e < E; ++e) {
      dqt[e] = g[e] * gk[e] * p.scale;
      g[e] = is_q ? dqt[e] * gm[e] : g[e] * (1.0f / kLog2e);
    }
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) ss = fmaf(x[e], x[e], ss);
    const float rinv = rsqrtf(warp_sum(ss) * (1.0f / D) + p.eps);
    float cs[E], sn[E], y[E];
    if (rope != nullptr) {   // warp-uniform
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const float xp = __shfl_xor_sync(0xffffffffu, x[e], 16);
        sincosf(__ldg(rope + tok * (D / 2) + (lane & 15) * E + e), &sn[e], &cs[e]);
        y[e] = lane < 16 ? rope_first(x[e], xp, cs[e], sn[e]) : rope_second(xp, x[e], cs[e], sn[e]);
        x[e] = y[e];
      }
    }
    float dot = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      x[e] *= rinv;   // x^
      dot = fmaf(g[e], x[e], dot);
    }
    const float mean_dot = warp_sum(dot) * (1.0f / D);
    float o[E];
#pragma unroll
    for (int e = 0; e < E; ++e) o[e] = rinv * (g[e] - x[e] * mean_dot);
    if (rope != nullptr) {
      // o = gradient w.r.t. y = rope(raw); pair (a, b) = (lane < 16, lane ^ 16):
      // d angle = -o_a y_b + o_b y_a, d raw_a = o_a c + o_b s, d raw_b = o_b c - o_a s
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const float op = __shfl_xor_sync(0xffffffffu, o[e], 16);
        const float yp = __shfl_xor_sync(0xffffffffu, y[e], 16);
        if constexpr (kDet)
          dr[e] += op * y[e] - o[e] * yp;
        else if (drope != nullptr && lane < 16)
          atomicAdd(drope + tok * (D / 2) + lane * E + e, op * y[e] - o[e] * yp);
        o[e] = lane < 16 ? fmaf(op, sn[e], o[e] * cs[e]) : fmaf(-op, sn[e], o[e] * cs[e]);
      }
    }
    if (is_q) {
      IO::store_bf16(p.dq + r * D, lane, o);
#pragma unroll
      for (int e = 0; e < E; ++e) gacc_q[e] = fmaf(dqt[e], x[e], gacc_q[e]);
    } else {
      IO::store_bf16(p.dk + r * D, lane, o);
      IO::store_bf16(p.dv + r * D, lane, dvv);
#pragma unroll
      for (int e = 0; e < E; ++e) gacc_k[e] = fmaf(g[e] / gk[e], x[e], gacc_k[e]);
    }
  };
  auto load_row = [&](int64_t rr, float (&x)[E], float (&g)[E], float (&dvv)[E]) {
    const bool is_q = rr < n_q;
    const int64_t r = is_q ? rr : rr - n_q;
    IO::load_bf16((is_q ? p.q : p.k) + r * D, lane, x);
    IO::load_f32((is_q ? p.dqacc : p.dkacc) + r * D, lane, g);
    if (!is_q) IO::load_f32(p.dvacc + r * D, lane, dvv);
  };
  if constexpr (!kDet) {
    const int64_t total = n_q + n_k;
    float dr[E];   // (unused: angle gradients go out by atomics)
    for (int64_t rr = (int64_t)blockIdx.x * 8 + wid; rr < total; rr += 2 * warps) {
      const int64_t rr2 = rr + warps;
      float x0[E], g0[E], v0[E], x1[E], g1[E], v1[E];
      load_row(rr, x0, g0, v0);
      if (rr2 < total) load_row(rr2, x1, g1, v1);
      finish_row(rr, x0, g0, v0, dr);
      if (rr2 < total) finish_row(rr2, x1, g1, v1, dr);
    }
  } else {
    // tokens [0, Sq) are query tokens, [Sq, Sq + Skv) key tokens
    const int64_t tokens = (int64_t)p.seqlen_q + p.seqlen_kv;
    for (int64_t tt = (int64_t)blockIdx.x * 8 + wid; tt < tokens; tt += warps) {
      const bool is_q = tt < p.seqlen_q;
      const int64_t s_tok = is_q ? tt : tt - p.seqlen_q;
      const int H = is_q ? p.heads_q : p.heads_kv;
      const int64_t S = is_q ? p.seqlen_q : p.seqlen_kv;
      const int n = p.batch * H;
      auto row_of = [&](int i) {   // i-th (batch, head) row of the token, in the finalize's row numbering
        const int64_t r = ((int64_t)(i / H) * S + s_tok) * H + i % H;
        return is_q ? r : n_q + r;
      };
      float dr[E];
#pragma unroll
      for (int e = 0; e < E; ++e) dr[e] = 0.f;
      for (int i = 0; i < n; i += 2) {
        float x0[E], g0[E], v0[E], x1[E], g1[E], v1[E];
        load_row(row_of(i), x0, g0, v0);
        if (i + 1 < n) load_row(row_of(i + 1), x1, g1, v1);
        finish_row(row_of(i), x0, g0, v0, dr);
        if (i + 1 < n) finish_row(row_of(i + 1), x1, g1, v1, dr);
      }
      if constexpr (kRope) {
        float* drope = is_q ? p.drope_q : p.drope_k;
        if (drope != nullptr && lane < 16) {
#pragma unroll
          for (int e = 0; e < E; ++e) drope[s_tok * (D / 2) + lane * E + e] = dr[e];
        }
      }
    }
  }
  if (p.dgamma_q != nullptr || p.dgamma_k != nullptr) {
#pragma unroll
    for (int e = 0; e < E; ++e) {
      red[0][wid][lane * E + e] = gacc_q[e];
      red[1][wid][lane * E + e] = gacc_k[e];
    }
    __syncthreads();
    if (threadIdx.x < D) {
      float aq = 0.f, ak = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        aq += red[0][w][threadIdx.x];
        ak += red[1][w][threadIdx.x];
      }
      if constexpr (kDet) {
        p.dgamma_part[(size_t)blockIdx.x * 2 * D + threadIdx.x] = aq;
        p.dgamma_part[(size_t)blockIdx.x * 2 * D + D + threadIdx.x] = ak;
      } else {
        if (p.dgamma_q != nullptr) atomicAdd(p.dgamma_q + threadIdx.x, aq);
        if (p.dgamma_k != nullptr) atomicAdd(p.dgamma_k + threadIdx.x, ak);
      }
    }
  }
}

// dgamma of the deterministic backward: thread d adds slot d of every
// finalize block's partials in block order.
template <int D>
__global__ void __launch_bounds__(2 * D) bca_bwd_dgamma_reduce_kernel(const BwdParams p, int blocks) {
  const int d = threadIdx.x % D;
  const bool is_k = threadIdx.x >= D;
  float acc = 0.f;
  for (int i = 0; i < blocks; ++i) acc += p.dgamma_part[(size_t)i * 2 * D + threadIdx.x];
  float* dst = is_k ? p.dgamma_k : p.dgamma_q;
  if (dst != nullptr) dst[d] = acc;
}

// Largest finalize grid of the deterministic backward (its dgamma slots).
constexpr int kMaxFinBlocks = 2048;

template <int D>
cudaError_t launch_bwd_d(const CUtensorMap& t_k, const CUtensorMap& t_v, const CUtensorMap& t_qn,
                         const CUtensorMap& t_do, const CUtensorMap& t_dq, const CUtensorMap& t_dv,
                         const CUtensorMap& t_dk, const BwdParams& p, int n_units, int n_dq_units,
                         cudaStream_t stream) {
  using L = BwdLayout<D>;
  static uint64_t configured = 0;
  const bool det = p.deterministic != 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  int max_optin = 0;
  e = cudaDeviceGetAttribute(&max_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e != cudaSuccess) return e;
  const int alloc = L::kTotal + 1024 <= max_optin ? L::kTotal + 1024 : max_optin;
  if (alloc < L::kTotal) return cudaErrorInvalidConfiguration;
  if (!det) {
    e = set_smem_once(configured, dev, bca_bwd_main_kernel<D>, alloc);
    if (e != cudaSuccess) return e;
  }
  int sms = 148;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t rows = (int64_t)p.batch * p.seqlen_q * p.heads_q + (int64_t)p.batch * p.seqlen_kv * p.heads_kv;
  // one wave of the row kernels (grid-stride loops over one warp per row or token)
  static int prep_per_sm[2] = {0, 0}, fin_per_sm[2][2][2] = {};
  const bool rope = p.rope_q != nullptr || p.rope_k != nullptr;
  int& prep_occ = prep_per_sm[D == 128];
  int& fin_occ = fin_per_sm[D == 128][rope][det];
  if (prep_occ == 0) {
    int n = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, bca_bwd_prep_kernel<D>, 256, 0);
    prep_occ = std::max(n, 1);
  }
  auto finalize_kernel = [&]() {
    if (det) return rope ? bca_bwd_finalize_kernel<D, true, true> : bca_bwd_finalize_kernel<D, false, true>;
    return rope ? bca_bwd_finalize_kernel<D, true, false> : bca_bwd_finalize_kernel<D, false, false>;
  };
  if (fin_occ == 0) {
    int n = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, finalize_kernel(), 256, 0);
    fin_occ = std::max(n, 1);
  }
  const int prep_blocks = (int)std::min<int64_t>((rows + 7) / 8, (int64_t)sms * prep_occ);
  if (p.seqlen_q_pad != p.seqlen_q) {
    // padding entries of the {lse, Delta} pairs are read by full-tile loads
    e = cudaMemsetAsync(p.ld, 0, (size_t)p.batch * p.heads_q * p.seqlen_q_pad * 16, stream);
    if (e != cudaSuccess) return e;
  }
  bca_bwd_prep_kernel<D><<<prep_blocks, 256, 0, stream>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  profile_mark(0, stream);
  if (det) {
    // the dq pass, then the dK/dV pass (bca_bwd_split.cu)
    e = launch_bwd_split(t_k, t_v, t_qn, t_do, t_dv, t_dk, p, D, n_units, n_dq_units, stream);
    if (e != cudaSuccess) return e;
  } else if (n_units > 0) {
    bca_bwd_main_kernel<D><<<n_units, kThreads, alloc, stream>>>(t_k, t_v, t_qn, t_do, t_dq, t_dv, t_dk, p, alloc);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  profile_mark(1, stream);
  // a deterministic finalize takes whole tokens; its grid also fixes the dgamma slots
  const int64_t work = det ? (int64_t)p.seqlen_q + p.seqlen_kv : rows;
  int fin_blocks = (int)std::min<int64_t>((work + 7) / 8, (int64_t)sms * fin_occ);
  if (det) fin_blocks = std::min(fin_blocks, kMaxFinBlocks);
  finalize_kernel()<<<fin_blocks, 256, 0, stream>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (det && (p.dgamma_q != nullptr || p.dgamma_k != nullptr)) {
    bca_bwd_dgamma_reduce_kernel<D><<<1, 2 * D, 0, stream>>>(p, fin_blocks);
    e = cudaGetLastError();
  }
  return e;
}

}  // namespace

BwdWorkspace bwd_workspace_layout(int B, int Sq, int Skv, int Hq, int Hkv, int D) {
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  const size_t sq_pad = (size_t)((Sq + 127) / 128) * 128;
  BwdWorkspace w;
  w.qn = 0;
  w.kn = w.qn + up((size_t)B * Sq * Hq * D * 2);
  w.ld = w.kn + up((size_t)B * Skv * Hkv * D * 2);
  w.dqacc = w.ld + up((size_t)B * Hq * sq_pad * 16);
  w.dvacc = w.dqacc + up((size_t)B * Sq * Hq * D * 4);
  w.dkacc = w.dvacc + up((size_t)B * Skv * Hkv * D * 4);
  w.dgpart = w.dkacc + up((size_t)B * Skv * Hkv * D * 4);
  w.total = w.dgpart + up((size_t)kMaxFinBlocks * 2 * D * 4);
  return w;
}

cudaError_t launch_bwd(const CUtensorMap& t_k, const CUtensorMap& t_v, const CUtensorMap& t_qn,
                       const CUtensorMap& t_do, const CUtensorMap& t_dq, const CUtensorMap& t_dv,
                       const CUtensorMap& t_dk, const BwdParams& p, int head_dim, int n_units, int n_dq_units,
                       cudaStream_t stream) {
  if (head_dim == 128)
    return launch_bwd_d<128>(t_k, t_v, t_qn, t_do, t_dq, t_dv, t_dk, p, n_units, n_dq_units, stream);
  return launch_bwd_d<64>(t_k, t_v, t_qn, t_do, t_dq, t_dv, t_dk, p, n_units, n_dq_units, stream);
}

}  // namespace magi
