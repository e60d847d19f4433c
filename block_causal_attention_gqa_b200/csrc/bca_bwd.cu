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
// Deterministic backward (dims.deterministic): no sum depends on timing.  The
// dq pass (bca_bwd_dq_kernel, query-major, one CTA per query tile) computes
// G_q before the main kernel, which then skips its G_q product and drain;
// every kv tile is one main-kernel unit, so dV and G_k are added once onto
// zero; the finalize takes whole tokens (angle gradients summed in registers)
// and writes per-block dgamma partials that one small kernel adds in block
// order.  The dq pass recomputes S and dP, so the tensor work is 7/5 of the
// default path's.
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

#include "bca_kernels.h"
#include "bca_norm.cuh"
#include "sm100.cuh"

namespace magi {
namespace {

using namespace sm100;

constexpr int kComputeWarpgroups = 4;               // each owns 32 of the 128 query columns
constexpr int kMmaWarp = 4 * kComputeWarpgroups;      // warp 16
constexpr int kTmaWarp = kMmaWarp + 1;                // warp 17
constexpr int kThreads = 32 * (kTmaWarp + 1);         // 576
constexpr float kLog2e = 1.4426950408889634f;

enum : int {
  kErrKv = 2001, kErrQFull = 2002, kErrQEmpty = 2003, kErrSFull = 2004, kErrDsReady = 2005,
  kErrDqFull = 2006, kErrDqDrained = 2007, kErrAcc = 2008, kErrSmem = 2009, kErrLdEmpty = 2010,
  kErrDqQ = 2011, kErrDqK = 2012, kErrDqV = 2013, kErrDqKEmpty = 2014, kErrDqVEmpty = 2015,
  kErrDqSFull = 2016, kErrDqDpFree = 2017, kErrDqDsReady = 2018, kErrDqGq = 2019
};

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, bool ok, int* status, int code) {
  if (ok) ok = mbar_wait(bar, parity, status, code);
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}


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
  const int32_t* u = p.units + (size_t)blockIdx.x * 8;
  const int b = __ldg(u + 0), hk = __ldg(u + 1), n0 = __ldg(u + 2);
  // steps [s_begin, s_end) of this kv tile; step s = (query tile s / group,
  // head s % group of the kv head's group); query tiles below diag_end or from
  // diag_hi_begin on (KV range) need the mask
  const int s_begin = __ldg(u + 3), s_end = __ldg(u + 4), diag_end = __ldg(u + 5);
  const int diag_hi_begin = __ldg(u + 6);
  const int group = p.heads_q / p.heads_kv;
  const int n_steps = s_end - s_begin;
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
        const int qt = (s_begin + t) / group, h = hk * group + ((s_begin + t) % group + rot) % group;
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
          const int qt1 = (s_begin + t + 1) / group, h1 = hk * group + ((s_begin + t + 1) % group + rot) % group;
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
    // First query row that sees key n0 + j: query chunk c sees keys below
    // kv_offsets[n_kv - n_q + c + 1], so it is the first chunk whose end exceeds the key.
    int row_min = p.seqlen_q;
    {
      const int key = n0 + j;
      if (key < p.seqlen_kv) {
        const int shift = p.n_kv_chunks - p.n_q_chunks;
        int lo = 0, hi = p.n_q_chunks;  // first c in [0, n_q) with kv_offsets[shift + c + 1] > key
        while (lo < hi) {
          const int mid = (lo + hi) >> 1;
          if (__ldg(p.kv_offsets + shift + mid + 1) > key) hi = mid; else lo = mid + 1;
        }
        row_min = lo < p.n_q_chunks ? __ldg(p.q_offsets + lo) : p.seqlen_q;
      }
    }
    // First query row that no longer sees key n0 + j (KV range R): query chunk
    // c's first visible key is kv_offsets[max(0, n_kv - n_q + c - R + 1)].
    int row_max = p.seqlen_q;
    if (p.kv_range > 0) {
      const int key = n0 + j;
      const int shift = p.n_kv_chunks - p.n_q_chunks - p.kv_range + 1;
      int lo = 0, hi = p.n_q_chunks;  // first c with a first visible key above `key`
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (__ldg(p.kv_offsets + max(shift + mid, 0)) > key) hi = mid; else lo = mid + 1;
      }
      row_max = lo < p.n_q_chunks ? __ldg(p.q_offsets + lo) : p.seqlen_q;
    }
    // G_q drain: warpgroup w owns G_q columns [32 w, 32 w + 32); with D = 64 only
    // warpgroups 0 and 1 have columns.  Staging chunks are [128 rows][32 floats]
    // with the 128-byte swizzle (16 KB) in this step's Q^ and dO stage buffers.
    const bool drains = wg * 32 < D;
    bool ok = true;
    for (int t = 0; t < n_steps; ++t) {
      const int st = t & 1;
      const int qt = (s_begin + t) / group, h = hk * group + ((s_begin + t) % group + rot) % group;
      const int q0 = qt * 128;
      const bool diag = qt < diag_end || qt >= diag_hi_begin;
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
            // columns c < lim and c >= hi_lim cannot see key j
            const int lim = row_min - (q0 + col0), hi_lim = row_max - (q0 + col0);
#pragma unroll
            for (int c = 0; c < 16; c += 2) {
              const float p0 = c < lim || c >= hi_lim ? 0.f : fast_exp2(__uint_as_float(sr[c]));
              const float p1 = c + 1 < lim || c + 1 >= hi_lim ? 0.f : fast_exp2(__uint_as_float(sr[c + 1]));
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
  const int32_t* u = p.units + (size_t)blockIdx.x * 8;
  const int b = __ldg(u + 0), hk = __ldg(u + 1), n0 = __ldg(u + 2);
  const int s_begin = __ldg(u + 3), s_end = __ldg(u + 4), diag_end = __ldg(u + 5);
  const int diag_hi_begin = __ldg(u + 6);
  const int group = p.heads_q / p.heads_kv;
  const int n_steps = s_end - s_begin;

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
        const int qt = (s_begin + t) / group, h = hk * group + (s_begin + t) % group;
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
          const int qt1 = (s_begin + t + 1) / group, h1 = hk * group + (s_begin + t + 1) % group;
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
    // first query row that sees key n0 + j, and (KV range) the first that no longer does
    int row_min = p.seqlen_q;
    {
      const int key = n0 + j;
      if (key < p.seqlen_kv) {
        const int shift = p.n_kv_chunks - p.n_q_chunks;
        int lo = 0, hi = p.n_q_chunks;
        while (lo < hi) {
          const int mid = (lo + hi) >> 1;
          if (__ldg(p.kv_offsets + shift + mid + 1) > key) hi = mid; else lo = mid + 1;
        }
        row_min = lo < p.n_q_chunks ? __ldg(p.q_offsets + lo) : p.seqlen_q;
      }
    }
    int row_max = p.seqlen_q;
    if (p.kv_range > 0) {
      const int key = n0 + j;
      const int shift = p.n_kv_chunks - p.n_q_chunks - p.kv_range + 1;
      int lo = 0, hi = p.n_q_chunks;
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (__ldg(p.kv_offsets + max(shift + mid, 0)) > key) hi = mid; else lo = mid + 1;
      }
      row_max = lo < p.n_q_chunks ? __ldg(p.q_offsets + lo) : p.seqlen_q;
    }
    const bool drains = wg * 32 < D;
    bool ok = true;
    for (int t = 0; t < n_steps; ++t) {
      const int qt = (s_begin + t) / group;
      const int q0 = qt * 128;
      const bool diag = qt < diag_end || qt >= diag_hi_begin;
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
            const int lim = row_min - (q0 + col0), hi_lim = row_max - (q0 + col0);
#pragma unroll
            for (int c = 0; c < 16; c += 2) {
              const float p0 = c < lim || c >= hi_lim ? 0.f : fast_exp2(__uint_as_float(sr[c]));
              const float p1 = c + 1 < lim || c + 1 >= hi_lim ? 0.f : fast_exp2(__uint_as_float(sr[c + 1]));
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

// chunk c with offs[c] <= row < offs[c + 1]
__device__ __forceinline__ int find_chunk(const int32_t* offs, int n, int row) {
  int lo = 0, hi = n;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(offs + mid) <= row) lo = mid; else hi = mid;
  }
  return lo;
}

template <int D>
__global__ void __launch_bounds__(kDqThreads, 1)
bca_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_qn, const __grid_constant__ CUtensorMap tm_do,
                  const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                  const BwdParams p, const int smem_alloc) {
  using L = DqLayout<D>;
  const int32_t* u = p.dq_units + (size_t)(blockIdx.x >> 1) * 12;
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
  const int n_full = __ldg(u + 6), n_tiles = __ldg(u + 7);
  const int t_begin = __ldg(u + 8), t_full_begin = __ldg(u + 9);
  const int n_vis = n_tiles - t_begin;

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
        const int n0 = (t_begin + j) * 128;
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
    // visible keys [kv_first, limit) of the row
    int limit = p.seqlen_kv, kv_first = 0;
    if (row < p.seqlen_q) {
      const int c = find_chunk(p.q_offsets, p.n_q_chunks, row);
      limit = __ldg(p.kv_offsets + p.n_kv_chunks - p.n_q_chunks + c + 1);
      if (p.kv_range > 0)
        kv_first = __ldg(p.kv_offsets + max(p.n_kv_chunks - p.n_q_chunks + c - p.kv_range + 1, 0));
    }
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
        const int tile = t_begin + j;
        const bool masked = tile < t_full_begin || tile >= n_full;
        uint32_t pk[32];
        auto sval = [&](int c) { return __uint_as_float(c < 32 ? sa[c] : sb[c - 32]); };
        auto dval = [&](int c) { return __uint_as_float(c < 32 ? da[c] : db[c - 32]); };
        if (masked) {
          const int c0 = tile * 128 + 64 * wg;
          const int lim = limit - c0, lo = kv_first - c0;   // columns [lo, lim) are visible
#pragma unroll
          for (int c = 0; c < 64; c += 2) {
            const float p0 = c >= lo && c < lim ? fast_exp2(sval(c) + nl) : 0.f;
            const float p1 = c + 1 >= lo && c + 1 < lim ? fast_exp2(sval(c + 1) + nl) : 0.f;
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

// cudaFuncSetAttribute once per (kernel, device); bit `dev` of `mask`.
template <typename K>
cudaError_t set_smem_once(uint64_t& mask, int dev, K kernel, int bytes) {
  if (dev < 64 && ((mask >> dev) & 1u)) return cudaSuccess;
  const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && dev < 64) mask |= uint64_t(1) << dev;
  return e;
}

template <int D>
cudaError_t launch_bwd_d(const CUtensorMap& t_k, const CUtensorMap& t_v, const CUtensorMap& t_qn,
                         const CUtensorMap& t_do, const CUtensorMap& t_dq, const CUtensorMap& t_dv,
                         const CUtensorMap& t_dk, const BwdParams& p, int n_units, int n_dq_units,
                         cudaStream_t stream) {
  using L = BwdLayout<D>;
  using LD = DqLayout<D>;
  static uint64_t configured[2] = {0, 0}, configured_dq = 0;
  const bool det = p.deterministic != 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  int max_optin = 0;
  e = cudaDeviceGetAttribute(&max_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e != cudaSuccess) return e;
  const int alloc = L::kTotal + 1024 <= max_optin ? L::kTotal + 1024 : max_optin;
  if (alloc < L::kTotal) return cudaErrorInvalidConfiguration;
  using LK = DkdvLayout<D>;
  const int alloc_kv = LK::kTotal + 1024 <= max_optin ? LK::kTotal + 1024 : max_optin;
  if (det) {
    if (alloc_kv < LK::kTotal) return cudaErrorInvalidConfiguration;
    e = set_smem_once(configured[0], dev, bca_bwd_dkdv_kernel<D>, alloc_kv);
  } else {
    e = set_smem_once(configured[1], dev, bca_bwd_main_kernel<D>, alloc);
  }
  if (e != cudaSuccess) return e;
  const int alloc_dq = LD::kTotal + 1024 <= max_optin ? LD::kTotal + 1024 : max_optin;
  if (det) {
    if (alloc_dq < LD::kTotal) return cudaErrorInvalidConfiguration;
    e = set_smem_once(configured_dq, dev, bca_bwd_dq_kernel<D>, alloc_dq);
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
  if (det && n_dq_units > 0) {
    // G_q of every query row, summed in tile order inside one CTA
    bca_bwd_dq_kernel<D><<<2 * n_dq_units, kDqThreads, alloc_dq, stream>>>(t_qn, t_do, t_k, t_v, p, alloc_dq);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (n_units > 0) {
    if (det)
      bca_bwd_dkdv_kernel<D><<<n_units, kThreads, alloc_kv, stream>>>(t_k, t_v, t_qn, t_do, t_dv, t_dk, p, alloc_kv);
    else
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
