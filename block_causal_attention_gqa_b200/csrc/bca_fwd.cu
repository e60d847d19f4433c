// Forward kernel: block-causal GQA attention with fused QK-RMSNorm, sm_100a.
//
// One CTA runs one work unit: up to two 128-row query tiles ("sub-tiles")
// that share a key/value head and a kv extent (bca_sched.h).  Roles:
//   warps 0-3  softmax warpgroup for sub-tile 0 (thread i owns query row i,
//              which is TMEM lane i)
//   warps 4-7  softmax warpgroup for sub-tile 1
//   warp  8    tcgen05 MMA issue (one elected thread)
//   warp  9    TMA producer (one elected thread)
// TMEM (512 columns): S_s at 256*s, O_s at 256*s + 128.  P_s (bf16 pairs)
// overwrites the first 64 columns of S_s once S_s has been read.
//
// Per kv tile j the MMA thread issues, for each sub-tile s,
//   O_s += P_s(j) V_j      (A from TMEM, V as an MN-major B operand)
//   S_s  = Q_s K_{j+1}^T   (both K-major)
// and commits s_full[s]; a commit completes only when every earlier tcgen05
// operation of the thread has, so s_full also says "O_s is up to date".
//
// QK-RMSNorm fold.  With r_q = rsqrt(mean q^2 + eps), r_k likewise,
//   scale * q~.k~ = sum_d (q_d r_q gamma_q[d] gamma_k[d] scale) (k_d r_k).
// bca_knorm_kernel writes K^ = bf16(k r_k) once per call (one warp per key
// row), the TMA streams K^, and the softmax warps scale each Q row once in
// shared memory by r_q gamma_q gamma_k scale log2(e); the MMA then produces
// the logits directly in log2 units, with nothing left to apply per element.

// Online softmax with a lazy maximum: a row's reference maximum moves only
// when a tile's maximum exceeds it by more than 8 (log2 units), so P <= 256
// and the O rescale (TMEM load, multiply, store) is rare after the first
// tiles.  The result is exact: O and l are always scaled by the same factor.
//
// Throughput of the softmax: the row is processed as fp32 pairs with the
// .f32x2 instructions, the row maximum with three-input max, and on unmasked
// tiles one exponential in four is computed by a cubic on the FMA pipe
// instead of MUFU (exp2_poly_pair).  The masked and unmasked exponential
// loops are separate straight-line code: a per-pair branch on the mask flag
// split the loop into small blocks the compiler could not interleave, which
// had made the exponential phase three times its MUFU time.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <type_traits>

#include "bca_kernels.h"
#include "bca_mask.cuh"
#include "bca_norm.cuh"
#include "sm100.cuh"

namespace magi {
namespace {

using namespace sm100;

constexpr int kThreads = 320;
constexpr int kStages = 2;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;

enum : int {
  kErrQ = 1001, kErrKFull = 1002, kErrVFull = 1003, kErrKEmpty = 1004, kErrVEmpty = 1005,
  kErrSFull = 1006, kErrPReady = 1007, kErrQReady = 1008, kErrKSoft = 1009
};

template <int D>
struct FwdLayout {
  static constexpr int kTileBytes = 128 * D * 2;  // one [128][D] bf16 tile
  static constexpr int kQ = 0;                     // 2 sub-tiles
  static constexpr int kK = kQ + 2 * kTileBytes;   // kStages
  static constexpr int kV = kK + kStages * kTileBytes;
  static constexpr int kQScale = kV + kStages * kTileBytes;  // float [D]
  static constexpr int kBars = kQScale + D * 4;
  static constexpr int kNumBars = 16;
  static constexpr int kTmemSlot = kBars + kNumBars * 8;
  static constexpr int kTotal = kTmemSlot + 16;
  static constexpr int kAlloc = kTotal + 1024;  // slack for 1024-byte alignment
};

struct Bars {
  uint64_t q_full[2], q_ready[2], s_full[2], p_ready[2];
  uint64_t k_full[kStages], k_empty[kStages], v_full[kStages], v_empty[kStages];
};

// Bounded wait whose outcome every lane of the warp agrees on, so warp-wide
// tcgen05 instructions are executed by all lanes or by none.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, bool ok, int* status, int code) {
  if (ok) ok = mbar_wait(bar, parity, status, code);
  return __all_sync(0xffffffffu, ok);
}

// kGlobal: the schedule has units with a second range of kv tiles (a global
// block); without it the tile of visited step j is t_begin + j and the mask
// test is the first range's, which keeps the per-tile state (and the register
// pressure of the softmax loop) as small as possible.
template <int D, bool kRope, bool kGlobal>
__global__ void __launch_bounds__(kThreads, 1)
bca_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using L = FwdLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + L::kBars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kTmemSlot);
  float* qscale = reinterpret_cast<float*>(smem + L::kQScale);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int32_t* u = p.units + (size_t)blockIdx.x * kFwdUnitInts;
  if constexpr (kDebugChecks) {
    if (!fwd_unit_in_range(u, p.batch, p.heads_q, p.heads_kv, p.seqlen_q, p.seqlen_kv, p.status)) return;
  }
  const int b = __ldg(u + 0), hk = __ldg(u + 1);
  const int head0 = __ldg(u + 2), head1 = __ldg(u + 4);
  const int m00 = __ldg(u + 3), m01 = __ldg(u + 5);
  const FwdTiles ft = fwd_tiles(u);
  const int n_vis = kGlobal ? ft.count() : ft.n_tiles - ft.t_begin;
  auto tile_of = [&](int j) { return kGlobal ? ft.tile(j) : ft.t_begin + j; };
  const int n_sub = head1 >= 0 ? 2 : 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->q_full[s], 1);
      mbar_init(&bars->q_ready[s], 1);
      mbar_init(&bars->s_full[s], 1);
      mbar_init(&bars->p_ready[s], 1);
    }
    for (int st = 0; st < kStages; ++st) {
      mbar_init(&bars->k_full[st], 1);
      mbar_init(&bars->k_empty[st], 1);
      mbar_init(&bars->v_full[st], 1);
      mbar_init(&bars->v_empty[st], 1);
    }
    fence_mbar_init();
  }
  if (warp == 9 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 8) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  for (int d = threadIdx.x; d < D; d += kThreads) qscale[d] = qscale_of(p.gamma_q, p.gamma_k, p.scale_log2, d);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 9) {
    // ------------------------------------------------------------ TMA producer
    if (elect_one()) {
      for (int s = 0; s < n_sub; ++s) {
        mbar_arrive_expect_tx(&bars->q_full[s], L::kTileBytes);
        for (int box = 0; box < D / 64; ++box)
          tma_load_4d(smem + L::kQ + s * L::kTileBytes + box * 16384, &tm_q, &bars->q_full[s], box * 64,
                      s ? head1 : head0, s ? m01 : m00, b);
      }
      for (int j = 0; j < n_vis; ++j) {
        const int st = j % kStages;
        const uint32_t par = ((j / kStages) & 1) ^ 1;
        if (!mbar_wait(&bars->k_empty[st], par, p.status, kErrKEmpty)) break;
        mbar_arrive_expect_tx(&bars->k_full[st], L::kTileBytes);
        for (int box = 0; box < D / 64; ++box)
          tma_load_4d(smem + L::kK + st * L::kTileBytes + box * 16384, &tm_k, &bars->k_full[st], box * 64, hk,
                      tile_of(j) * 128, b);
        if (!mbar_wait(&bars->v_empty[st], par, p.status, kErrVEmpty)) break;
        mbar_arrive_expect_tx(&bars->v_full[st], L::kTileBytes);
        for (int box = 0; box < D / 64; ++box)
          tma_load_4d(smem + L::kV + st * L::kTileBytes + box * 16384, &tm_v, &bars->v_full[st], box * 64, hk,
                      tile_of(j) * 128, b);
      }
    }
  } else if (warp == 8) {
    // ------------------------------------------------------------ MMA issuer
    if (elect_one()) {
      constexpr uint32_t idesc_s = make_idesc_bf16(128, 128, false, false);
      constexpr uint32_t idesc_o = make_idesc_bf16(128, D, false, true);
      const uint32_t q_base = smem_u32(smem + L::kQ);
      const uint32_t k_base = smem_u32(smem + L::kK);
      const uint32_t v_base = smem_u32(smem + L::kV);
      bool ok = true;
      auto issue_s = [&](int s, int st) {
        const uint32_t qa = q_base + s * L::kTileBytes, ka = k_base + st * L::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_bf16_ss(tmem + 256 * s, make_sw128_desc(qa + off, 16, 1024), make_sw128_desc(ka + off, 16, 1024),
                      idesc_s, kk > 0);
        }
      };
      for (int s = 0; s < n_sub && ok; ++s) ok = mbar_wait(&bars->q_ready[s], 0, p.status, kErrQReady);
      ok = ok && mbar_wait(&bars->k_full[0], 0, p.status, kErrKFull);
      if (ok) {
        tc_fence_after();
        for (int s = 0; s < n_sub; ++s) {
          issue_s(s, 0);
          mma_commit(&bars->s_full[s]);
        }
        mma_commit(&bars->k_empty[0]);
      }
      for (int j = 0; j < n_vis && ok; ++j) {
        const int st = j % kStages;
        if (!mbar_wait(&bars->v_full[st], (j / kStages) & 1, p.status, kErrVFull)) break;
        const bool has_next = j + 1 < n_vis;
        const int st1 = (j + 1) % kStages;
        for (int s = 0; s < n_sub; ++s) {
          if (!mbar_wait(&bars->p_ready[s], j & 1, p.status, kErrPReady)) { ok = false; break; }
          tc_fence_after();
          const uint32_t va = v_base + st * L::kTileBytes;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_bf16_ts(tmem + 256 * s + 128, tmem + 256 * s + kk * 8,
                        make_sw128_desc(va + kk * 2048, 16384, 1024), idesc_o, j > 0 || kk > 0);
          if (has_next) {
            if (s == 0 && !mbar_wait(&bars->k_full[st1], ((j + 1) / kStages) & 1, p.status, kErrKFull)) {
              ok = false;
              break;
            }
            issue_s(s, st1);
          }
          mma_commit(&bars->s_full[s]);
        }
        if (!ok) break;
        mma_commit(&bars->v_empty[st]);
        if (has_next) mma_commit(&bars->k_empty[st1]);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax warpgroups
    const int s = warp >> 2;           // sub-tile
    const int r = threadIdx.x & 127;   // row within the tile == TMEM lane
    if (s < n_sub) {
      const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
      const uint32_t t_s = tmem + lane_base + 256 * s;        // S_s / P_s
      const uint32_t t_o = tmem + lane_base + 256 * s + 128;  // O_s
      uint8_t* q_tile = smem + L::kQ + s * L::kTileBytes;
      const int bar_id = 1 + s;
      bool ok = true;

      // Q prologue: RMSNorm the row and fold gains, scale and log2(e) into it;
      // with rotary angles the row is rotated first (the RMS is the raw row's:
      // a rotation keeps it).
      ok = warp_wait(&bars->q_full[s], 0, ok, p.status, kErrQ);
      const int row = (s ? m01 : m00) + r;
      if (ok) {
        const float rq = rms_inv<D>(row_sumsq_swizzled_warp_order<D>(q_tile, r), p.eps);
        if (kRope && row < p.seqlen_q) {
          const float* ang = p.rope_q + (size_t)row * (D / 2);
#pragma unroll
          for (int pc = 0; pc < D / 16; ++pc) {
            const int fa = pc * 8, fb = fa + D / 2;
            uint4* pa = reinterpret_cast<uint4*>(q_tile + (fa / 64) * 16384 + sw128_offset(r, fa % 64));
            uint4* pb = reinterpret_cast<uint4*>(q_tile + (fb / 64) * 16384 + sw128_offset(r, fb % 64));
            uint4 va = *pa, vb = *pb;
            fold_q_pair<D>(va, vb, rq, qscale, fa, ang + fa);
            *pa = va;
            *pb = vb;
          }
        } else {
#pragma unroll
          for (int box = 0; box < D / 64; ++box) {
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              uint4* ptr = reinterpret_cast<uint4*>(q_tile + box * 16384 + sw128_offset(r, c * 8));
              *ptr = fold_q_chunk(*ptr, rq, qscale, box * 64 + c * 8);
            }
          }
        }
        fence_proxy_async_smem();
      }
      named_bar_sync(bar_id, 128);
      if (r == 0 && ok) mbar_arrive(&bars->q_ready[s]);

      int limit = p.seqlen_kv, kv_first = 0;
      if (row < p.seqlen_q) row_keys(p.mask, row, kv_first, limit);

      float m_ref = -INFINITY, l_sum = 0.f;
      // Every thread runs all n_vis iterations and reaches every named
      // barrier even after a failed wait; only the work is skipped.
      for (int j = 0; j < n_vis; ++j) {
        ok = warp_wait(&bars->s_full[s], j & 1, ok, p.status, kErrSFull);
        if (ok) {
          tc_fence_after();
          // S row (log2-unit logits) as 64 fp32 pairs
          uint64_t x2[64];
          {
            uint32_t raw[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld32(t_s + c * 32, raw[c]);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 4; ++c)
#pragma unroll
              for (int i = 0; i < 16; ++i)
                x2[c * 16 + i] = f2_pack(__uint_as_float(raw[c][2 * i]), __uint_as_float(raw[c][2 * i + 1]));
          }
          const int tile = tile_of(j);
          const bool masked = kGlobal ? ft.masked(j, p.mask.global_key, p.seqlen_kv)
                                      : tile < ft.t_full_begin || tile >= ft.n_full;
          if (masked) {
            // columns [lo, lim) and, with a global block, its keys [glo, ghi) are visible
            const int lim = limit - tile * 128, lo = kv_first - tile * 128;
            const int glo = kGlobal ? p.mask.global_key - tile * 128 : 0;
            const int ghi = kGlobal ? p.seqlen_kv - tile * 128 : 0;
#pragma unroll
            for (int c = 0; c < 64; ++c) {
              float a0, a1;
              f2_unpack(x2[c], a0, a1);
              const bool v0 = (2 * c >= lo && 2 * c < lim) || (2 * c >= glo && 2 * c < ghi);
              const bool v1 = (2 * c + 1 >= lo && 2 * c + 1 < lim) || (2 * c + 1 >= glo && 2 * c + 1 < ghi);
              x2[c] = f2_pack(v0 ? a0 : -INFINITY, v1 ? a1 : -INFINITY);
            }
          }
          // row maximum as a tree (short dependency chains)
          float mx[8];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            float a0, a1, b0, b1;
            f2_unpack(x2[i], a0, a1);
            f2_unpack(x2[4 + i], b0, b1);
            mx[2 * i] = fmaxf(a0, b0);
            mx[2 * i + 1] = fmaxf(a1, b1);
          }
#pragma unroll
          for (int c = 8; c < 64; c += 8)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              float a0, a1, b0, b1;
              f2_unpack(x2[c + i], a0, a1);
              f2_unpack(x2[c + 4 + i], b0, b1);
              mx[2 * i] = fmax3(mx[2 * i], a0, b0);
              mx[2 * i + 1] = fmax3(mx[2 * i + 1], a1, b1);
            }
          const float m_tile = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                                     fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
          // Lazy maximum: move the reference only when P could exceed 2^8.
          float alpha = 1.f;
          if (m_tile > m_ref + kRescaleThreshold) {
            alpha = fast_exp2(m_ref - m_tile);  // 0 on the first tile (m_ref = -inf)
            m_ref = m_tile;
            l_sum *= alpha;
          }
          // (a row whose visited tiles so far were all masked keeps m_ref = -inf
          // and gets P = 0 from exp2(-inf - 0))
          const float nm = m_ref == -INFINITY ? 0.f : -m_ref;
          const uint64_t negm = f2_pack(nm, nm);
          uint64_t ls2[4] = {0, 0, 0, 0};
          // P = exp2(S - m) -> bf16 pairs in TMEM.  The two variants are
          // separate straight-line loops (no per-pair branch), so the
          // compiler can interleave the exponentials of many pairs.
          auto exp_row = [&](auto use_poly) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              uint32_t pk[16];
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const uint64_t a2 = f2_add(x2[c * 16 + i], negm);
                float p0, p1;
                if (decltype(use_poly)::value && (i & 3) == 3) {
                  exp2_poly_pair(a2, p0, p1);
                } else {
                  float a0, a1;
                  f2_unpack(a2, a0, a1);
                  p0 = fast_exp2(a0);
                  p1 = fast_exp2(a1);
                }
                const uint64_t p2 = f2_pack(p0, p1);
                ls2[i & 3] = f2_add(ls2[i & 3], p2);
                pk[i] = pack_bf16x2(p0, p1);
              }
              tmem_st16(t_s + c * 16, pk);
            }
          };
          if (masked)
            exp_row(std::false_type{});
          else
            exp_row(std::true_type{});
          {
            float s[8];
#pragma unroll
            for (int i = 0; i < 4; ++i) f2_unpack(ls2[i], s[2 * i], s[2 * i + 1]);
            l_sum += ((s[0] + s[1]) + (s[2] + s[3])) + ((s[4] + s[5]) + (s[6] + s[7]));
          }
          if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
            // PV(j-1) is complete (s_full of tile j is committed after it); PV(j) is
            // issued only after p_ready below, so O can be rescaled here.
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
              uint32_t o[32];
              tmem_ld32(t_o + c * 32, o);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
              tmem_st32(t_o + c * 32, o);
            }
          }
          tmem_wait_st();
          tc_fence_before();
        }
        named_bar_sync(bar_id, 128);
        if (r == 0 && ok) mbar_arrive(&bars->p_ready[s]);
      }

      // Epilogue: wait for the last PV, then O / l -> bf16, and the LSE.
      ok = warp_wait(&bars->s_full[s], n_vis & 1, ok, p.status, kErrSFull);
      if (ok) {
        tc_fence_after();
        const float inv_l = 1.f / l_sum;
        const bool live = row < p.seqlen_q;
        const int hs = s ? head1 : head0;
        uint4* dst = reinterpret_cast<uint4*>(p.out + (((size_t)b * p.seqlen_q + row) * p.heads_q + hs) * D);
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(t_o + c * 32, o);
          tmem_wait_ld();
          if (live) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              uint4 w;
              w.x = pack_bf16x2(__uint_as_float(o[8 * i + 0]) * inv_l, __uint_as_float(o[8 * i + 1]) * inv_l);
              w.y = pack_bf16x2(__uint_as_float(o[8 * i + 2]) * inv_l, __uint_as_float(o[8 * i + 3]) * inv_l);
              w.z = pack_bf16x2(__uint_as_float(o[8 * i + 4]) * inv_l, __uint_as_float(o[8 * i + 5]) * inv_l);
              w.w = pack_bf16x2(__uint_as_float(o[8 * i + 6]) * inv_l, __uint_as_float(o[8 * i + 7]) * inv_l);
              dst[c * 4 + i] = w;
            }
          }
        }
        if (live && p.lse != nullptr)
          p.lse[((size_t)b * p.heads_q + hs) * p.seqlen_q + row] = (m_ref + log2f(l_sum)) * kLn2;
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

}  // namespace

// K^ = bf16(k r_k), r_k = rsqrt(mean_d k^2 + eps): one warp per key row, lane l
// holding features [l*D/32, (l+1)*D/32).  The backward runs the same kernel,
// so both passes see identical key operands.
template <int D>
__global__ void __launch_bounds__(256) bca_knorm_kernel(const uint16_t* __restrict__ k, uint16_t* __restrict__ kn,
                                                         int64_t rows, float eps, const float* __restrict__ rope,
                                                         int heads, int seqlen) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x / 32);
  for (int64_t r = (int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5); r < rows; r += warps) {
    // row r = (b * seqlen + token) * heads + h; the angles are the token's
    const float* ang = rope != nullptr ? rope + ((r / heads) % seqlen) * (D / 2) : nullptr;
    knorm_row<D>(k + r * D, kn + r * D, lane, eps, ang);
  }
}

cudaError_t launch_knorm(const uint16_t* k, uint16_t* kn, int64_t rows, int head_dim, float eps, cudaStream_t stream,
                         const float* rope, int heads, int seqlen) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int blocks = (int)std::min<int64_t>((rows + 7) / 8, (int64_t)sms * 16);
  if (blocks <= 0) return cudaSuccess;
  if (head_dim == 128)
    bca_knorm_kernel<128><<<blocks, 256, 0, stream>>>(k, kn, rows, eps, rope, heads, seqlen);
  else
    bca_knorm_kernel<64><<<blocks, 256, 0, stream>>>(k, kn, rows, eps, rope, heads, seqlen);
  return cudaGetLastError();
}

template <int D, bool kRope, bool kGlobal>
static cudaError_t launch_fwd_d(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                const FwdParams& p, int n_units, cudaStream_t stream) {
  using L = FwdLayout<D>;
  static uint64_t configured = 0;  // one bit per device ordinal that has the attribute set (per variant)
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !((configured >> dev) & 1u)) {
    e = cudaFuncSetAttribute(bca_fwd_kernel<D, kRope, kGlobal>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             L::kAlloc);
    if (e != cudaSuccess) return e;
    if (dev < 64) configured |= uint64_t(1) << dev;
  }
  bca_fwd_kernel<D, kRope, kGlobal><<<n_units, kThreads, L::kAlloc, stream>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

cudaError_t launch_fwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const FwdParams& p,
                       int head_dim, int n_units, cudaStream_t stream) {
  if (n_units <= 0) return cudaSuccess;
  const bool rope = p.rope_q != nullptr;
  const bool global = p.mask.global_key < p.seqlen_kv;
  if (head_dim == 128) {
    if (global)
      return rope ? launch_fwd_d<128, true, true>(tq, tk, tv, p, n_units, stream)
                  : launch_fwd_d<128, false, true>(tq, tk, tv, p, n_units, stream);
    return rope ? launch_fwd_d<128, true, false>(tq, tk, tv, p, n_units, stream)
                : launch_fwd_d<128, false, false>(tq, tk, tv, p, n_units, stream);
  }
  if (global)
    return rope ? launch_fwd_d<64, true, true>(tq, tk, tv, p, n_units, stream)
                : launch_fwd_d<64, false, true>(tq, tk, tv, p, n_units, stream);
  return rope ? launch_fwd_d<64, true, false>(tq, tk, tv, p, n_units, stream)
              : launch_fwd_d<64, false, false>(tq, tk, tv, p, n_units, stream);
}

size_t fwd_smem_bytes(int head_dim) {
  return head_dim == 128 ? FwdLayout<128>::kAlloc : FwdLayout<64>::kAlloc;
}

}  // namespace magi
