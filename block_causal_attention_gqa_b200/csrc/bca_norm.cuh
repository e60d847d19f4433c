// RMSNorm pieces shared by the forward and the backward.
//
// The backward recomputes the forward's logits, so both must produce the
// same fp32 row statistics and the same bf16 query operand bit for bit:
// every function here fixes its summation order (feature 0, 1, 2, ... in
// sequence) and its rounding points, whether the row sits in a 128-byte
// swizzled shared-memory tile or in global memory.
#pragma once
#include <cstdint>

#include "sm100.cuh"

namespace magi {

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// The same sum in the order a warp computes it when lane l holds features
// [l*E, l*E + E) (E = D/32): per-lane fmaf chains, then an xor butterfly
// (offsets 16, 8, 4, 2, 1).  Floating-point addition is commutative, so every
// lane of the warp ends with this value; warp_sumsq_row below is the warp side.
template <int D>
__device__ __forceinline__ float row_sumsq_swizzled_warp_order(const uint8_t* tile, int row) {
  constexpr int E = D / 32;
  float part[32];
#pragma unroll
  for (int box = 0; box < D / 64; ++box)
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const uint4 v = *reinterpret_cast<const uint4*>(tile + box * 16384 + sm100::sw128_offset(row, c * 8));
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const float x = (k & 1) ? bf16_hi(w[k >> 1]) : bf16_lo(w[k >> 1]);
        const int d = box * 64 + c * 8 + k;
        part[d / E] = (d % E == 0) ? x * x : fmaf(x, x, part[d / E]);
      }
    }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1)
#pragma unroll
    for (int i = 0; i < o; ++i) part[i] = part[i] + part[i + o];
  return part[0];
}

// Warp side of the above: lane holds x[0..E) of the row; returns the sum in every lane.
template <int E>
__device__ __forceinline__ float warp_sumsq_row(const float (&x)[E]) {
  float s = x[0] * x[0];
#pragma unroll
  for (int e = 1; e < E; ++e) s = fmaf(x[e], x[e], s);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s = s + __shfl_xor_sync(0xffffffffu, s, o);
  return s;
}

// 1 / RMS of a row from its sum of squares.
template <int D>
__device__ __forceinline__ float rms_inv(float sumsq, float eps) {
  return rsqrtf(sumsq * (1.0f / D) + eps);
}

// Rotary pair: (a, b) = (x_i, x_{i+D/2}) rotated by the angle whose cosine and
// sine are c, s.  Explicit roundings, so every kernel that rotates a row (the
// forward's Q prologue and key pre-pass, the backward's prep and finalize)
// gets the same bits.
__device__ __forceinline__ float rope_first(float a, float b, float c, float s) {
  return __fmaf_rn(-b, s, __fmul_rn(a, c));
}
__device__ __forceinline__ float rope_second(float a, float b, float c, float s) {
  return __fmaf_rn(a, s, __fmul_rn(b, c));
}

// Warp form: lane holds features [lane*E, lane*E + E) (E = D/32), so the pair
// partner of its features (i +- D/2) sits in lane ^ 16.  `ang` is the row's
// D/2 angles (nullptr: no rotation); y receives the rotated features.
template <int D>
__device__ __forceinline__ void rope_warp(const float (&x)[D / 32], const float* ang, int lane, float (&y)[D / 32]) {
  constexpr int E = D / 32;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const float xp = __shfl_xor_sync(0xffffffffu, x[e], 16);
    float sn, cs;
    sincosf(__ldg(ang + (lane & 15) * E + e), &sn, &cs);
    y[e] = lane < 16 ? rope_first(x[e], xp, cs, sn) : rope_second(xp, x[e], cs, sn);
  }
}

// One key row: dst = bf16(rope(src) * r_k), r_k = 1 / RMS(src) (a rotation
// keeps the RMS), by one warp (lane holds features [lane*D/32, lane*D/32 +
// D/32)); `ang` = the token's rotary angles or nullptr.  The forward's key
// pre-pass and the backward's prep both call this, so both see the same K^ bits.
template <int D>
__device__ __forceinline__ void knorm_row(const uint16_t* src, uint16_t* dst, int lane, float eps,
                                          const float* ang = nullptr) {
  constexpr int E = D / 32;
  float x[E];
  if constexpr (E == 4) {
    const uint2 w = *reinterpret_cast<const uint2*>(src + lane * E);
    x[0] = bf16_lo(w.x); x[1] = bf16_hi(w.x); x[2] = bf16_lo(w.y); x[3] = bf16_hi(w.y);
  } else {
    const uint32_t w = *reinterpret_cast<const uint32_t*>(src + lane * E);
    x[0] = bf16_lo(w); x[1] = bf16_hi(w);
  }
  float ss = 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e) ss = fmaf(x[e], x[e], ss);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float rk = rms_inv<D>(ss, eps);
  if (ang != nullptr) {   // warp-uniform
    float y[E];
    rope_warp<D>(x, ang, lane, y);
#pragma unroll
    for (int e = 0; e < E; ++e) x[e] = y[e];
  }
  if constexpr (E == 4) {
    uint2 w;
    w.x = sm100::pack_bf16x2(x[0] * rk, x[1] * rk);
    w.y = sm100::pack_bf16x2(x[2] * rk, x[3] * rk);
    *reinterpret_cast<uint2*>(dst + lane * E) = w;
  } else {
    *reinterpret_cast<uint32_t*>(dst + lane * E) = sm100::pack_bf16x2(x[0] * rk, x[1] * rk);
  }
}

// The forward's query operand for one 16-byte chunk (8 features starting at d0):
// bf16(q * r_q * qscale[d]) with qscale = gamma_q * gamma_k * softmax_scale * log2(e).
__device__ __forceinline__ uint4 fold_q_chunk(uint4 v, float rq, const float* qscale, int d0) {
  uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float lo = bf16_lo(w[i]) * rq * qscale[d0 + 2 * i];
    const float hi = bf16_hi(w[i]) * rq * qscale[d0 + 2 * i + 1];
    w[i] = sm100::pack_bf16x2(lo, hi);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// The forward's query operand for a rotary pair of 16-byte chunks: va holds
// features [d0, d0 + 8) and vb features [d0 + D/2, d0 + D/2 + 8); `ang` the
// row's angles for d0 .. d0 + 7.  bf16(rope(q) * r_q * qscale[d]).
template <int D>
__device__ __forceinline__ void fold_q_pair(uint4& va, uint4& vb, float rq, const float* qscale, int d0,
                                            const float* ang) {
  uint32_t wa[4] = {va.x, va.y, va.z, va.w}, wb[4] = {vb.x, vb.y, vb.z, vb.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float a[2] = {bf16_lo(wa[i]), bf16_hi(wa[i])}, b[2] = {bf16_lo(wb[i]), bf16_hi(wb[i])};
    float ya[2], yb[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float sn, cs;
      sincosf(__ldg(ang + 2 * i + h), &sn, &cs);
      ya[h] = rope_first(a[h], b[h], cs, sn) * rq * qscale[d0 + 2 * i + h];
      yb[h] = rope_second(a[h], b[h], cs, sn) * rq * qscale[d0 + D / 2 + 2 * i + h];
    }
    wa[i] = sm100::pack_bf16x2(ya[0], ya[1]);
    wb[i] = sm100::pack_bf16x2(yb[0], yb[1]);
  }
  va = make_uint4(wa[0], wa[1], wa[2], wa[3]);
  vb = make_uint4(wb[0], wb[1], wb[2], wb[3]);
}

__device__ __forceinline__ float qscale_of(const float* gamma_q, const float* gamma_k, float scale_log2, int d) {
  return __ldg(gamma_q + d) * __ldg(gamma_k + d) * scale_log2;
}

}  // namespace magi
