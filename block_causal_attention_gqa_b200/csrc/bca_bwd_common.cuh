// Definitions shared by the backward's translation units (bca_bwd.cu: prep,
// fused main kernel, finalize; bca_bwd_split.cu: the dq and dK/dV passes of
// the deterministic backward): warp roles of the 576-thread kv-major kernels,
// device status codes of their bounded waits, and small helpers.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include "bca_kernels.h"
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

// cudaFuncSetAttribute once per (kernel, device); bit `dev` of `mask`.
template <typename K>
cudaError_t set_smem_once(uint64_t& mask, int dev, K kernel, int bytes) {
  if (dev < 64 && ((mask >> dev) & 1u)) return cudaSuccess;
  const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && dev < 64) mask |= uint64_t(1) << dev;
  return e;
}

}  // namespace
}  // namespace magi
