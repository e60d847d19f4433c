// Test kernel: evaluates the kernels' exp2 cubic (exp2_poly_pair) and CUDA's
// exp2f on the same inputs, for tests/test_exp2_poly.py.  Not part of the
// library.
#include <cuda_runtime.h>

#include "../block_causal_attention_gqa_b200/csrc/sm100.cuh"

__global__ void exp2_poly_probe_kernel(const float* x, float* poly, float* ref, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float a0 = x[i], a1 = i + 1 < n ? x[i + 1] : x[i];
  float p0, p1;
  magi::sm100::exp2_poly_pair(magi::sm100::f2_pack(a0, a1), p0, p1);
  poly[i] = p0;
  ref[i] = exp2f(a0);
  if (i + 1 < n) {
    poly[i + 1] = p1;
    ref[i + 1] = exp2f(a1);
  }
}

extern "C" int exp2_poly_probe(const float* x, float* poly, float* ref, int n) {
  if (n <= 0) return 0;
  const int pairs = (n + 1) / 2;
  exp2_poly_probe_kernel<<<(pairs + 255) / 256, 256>>>(x, poly, ref, n);
  return cudaGetLastError() == cudaSuccess ? 0 : 1;
}
