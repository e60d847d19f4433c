// Internal interface between the C ABI (bca_api.cu) and the kernels.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

namespace magi {

struct FwdParams {
  const int32_t* units;       // device, 8 int32 per unit (see magi_bca_fwd_schedule)
  const int32_t* q_offsets;   // device copy of the query chunk offsets
  const int32_t* kv_offsets;  // device copy of the kv chunk offsets
  int n_q_chunks, n_kv_chunks;
  const float* gamma_q;
  const float* gamma_k;
  uint16_t* out;              // [B, Sq, Hq, D] bf16
  float* lse;                 // [B, Hq, Sq] or nullptr
  int seqlen_q, seqlen_kv, heads_q;
  float scale_log2;           // softmax_scale * log2(e)
  float eps;
  int* status;                // device status word (bounded waits)
};

cudaError_t launch_fwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const FwdParams& p,
                       int head_dim, int n_units, cudaStream_t stream);
size_t fwd_smem_bytes(int head_dim);

}  // namespace magi
