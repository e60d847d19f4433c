// Internal interface between the C ABI (bca_api.cu) and the kernels.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>
#include <vector>

#include "../../include/magi_bca.h"

namespace magi {

// Which keys each query row sees, as the kernels read it (built on the host
// from the chunk offsets, the KV range, the packed samples and the global
// block; see MaskSpec in bca_sched.h).  A query row of chunk c sees the keys
// [q_lo[c], q_hi[c]) and the global keys [global_key, seqlen_kv).
struct MaskArgs {
  const int32_t* q_offsets;   // device copy of the query chunk offsets [n_q_chunks + 1]
  const int32_t* q_lo;        // device [n_q_chunks]: first visible key by the block-causal rule
  const int32_t* q_hi;        // device [n_q_chunks]: end of those keys
  int n_q_chunks;
  int n_normal_q;             // chunks [0, n_normal_q) are not global (lo, hi non-decreasing there)
  int global_q_row;           // rows from here on see every key (seqlen_q: none)
  int global_key;             // keys from here on are seen by every row (seqlen_kv: none)
};

struct FwdParams {
  const int32_t* units;       // device, 12 int32 per unit (see magi_bca_fwd_schedule)
  MaskArgs mask;
  const float* rope_q;        // rotary angles of the query tokens [Sq, D/2] or nullptr
  const float* gamma_q;
  const float* gamma_k;
  uint16_t* out;              // [B, Sq, Hq, D] bf16
  float* lse;                 // [B, Hq, Sq] or nullptr
  int batch, seqlen_q, seqlen_kv, heads_q, heads_kv;
  float scale_log2;           // softmax_scale * log2(e)
  float eps;
  int* status;                // device status word (bounded waits, debug checks)
};

struct BwdParams {
  // inputs
  const uint16_t* q;          // [B, Sq, Hq, D] raw
  const uint16_t* k;          // [B, Skv, Hkv, D] raw
  const uint16_t* out;        // forward output
  const uint16_t* dout;
  const float* lse;           // [B, Hq, Sq] natural log
  const float* gamma_q;
  const float* gamma_k;
  const int32_t* units;       // device schedule, 12 int32 per unit (see magi_bca_bwd_schedule)
  MaskArgs mask;
  const float* rope_q;        // rotary angles [Sq, D/2] / [Skv, D/2], or nullptr
  const float* rope_k;
  float* drope_q;             // their gradients (summed over batch and heads), or nullptr
  float* drope_k;
  // outputs
  uint16_t* dq;
  uint16_t* dk;
  uint16_t* dv;
  float* dgamma_q;            // may be null
  float* dgamma_k;            // may be null
  // workspace
  uint16_t* qn;               // forward query operand Q^       [B, Sq, Hq, D]
  uint16_t* kn;               // forward key operand K^ = bf16(k r_k) [B, Skv, Hkv, D]
  float* ld;                  // 16-byte rows of bf16 pieces of -lse*log2(e), -Delta [B, Hq, Sq_pad, 8 x bf16]
  float* dqacc;               // fp32 G_q accumulator          [B, Sq, Hq, D]
  float* dvacc;               // fp32 dV accumulator           [B, Skv, Hkv, D]
  float* dkacc;               // fp32 G_k accumulator          [B, Skv, Hkv, D]
  // deterministic backward
  int deterministic;          // 0 or 1
  const int32_t* dq_units;    // query-major units of the dq pass (forward schedule, 12 int32 each)
  float* dgamma_part;         // per finalize block: dgamma_q [D] then dgamma_k [D], summed in block order
  int batch, seqlen_q, seqlen_kv, heads_q, heads_kv, seqlen_q_pad;
  float scale;                // softmax scale
  float scale_log2;           // softmax scale * log2(e)
  float eps;
  int* status;
};

struct BwdWorkspace {
  size_t qn, kn, ld, dqacc, dvacc, dkacc, dgpart, total;  // byte offsets and total size
};
BwdWorkspace bwd_workspace_layout(int B, int Sq, int Skv, int Hq, int Hkv, int D);

cudaError_t launch_bwd(const CUtensorMap& t_k, const CUtensorMap& t_v, const CUtensorMap& t_qn,
                       const CUtensorMap& t_do, const CUtensorMap& t_dq, const CUtensorMap& t_dv,
                       const CUtensorMap& t_dk, const BwdParams& p, int head_dim, int n_units, int n_dq_units,
                       cudaStream_t stream);
int make_tensor_map_f32_dq(CUtensorMap* m, const void* base, int B, int S, int H, int D);
// The deterministic backward's dq pass and dK/dV pass (bca_bwd_split.cu), launched
// by launch_bwd between the prep and finalize kernels.
cudaError_t launch_bwd_split(const CUtensorMap& t_k, const CUtensorMap& t_v, const CUtensorMap& t_qn,
                             const CUtensorMap& t_do, const CUtensorMap& t_dv, const CUtensorMap& t_dk,
                             const BwdParams& p, int head_dim, int n_units, int n_dq_units, cudaStream_t stream);

// K^ = bf16(rope(k) rsqrt(mean k^2 + eps)) for `rows` rows [B, seqlen, heads] of head_dim
// features; `rope` = per-token angles [seqlen, head_dim / 2] or nullptr (no rotation).
cudaError_t launch_knorm(const uint16_t* k, uint16_t* kn, int64_t rows, int head_dim, float eps, cudaStream_t stream,
                         const float* rope, int heads, int seqlen);

cudaError_t launch_fwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const FwdParams& p,
                       int head_dim, int n_units, cudaStream_t stream);
size_t fwd_smem_bytes(int head_dim);

// Records the diagnostic timing events (magi_bca_profile_events) on `stream`:
// which = 0 before a main-kernel launch, 1 after it.  No-op when unset.
void profile_mark(int which, cudaStream_t stream);

// The mask part of a device schedule blob: query offsets, then lo, then hi
// (3 n_q_chunks + 1 int32), and the MaskArgs that point into it at `dev`.
struct MaskSpec;
void append_mask_blob(std::vector<int32_t>& blob, const int32_t* q_offsets, const MaskSpec& m, int n_q_chunks);
MaskArgs mask_args_at(const int32_t* dev, const MaskSpec& m, int n_q_chunks);

// Shared host helpers (bca_api.cu).
int make_tensor_map_bf16(CUtensorMap* m, const void* base, int B, int S, int H, int D);
float resolve_softmax_scale(const magi_bca_dims& d);
int device_status_word(int** out);  // the status word of the current device (checks the device once)
int record_cuda_failure(const char* what, cudaError_t e);  // sets the error detail, returns MAGI_BCA_CUDA_ERROR

}  // namespace magi
