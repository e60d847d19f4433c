// magi_bca_bwd_noalloc: the backward without any device allocation.
//
// Some callers cannot hand this library device memory or let it allocate:
// processes whose device memory is owned up front by a pooled allocator (an
// inference or training server that reserves the GPU's memory at start-up and
// grants nothing outside its pool), plugin interfaces whose execute callback
// must not allocate, and latency-critical loops that cannot afford
// cudaMalloc's implicit device synchronisation.  This entry point serves them:
// the backward's workspace and its tile schedule live in one file-scope
// device array, so a call allocates nothing.
//
// The array is kNoallocScratchBytes (96 MiB) per device.  Every GPU that loads
// this library holds it until the process exits.  Problems whose workspace
// plus schedule do not fit are rejected with MAGI_BCA_WORKSPACE_TOO_SMALL.
//
// The host code of this file cannot pass the array's name to a kernel: on the
// host the name is only a stand-in, not a device address.  The first call on a
// device looks up the array's device address with cudaGetSymbolAddress (with
// that device current) and keeps it; make that first call before any stream
// capture.  Each call copies its tile schedule into the array from host
// memory, so while its stream is capturing the call returns
// MAGI_BCA_UNSUPPORTED with nothing enqueued.  All calls share the array and
// it keeps the last call's contents, so calls that overlap on the GPU (other
// streams, other threads) race; the kernels clear everything that must start
// at zero.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/magi_bca.h"
#include "bca_kernels.h"
#include "bca_sched.h"

namespace magi {

constexpr size_t kNoallocScratchBytes = size_t(96) << 20;

namespace {

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[64] = {};  // device address of the array, per device ordinal

// Device address of the scratch array on the current device (set up once).
int scratch_address(int dev, unsigned char** out) {
  if (dev < 0 || dev >= 64) return MAGI_BCA_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr)
      return MAGI_BCA_CUDA_ERROR;
    g_noalloc_ptr[dev] = ptr;
  }
  *out = static_cast<unsigned char*>(g_noalloc_ptr[dev]);
  return MAGI_BCA_OK;
}

int make_bf16_map(CUtensorMap* m, const void* base, int B, int S, int H, int D) {
  return make_tensor_map_bf16(m, base, B, S, H, D);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace magi

using namespace magi;

extern "C" int magi_bca_bwd_noalloc(const magi_bca_bf16* q, const magi_bca_bf16* k, const magi_bca_bf16* v,
                                    const magi_bca_bf16* out, const magi_bca_bf16* dout, const float* lse,
                                    const int32_t* q_chunk_offsets, const int32_t* kv_chunk_offsets,
                                    const float* gamma_q, const float* gamma_k, magi_bca_bf16* dq,
                                    magi_bca_bf16* dk, magi_bca_bf16* dv, float* dgamma_q, float* dgamma_k,
                                    const magi_bca_dims* dims, void* stream) {
  int st = validate_dims(dims);
  if (st != MAGI_BCA_OK) return st;
  const magi_bca_dims& d = *dims;
  if (!q || !k || !v || !out || !dout || !lse || !gamma_q || !gamma_k || !dq || !dk || !dv)
    return MAGI_BCA_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(dout) || !aligned16(dq) ||
      !aligned16(dk) || !aligned16(dv) || !aligned16(lse))
    return MAGI_BCA_INVALID_ARG;
  st = validate_offsets(q_chunk_offsets, kv_chunk_offsets, d);
  if (st != MAGI_BCA_OK) return st;

  // Layout inside the array: [workspace][schedule units][mask blob: query
  // offsets, lo, hi] and, for the deterministic backward, [dq-pass units].
  const BwdWorkspace ws = bwd_workspace_layout(d.batch, d.seqlen_q, d.seqlen_kv, d.heads_q, d.heads_kv, d.head_dim);
  int sms = 148;
  {
    int dev0 = 0;
    if (cudaGetDevice(&dev0) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev0);
  }
  std::vector<int32_t> blob = build_bwd_schedule(q_chunk_offsets, kv_chunk_offsets, d, sms);
  const int n_units = static_cast<int>(blob.size() / kUnitInts);
  const MaskSpec mask = build_mask_spec(q_chunk_offsets, kv_chunk_offsets, d);
  append_mask_blob(blob, q_chunk_offsets, mask, d.n_q_chunks);
  const size_t dq_units_off = blob.size();
  int n_dq_units = 0;
  if (d.deterministic) {
    const std::vector<int32_t> fwd = build_fwd_schedule(q_chunk_offsets, kv_chunk_offsets, d);
    n_dq_units = static_cast<int>(fwd.size() / kFwdUnitInts);
    blob.insert(blob.end(), fwd.begin(), fwd.end());
  }
  const size_t sched_off = ws.total;  // a multiple of 256
  const size_t need = sched_off + blob.size() * sizeof(int32_t);
  if (need > kNoallocScratchBytes) return MAGI_BCA_WORKSPACE_TOO_SMALL;

  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return MAGI_BCA_CUDA_ERROR;
  int* status = nullptr;
  st = device_status_word(&status);
  if (st != MAGI_BCA_OK) return st;
  unsigned char* scratch = nullptr;
  st = scratch_address(dev, &scratch);
  if (st != MAGI_BCA_OK) return st;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // Every call uploads its schedule from a host vector that is gone when the
  // call returns, so a capture would record a copy from freed host memory:
  // refuse while the stream is capturing, before anything is enqueued.
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  const cudaError_t ce = cudaStreamIsCapturing(s, &cap);
  if (ce != cudaSuccess) return record_cuda_failure("cudaStreamIsCapturing", ce);
  if (cap != cudaStreamCaptureStatusNone) return MAGI_BCA_UNSUPPORTED;
  int32_t* sched = reinterpret_cast<int32_t*>(scratch + sched_off);
  // From pageable host memory the copy is staged before this call returns, so
  // the local vector may go out of scope afterwards.
  if (cudaMemcpyAsync(sched, blob.data(), blob.size() * sizeof(int32_t), cudaMemcpyHostToDevice, s) != cudaSuccess)
    return MAGI_BCA_CUDA_ERROR;

  BwdParams p;
  p.q = q;
  p.k = k;
  p.out = out;
  p.dout = dout;
  p.lse = lse;
  p.gamma_q = gamma_q;
  p.gamma_k = gamma_k;
  p.units = sched;
  p.mask = mask_args_at(sched + (size_t)n_units * kUnitInts, mask, d.n_q_chunks);
  p.rope_q = p.rope_k = nullptr;
  p.drope_q = p.drope_k = nullptr;
  p.deterministic = d.deterministic;
  p.dq_units = d.deterministic ? sched + dq_units_off : nullptr;
  p.dgamma_part = reinterpret_cast<float*>(scratch + ws.dgpart);
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  p.dgamma_q = dgamma_q;
  p.dgamma_k = dgamma_k;
  p.qn = reinterpret_cast<uint16_t*>(scratch + ws.qn);
  p.kn = reinterpret_cast<uint16_t*>(scratch + ws.kn);
  p.ld = reinterpret_cast<float*>(scratch + ws.ld);
  p.dqacc = reinterpret_cast<float*>(scratch + ws.dqacc);
  p.dvacc = reinterpret_cast<float*>(scratch + ws.dvacc);
  p.dkacc = reinterpret_cast<float*>(scratch + ws.dkacc);
  p.batch = d.batch;
  p.seqlen_q = d.seqlen_q;
  p.seqlen_kv = d.seqlen_kv;
  p.heads_q = d.heads_q;
  p.heads_kv = d.heads_kv;
  p.seqlen_q_pad = (d.seqlen_q + 127) / 128 * 128;
  p.scale = resolve_softmax_scale(d);
  p.scale_log2 = p.scale * 1.4426950408889634f;
  p.eps = d.rms_eps;
  p.status = status;
  CUtensorMap t_k, t_v, t_qn, t_do, t_dq, t_dv, t_dk;
  if (make_tensor_map_f32_dq(&t_dq, p.dqacc, d.batch, d.seqlen_q, d.heads_q, d.head_dim) != MAGI_BCA_OK ||
      make_tensor_map_f32_dq(&t_dv, p.dvacc, d.batch, d.seqlen_kv, d.heads_kv, d.head_dim) != MAGI_BCA_OK ||
      make_tensor_map_f32_dq(&t_dk, p.dkacc, d.batch, d.seqlen_kv, d.heads_kv, d.head_dim) != MAGI_BCA_OK ||
      make_bf16_map(&t_k, p.kn, d.batch, d.seqlen_kv, d.heads_kv, d.head_dim) != MAGI_BCA_OK ||
      make_bf16_map(&t_v, v, d.batch, d.seqlen_kv, d.heads_kv, d.head_dim) != MAGI_BCA_OK ||
      make_bf16_map(&t_qn, p.qn, d.batch, d.seqlen_q, d.heads_q, d.head_dim) != MAGI_BCA_OK ||
      make_bf16_map(&t_do, dout, d.batch, d.seqlen_q, d.heads_q, d.head_dim) != MAGI_BCA_OK)
    return MAGI_BCA_CUDA_ERROR;
  const cudaError_t e = launch_bwd(t_k, t_v, t_qn, t_do, t_dq, t_dv, t_dk, p, d.head_dim, n_units, n_dq_units, s);
  return e == cudaSuccess ? MAGI_BCA_OK : record_cuda_failure("allocation-free backward launch", e);
}
