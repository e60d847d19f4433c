// C ABI of libmagi_bca: argument checks, the schedule cache, TMA descriptors
// and kernel dispatch.  See include/magi_bca.h for the contract.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>
#include <vector>

#include "../../include/magi_bca.h"
#include "bca_kernels.h"
#include "bca_sched.h"
#include "sm100.cuh"

namespace magi {

// Device status word written by bounded waits that give up (0 = fine).
__device__ int g_device_status;

// Diagnostic timing events (magi_bca_profile_events); null when unset.
std::atomic<void*> g_profile_begin{nullptr}, g_profile_end{nullptr};

// Self-test of the bounded-wait path: one thread waits, with a short poll
// limit, on an mbarrier that nothing arrives at, so the wait gives up and
// records `code` in the status word as a stalled pipeline stage would.
__global__ void bca_wait_selftest_kernel(int* status, int code, uint32_t limit) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    sm100::mbar_init(&bar, 1);
    sm100::fence_mbar_init();
    sm100::mbar_wait_limit(&bar, 0, status, code, limit);
  }
}

void profile_mark(int which, cudaStream_t stream) {
  void* ev = which == 0 ? g_profile_begin.load() : g_profile_end.load();
  if (ev != nullptr) cudaEventRecord(static_cast<cudaEvent_t>(ev), stream);
}

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

std::mutex g_mutex;

// Text of the most recent failure on this thread (CUDA call and its error).
thread_local char g_last_detail[256] = "";

int cuda_fail(const char* what, cudaError_t e) {
  std::snprintf(g_last_detail, sizeof(g_last_detail), "%s: %s", what, cudaGetErrorString(e));
  return MAGI_BCA_CUDA_ERROR;
}

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!tried) {
    tried = true;
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

struct DeviceState {
  int* status = nullptr;
  bool checked = false;
  bool supported = false;
};

struct ScheduleEntry {
  int32_t* dev = nullptr;  // units, then q offsets, then kv offsets
  int n_units = 0;
};

std::map<int, DeviceState> g_devices;
std::map<std::vector<int32_t>, ScheduleEntry> g_schedules;
// Normalised-key buffers of the forward, one per (device, stream, bytes), so
// calls on different streams never share one.
std::map<std::tuple<int, uintptr_t, size_t>, void*> g_knorm_bufs;

int knorm_buffer(int dev, cudaStream_t stream, size_t bytes, void** out) {
  std::lock_guard<std::mutex> lock(g_mutex);
  auto key = std::make_tuple(dev, reinterpret_cast<uintptr_t>(stream), bytes);
  auto it = g_knorm_bufs.find(key);
  if (it != g_knorm_bufs.end()) {
    *out = it->second;
    return MAGI_BCA_OK;
  }
  void* ptr = nullptr;
  const cudaError_t e = cudaMalloc(&ptr, bytes);
  if (e != cudaSuccess) return cuda_fail("cudaMalloc (normalised-key buffer)", e);
  g_knorm_bufs[key] = ptr;
  *out = ptr;
  return MAGI_BCA_OK;
}

// Checks the current device once (sm_100 family) and resolves the status word.
int device_state(int* device_out, DeviceState** st_out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return MAGI_BCA_CUDA_ERROR;
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceState& st = g_devices[dev];
  if (!st.checked) {
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return MAGI_BCA_CUDA_ERROR;
    st.supported = (prop.major == 10 && prop.minor == 0);
    void* addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_device_status) != cudaSuccess) return MAGI_BCA_CUDA_ERROR;
    st.status = static_cast<int*>(addr);
    st.checked = true;
  }
  if (!st.supported) return MAGI_BCA_UNSUPPORTED;
  *device_out = dev;
  *st_out = &st;
  return MAGI_BCA_OK;
}

std::vector<int32_t> schedule_key(int dev, int kind, const magi_bca_dims& d, const int32_t* qo, const int32_t* ko) {
  std::vector<int32_t> key = {dev,        kind,         d.batch,       d.seqlen_q,  d.seqlen_kv,
                              d.heads_q,  d.heads_kv,   d.head_dim,    d.n_q_chunks, d.n_kv_chunks,
                              d.kv_range, kind == 0 ? 0 : d.deterministic};
  key.insert(key.end(), qo, qo + d.n_q_chunks + 1);
  key.insert(key.end(), ko, ko + d.n_kv_chunks + 1);
  return key;
}

// Returns the cached device schedule, building and uploading it on first use.
int get_schedule(int dev, int kind, const magi_bca_dims& d, const int32_t* qo, const int32_t* ko,
                 ScheduleEntry* out) {
  std::vector<int32_t> key = schedule_key(dev, kind, d, qo, ko);
  std::lock_guard<std::mutex> lock(g_mutex);
  auto it = g_schedules.find(key);
  if (it != g_schedules.end()) {
    *out = it->second;
    return MAGI_BCA_OK;
  }
  int sms = 148;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  std::vector<int32_t> units = kind == 0 ? build_fwd_schedule(qo, ko, d) : build_bwd_schedule(qo, ko, d, sms);
  ScheduleEntry e;
  e.n_units = static_cast<int>(units.size() / (kind == 0 ? kFwdUnitInts : kUnitInts));
  std::vector<int32_t> blob = units;
  blob.insert(blob.end(), qo, qo + d.n_q_chunks + 1);
  blob.insert(blob.end(), ko, ko + d.n_kv_chunks + 1);
  if (cudaMalloc(&e.dev, blob.size() * sizeof(int32_t)) != cudaSuccess) return MAGI_BCA_CUDA_ERROR;
  if (cudaMemcpy(e.dev, blob.data(), blob.size() * sizeof(int32_t), cudaMemcpyHostToDevice) != cudaSuccess) {
    cudaFree(e.dev);
    return MAGI_BCA_CUDA_ERROR;
  }
  g_schedules[key] = e;
  *out = e;
  return MAGI_BCA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// 4-D map over a [B, S, H, D] bf16 tensor with a {64, 1, 128, 1} box and the
// 128-byte swizzle, so one load brings 128 tokens x 64 features of one head.
int make_map(CUtensorMap* m, const void* base, int B, int S, int H, int D) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return MAGI_BCA_CUDA_ERROR;
  cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)S, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2, (cuuint64_t)S * H * D * 2};
  cuuint32_t box[4] = {64, 1, 128, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    std::snprintf(g_last_detail, sizeof(g_last_detail), "cuTensorMapEncodeTiled (bf16) failed: CUresult %d", (int)r);
    return MAGI_BCA_CUDA_ERROR;
  }
  return MAGI_BCA_OK;
}

// 4-D map over the fp32 [B, S, H, D] dq accumulator with a {32, 1, 128, 1} box
// (128 bytes wide) and the 128-byte swizzle, for bulk reduce-adds.
int make_map_f32(CUtensorMap* m, const void* base, int B, int S, int H, int D) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return MAGI_BCA_CUDA_ERROR;
  cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)S, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)D * 4, (cuuint64_t)H * D * 4, (cuuint64_t)S * H * D * 4};
  cuuint32_t box[4] = {32, 1, 128, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, const_cast<void*>(base), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    std::snprintf(g_last_detail, sizeof(g_last_detail), "cuTensorMapEncodeTiled (fp32) failed: CUresult %d", (int)r);
    return MAGI_BCA_CUDA_ERROR;
  }
  return MAGI_BCA_OK;
}

float resolve_scale(const magi_bca_dims& d) {
  return d.softmax_scale > 0.f ? d.softmax_scale : 1.0f / std::sqrt((float)d.head_dim);
}

}  // namespace

// Entry points for other translation units of the library.
int make_tensor_map_bf16(CUtensorMap* m, const void* base, int B, int S, int H, int D) {
  return make_map(m, base, B, S, H, D);
}

int make_tensor_map_f32_dq(CUtensorMap* m, const void* base, int B, int S, int H, int D) {
  return make_map_f32(m, base, B, S, H, D);
}

float resolve_softmax_scale(const magi_bca_dims& d) { return resolve_scale(d); }

int record_cuda_failure(const char* what, cudaError_t e) { return cuda_fail(what, e); }

int device_status_word(int** out) {
  int dev;
  DeviceState* ds;
  const int st = device_state(&dev, &ds);
  if (st != MAGI_BCA_OK) return st;
  *out = ds->status;
  return MAGI_BCA_OK;
}

}  // namespace magi

using namespace magi;

extern "C" {

const char* magi_bca_version(void) { return "magi_bca 0.1 (sm_100a)"; }

int magi_bca_profile_events(void* event_begin, void* event_end) {
  if ((event_begin == nullptr) != (event_end == nullptr)) return MAGI_BCA_INVALID_ARG;
  magi::g_profile_begin.store(event_begin);
  magi::g_profile_end.store(event_end);
  return MAGI_BCA_OK;
}

const char* magi_bca_status_string(int status) {
  switch (status) {
    case MAGI_BCA_OK: return "ok";
    case MAGI_BCA_INVALID_ARG: return "invalid argument";
    case MAGI_BCA_UNSUPPORTED: return "unsupported configuration or device";
    case MAGI_BCA_BAD_OFFSETS: return "bad chunk offsets";
    case MAGI_BCA_WORKSPACE_TOO_SMALL: return "workspace too small";
    case MAGI_BCA_CUDA_ERROR: return "CUDA runtime error";
    case MAGI_BCA_DEVICE_TIMEOUT: return "device-side wait timed out";
    default: return "unknown status";
  }
}

int64_t magi_bca_fwd_schedule(const int32_t* q_chunk_offsets, const int32_t* kv_chunk_offsets,
                              const magi_bca_dims* dims, int32_t* units, int64_t capacity) {
  int st = validate_dims(dims);
  if (st != MAGI_BCA_OK) return st;
  st = validate_offsets(q_chunk_offsets, kv_chunk_offsets, *dims);
  if (st != MAGI_BCA_OK) return st;
  if (capacity > 0 && units == nullptr) return MAGI_BCA_INVALID_ARG;
  std::vector<int32_t> s = build_fwd_schedule(q_chunk_offsets, kv_chunk_offsets, *dims);
  const int64_t n = (int64_t)(s.size() / kFwdUnitInts);
  const int64_t w = n < capacity ? n : capacity;
  if (w > 0) std::memcpy(units, s.data(), (size_t)w * kFwdUnitInts * sizeof(int32_t));
  return n;
}

int64_t magi_bca_bwd_schedule(const int32_t* q_chunk_offsets, const int32_t* kv_chunk_offsets,
                              const magi_bca_dims* dims, int32_t num_sms, int32_t* units, int64_t capacity) {
  int st = validate_dims(dims);
  if (st != MAGI_BCA_OK) return st;
  st = validate_offsets(q_chunk_offsets, kv_chunk_offsets, *dims);
  if (st != MAGI_BCA_OK) return st;
  if ((capacity > 0 && units == nullptr) || num_sms <= 0) return MAGI_BCA_INVALID_ARG;
  std::vector<int32_t> s = build_bwd_schedule(q_chunk_offsets, kv_chunk_offsets, *dims, num_sms);
  const int64_t n = (int64_t)(s.size() / kUnitInts);
  const int64_t w = n < capacity ? n : capacity;
  if (w > 0) std::memcpy(units, s.data(), (size_t)w * kUnitInts * sizeof(int32_t));
  return n;
}

int magi_bca_fwd(const magi_bca_bf16* q, const magi_bca_bf16* k, const magi_bca_bf16* v,
                 const int32_t* q_chunk_offsets, const int32_t* kv_chunk_offsets, const float* gamma_q,
                 const float* gamma_k, magi_bca_bf16* out, float* lse, const magi_bca_dims* dims, void* stream) {
  return magi_bca_fwd_rope(q, k, v, q_chunk_offsets, kv_chunk_offsets, gamma_q, gamma_k, nullptr, nullptr, out, lse,
                           dims, stream);
}

int magi_bca_fwd_rope(const magi_bca_bf16* q, const magi_bca_bf16* k, const magi_bca_bf16* v,
                      const int32_t* q_chunk_offsets, const int32_t* kv_chunk_offsets, const float* gamma_q,
                      const float* gamma_k, const float* rope_q, const float* rope_k, magi_bca_bf16* out, float* lse,
                      const magi_bca_dims* dims, void* stream) {
  int st = validate_dims(dims);
  if (st != MAGI_BCA_OK) return st;
  const magi_bca_dims& d = *dims;
  if (!q || !k || !v || !gamma_q || !gamma_k || !out) return MAGI_BCA_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return MAGI_BCA_INVALID_ARG;
  st = validate_offsets(q_chunk_offsets, kv_chunk_offsets, d);
  if (st != MAGI_BCA_OK) return st;
  int dev;
  DeviceState* ds;
  st = device_state(&dev, &ds);
  if (st != MAGI_BCA_OK) return st;
  ScheduleEntry sched;
  st = get_schedule(dev, 0, d, q_chunk_offsets, kv_chunk_offsets, &sched);
  if (st != MAGI_BCA_OK) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const int64_t kv_rows = (int64_t)d.batch * d.seqlen_kv * d.heads_kv;
  void* kn = nullptr;
  st = knorm_buffer(dev, cs, (size_t)kv_rows * d.head_dim * 2, &kn);
  if (st != MAGI_BCA_OK) return st;
  cudaError_t ke = launch_knorm(k, static_cast<uint16_t*>(kn), kv_rows, d.head_dim, d.rms_eps, cs, rope_k,
                                d.heads_kv, d.seqlen_kv);
  if (ke != cudaSuccess) return cuda_fail("key normalisation launch", ke);
  CUtensorMap tq, tk, tv;
  if (make_map(&tq, q, d.batch, d.seqlen_q, d.heads_q, d.head_dim) != MAGI_BCA_OK ||
      make_map(&tk, kn, d.batch, d.seqlen_kv, d.heads_kv, d.head_dim) != MAGI_BCA_OK ||
      make_map(&tv, v, d.batch, d.seqlen_kv, d.heads_kv, d.head_dim) != MAGI_BCA_OK)
    return MAGI_BCA_CUDA_ERROR;
  FwdParams p;
  p.units = sched.dev;
  p.q_offsets = sched.dev + (size_t)sched.n_units * kFwdUnitInts;
  p.kv_offsets = p.q_offsets + d.n_q_chunks + 1;
  p.n_q_chunks = d.n_q_chunks;
  p.n_kv_chunks = d.n_kv_chunks;
  p.kv_range = d.kv_range;
  p.rope_q = rope_q;
  p.gamma_q = gamma_q;
  p.gamma_k = gamma_k;
  p.out = out;
  p.lse = lse;
  p.seqlen_q = d.seqlen_q;
  p.seqlen_kv = d.seqlen_kv;
  p.heads_q = d.heads_q;
  p.scale_log2 = resolve_scale(d) * 1.4426950408889634f;
  p.eps = d.rms_eps;
  p.status = ds->status;
  profile_mark(0, cs);
  cudaError_t e = launch_fwd(tq, tk, tv, p, d.head_dim, sched.n_units, cs);
  profile_mark(1, cs);
  return e == cudaSuccess ? MAGI_BCA_OK : cuda_fail("forward launch", e);
}

size_t magi_bca_bwd_workspace_size(const magi_bca_dims* dims) {
  if (validate_dims(dims) != MAGI_BCA_OK) return 0;
  const magi_bca_dims& d = *dims;
  return bwd_workspace_layout(d.batch, d.seqlen_q, d.seqlen_kv, d.heads_q, d.heads_kv, d.head_dim).total;
}

int magi_bca_bwd(const magi_bca_bf16* q, const magi_bca_bf16* k, const magi_bca_bf16* v, const magi_bca_bf16* out,
                 const magi_bca_bf16* dout, const float* lse, const int32_t* q_chunk_offsets,
                 const int32_t* kv_chunk_offsets, const float* gamma_q, const float* gamma_k, magi_bca_bf16* dq,
                 magi_bca_bf16* dk, magi_bca_bf16* dv, float* dgamma_q, float* dgamma_k, void* workspace,
                 size_t workspace_bytes, const magi_bca_dims* dims, void* stream) {
  return magi_bca_bwd_rope(q, k, v, out, dout, lse, q_chunk_offsets, kv_chunk_offsets, gamma_q, gamma_k, nullptr,
                           nullptr, dq, dk, dv, dgamma_q, dgamma_k, nullptr, nullptr, workspace, workspace_bytes, dims,
                           stream);
}

int magi_bca_bwd_rope(const magi_bca_bf16* q, const magi_bca_bf16* k, const magi_bca_bf16* v,
                      const magi_bca_bf16* out, const magi_bca_bf16* dout, const float* lse,
                      const int32_t* q_chunk_offsets, const int32_t* kv_chunk_offsets, const float* gamma_q,
                      const float* gamma_k, const float* rope_q, const float* rope_k, magi_bca_bf16* dq,
                      magi_bca_bf16* dk, magi_bca_bf16* dv, float* dgamma_q, float* dgamma_k, float* drope_q,
                      float* drope_k, void* workspace, size_t workspace_bytes, const magi_bca_dims* dims,
                      void* stream) {
  int st = validate_dims(dims);
  if (st != MAGI_BCA_OK) return st;
  const magi_bca_dims& d = *dims;
  if (!q || !k || !v || !out || !dout || !lse || !gamma_q || !gamma_k || !dq || !dk || !dv || !workspace)
    return MAGI_BCA_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(dout) || !aligned16(dq) ||
      !aligned16(dk) || !aligned16(dv) || !aligned16(lse) || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return MAGI_BCA_INVALID_ARG;
  st = validate_offsets(q_chunk_offsets, kv_chunk_offsets, d);
  if (st != MAGI_BCA_OK) return st;
  const BwdWorkspace ws = bwd_workspace_layout(d.batch, d.seqlen_q, d.seqlen_kv, d.heads_q, d.heads_kv, d.head_dim);
  if (workspace_bytes < ws.total) return MAGI_BCA_WORKSPACE_TOO_SMALL;
  int dev;
  DeviceState* ds;
  st = device_state(&dev, &ds);
  if (st != MAGI_BCA_OK) return st;
  ScheduleEntry sched, dq_sched;
  st = get_schedule(dev, 1, d, q_chunk_offsets, kv_chunk_offsets, &sched);
  if (st != MAGI_BCA_OK) return st;
  if (d.deterministic) {   // the dq pass runs the forward's query-major units
    st = get_schedule(dev, 0, d, q_chunk_offsets, kv_chunk_offsets, &dq_sched);
    if (st != MAGI_BCA_OK) return st;
  }
  uint8_t* w = static_cast<uint8_t*>(workspace);
  BwdParams p;
  p.q = q;
  p.k = k;
  p.out = out;
  p.dout = dout;
  p.lse = lse;
  p.gamma_q = gamma_q;
  p.gamma_k = gamma_k;
  p.units = sched.dev;
  p.q_offsets = sched.dev + (size_t)sched.n_units * kUnitInts;
  p.kv_offsets = p.q_offsets + d.n_q_chunks + 1;
  p.n_q_chunks = d.n_q_chunks;
  p.n_kv_chunks = d.n_kv_chunks;
  p.kv_range = d.kv_range;
  p.rope_q = rope_q;
  p.rope_k = rope_k;
  p.drope_q = rope_q != nullptr ? drope_q : nullptr;
  p.drope_k = rope_k != nullptr ? drope_k : nullptr;
  p.deterministic = d.deterministic;
  p.dq_units = d.deterministic ? dq_sched.dev : nullptr;
  p.dgamma_part = reinterpret_cast<float*>(w + ws.dgpart);
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  p.dgamma_q = dgamma_q;
  p.dgamma_k = dgamma_k;
  p.qn = reinterpret_cast<uint16_t*>(w + ws.qn);
  p.kn = reinterpret_cast<uint16_t*>(w + ws.kn);
  p.ld = reinterpret_cast<float*>(w + ws.ld);
  p.dqacc = reinterpret_cast<float*>(w + ws.dqacc);
  p.dvacc = reinterpret_cast<float*>(w + ws.dvacc);
  p.dkacc = reinterpret_cast<float*>(w + ws.dkacc);
  p.batch = d.batch;
  p.seqlen_q = d.seqlen_q;
  p.seqlen_kv = d.seqlen_kv;
  p.heads_q = d.heads_q;
  p.heads_kv = d.heads_kv;
  p.seqlen_q_pad = (d.seqlen_q + 127) / 128 * 128;
  p.scale = resolve_scale(d);
  p.scale_log2 = p.scale * 1.4426950408889634f;
  p.eps = d.rms_eps;
  p.status = ds->status;
  CUtensorMap t_k, t_v, t_qn, t_do, t_dq, t_dv, t_dk;
  if (make_map_f32(&t_dq, p.dqacc, d.batch, d.seqlen_q, d.heads_q, d.head_dim) != MAGI_BCA_OK ||
      make_map_f32(&t_dv, p.dvacc, d.batch, d.seqlen_kv, d.heads_kv, d.head_dim) != MAGI_BCA_OK ||
      make_map_f32(&t_dk, p.dkacc, d.batch, d.seqlen_kv, d.heads_kv, d.head_dim) != MAGI_BCA_OK ||
      make_map(&t_k, p.kn, d.batch, d.seqlen_kv, d.heads_kv, d.head_dim) != MAGI_BCA_OK ||
      make_map(&t_v, v, d.batch, d.seqlen_kv, d.heads_kv, d.head_dim) != MAGI_BCA_OK ||
      make_map(&t_qn, p.qn, d.batch, d.seqlen_q, d.heads_q, d.head_dim) != MAGI_BCA_OK ||
      make_map(&t_do, dout, d.batch, d.seqlen_q, d.heads_q, d.head_dim) != MAGI_BCA_OK)
    return MAGI_BCA_CUDA_ERROR;
  cudaError_t e =
      launch_bwd(t_k, t_v, t_qn, t_do, t_dq, t_dv, t_dk, p, d.head_dim, sched.n_units,
                 d.deterministic ? dq_sched.n_units : 0, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MAGI_BCA_OK : cuda_fail("backward launch", e);
}

const char* magi_bca_last_error_detail(void) { return g_last_detail; }

int magi_bca_selftest_wait_timeout(void* stream) {
  int dev;
  DeviceState* ds;
  const int st = device_state(&dev, &ds);
  if (st != MAGI_BCA_OK) return st;
  bca_wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(ds->status, 9001, 4096u);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? MAGI_BCA_OK : cuda_fail("wait self-test launch", e);
}

int magi_bca_last_device_status(void) {
  int host = 0;
  if (cudaMemcpyFromSymbol(&host, g_device_status, sizeof(int)) != cudaSuccess) return MAGI_BCA_CUDA_ERROR;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int)) != cudaSuccess) return MAGI_BCA_CUDA_ERROR;
  return host == 0 ? MAGI_BCA_OK : MAGI_BCA_DEVICE_TIMEOUT;
}

}  // extern "C"
