// C ABI of libmagi_bca: argument checks, the schedule cache, TMA descriptors
// and kernel dispatch.  See include/magi_bca.h for the contract.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <algorithm>
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

// The library's own device memory: tile schedules (per device, shape and
// mask) and the forward's normalised-key buffers (per device and stream).
// Both are bounded: at most kScheduleCacheEntries schedules per device (least
// recently used evicted), and one key buffer per stream that grows to the
// largest shape seen.  New memory comes from cudaMallocAsync on the caller's
// stream and schedules are uploaded with cudaMemcpyAsync from pinned staging,
// so no call waits for the device.  Entries and buffers used while a stream
// was being captured are kept until magi_bca_release_caches(): a graph holds
// their addresses.
constexpr int kScheduleCacheEntries = 64;

struct ScheduleEntry {
  int32_t* dev = nullptr;  // units, then the mask blob (query offsets, lo, hi)
  size_t bytes = 0;
  int device = 0;
  int n_units = 0;
  MaskSpec mask;           // its scalars go into the kernels' MaskArgs
  uint64_t last_use = 0;   // LRU clock
  int refs = 0;            // calls between lookup and launch
  bool pinned = false;     // used under stream capture: kept until release
  // Events recorded on the caller's stream after each call's launches, so an
  // eviction can wait for the reads without touching the callers' streams
  // (which may have been destroyed since).  Completed ones are dropped as new
  // ones are added; `untracked` is set if an event could not be recorded.
  std::vector<cudaEvent_t> uses;
  bool untracked = false;
};

struct KnormBuffer {
  void* ptr = nullptr;
  size_t bytes = 0;
  bool pinned = false;     // used under stream capture
  // recorded after each forward's launches: growing the buffer frees the old
  // one only after it, even if the stream handle now names a new stream
  cudaEvent_t last_use = nullptr;
};

// Pinned staging of a schedule upload, freed once its copy has completed.
struct Staging {
  void* host;
  cudaEvent_t done;
};

std::map<int, DeviceState> g_devices;
std::map<std::vector<int32_t>, ScheduleEntry> g_schedules;
std::map<std::pair<int, uintptr_t>, KnormBuffer> g_knorm_bufs;
std::vector<void*> g_retired;     // device buffers replaced while pinned (freed on release)
std::vector<Staging> g_staging;
uint64_t g_clock = 0;

bool capturing(cudaStream_t s) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  return cudaStreamIsCapturing(s, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone;
}

// Frees the staging of uploads that have completed (caller holds g_mutex).
void reap_staging() {
  for (size_t i = 0; i < g_staging.size();) {
    if (cudaEventQuery(g_staging[i].done) == cudaSuccess) {
      cudaFreeHost(g_staging[i].host);
      cudaEventDestroy(g_staging[i].done);
      g_staging[i] = g_staging.back();
      g_staging.pop_back();
    } else {
      ++i;
    }
  }
}

// Frees a schedule's device memory in the order of `stream`, after the calls
// that read it (their events), and destroys those events (caller holds
// g_mutex, device current).
void free_schedule(ScheduleEntry& e, cudaStream_t stream) {
  bool waited = !e.untracked;
  for (cudaEvent_t ev : e.uses) {
    if (cudaStreamWaitEvent(stream, ev, 0) != cudaSuccess) waited = false;
    cudaEventDestroy(ev);
  }
  e.uses.clear();
  if (!waited) cudaDeviceSynchronize();   // a use is not covered by an event: the slow, safe way
  cudaFreeAsync(e.dev, stream);
}

int knorm_buffer(int dev, cudaStream_t stream, size_t bytes, void** out) {
  std::lock_guard<std::mutex> lock(g_mutex);
  KnormBuffer& kb = g_knorm_bufs[std::make_pair(dev, reinterpret_cast<uintptr_t>(stream))];
  const bool cap = capturing(stream);
  if (kb.ptr != nullptr && kb.bytes >= bytes) {
    kb.pinned = kb.pinned || cap;
    *out = kb.ptr;
    return MAGI_BCA_OK;
  }
  if (cap) {
    std::snprintf(g_last_detail, sizeof(g_last_detail),
                  "the first forward call for a key length must come before stream capture");
    return MAGI_BCA_UNSUPPORTED;
  }
  // grow: the old buffer is freed in this stream's order after its last use
  cudaEvent_t last_use = kb.last_use;
  if (kb.ptr != nullptr) {
    if (kb.pinned) {
      g_retired.push_back(kb.ptr);
    } else {
      if (last_use != nullptr && cudaStreamWaitEvent(stream, last_use, 0) != cudaSuccess) cudaDeviceSynchronize();
      cudaFreeAsync(kb.ptr, stream);
    }
  }
  kb = KnormBuffer();
  kb.last_use = last_use;
  void* ptr = nullptr;
  const cudaError_t e = cudaMallocAsync(&ptr, bytes, stream);
  if (e != cudaSuccess) return cuda_fail("cudaMallocAsync (normalised-key buffer)", e);
  kb.ptr = ptr;
  kb.bytes = bytes;
  *out = ptr;
  return MAGI_BCA_OK;
}

// Records the end of a forward's use of its key buffer (not under capture: a
// buffer used there is pinned and never freed before release).
void knorm_mark_use(int dev, cudaStream_t stream) {
  std::lock_guard<std::mutex> lock(g_mutex);
  auto it = g_knorm_bufs.find(std::make_pair(dev, reinterpret_cast<uintptr_t>(stream)));
  if (it == g_knorm_bufs.end() || capturing(stream)) return;
  KnormBuffer& kb = it->second;
  if (kb.last_use == nullptr && cudaEventCreateWithFlags(&kb.last_use, cudaEventDisableTiming) != cudaSuccess) {
    kb.last_use = nullptr;
    return;
  }
  cudaEventRecord(kb.last_use, stream);
}

struct KnormUse {
  int dev = 0;
  cudaStream_t stream = nullptr;
  bool held = false;
  ~KnormUse() {
    if (held) knorm_mark_use(dev, stream);
  }
};

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
  const int n_samples = d.n_samples > 1 ? d.n_samples : 1;
  std::vector<int32_t> key = {dev,        kind,         d.batch,       d.seqlen_q,  d.seqlen_kv,
                              d.heads_q,  d.heads_kv,   d.head_dim,    d.n_q_chunks, d.n_kv_chunks,
                              d.kv_range, kind == 0 ? 0 : d.deterministic, n_samples, d.n_global_chunks};
  key.insert(key.end(), qo, qo + d.n_q_chunks + 1);
  key.insert(key.end(), ko, ko + d.n_kv_chunks + 1);
  if (n_samples > 1) key.insert(key.end(), d.sample_chunk_offsets, d.sample_chunk_offsets + n_samples + 1);
  return key;
}

// Returns the cached device schedule, building and uploading it (on `stream`)
// on first use.  The entry stays referenced until release_schedule(key).
int get_schedule(int dev, int kind, const magi_bca_dims& d, const int32_t* qo, const int32_t* ko,
                 cudaStream_t stream, ScheduleEntry* out, std::vector<int32_t>* key_out) {
  std::vector<int32_t> key = schedule_key(dev, kind, d, qo, ko);
  std::lock_guard<std::mutex> lock(g_mutex);
  // under capture only lookups happen: event queries, allocations and frees
  // would invalidate the capture
  const bool cap = capturing(stream);
  if (!cap) reap_staging();
  auto it = g_schedules.find(key);
  if (it == g_schedules.end()) {
    if (cap) {
      std::snprintf(g_last_detail, sizeof(g_last_detail),
                    "the first call for a shape must come before stream capture");
      return MAGI_BCA_UNSUPPORTED;
    }
    // evict the least recently used idle entries of this device beyond the limit
    int count = 0;
    for (auto& kv : g_schedules) count += kv.second.device == dev;
    while (count >= kScheduleCacheEntries) {
      auto victim = g_schedules.end();
      for (auto v = g_schedules.begin(); v != g_schedules.end(); ++v)
        if (v->second.device == dev && v->second.refs == 0 && !v->second.pinned &&
            (victim == g_schedules.end() || v->second.last_use < victim->second.last_use))
          victim = v;
      if (victim == g_schedules.end()) break;   // everything is in use or pinned
      free_schedule(victim->second, stream);
      g_schedules.erase(victim);
      --count;
    }
    int sms = 148;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    std::vector<int32_t> units = kind == 0 ? build_fwd_schedule(qo, ko, d) : build_bwd_schedule(qo, ko, d, sms);
    ScheduleEntry e;
    e.device = dev;
    e.n_units = static_cast<int>(units.size() / (kind == 0 ? kFwdUnitInts : kUnitInts));
    e.mask = build_mask_spec(qo, ko, d);
    std::vector<int32_t> blob = units;
    append_mask_blob(blob, qo, e.mask, d.n_q_chunks);
    e.bytes = blob.size() * sizeof(int32_t);
    Staging stg{nullptr, nullptr};
    cudaError_t ce = cudaMallocHost(&stg.host, e.bytes);
    if (ce != cudaSuccess) return cuda_fail("cudaMallocHost (schedule staging)", ce);
    std::memcpy(stg.host, blob.data(), e.bytes);
    ce = cudaMallocAsync(reinterpret_cast<void**>(&e.dev), e.bytes, stream);
    if (ce == cudaSuccess) ce = cudaMemcpyAsync(e.dev, stg.host, e.bytes, cudaMemcpyHostToDevice, stream);
    if (ce == cudaSuccess) ce = cudaEventCreateWithFlags(&stg.done, cudaEventDisableTiming);
    if (ce == cudaSuccess) ce = cudaEventRecord(stg.done, stream);
    if (ce != cudaSuccess) {
      cudaStreamSynchronize(stream);
      if (e.dev != nullptr) cudaFree(e.dev);
      cudaFreeHost(stg.host);
      return cuda_fail("schedule upload", ce);
    }
    g_staging.push_back(stg);
    it = g_schedules.emplace(key, std::move(e)).first;
  }
  ScheduleEntry& e = it->second;
  e.last_use = ++g_clock;
  e.refs += 1;
  e.pinned = e.pinned || cap;
  out->dev = e.dev;
  out->n_units = e.n_units;
  out->mask = e.mask;
  *key_out = std::move(key);
  return MAGI_BCA_OK;
}

// Ends the reference get_schedule took, after the launches that use it, and
// records on `stream` the event an eviction will wait for.  Under stream
// capture the entry is pinned (never evicted), so nothing is recorded.
void release_schedule(const std::vector<int32_t>& key, cudaStream_t stream) {
  std::lock_guard<std::mutex> lock(g_mutex);
  auto it = g_schedules.find(key);
  if (it == g_schedules.end()) return;
  ScheduleEntry& e = it->second;
  if (e.refs > 0) e.refs -= 1;
  if (capturing(stream)) return;
  for (size_t i = 0; i < e.uses.size();) {
    if (cudaEventQuery(e.uses[i]) == cudaSuccess) {
      cudaEventDestroy(e.uses[i]);
      e.uses[i] = e.uses.back();
      e.uses.pop_back();
    } else {
      ++i;
    }
  }
  cudaEvent_t ev;
  if (cudaEventCreateWithFlags(&ev, cudaEventDisableTiming) != cudaSuccess) {
    e.untracked = true;
    return;
  }
  if (cudaEventRecord(ev, stream) != cudaSuccess) {
    cudaEventDestroy(ev);
    e.untracked = true;
    return;
  }
  e.uses.push_back(ev);
}

// Holds a schedule reference for the scope of an entry point.
struct ScheduleRef {
  std::vector<int32_t> key;
  cudaStream_t stream = nullptr;
  bool held = false;
  ~ScheduleRef() {
    if (held) release_schedule(key, stream);
  }
};

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
    case MAGI_BCA_DEVICE_CHECK: return "device-side bounds check failed (debug build)";
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
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  ScheduleEntry sched;
  ScheduleRef ref;
  st = get_schedule(dev, 0, d, q_chunk_offsets, kv_chunk_offsets, cs, &sched, &ref.key);
  if (st != MAGI_BCA_OK) return st;
  ref.held = true;
  ref.stream = cs;
  const int64_t kv_rows = (int64_t)d.batch * d.seqlen_kv * d.heads_kv;
  void* kn = nullptr;
  st = knorm_buffer(dev, cs, (size_t)kv_rows * d.head_dim * 2, &kn);
  if (st != MAGI_BCA_OK) return st;
  KnormUse kuse;
  kuse.dev = dev;
  kuse.stream = cs;
  kuse.held = true;
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
  p.mask = mask_args_at(sched.dev + (size_t)sched.n_units * kFwdUnitInts, sched.mask, d.n_q_chunks);
  p.rope_q = rope_q;
  p.gamma_q = gamma_q;
  p.gamma_k = gamma_k;
  p.out = out;
  p.lse = lse;
  p.batch = d.batch;
  p.seqlen_q = d.seqlen_q;
  p.seqlen_kv = d.seqlen_kv;
  p.heads_q = d.heads_q;
  p.heads_kv = d.heads_kv;
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
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  ScheduleEntry sched, dq_sched;
  ScheduleRef ref, dq_ref;
  st = get_schedule(dev, 1, d, q_chunk_offsets, kv_chunk_offsets, cs, &sched, &ref.key);
  if (st != MAGI_BCA_OK) return st;
  ref.held = true;
  ref.stream = cs;
  if (d.deterministic) {   // the dq pass runs the forward's query-major units
    st = get_schedule(dev, 0, d, q_chunk_offsets, kv_chunk_offsets, cs, &dq_sched, &dq_ref.key);
    if (st != MAGI_BCA_OK) return st;
    dq_ref.held = true;
    dq_ref.stream = cs;
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
  p.mask = mask_args_at(sched.dev + (size_t)sched.n_units * kUnitInts, sched.mask, d.n_q_chunks);
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
  cudaError_t e = launch_bwd(t_k, t_v, t_qn, t_do, t_dq, t_dv, t_dk, p, d.head_dim, sched.n_units,
                             d.deterministic ? dq_sched.n_units : 0, cs);
  return e == cudaSuccess ? MAGI_BCA_OK : cuda_fail("backward launch", e);
}

const char* magi_bca_last_error_detail(void) { return g_last_detail; }

int magi_bca_release_caches(void) {
  std::lock_guard<std::mutex> lock(g_mutex);
  int prev = -1;
  if (cudaGetDevice(&prev) != cudaSuccess) return MAGI_BCA_CUDA_ERROR;
  int status = MAGI_BCA_OK;
  // every device that holds cached memory: wait for its work, then free
  std::vector<int> devs;
  for (auto& kv : g_schedules) devs.push_back(kv.second.device);
  for (auto& kv : g_knorm_bufs) devs.push_back(kv.first.first);
  if (!g_retired.empty()) devs.push_back(prev);
  std::sort(devs.begin(), devs.end());
  devs.erase(std::unique(devs.begin(), devs.end()), devs.end());
  for (int dv : devs) {
    if (cudaSetDevice(dv) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess) status = MAGI_BCA_CUDA_ERROR;
    for (auto& kv : g_schedules) {
      if (kv.second.device != dv) continue;
      for (cudaEvent_t ev : kv.second.uses) cudaEventDestroy(ev);
      kv.second.uses.clear();
      if (cudaFree(kv.second.dev) != cudaSuccess) status = MAGI_BCA_CUDA_ERROR;
    }
    for (auto& kv : g_knorm_bufs) {
      if (kv.first.first != dv) continue;
      if (kv.second.last_use != nullptr) cudaEventDestroy(kv.second.last_use);
      if (kv.second.ptr != nullptr && cudaFree(kv.second.ptr) != cudaSuccess) status = MAGI_BCA_CUDA_ERROR;
    }
    if (dv == prev) {
      for (void* ptr : g_retired) cudaFree(ptr);
      g_retired.clear();
    }
  }
  g_schedules.clear();
  g_knorm_bufs.clear();
  cudaSetDevice(prev);
  for (Staging& stg : g_staging) {
    cudaEventSynchronize(stg.done);
    cudaFreeHost(stg.host);
    cudaEventDestroy(stg.done);
  }
  g_staging.clear();
  return status;
}

size_t magi_bca_cache_bytes(void) {
  std::lock_guard<std::mutex> lock(g_mutex);
  size_t total = 0;
  for (auto& kv : g_schedules) total += kv.second.bytes;
  for (auto& kv : g_knorm_bufs) total += kv.second.bytes;
  return total;
}

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
  if (host == 0) return MAGI_BCA_OK;
  return host >= 3000 && host < 3100 ? MAGI_BCA_DEVICE_CHECK : MAGI_BCA_DEVICE_TIMEOUT;
}

}  // extern "C"
