/*
 * magi_bca — block-causal grouped-query attention with QK-RMSNorm for
 * NVIDIA B200 (sm_100a).  Plain C ABI: device pointers, host arrays, sizes.
 *
 * The operation (MAGI-1: Autoregressive Video Generation at Scale):
 *   - A latent video is a sequence of fixed-length chunks.  A query token
 *     attends to every token of its own chunk (bidirectional) and of every
 *     earlier chunk, and never to a later chunk ("block-causal attention",
 *     MAGI-1 §2 and Figure 1; notes page §2 and Figure 1).
 *   - Query and key heads are normalised per head before the dot product
 *     ("QK normalization", MAGI-1 §2.2.2); the norm is RMSNorm with a
 *     learnable gain gamma of length head_dim:
 *         x~ = x / sqrt(mean_d x^2 + eps) * gamma.
 *   - Grouped-query attention (MAGI-1 §2.2.2; notes §3.2.2 model table):
 *     query head h reads key/value head h / (heads_q / heads_kv).
 *   - O = softmax(softmax_scale * q~ k~^T + mask) v, and
 *     lse = ln sum_j exp(softmax_scale * q~_i . k~_j) over unmasked j.
 *   - Streaming inference (MAGI-1 §2: up to four chunks denoised at once;
 *     §2.4.4: KV cache of clean chunks): the query sequence holds the LAST
 *     n_q_chunks chunks of the key/value sequence, so query chunk c is
 *     key/value chunk n_kv_chunks - n_q_chunks + c.  With n_q == n_kv this
 *     is the training layout.
 *   - Backward: FLOP convention of MAGI-1 App. B.2.1 (the backward
 *     recomputes attention; 2.5x the forward).
 *
 * Layouts (all contiguous, row-major):
 *   q, out, dout, dq : [batch, seqlen_q,  heads_q,  head_dim]  bf16
 *   k, v, dk, dv     : [batch, seqlen_kv, heads_kv, head_dim]  bf16
 *   lse              : [batch, heads_q, seqlen_q]              fp32 (natural log)
 *   gamma_q, gamma_k : [head_dim]                              fp32 (shared by all heads)
 *   dgamma_q/_k      : [head_dim]                              fp32
 *   *_chunk_offsets  : host int32 [n_chunks + 1], offsets[0] = 0, strictly
 *                      increasing, offsets[n] = seqlen; the same chunking
 *                      applies to every batch element.  Matched chunks
 *                      (query chunk c and kv chunk n_kv - n_q + c) may differ
 *                      in length: self-attention has them equal; one query
 *                      chunk against one key/value chunk of another length is
 *                      cross-attention (MAGI-1 §2.2.2, text K/V), and with
 *                      kv_range = 1 each query chunk attends only to its own
 *                      key/value chunk (chunk-wise text conditioning, MAGI-1 §7).
 *
 * Ownership: every tensor pointer is caller-owned device memory; the chunk
 * offsets are host memory read during the call.  The library's own device
 * memory is bounded: a schedule cache (per device, shape and mask; at most 64
 * entries per device, least recently used evicted; mutex-guarded) and, for the
 * forward, one normalised-key buffer per stream, grown to the largest key
 * length seen on it.  It allocates with cudaMallocAsync on the caller's stream
 * and uploads schedules with cudaMemcpyAsync from pinned staging, and frees in
 * stream order, so no call waits for the device.  Allocation happens only
 * when a new shape (or a longer key sequence on a stream) is first seen: make
 * that first call before any CUDA-graph capture of later calls; on a capturing
 * stream a call that would need new memory returns MAGI_BCA_UNSUPPORTED.
 * Schedules and buffers used under capture are kept until
 * magi_bca_release_caches(), since a graph holds their addresses.
 *
 * Errors: every entry point returns MAGI_BCA_OK (0) or a negative status.
 * No exception crosses the ABI and no call synchronises the host with the
 * device.  Faults that happen on the device surface on the stream; a device
 * wait that times out is reported by magi_bca_last_device_status().
 *
 * Streams: `stream` is a cudaStream_t (NULL = legacy default stream).  All
 * work of a call is enqueued on it.
 */
#ifndef MAGI_BCA_H_
#define MAGI_BCA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t magi_bca_bf16; /* raw bfloat16 bits */

enum {
  MAGI_BCA_OK = 0,
  MAGI_BCA_INVALID_ARG = -1,        /* null pointer, non-positive size, bad dims struct */
  MAGI_BCA_UNSUPPORTED = -2,        /* head_dim not 64/128, heads_q % heads_kv != 0, device not sm_100,
                                     * magi_bca_bwd_noalloc on a capturing stream */
  MAGI_BCA_BAD_OFFSETS = -3,        /* chunk or sample offsets violate the rules above */
  MAGI_BCA_WORKSPACE_TOO_SMALL = -4,
  MAGI_BCA_CUDA_ERROR = -5,         /* a CUDA runtime call failed (launch, copy, ...) */
  MAGI_BCA_DEVICE_TIMEOUT = -6,     /* a bounded device-side wait gave up */
  MAGI_BCA_DEVICE_CHECK = -7        /* a device-side bounds check failed (library built with
                                     * -DMAGI_BCA_DEBUG: a work unit outside the problem) */
};

typedef struct {
  int32_t batch;
  int32_t seqlen_q;     /* total query tokens per batch element */
  int32_t seqlen_kv;    /* total key/value tokens per batch element */
  int32_t heads_q;
  int32_t heads_kv;     /* heads_q % heads_kv == 0 */
  int32_t head_dim;     /* 64 or 128 */
  int32_t n_q_chunks;   /* 1 <= n_q_chunks <= n_kv_chunks */
  int32_t n_kv_chunks;
  float softmax_scale;  /* 0 selects 1/sqrt(head_dim) */
  float rms_eps;        /* RMSNorm epsilon; must be >= 0 (1e-6 is the usual value) */
  int32_t kv_range;     /* KV range in chunks (MAGI-1 §2.4.4, §2.6, Fig. 12): > 0 limits the query
                         * chunk matched to kv chunk c to kv chunks [c - kv_range + 1, c] (1 = its
                         * own chunk only); 0 = no limit (every kv chunk up to c).  Must be >= 0. */
  int32_t deterministic; /* backward only: 1 = every gradient is summed in a fixed order, so two calls
                          * with the same inputs on the same device give the same bits (dq comes from
                          * a query-major pass that owns each query tile, no dq reductions across
                          * CTAs; each kv tile is one work unit; dgamma and the angle gradients are
                          * reduced in a fixed order).  Costs about 7/5 of the tensor work of 0.
                          * 0 = fastest (fp32 reductions whose order depends on timing).  The
                          * forward is always deterministic and ignores it.  Must be 0 or 1. */
  int32_t n_samples;     /* packed samples (MAGI-1 §4.1.2, Figure 15 (f), "varlen block-causal"): 0 or 1 =
                          * the whole sequence is one sample; > 1 = sample_chunk_offsets lists the samples
                          * packed one after another, and a query sees only keys of its own sample (the
                          * sample of its matched kv chunk). */
  int32_t n_global_chunks; /* global block (MAGI-1 §4.1.2, Figure 15 (g); App. B.1, Figure 23, a last
                          * global block): the last n_global_chunks kv chunks.  Every query sees their
                          * keys, and the query chunks matched to them see every key, whatever the
                          * sample or the KV range.  0 = none; at most n_kv_chunks. */
  const int32_t* sample_chunk_offsets; /* host int32 [n_samples + 1], read during the call: cumulative kv-chunk
                          * counts of the samples, 0 = s[0] < s[1] < ... < s[n_samples] = n_kv_chunks.
                          * Ignored (may be NULL) when n_samples <= 1. */
} magi_bca_dims;

/* Forward.  Writes out (bf16) and lse (fp32; may be NULL when the caller
 * does not need it, e.g. inference).  The call is asynchronous on `stream`. */
int magi_bca_fwd(const magi_bca_bf16* q, const magi_bca_bf16* k, const magi_bca_bf16* v,
                 const int32_t* q_chunk_offsets, const int32_t* kv_chunk_offsets,
                 const float* gamma_q, const float* gamma_k,
                 magi_bca_bf16* out, float* lse,
                 const magi_bca_dims* dims, void* stream);

/* Forward with rotary position embedding on q and k before the norm
 * (MAGI-1 §2.2.2 and the notes' DiT-block sketch: learnable 3D RoPE, then
 * QK-norm).  rope_q [seqlen_q, head_dim/2] and rope_k [seqlen_kv,
 * head_dim/2] are fp32 device arrays of per-token rotation angles (radians),
 * shared by every head and batch element; feature pair (i, i + head_dim/2) of
 * token s rotates by angle[s][i]: y_i = x_i cos - x_{i+D/2} sin,
 * y_{i+D/2} = x_{i+D/2} cos + x_i sin.  The 3D split (time, height, width)
 * and the learnable frequencies live in the caller, which computes the
 * angles.  Either table may be NULL (no rotation of that side).  Otherwise
 * as magi_bca_fwd (which is this call with both tables NULL). */
int magi_bca_fwd_rope(const magi_bca_bf16* q, const magi_bca_bf16* k, const magi_bca_bf16* v,
                      const int32_t* q_chunk_offsets, const int32_t* kv_chunk_offsets,
                      const float* gamma_q, const float* gamma_k,
                      const float* rope_q, const float* rope_k,
                      magi_bca_bf16* out, float* lse,
                      const magi_bca_dims* dims, void* stream);

/* Bytes of device workspace magi_bca_bwd / magi_bca_bwd_rope need for `dims`
 * (either value of dims->deterministic); 0 if dims is NULL or invalid. */
size_t magi_bca_bwd_workspace_size(const magi_bca_dims* dims);

/* Backward of the training layout (any layout the forward accepts works).
 * Inputs: q, k, v, the forward's out and lse, and dout.  Outputs: dq, dk (the
 * gradients with respect to the RAW, un-normalised q and k, because the
 * RMSNorm is part of the operation), dv, and optionally dgamma_q / dgamma_k
 * (NULL to skip).  `workspace` is caller-owned device memory of at least
 * magi_bca_bwd_workspace_size(dims) bytes, 256-byte aligned; its contents on
 * entry do not matter. */
int magi_bca_bwd(const magi_bca_bf16* q, const magi_bca_bf16* k, const magi_bca_bf16* v,
                 const magi_bca_bf16* out, const magi_bca_bf16* dout, const float* lse,
                 const int32_t* q_chunk_offsets, const int32_t* kv_chunk_offsets,
                 const float* gamma_q, const float* gamma_k,
                 magi_bca_bf16* dq, magi_bca_bf16* dk, magi_bca_bf16* dv,
                 float* dgamma_q, float* dgamma_k,
                 void* workspace, size_t workspace_bytes,
                 const magi_bca_dims* dims, void* stream);

/* Backward that allocates nothing.  Same arguments and results as
 * magi_bca_bwd, without the workspace: the workspace and the tile schedule live
 * in a 96 MiB array that the library keeps in every GPU's memory from load
 * until exit.  It is for callers that cannot allocate or pass device memory,
 * e.g. processes whose GPU memory is owned up front by a pooled allocator,
 * plugin hooks that must not allocate, or loops that cannot take
 * cudaMalloc's implicit synchronisation.  (The paper has no counterpart; this
 * is a deployment variant.)
 *   - Problems needing more than the array (workspace + schedule) return
 *     MAGI_BCA_WORKSPACE_TOO_SMALL; e.g. 4 chunks x 1024 tokens, 16 query heads,
 *     head_dim 128 fits.
 *   - The first call on a device looks up the array's device address; make that
 *     first call before any stream capture.
 *   - Every call copies its tile schedule from host memory into the array, so
 *     while `stream` is capturing the call returns MAGI_BCA_UNSUPPORTED and
 *     enqueues nothing.
 *   - All calls share the array and it keeps the last call's contents, so calls
 *     that overlap on the GPU (several streams or threads) race.  Run them in
 *     one stream, one at a time. */
int magi_bca_bwd_noalloc(const magi_bca_bf16* q, const magi_bca_bf16* k, const magi_bca_bf16* v,
                         const magi_bca_bf16* out, const magi_bca_bf16* dout, const float* lse,
                         const int32_t* q_chunk_offsets, const int32_t* kv_chunk_offsets,
                         const float* gamma_q, const float* gamma_k,
                         magi_bca_bf16* dq, magi_bca_bf16* dk, magi_bca_bf16* dv,
                         float* dgamma_q, float* dgamma_k,
                         const magi_bca_dims* dims, void* stream);

/* Frees every schedule and buffer the library holds (the paper has no
 * counterpart; memory management of this library).  Synchronises each device
 * that holds any (the one call that does), so no launched kernel is still
 * reading them; CUDA graphs captured earlier that used them must not be
 * replayed afterwards.  Returns MAGI_BCA_OK or MAGI_BCA_CUDA_ERROR. */
int magi_bca_release_caches(void);

/* Bytes of device memory the library holds in its caches (schedules and
 * normalised-key buffers, all devices); host-only, no synchronisation. */
size_t magi_bca_cache_bytes(void);

/* Static text for a status code. */
const char* magi_bca_status_string(int status);

/* Text describing the most recent MAGI_BCA_CUDA_ERROR on the calling thread
 * (which CUDA call failed and its error string); "" if none.  Owned by the
 * library, valid until the thread's next failing call. */
const char* magi_bca_last_error_detail(void);

/* Backward of magi_bca_fwd_rope.  dq and dk are gradients with respect to
 * the raw (pre-rotation, pre-norm) q and k.  drope_q [seqlen_q, head_dim/2]
 * and drope_k [seqlen_kv, head_dim/2] (fp32, nullable; ignored where the
 * matching angle table is NULL) receive the angle gradients summed over
 * batch and heads, so the caller can continue into its learnable
 * frequencies.  Otherwise as magi_bca_bwd (this call with NULL tables). */
int magi_bca_bwd_rope(const magi_bca_bf16* q, const magi_bca_bf16* k, const magi_bca_bf16* v,
                      const magi_bca_bf16* out, const magi_bca_bf16* dout, const float* lse,
                      const int32_t* q_chunk_offsets, const int32_t* kv_chunk_offsets,
                      const float* gamma_q, const float* gamma_k,
                      const float* rope_q, const float* rope_k,
                      magi_bca_bf16* dq, magi_bca_bf16* dk, magi_bca_bf16* dv,
                      float* dgamma_q, float* dgamma_k, float* drope_q, float* drope_k,
                      void* workspace, size_t workspace_bytes,
                      const magi_bca_dims* dims, void* stream);

/* Reads (and clears) the device status word that bounded waits write when
 * they give up (and, in a -DMAGI_BCA_DEBUG build, the kernels' bounds checks).
 * Synchronises with the device; returns MAGI_BCA_OK, MAGI_BCA_DEVICE_TIMEOUT or
 * MAGI_BCA_DEVICE_CHECK (or MAGI_BCA_CUDA_ERROR if the read itself fails).
 * Meant for tests and diagnostics, not for the hot path. */
int magi_bca_last_device_status(void);

/* Diagnostic timing hook (the paper has no counterpart).  `event_begin` and
 * `event_end` are cudaEvent_t handles created by the caller.  While both are
 * non-NULL, every magi_bca_fwd / magi_bca_bwd / magi_bca_bwd_noalloc call
 * records event_begin on its stream immediately before launching its main
 * kernel (bca_fwd_kernel or bca_bwd_main_kernel; with dims->deterministic the
 * backward's dq and dK/dV passes together) and event_end immediately after, so
 * the caller can time that work alone with cudaEventElapsedTime.
 * Pass NULL, NULL to stop.  Process-wide setting; not for concurrent calls on
 * several streams.  Returns MAGI_BCA_OK, or MAGI_BCA_INVALID_ARG if exactly
 * one handle is NULL. */
int magi_bca_profile_events(void* event_begin, void* event_end);

/* Self-test of the device-timeout path (diagnostic; the paper has no
 * counterpart).  Launches one small kernel on `stream` whose bounded wait, on
 * an mbarrier that nothing arrives at, gives up after a short poll limit and
 * records a device status code, as a stalled pipeline stage in the attention
 * kernels would.  A following magi_bca_last_device_status() returns
 * MAGI_BCA_DEVICE_TIMEOUT (and clears the word); the CUDA context stays
 * usable.  Returns MAGI_BCA_OK, MAGI_BCA_UNSUPPORTED (device) or
 * MAGI_BCA_CUDA_ERROR (launch failure). */
int magi_bca_selftest_wait_timeout(void* stream);

/* Host-only view of the tile schedule the kernels run (no device needed).
 * A work unit is up to two 128-row query tiles ("sub-tiles") that read the
 * same key/value head and visit the same kv tiles, so every K/V tile the
 * unit loads into shared memory serves both.  For every unit the scheduler
 * emits 12 int32 values:
 *   {batch, kv_head, head_0, m0_0, head_1, m0_1, n_full, n_tiles,
 *    t_begin, t_full_begin, g_begin, g_end}
 * where (head_s, m0_s) is sub-tile s's query head and first query row
 * (head_1 = -1 when the unit has one sub-tile); kv tiles [t_begin, n_tiles)
 * are visited (t_begin > 0 under a KV range or packed samples) and tiles below
 * t_full_begin or from n_full on need the per-row mask; then, with a global
 * block, the tiles [g_begin, g_end) of its keys that the first range does not
 * hold (g_begin = g_end = 0 otherwise; masked only where they straddle the
 * block's start or the sequence's end).  Units are listed in launch order:
 * longest first.  The deterministic backward's query-major dq
 * pass runs the same units, one CTA per sub-tile.
 * Returns the number of units (even if larger than `capacity`, in which case
 * only `capacity` units are written), or a negative status. */
int64_t magi_bca_fwd_schedule(const int32_t* q_chunk_offsets, const int32_t* kv_chunk_offsets,
                              const magi_bca_dims* dims, int32_t* units, int64_t capacity);

/* Host-only view of the backward schedule (no device needed).  A unit is one
 * 128-key tile of one (batch, kv head) and a contiguous range of its "steps":
 * a step is one (query tile qt, query head g of the kv head's group) that sees
 * the tile, numbered qt * G + g with G = heads_q / heads_kv.  Each tile's steps
 * are cut into near-equal pieces whose length is chosen by simulating how
 * `num_sms` SMs would run them (with dims->deterministic = 1 every tile is
 * one unit).  Per unit 12 int32:
 *   {batch, kv_head, n0 (first key), step_begin, step_end,
 *    diag_end, diag_hi_begin, split, jump, diag_global, 0, 0}
 * A unit runs steps v in [step_begin, step_end); step v is the absolute step
 * v (query tile v / G) below `split` and v + jump from `split` on, so with a
 * global block a kv tile's steps can be two runs of query tiles: the rows that
 * see its keys by the block-causal rule, then the global block's query rows
 * (split = INT32_MAX, jump = 0 when there is one run).  Query tiles of the
 * first run below diag_end or from diag_hi_begin on (KV range, packed samples)
 * need the mask; in the second run only query tile diag_global does (-1:
 * none).  Units are in launch order (longest first).  Returns the number of
 * units (writing at most `capacity`), or a negative status. */
int64_t magi_bca_bwd_schedule(const int32_t* q_chunk_offsets, const int32_t* kv_chunk_offsets,
                              const magi_bca_dims* dims, int32_t num_sms, int32_t* units, int64_t capacity);

/* Library version string. */
const char* magi_bca_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MAGI_BCA_H_ */
