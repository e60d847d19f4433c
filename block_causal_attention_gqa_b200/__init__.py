"""Block-causal grouped-query attention with QK-RMSNorm on B200 (sm_100a).

Thin ctypes binding over ``libmagi_bca.so`` (C ABI in ``include/magi_bca.h``).
This module only marshals arguments: PyTorch provides device memory and the
current stream; every step of the computation runs in the library's CUDA
kernels.  There is no CPU or PyTorch fallback: if the library is missing or
the device is not an sm_100 GPU, the calls raise.

The operation (MAGI-1: Autoregressive Video Generation at Scale, §2 and
Figure 1; §2.2.2): every query token attends to all tokens of its own chunk
and of every earlier chunk; q and k are RMS-normalised per head with gains
gamma_q / gamma_k; query head h reads kv head h // (Hq // Hkv).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence, Tuple

import numpy as np

__all__ = ["magi_bca_fwd", "magi_bca_bwd", "magi_bca_fwd_rope", "magi_bca_bwd_rope", "magi_bca_bwd_noalloc",
           "magi_bca_bwd_workspace_size", "magi_bca_fwd_schedule", "magi_bca_release_caches", "magi_bca_cache_bytes",
           "magi_bca_status_string", "magi_bca_last_device_status", "magi_bca_profile_events", "MagiBcaError",
           "Dims", "library",
           "library_path", "EXPORTED_SYMBOLS"]

_HERE = os.path.dirname(os.path.abspath(__file__))
# MAGI_BCA_LIBRARY selects another build of the library (e.g. the bounds-checked
# libmagi_bca_debug.so from `build.py --debug`); the default is the in-tree build.
library_path = os.environ.get("MAGI_BCA_LIBRARY") or os.path.join(_HERE, "libmagi_bca.so")

EXPORTED_SYMBOLS = ["magi_bca_fwd", "magi_bca_bwd", "magi_bca_bwd_workspace_size", "magi_bca_status_string",
                    "magi_bca_last_device_status", "magi_bca_fwd_schedule", "magi_bca_version",
                    "magi_bca_bwd_noalloc", "magi_bca_last_error_detail", "magi_bca_bwd_schedule",
                    "magi_bca_profile_events", "magi_bca_fwd_rope", "magi_bca_bwd_rope",
                    "magi_bca_selftest_wait_timeout", "magi_bca_release_caches", "magi_bca_cache_bytes"]


class MagiBcaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        detail = ""
        if status == -5:
            detail = "; " + library().magi_bca_last_error_detail().decode()
        super().__init__(f"{where} failed: status {status} ({magi_bca_status_string(status)}{detail})")


class Dims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("seqlen_q", ctypes.c_int32), ("seqlen_kv", ctypes.c_int32),
                ("heads_q", ctypes.c_int32), ("heads_kv", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("n_q_chunks", ctypes.c_int32), ("n_kv_chunks", ctypes.c_int32),
                ("softmax_scale", ctypes.c_float), ("rms_eps", ctypes.c_float), ("kv_range", ctypes.c_int32),
                ("deterministic", ctypes.c_int32), ("n_samples", ctypes.c_int32), ("n_global_chunks", ctypes.c_int32),
                ("sample_chunk_offsets", ctypes.POINTER(ctypes.c_int32))]


_lib = None


def library() -> ctypes.CDLL:
    """Loads libmagi_bca.so (built in-tree by ``build.py``); raises if absent."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(library_path):
        raise RuntimeError(f"{library_path} is missing: build it with "
                           "`python -m block_causal_attention_gqa_b200.build` (no fallback exists)")
    lib = ctypes.CDLL(library_path)
    vp, i32p, f32p = ctypes.c_void_p, ctypes.POINTER(ctypes.c_int32), ctypes.c_void_p
    dp = ctypes.POINTER(Dims)
    lib.magi_bca_fwd.argtypes = [vp, vp, vp, i32p, i32p, f32p, f32p, vp, f32p, dp, vp]
    lib.magi_bca_fwd.restype = ctypes.c_int
    lib.magi_bca_bwd.argtypes = [vp, vp, vp, vp, vp, f32p, i32p, i32p, f32p, f32p, vp, vp, vp, f32p, f32p, vp,
                                 ctypes.c_size_t, dp, vp]
    lib.magi_bca_bwd.restype = ctypes.c_int
    lib.magi_bca_bwd_noalloc.argtypes = [vp, vp, vp, vp, vp, f32p, i32p, i32p, f32p, f32p, vp, vp, vp, f32p, f32p,
                                         dp, vp]
    lib.magi_bca_bwd_noalloc.restype = ctypes.c_int
    lib.magi_bca_bwd_workspace_size.argtypes = [dp]
    lib.magi_bca_bwd_workspace_size.restype = ctypes.c_size_t
    lib.magi_bca_status_string.argtypes = [ctypes.c_int]
    lib.magi_bca_status_string.restype = ctypes.c_char_p
    lib.magi_bca_last_device_status.argtypes = []
    lib.magi_bca_last_device_status.restype = ctypes.c_int
    lib.magi_bca_fwd_schedule.argtypes = [i32p, i32p, dp, i32p, ctypes.c_int64]
    lib.magi_bca_fwd_schedule.restype = ctypes.c_int64
    lib.magi_bca_last_error_detail.argtypes = []
    lib.magi_bca_last_error_detail.restype = ctypes.c_char_p
    lib.magi_bca_bwd_schedule.argtypes = [i32p, i32p, dp, ctypes.c_int32, i32p, ctypes.c_int64]
    lib.magi_bca_bwd_schedule.restype = ctypes.c_int64
    lib.magi_bca_version.argtypes = []
    lib.magi_bca_version.restype = ctypes.c_char_p
    lib.magi_bca_fwd_rope.argtypes = [vp, vp, vp, i32p, i32p, f32p, f32p, vp, vp, vp, f32p, dp, vp]
    lib.magi_bca_fwd_rope.restype = ctypes.c_int
    lib.magi_bca_bwd_rope.argtypes = [vp, vp, vp, vp, vp, f32p, i32p, i32p, f32p, f32p, vp, vp, vp, vp, vp, f32p,
                                      f32p, vp, vp, vp, ctypes.c_size_t, dp, vp]
    lib.magi_bca_bwd_rope.restype = ctypes.c_int
    lib.magi_bca_profile_events.argtypes = [vp, vp]
    lib.magi_bca_profile_events.restype = ctypes.c_int
    lib.magi_bca_selftest_wait_timeout.argtypes = [vp]
    lib.magi_bca_selftest_wait_timeout.restype = ctypes.c_int
    lib.magi_bca_release_caches.argtypes = []
    lib.magi_bca_release_caches.restype = ctypes.c_int
    lib.magi_bca_cache_bytes.argtypes = []
    lib.magi_bca_cache_bytes.restype = ctypes.c_size_t
    _lib = lib
    return lib


def magi_bca_release_caches() -> None:
    """Frees the library's cached schedules and key buffers (synchronises the
    devices that hold any)."""
    st = library().magi_bca_release_caches()
    if st != 0:
        raise MagiBcaError(st, "magi_bca_release_caches")


def magi_bca_cache_bytes() -> int:
    """Device bytes held by the library's caches."""
    return int(library().magi_bca_cache_bytes())


def magi_bca_status_string(status: int) -> str:
    return library().magi_bca_status_string(int(status)).decode()


def magi_bca_last_device_status() -> int:
    return int(library().magi_bca_last_device_status())


def magi_bca_selftest_wait_timeout(stream=None) -> None:
    """Diagnostic: one kernel whose bounded wait on an mbarrier that nothing
    arrives at gives up; magi_bca_last_device_status() then reports the
    device timeout (-6) without any fault."""
    import torch
    dev = torch.device("cuda", torch.cuda.current_device())
    st = library().magi_bca_selftest_wait_timeout(_stream_handle(stream, dev))
    if st != 0:
        raise MagiBcaError(st, "magi_bca_selftest_wait_timeout")


def magi_bca_profile_events(begin=None, end=None) -> None:
    """Diagnostic: while set, each forward/backward call records the two
    events (torch.cuda.Event with timing enabled, or raw cudaEvent_t handles)
    around its main kernel's launch.  ``magi_bca_profile_events()`` clears."""
    def handle(ev):
        if ev is None:
            return None
        if hasattr(ev, "cuda_event"):
            if ev.cuda_event == 0:   # torch creates the CUDA event on its first record
                ev.record()
            return ev.cuda_event
        return int(ev)
    st = library().magi_bca_profile_events(handle(begin), handle(end))
    if st != 0:
        raise MagiBcaError(st, "magi_bca_profile_events")


def _offsets(x) -> np.ndarray:
    if hasattr(x, "detach"):
        x = x.detach().cpu().numpy()
    a = np.ascontiguousarray(np.asarray(x, dtype=np.int32))
    if a.ndim != 1:
        raise ValueError("chunk offsets must be a 1-D array")
    return a


def _i32p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))


def make_dims(batch, seqlen_q, seqlen_kv, heads_q, heads_kv, head_dim, n_q_chunks, n_kv_chunks,
              softmax_scale=0.0, rms_eps=1e-6, kv_range=0, deterministic=False, samples=None,
              n_global=0) -> Dims:
    """The dims struct.  samples: cumulative kv-chunk counts [0, ..., n_kv_chunks]
    of packed samples (None: one sample); n_global: the last n_global kv chunks
    form a global block.  The struct keeps a reference to the samples array it
    points at."""
    d = Dims(batch, seqlen_q, seqlen_kv, heads_q, heads_kv, head_dim, n_q_chunks, n_kv_chunks,
             float(softmax_scale), float(rms_eps), int(kv_range), int(bool(deterministic)), 0, int(n_global), None)
    if samples is not None:
        so = _offsets(samples)
        d.n_samples = len(so) - 1
        d.sample_chunk_offsets = _i32p(so)
        d.keep_samples = so
    return d


def _check_bf16(name, t, shape=None):
    import torch
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != torch.bfloat16:
        raise TypeError(f"{name} must be bfloat16 (got {t.dtype})")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _check_f32(name, t, shape):
    import torch
    if not isinstance(t, torch.Tensor) or not t.is_cuda or t.dtype != torch.float32 or not t.is_contiguous():
        raise TypeError(f"{name} must be a contiguous float32 CUDA tensor")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _check_same_device(device, named):
    """Every tensor of a call must live on the device the call runs on: the
    kernels dereference each pointer there."""
    for name, t in named:
        if t is not None and t.device != device:
            raise ValueError(f"{name} is on {t.device}, the call runs on {device}")


def _stream_handle(stream, device):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def _fwd(q, k, v, q_chunk_offsets, kv_chunk_offsets, gamma_q, gamma_k, out, lse, softmax_scale, rms_eps, stream,
         want_lse, kv_range, rope=None, samples=None, n_global=0):
    import torch
    _check_bf16("q", q)
    B, Sq, Hq, D = q.shape
    _check_bf16("k", k)                     # a CUDA bf16 tensor before its shape is read
    Skv, Hkv = k.shape[1], k.shape[2]
    _check_bf16("k", k, (B, Skv, Hkv, D))
    _check_bf16("v", v, (B, Skv, Hkv, D))
    _check_f32("gamma_q", gamma_q, (D,))
    _check_f32("gamma_k", gamma_k, (D,))
    qo, ko = _offsets(q_chunk_offsets), _offsets(kv_chunk_offsets)
    if out is None:
        out = torch.empty_like(q)
    _check_bf16("out", out, q.shape)
    if lse is None and want_lse:
        lse = torch.empty(B, Hq, Sq, device=q.device, dtype=torch.float32)
    if lse is not None:
        _check_f32("lse", lse, (B, Hq, Sq))
    _check_same_device(q.device, (("k", k), ("v", v), ("gamma_q", gamma_q), ("gamma_k", gamma_k), ("out", out),
                                  ("lse", lse)) + ((("rope_q", rope[0]), ("rope_k", rope[1])) if rope else ()))
    dims = make_dims(B, Sq, Skv, Hq, Hkv, D, len(qo) - 1, len(ko) - 1, softmax_scale, rms_eps, kv_range,
                     samples=samples, n_global=n_global)
    ptr = lambda t: t.data_ptr() if t is not None else None
    with torch.cuda.device(q.device):
        if rope is None:
            st = library().magi_bca_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), _i32p(qo), _i32p(ko),
                                        gamma_q.data_ptr(), gamma_k.data_ptr(), out.data_ptr(), ptr(lse),
                                        ctypes.byref(dims), _stream_handle(stream, q.device))
        else:
            rq, rk = rope
            if rq is not None:
                _check_f32("rope_q", rq, (Sq, D // 2))
            if rk is not None:
                _check_f32("rope_k", rk, (Skv, D // 2))
            st = library().magi_bca_fwd_rope(q.data_ptr(), k.data_ptr(), v.data_ptr(), _i32p(qo), _i32p(ko),
                                             gamma_q.data_ptr(), gamma_k.data_ptr(), ptr(rq), ptr(rk),
                                             out.data_ptr(), ptr(lse), ctypes.byref(dims),
                                             _stream_handle(stream, q.device))
    if st != 0:
        raise MagiBcaError(st, "magi_bca_fwd" if rope is None else "magi_bca_fwd_rope")
    return out, lse


def magi_bca_fwd(q, k, v, q_chunk_offsets, kv_chunk_offsets, gamma_q, gamma_k, out=None, lse=None,
                 softmax_scale: float = 0.0, rms_eps: float = 1e-6, stream=None, want_lse: bool = True,
                 kv_range: int = 0, samples=None, n_global: int = 0):
    """Forward.  q [B,Sq,Hq,D], k/v [B,Skv,Hkv,D] bf16; gammas fp32 [D];
    offsets: host int arrays of chunk boundaries; samples: kv-chunk offsets of
    packed samples (None: one); n_global: trailing kv chunks that form a global
    block.  Returns (out, lse)."""
    return _fwd(q, k, v, q_chunk_offsets, kv_chunk_offsets, gamma_q, gamma_k, out, lse, softmax_scale, rms_eps,
                stream, want_lse, kv_range, samples=samples, n_global=n_global)


def magi_bca_fwd_rope(q, k, v, q_chunk_offsets, kv_chunk_offsets, gamma_q, gamma_k, rope_q, rope_k, out=None,
                      lse=None, softmax_scale: float = 0.0, rms_eps: float = 1e-6, stream=None,
                      want_lse: bool = True, kv_range: int = 0, samples=None, n_global: int = 0):
    """Forward with rotary angles (fp32 [Sq, D/2] / [Skv, D/2] per token, or
    None) applied to q and k before the norm.  Returns (out, lse)."""
    return _fwd(q, k, v, q_chunk_offsets, kv_chunk_offsets, gamma_q, gamma_k, out, lse, softmax_scale, rms_eps,
                stream, want_lse, kv_range, rope=(rope_q, rope_k), samples=samples, n_global=n_global)


def magi_bca_bwd_workspace_size(dims: Dims) -> int:
    return int(library().magi_bca_bwd_workspace_size(ctypes.byref(dims)))


def _bwd(q, k, v, out, dout, lse, q_chunk_offsets, kv_chunk_offsets, gamma_q, gamma_k, dq, dk, dv, dgamma_q,
         dgamma_k, want_dgamma, workspace, softmax_scale, rms_eps, stream, kv_range, rope=None,
         deterministic=False, samples=None, n_global=0):
    """Shared marshalling of magi_bca_bwd and (rope = (rope_q, rope_k, drope_q,
    drope_k)) magi_bca_bwd_rope."""
    import torch
    _check_bf16("q", q)
    B, Sq, Hq, D = q.shape
    Skv, Hkv = k.shape[1], k.shape[2]
    _check_bf16("k", k, (B, Skv, Hkv, D))
    _check_bf16("v", v, (B, Skv, Hkv, D))
    _check_bf16("out", out, q.shape)
    _check_bf16("dout", dout, q.shape)
    _check_f32("lse", lse, (B, Hq, Sq))
    _check_f32("gamma_q", gamma_q, (D,))
    _check_f32("gamma_k", gamma_k, (D,))
    qo, ko = _offsets(q_chunk_offsets), _offsets(kv_chunk_offsets)
    dims = make_dims(B, Sq, Skv, Hq, Hkv, D, len(qo) - 1, len(ko) - 1, softmax_scale, rms_eps, kv_range,
                     deterministic, samples=samples, n_global=n_global)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _check_bf16("dq", dq, q.shape)
    _check_bf16("dk", dk, k.shape)
    _check_bf16("dv", dv, v.shape)
    if want_dgamma:
        dgamma_q = torch.empty(D, device=q.device, dtype=torch.float32) if dgamma_q is None else dgamma_q
        dgamma_k = torch.empty(D, device=q.device, dtype=torch.float32) if dgamma_k is None else dgamma_k
    for nm, t in (("dgamma_q", dgamma_q), ("dgamma_k", dgamma_k)):
        if t is not None:
            _check_f32(nm, t, (D,))
    ws_bytes = magi_bca_bwd_workspace_size(dims)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 1), device=q.device, dtype=torch.uint8)
    elif not isinstance(workspace, torch.Tensor) or not workspace.is_cuda or not workspace.is_contiguous():
        raise TypeError("workspace must be a contiguous CUDA tensor")
    _check_same_device(q.device, (("k", k), ("v", v), ("out", out), ("dout", dout), ("lse", lse),
                                  ("gamma_q", gamma_q), ("gamma_k", gamma_k), ("dq", dq), ("dk", dk), ("dv", dv),
                                  ("dgamma_q", dgamma_q), ("dgamma_k", dgamma_k), ("workspace", workspace))
                       + tuple(zip(("rope_q", "rope_k", "drope_q", "drope_k"), rope or ())))
    ptr = lambda t: t.data_ptr() if t is not None else None
    common = (q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), dout.data_ptr(), lse.data_ptr(),
              _i32p(qo), _i32p(ko), gamma_q.data_ptr(), gamma_k.data_ptr())
    tail = (workspace.data_ptr(), workspace.numel() * workspace.element_size(), ctypes.byref(dims),
            _stream_handle(stream, q.device))
    with torch.cuda.device(q.device):
        if rope is None:
            st = library().magi_bca_bwd(*common, dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), ptr(dgamma_q),
                                        ptr(dgamma_k), *tail)
        else:
            rq, rk, drq, drk = rope
            st = library().magi_bca_bwd_rope(*common, ptr(rq), ptr(rk), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                                             ptr(dgamma_q), ptr(dgamma_k), ptr(drq), ptr(drk), *tail)
    if st != 0:
        raise MagiBcaError(st, "magi_bca_bwd" if rope is None else "magi_bca_bwd_rope")
    return dq, dk, dv, dgamma_q, dgamma_k


def magi_bca_bwd(q, k, v, out, dout, lse, q_chunk_offsets, kv_chunk_offsets, gamma_q, gamma_k,
                 dq=None, dk=None, dv=None, dgamma_q=None, dgamma_k=None, want_dgamma: bool = True,
                 workspace=None, softmax_scale: float = 0.0, rms_eps: float = 1e-6, stream=None,
                 kv_range: int = 0, deterministic: bool = False, samples=None, n_global: int = 0):
    """Backward.  Returns (dq, dk, dv, dgamma_q, dgamma_k); dq/dk are with
    respect to the raw (pre-norm) q and k.  deterministic=True sums every
    gradient in a fixed order (same bits on every call; more tensor work)."""
    return _bwd(q, k, v, out, dout, lse, q_chunk_offsets, kv_chunk_offsets, gamma_q, gamma_k, dq, dk, dv,
                dgamma_q, dgamma_k, want_dgamma, workspace, softmax_scale, rms_eps, stream, kv_range,
                deterministic=deterministic, samples=samples, n_global=n_global)


def magi_bca_bwd_rope(q, k, v, out, dout, lse, q_chunk_offsets, kv_chunk_offsets, gamma_q, gamma_k,
                      rope_q, rope_k, dq=None, dk=None, dv=None, dgamma_q=None, dgamma_k=None,
                      want_dgamma: bool = True, want_drope: bool = True, workspace=None,
                      softmax_scale: float = 0.0, rms_eps: float = 1e-6, stream=None, kv_range: int = 0,
                      deterministic: bool = False, samples=None, n_global: int = 0):
    """Backward of magi_bca_fwd_rope.  Returns (dq, dk, dv, dgamma_q, dgamma_k,
    drope_q, drope_k); dq/dk are with respect to the raw (pre-rotation,
    pre-norm) q and k; drope_* (fp32 [seqlen, D/2], summed over batch and
    heads) are None where the angle table is None or want_drope is False."""
    import torch
    D = q.shape[3]
    drq = drk = None
    if rope_q is not None:
        _check_f32("rope_q", rope_q, (q.shape[1], D // 2))
        if want_drope:
            drq = torch.empty_like(rope_q)
    if rope_k is not None:
        _check_f32("rope_k", rope_k, (k.shape[1], D // 2))
        if want_drope:
            drk = torch.empty_like(rope_k)
    res = _bwd(q, k, v, out, dout, lse, q_chunk_offsets, kv_chunk_offsets, gamma_q, gamma_k, dq, dk, dv,
               dgamma_q, dgamma_k, want_dgamma, workspace, softmax_scale, rms_eps, stream, kv_range,
               rope=(rope_q, rope_k, drq, drk), deterministic=deterministic, samples=samples, n_global=n_global)
    return res + (drq, drk)


def magi_bca_bwd_noalloc(q, k, v, out, dout, lse, q_chunk_offsets, kv_chunk_offsets, gamma_q, gamma_k,
                         dq, dk, dv, dgamma_q=None, dgamma_k=None, softmax_scale: float = 0.0,
                         rms_eps: float = 1e-6, stream=None, kv_range: int = 0, deterministic: bool = False,
                         samples=None, n_global: int = 0):
    """Backward through the allocation-free entry point.

    For callers that cannot allocate device memory or hand the library a
    workspace (a pooled allocator owns the GPU's memory, a plugin hook must
    not allocate, or cudaMalloc's implicit synchronisation is unaffordable).
    Every output is passed in by the caller; the library uses its own 96 MiB
    device array as workspace, so calls must not overlap on the GPU.  Problems
    too large for that array raise MagiBcaError (status -4)."""
    _check_bf16("q", q)
    B, Sq, Hq, D = q.shape
    Skv, Hkv = k.shape[1], k.shape[2]
    for nm, t, shp in (("k", k, (B, Skv, Hkv, D)), ("v", v, (B, Skv, Hkv, D)), ("out", out, q.shape),
                       ("dout", dout, q.shape), ("dq", dq, q.shape), ("dk", dk, k.shape), ("dv", dv, v.shape)):
        _check_bf16(nm, t, shp)
    _check_f32("lse", lse, (B, Hq, Sq))
    _check_f32("gamma_q", gamma_q, (D,))
    _check_f32("gamma_k", gamma_k, (D,))
    for nm, t in (("dgamma_q", dgamma_q), ("dgamma_k", dgamma_k)):
        if t is not None:
            _check_f32(nm, t, (D,))
    _check_same_device(q.device, (("k", k), ("v", v), ("out", out), ("dout", dout), ("lse", lse),
                                  ("gamma_q", gamma_q), ("gamma_k", gamma_k), ("dq", dq), ("dk", dk), ("dv", dv),
                                  ("dgamma_q", dgamma_q), ("dgamma_k", dgamma_k)))
    qo, ko = _offsets(q_chunk_offsets), _offsets(kv_chunk_offsets)
    dims = make_dims(B, Sq, Skv, Hq, Hkv, D, len(qo) - 1, len(ko) - 1, softmax_scale, rms_eps, kv_range,
                     deterministic, samples=samples, n_global=n_global)
    import torch
    with torch.cuda.device(q.device):
        st = library().magi_bca_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                            dout.data_ptr(), lse.data_ptr(), _i32p(qo), _i32p(ko),
                                            gamma_q.data_ptr(), gamma_k.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                                            dv.data_ptr(), dgamma_q.data_ptr() if dgamma_q is not None else None,
                                            dgamma_k.data_ptr() if dgamma_k is not None else None,
                                            ctypes.byref(dims), _stream_handle(stream, q.device))
    if st != 0:
        raise MagiBcaError(st, "magi_bca_bwd_noalloc")
    return dq, dk, dv, dgamma_q, dgamma_k


def magi_bca_fwd_schedule(q_chunk_offsets, kv_chunk_offsets, batch, heads_q, heads_kv, head_dim,
                          kv_range=0, samples=None, n_global=0) -> np.ndarray:
    """Host-only: the forward's work units as an int32 array [n_units, 12]."""
    qo, ko = _offsets(q_chunk_offsets), _offsets(kv_chunk_offsets)
    dims = make_dims(batch, int(qo[-1]), int(ko[-1]), heads_q, heads_kv, head_dim, len(qo) - 1, len(ko) - 1,
                     kv_range=kv_range, samples=samples, n_global=n_global)
    lib = library()
    n = lib.magi_bca_fwd_schedule(_i32p(qo), _i32p(ko), ctypes.byref(dims), None, 0)
    if n < 0:
        raise MagiBcaError(int(n), "magi_bca_fwd_schedule")
    buf = np.zeros((max(n, 1), 12), dtype=np.int32)
    n2 = lib.magi_bca_fwd_schedule(_i32p(qo), _i32p(ko), ctypes.byref(dims), _i32p(buf), n)
    assert n2 == n
    return buf[:n]


def magi_bca_bwd_schedule(q_chunk_offsets, kv_chunk_offsets, batch, heads_q, heads_kv, head_dim,
                          num_sms=148, kv_range=0, deterministic=False, samples=None, n_global=0) -> np.ndarray:
    """Host-only: the backward's work units as an int32 array [n_units, 12]
    (deterministic=True: one unit per kv tile)."""
    qo, ko = _offsets(q_chunk_offsets), _offsets(kv_chunk_offsets)
    dims = make_dims(batch, int(qo[-1]), int(ko[-1]), heads_q, heads_kv, head_dim, len(qo) - 1, len(ko) - 1,
                     kv_range=kv_range, deterministic=deterministic, samples=samples, n_global=n_global)
    lib = library()
    n = lib.magi_bca_bwd_schedule(_i32p(qo), _i32p(ko), ctypes.byref(dims), num_sms, None, 0)
    if n < 0:
        raise MagiBcaError(int(n), "magi_bca_bwd_schedule")
    buf = np.zeros((max(n, 1), 12), dtype=np.int32)
    n2 = lib.magi_bca_bwd_schedule(_i32p(qo), _i32p(ko), ctypes.byref(dims), num_sms, _i32p(buf), n)
    assert n2 == n
    return buf[:n]
