"""Seeded synthetic workloads for block-causal GQA attention with QK-RMSNorm.

This module only describes shapes and draws random numbers.  It holds none of
the attention arithmetic, so both the fp64 oracle (``oracle/``) and the CUDA
path (``block_causal_attention_gqa_b200``) can take their inputs from it
without sharing any code with each other.

The five workloads mirror the shapes of MAGI-1 (arXiv 2505.13211):

* a latent video is a sequence of fixed-length chunks, 24 frames per chunk
  which the VAE compresses 4x in time to 6 latent frames, so one chunk of
  24x40 latent patches is 6*24*40 = 5760 tokens (MAGI-1 §2 and §2.1);
* the model uses grouped-query attention with 8 key/value groups
  (MAGI-1 §2.2.2, model table: "128 heads (8 groups)");
* streaming inference denoises up to four chunks at once against the cached
  keys/values of earlier clean chunks (MAGI-1 §2, Fig. 1; §2.4.4 KV cache).

Random draws use a CPU ``torch.Generator`` seeded with the workload's seed,
in fp32, in the order q, k, v, gamma_q, gamma_k, dO and then (long-context
workload only) the per-token LogNormal scales of q and k.  ``device="cuda"``
draws the same distributions from a CUDA generator instead (fast, but not the
same numbers); parity tests always use the CPU stream.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import numpy as np
import torch

__all__ = ["Workload", "WORKLOADS", "ORDER", "workload", "custom", "uniform_offsets", "rope_angles",
           "make_inputs", "sample_rows"]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    q_chunks: tuple          # token counts of the query-side chunks
    kv_chunks: tuple         # token counts of the key/value-side chunks
    heads_q: int
    heads_kv: int
    head_dim: int
    seed: int
    backward: bool           # training layout (fwd+bwd) or inference (fwd only)
    input_dtype: str = "bf16"    # "fp32" = drawn fp32 then rounded to bf16 at the boundary
    gamma: str = "perturbed"     # "ones" or "perturbed" (1 + N(0, 0.1) per head-dim)
    token_scale: bool = False    # LogNormal(0, 0.5) per-token scale on q and k
    kv_range: int = 0            # KV range in chunks (0 = every earlier chunk); MAGI-1 §2.4.4, Fig. 12
    rope: bool = False           # rotary angles for q and k (3D positions, see rope_angles)
    deterministic: bool = False  # backward with every sum in a fixed order (same bits on every call)
    samples: Optional[tuple] = None  # packed samples: cumulative kv-chunk counts (None: one sample)
    n_global: int = 0            # the last n_global kv chunks form a global block
    shard_rank: int = 0          # with shard_world > 1: this workload is kv heads [r*Hkv, (r+1)*Hkv) (and
    shard_world: int = 1         # their query groups) of a problem with shard_world times the heads

    @property
    def seqlen_q(self) -> int:
        return int(sum(self.q_chunks))

    @property
    def seqlen_kv(self) -> int:
        return int(sum(self.kv_chunks))

    @property
    def mask_kw(self) -> dict:
        """The mask options as keyword arguments (the binding's entry points and
        the oracle take the same names)."""
        return dict(kv_range=self.kv_range, samples=None if self.samples is None else list(self.samples),
                    n_global=self.n_global)

    @property
    def q_offsets(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.q_chunks)]).astype(np.int32)

    @property
    def kv_offsets(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.kv_chunks)]).astype(np.int32)


def uniform_offsets(n_chunks: int, chunk_len: int) -> tuple:
    return tuple([chunk_len] * n_chunks)


WORKLOADS = {
    # 2 chunks x 64 tokens, 2 query heads sharing 1 kv head, head_dim 64.
    "tiny": Workload("tiny", 1, (64, 64), (64, 64), 2, 1, 64, seed=0, backward=False,
                     input_dtype="fp32", gamma="ones"),
    # training layout, 4 chunks x 1024 tokens, GQA 16/4, head_dim 128.
    "train4k": Workload("train4k", 1, uniform_offsets(4, 1024), uniform_offsets(4, 1024),
                        16, 4, 128, seed=1, backward=True),
    # model scale: 8 chunks x 5760 tokens (6 latent frames x 24x40 patches), GQA 24/8.
    "model46k": Workload("model46k", 1, uniform_offsets(8, 5760), uniform_offsets(8, 5760),
                         24, 8, 128, seed=2, backward=True),
    # streaming inference: 4 active chunks against 12 clean cached chunks + themselves.
    "stream4of16": Workload("stream4of16", 2, uniform_offsets(4, 5760), uniform_offsets(16, 5760),
                            24, 8, 128, seed=3, backward=False),
    # long context: 32 chunks x 8192 tokens, GQA 16/2, LogNormal per-token q/k scales.
    "long262k": Workload("long262k", 1, uniform_offsets(32, 8192), uniform_offsets(32, 8192),
                         16, 2, 128, seed=4, backward=True, token_scale=True),
    # a quarter of long262k (8 chunks of 8192 tokens, same heads and value recipe): its launches fit an
    # ncu capture, and long262k's DRAM traffic per launch is scaled from it by the units processed
    "long65k": Workload("long65k", 1, uniform_offsets(8, 8192), uniform_offsets(8, 8192),
                        16, 2, 128, seed=4, backward=True, token_scale=True),
    # long context with a KV range of 8 chunks (MAGI-1 §2.4.4 and §2.6: each chunk limited to
    # the preceding content, KV range 8 for long videos), otherwise as long262k.
    "window262k": Workload("window262k", 1, uniform_offsets(32, 8192), uniform_offsets(32, 8192),
                           16, 2, 128, seed=5, backward=True, token_scale=True, kv_range=8),

    # cross-attention of the model-scale video sequence (one chunk of 8 x 5760 tokens)
    # against 1024 text tokens (MAGI-1 §2.2.2: cross-attention with QK-norm and GQA
    # to the T5 text condition; the text length is a reading), GQA 24/8.
    "xattn46k": Workload("xattn46k", 1, (46080,), (1024,), 24, 8, 128, seed=6, backward=True),
    # model46k with rotary angles on q and k before the norm (MAGI-1 §2.2.2: learnable 3D
    # RoPE; angles from the 6 x 24 x 40 latent grid of each chunk, see rope_angles).
    "model46k_rope": Workload("model46k_rope", 1, uniform_offsets(8, 5760), uniform_offsets(8, 5760),
                              24, 8, 128, seed=7, backward=True, rope=True),
    # packed training sequence of model46k's size (MAGI-1 §4.1.2, Figure 15 (g)): three samples of
    # 3, 1 and 3 chunks of 5760 tokens packed one after another, and a last chunk that forms a global
    # block (every query sees it, its queries see everything), GQA 24/8
    "packed46k": Workload("packed46k", 1, uniform_offsets(8, 5760), uniform_offsets(8, 5760), 24, 8, 128,
                          seed=8, backward=True, samples=(0, 3, 4, 7, 8), n_global=1),
    # model46k through the deterministic backward (dq from a query-major pass, one unit
    # per kv tile, fixed-order dgamma): the reproducible-training setting
    "model46k_det": Workload("model46k_det", 1, uniform_offsets(8, 5760), uniform_offsets(8, 5760),
                             24, 8, 128, seed=2, backward=True, deterministic=True),
    "train4k_det": Workload("train4k_det", 1, uniform_offsets(4, 1024), uniform_offsets(4, 1024),
                            16, 4, 128, seed=1, backward=True, deterministic=True),
}

ORDER = ["tiny", "train4k", "model46k", "stream4of16", "long262k", "window262k", "xattn46k", "model46k_rope",
         "model46k_det", "train4k_det", "long65k", "packed46k"]


def workload(name_or_index) -> Workload:
    if isinstance(name_or_index, int):
        return WORKLOADS[ORDER[name_or_index]]
    return WORKLOADS[name_or_index]


def shard_heads(w: Workload, world: int, rank: int) -> Workload:
    """Rank `rank`'s share of `w` when its key/value heads (each with its whole
    group of query heads) are split over `world` ranks: the same chunks and
    head_dim with heads_kv / world kv heads and heads_q / world query heads.
    Each kv head's attention is independent of the others, so the shards need
    no exchange.  Every rank draws the whole problem's inputs (same seed) and
    keeps its own contiguous heads (make_inputs), so the shards' results put
    together are the unsharded result."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of {world}")
    if w.shard_world != 1:
        raise ValueError(f"{w.name} is already a shard")
    if w.heads_kv % world != 0:
        raise ValueError(f"{w.name}: {w.heads_kv} kv heads do not split over {world} ranks")
    return dataclasses.replace(w, name=f"{w.name}[heads {rank}/{world}]", heads_q=w.heads_q // world,
                               heads_kv=w.heads_kv // world, shard_rank=rank, shard_world=world)


def custom(name: str, batch: int, q_chunks: Sequence[int], kv_chunks: Optional[Sequence[int]],
           heads_q: int, heads_kv: int, head_dim: int, seed: int, backward: bool = True,
           gamma: str = "perturbed", token_scale: bool = False, kv_range: int = 0,
           rope: bool = False, samples: Optional[Sequence[int]] = None, n_global: int = 0,
           deterministic: bool = False) -> Workload:
    kv = tuple(kv_chunks) if kv_chunks is not None else tuple(q_chunks)
    return Workload(name, batch, tuple(q_chunks), kv, heads_q, heads_kv, head_dim, seed,
                    backward, gamma=gamma, token_scale=token_scale, kv_range=kv_range, rope=rope,
                    deterministic=deterministic, samples=None if samples is None else tuple(samples),
                    n_global=n_global)


def rope_angles(positions: np.ndarray, head_dim: int, grid=(6, 24, 40), base: float = 10000.0) -> np.ndarray:
    """Rotary angles [len(positions), head_dim/2] (fp32) for key/value token
    positions: token t of the sequence sits at latent frame, row and column
    (t // (H W), (t // W) % H, t % W) of a 6 x 24 x 40 grid per 5760-token
    chunk (frames continue across chunks), and the head_dim/2 frequency pairs
    are split into three near-equal groups, one per axis, with frequencies
    base^(-j / n) inside a group.  (A stand-in for MAGI-1's learnable 3D RoPE,
    whose learned frequencies the pages do not give.)"""
    t = np.asarray(positions, dtype=np.int64)
    _, H, W = grid
    axes = [t // (H * W), (t // W) % H, t % W]
    half = head_dim // 2
    sizes = [half - 2 * (half // 3), half // 3, half // 3]
    cols = []
    for a, n in zip(axes, sizes):
        freq = base ** (-np.arange(n) / max(n, 1))
        cols.append(a[:, None].astype(np.float64) * freq[None, :])
    return np.concatenate(cols, axis=1).astype(np.float32)


def make_inputs(w: Workload, device: str = "cpu", with_grad_out: Optional[bool] = None) -> dict:
    """Draw the workload's tensors.

    Returns a dict with q [B,Sq,Hq,D], k/v [B,Skv,Hkv,D] and dout [B,Sq,Hq,D]
    as bf16 (fp32 draws rounded to bf16, the values both sides consume), the
    unrounded fp32 q/k/v under ``*_f32`` when the workload is fp32-in, and
    gamma_q/gamma_k as fp32 [D].
    """
    want_dout = w.backward if with_grad_out is None else with_grad_out
    gen_dev = "cuda" if device.startswith("cuda") else "cpu"
    g = torch.Generator(device=gen_dev)
    g.manual_seed(w.seed)
    n, r = w.shard_world, w.shard_rank
    # a head shard draws the whole problem (n times the heads) and keeps its heads
    B, Sq, Skv, Hq, Hkv, D = w.batch, w.seqlen_q, w.seqlen_kv, w.heads_q * n, w.heads_kv * n, w.head_dim
    kw = dict(generator=g, device=gen_dev, dtype=torch.float32)
    q = torch.randn(B, Sq, Hq, D, **kw)
    k = torch.randn(B, Skv, Hkv, D, **kw)
    v = torch.randn(B, Skv, Hkv, D, **kw)
    if w.gamma == "ones":
        gq = torch.ones(D, device=gen_dev)
        gk = torch.ones(D, device=gen_dev)
    else:
        gq = 1.0 + 0.1 * torch.randn(D, **kw)
        gk = 1.0 + 0.1 * torch.randn(D, **kw)
    dout = torch.randn(B, Sq, Hq, D, **kw) if want_dout else None
    if w.token_scale:
        # one LogNormal(0, 0.5) draw per token per tensor, shared by all heads
        sq = torch.exp(0.5 * torch.randn(B, Sq, 1, 1, **kw))
        sk = torch.exp(0.5 * torch.randn(B, Skv, 1, 1, **kw))
        q.mul_(sq)
        k.mul_(sk)
    if n > 1:
        hq, hk = w.heads_q, w.heads_kv
        q = q[:, :, r * hq:(r + 1) * hq].contiguous()
        k = k[:, :, r * hk:(r + 1) * hk].contiguous()
        v = v[:, :, r * hk:(r + 1) * hk].contiguous()
        if dout is not None:
            dout = dout[:, :, r * hq:(r + 1) * hq].contiguous()
    out = dict(gamma_q=gq.float().to(device), gamma_k=gk.float().to(device))
    if w.input_dtype == "fp32":
        out.update(q_f32=q.to(device), k_f32=k.to(device), v_f32=v.to(device))
    out.update(q=q.to(torch.bfloat16).to(device), k=k.to(torch.bfloat16).to(device),
               v=v.to(torch.bfloat16).to(device))
    if dout is not None:
        out["dout"] = dout.to(torch.bfloat16).to(device)
    if w.rope:
        # query token i of query chunk c is kv token kv_offsets[n_kv - n_q + c] + (i - q_offsets[c])
        qo, ko = w.q_offsets, w.kv_offsets
        shift = len(ko) - len(qo)
        qpos = np.concatenate([ko[shift + c] + np.arange(qo[c + 1] - qo[c]) for c in range(len(qo) - 1)])
        out["rope_q"] = torch.from_numpy(rope_angles(qpos, D)).to(device)
        out["rope_k"] = torch.from_numpy(rope_angles(np.arange(Skv), D)).to(device)
    return out


def sample_rows(n_rows: int, offsets: np.ndarray, n_sample: int, seed: int, tile: int = 128) -> np.ndarray:
    """Stratified sample of row indices: the first and last row of every
    chunk, the rows on either side of every ``tile`` boundary, and the rest
    uniform from a fixed seed.  Returns a sorted unique int64 array."""
    if n_rows <= n_sample:
        return np.arange(n_rows, dtype=np.int64)
    must = set()
    for a, b in zip(offsets[:-1], offsets[1:]):
        must.update([int(a), int(b) - 1])
    for t in range(tile, n_rows, tile):
        must.update([t - 1, t])
    must = sorted(r for r in must if 0 <= r < n_rows)
    rng = np.random.default_rng(seed)
    if len(must) >= n_sample:
        pick = rng.choice(len(must), size=n_sample, replace=False)
        return np.sort(np.asarray(must, dtype=np.int64)[pick])
    rest = np.setdiff1d(np.arange(n_rows, dtype=np.int64), np.asarray(must, dtype=np.int64))
    extra = rng.choice(rest, size=n_sample - len(must), replace=False)
    return np.sort(np.concatenate([np.asarray(must, dtype=np.int64), extra]))
