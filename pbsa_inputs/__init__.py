"""Seeded synthetic workloads for Persistent Block-Sparse Attention (PBSA).

This module serves both the CUDA path and the CPU oracle.  It holds only the
workload recipes: the shapes of each workload and seeded random tensors drawn
per chunk.  It holds none of the method's arithmetic and none of its
definitions: no pooling, scoring, selection, memory update or attention, and
no window, candidate, block-tiling or pool-placement rule.  The engine and the
oracle each take those from their own code.

Workloads follow the shapes of a ~1.3B autoregressive video DiT layer as the
Sparse Forcing pages describe it (Wan2.1-T2V-1.3B base model, "Resultados
Experimentales"; chunked KV cache of the autoregressive rollout, "El Problema"):
latent frames of 1560 tokens, chunks of 3 frames, 128-token blocks, 12 heads of
dimension 128.  No trained weights or video data exist here, so Q/K/V are
N(0,1) with a random per-block "salience" offset of variance 2 added to a
fraction of key blocks (the pages' observation that attention concentrates on a
persistent subset of salient blocks, "Observación Empírica Clave").
"""
from __future__ import annotations

import dataclasses
import hashlib
import math
from typing import Dict, List

import numpy as np

POLICY_EVICT = 0
POLICY_MERGE_MEAN = 1
MASK_CHUNK = 0
MASK_TOKEN = 1


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    D: int
    bs: int                 # tokens per block
    dtype: str              # "bf16" or "f32" storage of Q/K/V
    chunk_tokens: int       # tokens per chunk (query chunk length)
    P: int                  # persistent-memory budget (blocks)
    n_sink: int             # pinned sink slots inside the budget
    W: int                  # local window, in chunks, current chunk included
    k: int                  # local top-k per query block
    policy: int             # POLICY_EVICT / POLICY_MERGE_MEAN
    mask: int               # MASK_CHUNK / MASK_TOKEN
    n_chunks: int           # snapshot: chunks in the cache (current included)
                            # rollout: number of chunk steps
    layers: int = 1
    salient_frac: float = 0.0
    salient_scope: str = "cache"   # "cache": one draw over the whole cache
                                   # "chunk": per chunk, redrawn every `redraw_every`
    redraw_every: int = 1
    rollout: bool = False
    seed: int = 0
    slots_in_pool: bool = True     # False: the persistent set references cache
                                   # blocks in place (trainable path), no slots


WORKLOADS: Dict[str, Workload] = {
    # Tiny CPU-checkable step (fp32): 16 cache blocks of 64 tokens, the query
    # chunk is the last 4 of them.
    "tiny": Workload("tiny", B=1, H=2, D=64, bs=64, dtype="f32", chunk_tokens=256,
                     P=4, n_sink=0, W=2, k=4, policy=POLICY_EVICT, mask=MASK_CHUNK,
                     n_chunks=4, seed=0),
    # Single-layer decode step of a 1.3B video DiT (bf16).
    "decode": Workload("decode", B=1, H=12, D=128, bs=128, dtype="bf16", chunk_tokens=4680,
                       P=24, n_sink=0, W=2, k=16, policy=POLICY_EVICT, mask=MASK_CHUNK,
                       n_chunks=5, salient_frac=0.10, salient_scope="cache", seed=1),
    # 20-second rollout with mean-compressed eviction.
    "rollout20s": Workload("rollout20s", B=1, H=12, D=128, bs=128, dtype="bf16",
                           chunk_tokens=4680, P=48, n_sink=0, W=2, k=16,
                           policy=POLICY_MERGE_MEAN, mask=MASK_CHUNK, n_chunks=27,
                           salient_frac=0.05, salient_scope="chunk", redraw_every=5,
                           rollout=True, seed=2),
    # 1-minute rollout over a 30-layer stack.
    "rollout1min": Workload("rollout1min", B=1, H=12, D=128, bs=128, dtype="bf16",
                            chunk_tokens=4680, P=64, n_sink=0, W=2, k=16,
                            policy=POLICY_EVICT, mask=MASK_CHUNK, n_chunks=80, layers=30,
                            salient_frac=0.10, salient_scope="chunk", redraw_every=1,
                            rollout=True, seed=3),
    # Trainable-path shape: 21 frames = 7 chunks, forward and backward.
    "train": Workload("train", B=2, H=12, D=128, bs=128, dtype="bf16", chunk_tokens=4680,
                      P=32, n_sink=0, W=2, k=16, policy=POLICY_EVICT, mask=MASK_CHUNK,
                      n_chunks=7, salient_frac=0.10, salient_scope="cache", seed=4,
                      slots_in_pool=False),
}

TRAIN_DENSITIES = (0.05, 0.10, 0.25, 0.50, 1.00)


def variant(w: Workload, **kw) -> Workload:
    return dataclasses.replace(w, **kw)


# ---------------------------------------------------------------------------
# seeded generators
# ---------------------------------------------------------------------------

def _rng(*key) -> np.random.Generator:
    """A numpy Generator keyed by an arbitrary tuple (stable across runs)."""
    h = hashlib.sha256(repr(key).encode()).digest()
    return np.random.default_rng(np.frombuffer(h[:16], dtype=np.uint32).tolist())


def round_to_storage(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round float32 samples to the storage type; returns float32 values.

    bf16 rounding is round-to-nearest-even on the float32 bit pattern (the
    samples are finite and far from overflow)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    if dtype == "f32":
        return x
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    u = ((u + 0x7FFF + lsb) >> 16) << 16
    return u.astype(np.uint32).view(np.float32)


def normal(shape, *key) -> np.ndarray:
    return _rng(*key).standard_normal(size=shape, dtype=np.float32)


def _salient_runs(w: Workload, layer: int, n_runs: int, scope_key) -> List[int]:
    """Indices (within ``n_runs``) of the salient row runs, floor(f*n + 1/2) of them."""
    n = int(math.floor(w.salient_frac * n_runs + 0.5))
    if n == 0:
        return []
    r = _rng(w.seed, "salient", layer, scope_key)
    return sorted(r.choice(n_runs, size=n, replace=False).tolist())


def chunk_tensors(w: Workload, t: int, layer: int = 0, with_q: bool = True):
    """Q, K, V of chunk ``t`` as float32 arrays [B, H, chunk_tokens, D] rounded to storage.

    Salience structure: the chunk's key rows are cut into runs of ``bs`` rows
    from its first row (the last run shorter), and every row of a salient run
    gets the same per-(b, h, run) offset vector drawn from N(0, 2)."""
    shape = (w.B, w.H, w.chunk_tokens, w.D)
    q = normal(shape, w.seed, "q", layer, t) if with_q else None
    k = normal(shape, w.seed, "k", layer, t)
    v = normal(shape, w.seed, "v", layer, t)
    runs = -(-w.chunk_tokens // w.bs)
    if w.salient_frac > 0:
        if w.salient_scope == "chunk":
            sal = _salient_runs(w, layer, runs, ("chunk", t // w.redraw_every))
        else:
            sal_all = _salient_runs(w, layer, w.n_chunks * runs, ("cache",))
            sal = [g - t * runs for g in sal_all if t * runs <= g < (t + 1) * runs]
        if sal:
            off = math.sqrt(2.0) * normal((w.B, w.H, len(sal), w.D), w.seed, "o", layer, t)
            for n, j in enumerate(sal):
                k[:, :, j * w.bs:(j + 1) * w.bs, :] += off[:, :, n:n + 1, :]
    if q is not None:
        q = round_to_storage(q, w.dtype)
    return q, round_to_storage(k, w.dtype), round_to_storage(v, w.dtype)


def snapshot_chunks(w: Workload, layer: int = 0):
    """Every chunk of a snapshot workload: {t: (q or None, k, v)}, with the
    queries drawn only for the current (last) chunk."""
    t_cur = w.n_chunks - 1
    return {t: chunk_tensors(w, t, layer, with_q=(t == t_cur)) for t in range(w.n_chunks)}


def grad_output(w: Workload, T: int, layer: int = 0) -> np.ndarray:
    return round_to_storage(normal((w.B, w.H, T, w.D), w.seed, "do", layer), w.dtype)


def chunk_tensors_device(w: Workload, t: int, layer: int = 0, device: str = "cuda"):
    """Q, K, V of chunk ``t`` as bf16 device tensors [B, H, chunk_tokens, D]
    drawn on the device from a generator keyed by (workload seed, layer, t),
    with the salience structure of ``chunk_tensors`` (the same salient runs;
    offsets drawn on the device).  Same distributions as ``chunk_tensors``,
    other values: for timing runs too large to draw on the host, where both
    sides of a comparison draw the same (layer, t) from this function."""
    import torch
    h = hashlib.sha256(repr((w.seed, "device", layer, t)).encode()).digest()
    g = torch.Generator(device=device).manual_seed(int.from_bytes(h[:8], "little") >> 1)
    shape = (w.B, w.H, w.chunk_tokens, w.D)
    q = torch.randn(shape, generator=g, device=device)
    k = torch.randn(shape, generator=g, device=device)
    v = torch.randn(shape, generator=g, device=device)
    runs = -(-w.chunk_tokens // w.bs)
    if w.salient_frac > 0:
        if w.salient_scope == "chunk":
            sal = _salient_runs(w, layer, runs, ("chunk", t // w.redraw_every))
        else:
            sal_all = _salient_runs(w, layer, w.n_chunks * runs, ("cache",))
            sal = [j - t * runs for j in sal_all if t * runs <= j < (t + 1) * runs]
        for j in sal:
            off = math.sqrt(2.0) * torch.randn((w.B, w.H, 1, w.D), generator=g, device=device)
            k[:, :, j * w.bs:(j + 1) * w.bs, :] += off
    return q.bfloat16(), k.bfloat16(), v.bfloat16()
