"""Seeded synthetic workloads for Persistent Block-Sparse Attention (PBSA).

This module is shared by the CUDA path, the CPU oracle, the tests and the
benchmark.  It holds only workload *recipes*: shapes, block tiling of a chunk,
the physical placement of blocks in the cache, and seeded random tensors.  It
holds none of the method's arithmetic (no pooling, scoring, selection, memory
update or attention).

Workloads follow the shapes of a ~1.3B autoregressive video DiT layer as the
Sparse Forcing pages describe it (Wan2.1-T2V-1.3B base model, "Resultados
Experimentales"; chunked KV cache of the autoregressive rollout, "El Problema"):
latent frames of 1560 tokens, chunks of 3 frames, 128-token blocks, 12 heads of
dimension 128.  No trained weights or video data exist here, so Q/K/V are
N(0,1) with a random per-block "salience" offset of variance 2 added to a
fraction of key blocks (the pages' observation that attention concentrates on a
persistent subset of salient blocks, "Observación Empírica Clave").

Physical layout of the block pool of one (batch, head):

* ids ``[0, P)``                    persistent-memory slots;
* snapshot workloads: ids ``P + t*nb_c + j`` hold block ``j`` of chunk ``t``;
* rollout workloads: a ring of ``W + 1`` chunk positions after the slots;
  chunk ``t`` lives at ring position ``t % (W + 1)``.  One position more than
  the window lets the chunk that leaves the window stay readable until the
  memory update of the step has consumed it.
"""
from __future__ import annotations

import dataclasses
import hashlib
import math
from typing import Dict, List, Optional

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
                                   # blocks in place (trainable path), no slot ids

    # ---- block tiling of a chunk -------------------------------------
    @property
    def nb_c(self) -> int:
        """Blocks per chunk: a chunk is tiled on its own, last block partial."""
        return -(-self.chunk_tokens // self.bs)

    def chunk_block_lens(self) -> List[int]:
        lens = [self.bs] * self.nb_c
        lens[-1] = self.chunk_tokens - (self.nb_c - 1) * self.bs
        return lens

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    # ---- physical placement ------------------------------------------
    @property
    def ring_chunks(self) -> int:
        return self.W + 1 if self.rollout else self.n_chunks

    @property
    def n_slots(self) -> int:
        return self.P if self.slots_in_pool else 0

    @property
    def NB_phys(self) -> int:
        return self.n_slots + self.ring_chunks * self.nb_c

    def chunk_phys_ids(self, t: int) -> List[int]:
        pos = (t % self.ring_chunks) if self.rollout else t
        base = self.n_slots + pos * self.nb_c
        return list(range(base, base + self.nb_c))

    def chunk_global_ids(self, t: int) -> List[int]:
        return list(range(t * self.nb_c, (t + 1) * self.nb_c))

    def window_chunks(self, t: int) -> List[int]:
        return [c for c in range(t - self.W + 1, t + 1) if c >= 0]

    def leaving_chunk(self, t: int) -> Optional[int]:
        """The chunk that leaves the local window when chunk ``t`` arrives."""
        c = t - self.W
        return c if c >= 0 else None

    def snapshot_candidate_chunks(self) -> List[int]:
        """Snapshot workloads: every chunk older than the window is a candidate."""
        t = self.n_chunks - 1
        return list(range(0, max(0, t - self.W + 1)))


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


def salient_blocks(w: Workload, layer: int, t: int, n_blocks: int, scope_key) -> List[int]:
    """Indices (within ``n_blocks``) of the salient key blocks, floor(f*n + 1/2) of them."""
    n = int(math.floor(w.salient_frac * n_blocks + 0.5))
    if n == 0:
        return []
    r = _rng(w.seed, "salient", layer, scope_key)
    return sorted(r.choice(n_blocks, size=n, replace=False).tolist())


def chunk_tensors(w: Workload, t: int, layer: int = 0, with_q: bool = True):
    """Q, K, V of chunk ``t`` as float32 arrays [B, H, chunk_tokens, D] rounded to storage.

    Key blocks that are salient get a per-(b, h, block) offset vector drawn
    from N(0, 2) added to every token of the block."""
    shape = (w.B, w.H, w.chunk_tokens, w.D)
    q = normal(shape, w.seed, "q", layer, t) if with_q else None
    k = normal(shape, w.seed, "k", layer, t)
    v = normal(shape, w.seed, "v", layer, t)
    lens = w.chunk_block_lens()
    if w.salient_frac > 0:
        if w.salient_scope == "chunk":
            sal = salient_blocks(w, layer, t, w.nb_c, ("chunk", t // w.redraw_every))
        else:
            total = w.n_chunks * w.nb_c
            sal_all = salient_blocks(w, layer, 0, total, ("cache",))
            sal = [g - t * w.nb_c for g in sal_all if t * w.nb_c <= g < (t + 1) * w.nb_c]
        if sal:
            off = math.sqrt(2.0) * normal((w.B, w.H, len(sal), w.D), w.seed, "o", layer, t)
            for n, j in enumerate(sal):
                r0 = j * w.bs
                k[:, :, r0:r0 + lens[j], :] += off[:, :, n:n + 1, :]
    if q is not None:
        q = round_to_storage(q, w.dtype)
    return q, round_to_storage(k, w.dtype), round_to_storage(v, w.dtype)


def grad_output(w: Workload, T: int, layer: int = 0) -> np.ndarray:
    return round_to_storage(normal((w.B, w.H, T, w.D), w.seed, "do", layer), w.dtype)


def pool_from_chunks(w: Workload, chunks: Dict[int, np.ndarray]) -> np.ndarray:
    """Scatter per-chunk token tensors [B,H,T_c,D] into a block pool [B,H,NB_phys,bs,D].

    Positions that hold no token (block padding, unused ids) are zero."""
    pool = np.zeros((w.B, w.H, w.NB_phys, w.bs, w.D), dtype=np.float32)
    lens = w.chunk_block_lens()
    for t, x in chunks.items():
        for j, pid in enumerate(w.chunk_phys_ids(t)):
            r0 = j * w.bs
            pool[:, :, pid, :lens[j], :] = x[:, :, r0:r0 + lens[j], :]
    return pool


def chunk_layout(w: Workload, chunks) -> Dict[str, np.ndarray]:
    """Per-(b,h) block metadata for the given resident chunks.

    Returns ``blk_len`` and ``blk_pos`` [B,H,NB_phys] int32 (global token
    position of a block's first token) for the chunk blocks; slot entries and
    unused ids are zero."""
    blk_len = np.zeros((w.B, w.H, w.NB_phys), dtype=np.int32)
    blk_pos = np.zeros((w.B, w.H, w.NB_phys), dtype=np.int32)
    lens = w.chunk_block_lens()
    for t in chunks:
        for j, pid in enumerate(w.chunk_phys_ids(t)):
            blk_len[:, :, pid] = lens[j]
            blk_pos[:, :, pid] = t * w.chunk_tokens + j * w.bs
    return blk_len, blk_pos


def empty_memory(w: Workload):
    """Slot metadata of an empty persistent memory: src -1, weight 0."""
    slot_src = np.full((w.B, w.H, w.n_slots), -1, dtype=np.int32)
    slot_w = np.zeros((w.B, w.H, w.n_slots), dtype=np.float32)
    return slot_src, slot_w


def snapshot(w: Workload):
    """Inputs of one snapshot step: the cache holds chunks 0..n_chunks-1, the
    query chunk is the last one, the persistent memory is empty."""
    qs, kc, vc = {}, {}, {}
    t_cur = w.n_chunks - 1
    for t in range(w.n_chunks):
        q, k, v = chunk_tensors(w, t, with_q=(t == t_cur))
        kc[t], vc[t] = k, v
        if t == t_cur:
            qs = q
    blk_len, blk_pos = chunk_layout(w, range(w.n_chunks))
    slot_src, slot_w = empty_memory(w)
    cand_chunks = w.snapshot_candidate_chunks()
    cand_ids = np.array([p for c in cand_chunks for p in w.chunk_phys_ids(c)], dtype=np.int32)
    cand_src = np.array([g for c in cand_chunks for g in w.chunk_global_ids(c)], dtype=np.int32)
    win = np.array([p for c in w.window_chunks(t_cur) for p in w.chunk_phys_ids(c)], dtype=np.int32)
    return dict(q=qs, kpool=pool_from_chunks(w, kc), vpool=pool_from_chunks(w, vc),
                blk_len=blk_len, blk_pos=blk_pos, slot_src=slot_src, slot_w=slot_w,
                cand_ids=cand_ids, cand_src=cand_src, win_ids=win,
                q_pos0=t_cur * w.chunk_tokens,
                new_ids=np.array(w.chunk_phys_ids(t_cur), dtype=np.int32),
                all_ids=np.array([p for c in range(w.n_chunks) for p in w.chunk_phys_ids(c)],
                                 dtype=np.int32))


def mem_ids_all_slots(w: Workload) -> np.ndarray:
    """Persistent-memory id list [B,H,P] naming every slot (empty slots are skipped by length)."""
    return np.broadcast_to(np.arange(w.P, dtype=np.int32), (w.B, w.H, w.P)).copy()


def amax(w: Workload) -> int:
    """Capacity of an attended-block list: all slots plus the local top-k."""
    return w.P + w.k
