"""Host-side bookkeeping of a layer's block pool: block tiling of a chunk,
where each chunk's blocks sit, the local window and the blocks that leave it.

The library addresses key/value blocks by physical id inside a pool
``[B, H, NB, bs, D]``.  ``PoolLayout`` fixes the convention the engine uses:

* ids ``[0, P)`` are the persistent slots (none on the trainable path);
* then one position of ``nb_c`` ids per chunk.  When every chunk stays
  resident (a snapshot, or the trainable path's whole sequence), chunk ``t``
  takes position ``t``; in a rollout, position ``t mod (W + 1)``: the ring
  holds one chunk more than the window, so the chunk that leaves the window
  stays readable while the memory update of the step consumes it;
* block ``j`` of chunk ``t`` has the global (source) id ``t * nb_c + j``.

Readings of the Sparse Forcing pages (gist.science/es, section 2
"Arquitectura Propuesta"):

* item "Ventana Local": the local window of chunk ``t`` is the ``W`` most
  recent chunks, ``t`` included;
* item "Mecanismo de Actualización": the memory's new candidates at step
  ``t`` are the blocks of chunk ``t - W``, the chunk that just left the window;
  a snapshot step offers every chunk older than the window at once;
* section 2 PBSA, item "Compresión de Bloques": a chunk of ``T_c`` tokens is
  cut into blocks of ``bs`` tokens on its own, the last block partial
  (4680 tokens = 36 x 128 + 72).
"""
from __future__ import annotations

from typing import List, Optional


class PoolLayout:
    def __init__(self, chunk_tokens: int, bs: int, P: int, W: int, n_chunks: int,
                 rollout: bool, slots_in_pool: bool = True):
        if chunk_tokens <= 0 or bs <= 0 or W <= 0:
            raise ValueError("chunk_tokens, bs and W must be positive")
        self.chunk_tokens = chunk_tokens
        self.bs = bs
        self.W = W
        self.rollout = rollout
        self.n_chunks = n_chunks
        self.P = P if slots_in_pool else 0
        self.nb_c = (chunk_tokens + bs - 1) // bs
        self.positions = W + 1 if rollout else n_chunks
        self.NB = self.P + self.positions * self.nb_c

    @classmethod
    def of(cls, cfg) -> "PoolLayout":
        return cls(cfg.chunk_tokens, cfg.bs, cfg.P, cfg.W, cfg.n_chunks, cfg.rollout,
                   getattr(cfg, "slots_in_pool", True))

    def block_lens(self) -> List[int]:
        """Valid rows of each block of a chunk, in order."""
        full, tail = divmod(self.chunk_tokens, self.bs)
        return [self.bs] * full + ([tail] if tail else [])

    def position(self, t: int) -> int:
        return t % self.positions if self.rollout else t

    def chunk_phys_ids(self, t: int) -> List[int]:
        base = self.P + self.position(t) * self.nb_c
        return list(range(base, base + self.nb_c))

    def chunk_global_ids(self, t: int) -> List[int]:
        return list(range(t * self.nb_c, (t + 1) * self.nb_c))

    def window_chunks(self, t: int) -> List[int]:
        return list(range(max(0, t - self.W + 1), t + 1))

    def leaving_chunk(self, t: int) -> Optional[int]:
        return t - self.W if t >= self.W else None

    def older_chunks(self, t: int) -> List[int]:
        return list(range(0, max(0, t - self.W + 1)))
