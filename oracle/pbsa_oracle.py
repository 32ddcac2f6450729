"""CPU oracle for Persistent Block-Sparse Attention (PBSA) -- TEST INFRASTRUCTURE.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module.  The product path (the CUDA library and
its Python binding) never calls it, and this module imports nothing of the
product.

What it computes is the hot path of Sparse Forcing's PBSA, restated step by
step in plain float64 numpy with Python loops over (batch, head, block):

* a1/a2  block compression by pooling and coarse block scoring
         (Sparse Forcing, gist.science/es, section 2 "Persistente Block-Sparse
         Attention (PBSA)", item "Compresión de Bloques"; the abstract on the
         shd-paper.top page: pooled routing is the PBSA kernel's job);
* a3     the persistent memory P_t: sink blocks, dynamic blocks chosen by
         coarse scoring, Top-C retention, and the learned compression,
         retention and refresh of the persistent blocks (same page, section 2 "Arquitectura
         Propuesta", items "Memoria Persistente", "Bloques Sumidero",
         "Bloques Dinámicos", "Mecanismo de Actualización"; the abstract);
* a4/a5  the local window L_t with a per-query-block Top-K of relevant blocks
         (section 2 "Arquitectura Propuesta", item "Ventana Local");
* a6     hybrid attention: dense over the persistent memory, sparse over the
         local window (section 2 PBSA, item "Atención Híbrida");
* a7     the backward pass of a6 for the trainable path (section 3
         "Contribuciones Clave", item "Kernel PBSA"; section 2 "Entrenamiento");
* the backward of a3 and the recurrent backward of a rollout, through the
         slots a block was copied or merged into (section 2 "Entrenamiento";
         the abstract).

The pages give no formulas.  Where they are silent this module takes the
plainest reading; each reading is named in the docstring of the function that
takes it (R1..R19 are the names used in the design notes).

Every function here is pinned by the tests under ``tests/test_oracle_*.py``
against closed forms, invariants, brute force and library routines (torch's
scaled-dot-product attention and autograd in float64); none is left unpinned.
"""
from __future__ import annotations

import math
from typing import Optional, Tuple

import numpy as np

EVICT = 0
MERGE_MEAN = 1
MASK_CHUNK = 0
MASK_TOKEN = 1


# ---------------------------------------------------------------------------
# storage rounding
# ---------------------------------------------------------------------------

def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 (ties to even), returned as float64.

    A bfloat16 keeps 8 significant bits.  ``frexp`` writes x = m * 2**e with
    0.5 <= |m| < 1, so m * 256 holds exactly the 8 kept bits left of the
    point; ``np.round`` rounds half to even."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)
    return np.ldexp(np.round(m * 256.0) / 256.0, e)


def round_storage(x: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "bf16":
        return round_bf16(x)
    if dtype == "f32":
        return np.asarray(x, dtype=np.float32).astype(np.float64)
    if dtype == "f64":
        return np.asarray(x, dtype=np.float64)
    raise ValueError(dtype)


# ---------------------------------------------------------------------------
# a1  block compression by pooling
# ---------------------------------------------------------------------------

def chunk_blocks(T_c: int, bs: int):
    """The blocks one chunk of T_c token rows is cut into (R9): runs of bs
    consecutive rows from the chunk's first row, the last run shorter when bs
    does not divide T_c.  Returns (first row within the chunk, length) per
    block.  Key chunks and query chunks are tiled alike; a 4680-token chunk in
    128-token blocks gives 36 full blocks and one of 72 rows."""
    out = []
    r0 = 0
    while r0 < T_c:
        n = min(bs, T_c - r0)
        out.append((r0, n))
        r0 += n
    return out


def query_blocks(Tq: int, bs: int, q_chunk: int = 0):
    """Query rows are a sequence of chunks of q_chunk rows (0: one chunk of Tq
    rows; the last chunk may be shorter), and each chunk is tiled into blocks
    on its own by ``chunk_blocks`` (R9), so no block crosses a chunk boundary.
    Returns the list of (first row, length) of every query block."""
    qc = q_chunk if q_chunk > 0 else Tq
    out = []
    c0 = 0
    while c0 < Tq:
        clen = min(qc, Tq - c0)
        out.extend((c0 + r0, n) for r0, n in chunk_blocks(clen, bs))
        c0 += clen
    return out


def query_block_lengths(Tq: int, bs: int, q_chunk: int = 0) -> np.ndarray:
    return np.array([n for _, n in query_blocks(Tq, bs, q_chunk)], dtype=np.int64)


def pool_queries(q: np.ndarray, bs: int, q_chunk: int = 0) -> np.ndarray:
    """Mean of the query rows of each query block (R1: mean over valid tokens).

    q: [B,H,Tq,D] -> q_bar [B,H,nQB,D] float64."""
    B, H, Tq, D = q.shape
    blocks = query_blocks(Tq, bs, q_chunk)
    out = np.zeros((B, H, len(blocks), D))
    for b in range(B):
        for h in range(H):
            for i, (r0, n) in enumerate(blocks):
                rows = q[b, h, r0:r0 + n].astype(np.float64)
                out[b, h, i] = rows.sum(axis=0) / n
    return out


def pool_keys(kpool: np.ndarray, blk_len: np.ndarray, ids, k_bar: np.ndarray) -> np.ndarray:
    """Mean of the valid key rows of each listed block; other entries of k_bar are kept.

    kpool: [B,H,NB,bs,D]; blk_len: [B,H,NB]; k_bar: [B,H,NB,D] (copied).
    A block of length 0 pools to the zero vector."""
    out = np.array(k_bar, dtype=np.float64, copy=True)
    B, H = kpool.shape[:2]
    for b in range(B):
        for h in range(H):
            for j in ids:
                n = int(blk_len[b, h, j])
                if n == 0:
                    out[b, h, j] = 0.0
                else:
                    out[b, h, j] = kpool[b, h, j, :n].astype(np.float64).sum(axis=0) / n
    return out


# ---------------------------------------------------------------------------
# a2  coarse block scores and the memory score
# ---------------------------------------------------------------------------

def block_scores(q_bar: np.ndarray, k_bar: np.ndarray, scale: float) -> np.ndarray:
    """S[b,h,i,j] = scale * <q_bar_i, k_bar_j> for every pair (R2)."""
    B, H, nQB, D = q_bar.shape
    NB = k_bar.shape[2]
    S = np.zeros((B, H, nQB, NB))
    for b in range(B):
        for h in range(H):
            S[b, h] = scale * (q_bar[b, h] @ k_bar[b, h].T)
    return S


def memory_scores(S: np.ndarray) -> np.ndarray:
    """Relevance of a block to the current step: mean of its scores over the
    query blocks of the chunk (R3).  S: [B,H,nQB,NB] -> m [B,H,NB]."""
    return S.sum(axis=2) / S.shape[2]


def score_blocks(q, kpool, blk_len, pool_ids, k_bar, scale, bs, q_chunk=0):
    """The whole scoring call: pool Q, (re)pool the listed key blocks, score all blocks."""
    q_bar = pool_queries(q, bs, q_chunk)
    k_bar = pool_keys(kpool, blk_len, pool_ids, k_bar)
    S = block_scores(q_bar, k_bar, scale)
    return q_bar, k_bar, S, memory_scores(S)


# ---------------------------------------------------------------------------
# a3  persistent-memory update
# ---------------------------------------------------------------------------

class _Item:
    """A candidate of the Top-C retention: an occupied slot or a block leaving the window."""

    def __init__(self, phys, src, w, m, old_slot):
        self.phys = int(phys)        # where its content lives now
        self.src = int(src)          # global id of the block it came from
        self.w = float(w)            # number of blocks merged into it
        self.m = float(m)            # memory score
        self.old_slot = old_slot     # slot index if it already is in memory


def _masked_rows(x: np.ndarray, n: int) -> np.ndarray:
    y = np.zeros_like(x, dtype=np.float64)
    y[:n] = x[:n]
    return y


def update_memory(kpool, vpool, blk_len, blk_pos, k_bar, slot_src, slot_w,
                  cand_ids, cand_src, mem_score, P: int, n_sink: int, policy: int,
                  store: str):
    """Top-C retention of the persistent memory P_t, in place on copies of the inputs.

    Sparse Forcing keeps a bounded set of historical blocks: fixed sink
    anchors plus dynamic blocks chosen by coarse scoring, refreshed by keeping
    the C best-scoring blocks and discarding the rest as they leave the local
    window (gist.science/es, section 2 "Arquitectura Propuesta"); per the
    abstract the mechanism also compresses persistent blocks, not only keeps them.

    Readings taken:
      R4  C = P - n_sink dynamic blocks besides the sinks.
      R6  slot s < n_sink is the sink of global block s: that block enters its
          sink slot when it leaves the window and is never ranked or merged into.
      R3  candidates are ranked by the memory score m (mean block score over the
          query blocks of the step); key (m descending, source id ascending).
      --  kept blocks already in memory stay in their slot; newly kept blocks
          fill the free non-sink slots in ascending slot order, taken in
          ascending source-id order.
      R5  policy MERGE_MEAN: each loser j is merged into the kept slot whose
          pre-merge pooled key has the largest dot product with j's pooled key
          (ties: lowest slot).  A slot's new content is the weight-averaged
          token-position-wise mean of its blocks, rows past a block's length
          counting as zero; weights add, the length is the maximum, the pooled
          key is recomputed from the stored result.  Policy EVICT drops losers.

    Shapes: kpool/vpool [B,H,NB,bs,D]; blk_len/blk_pos [B,H,NB]; k_bar
    [B,H,NB,D]; slot_src/slot_w [B,H,P]; cand_ids/cand_src [n]; mem_score
    [B,H,NB].  ``store`` is the storage type new slot rows are rounded to.

    Returns (kpool, vpool, blk_len, blk_pos, k_bar, slot_src, slot_w, info) with
    ``info[(b,h)] = dict(kept=[src...], losers=[src...], target={src: slot},
    compose={slot: [(pre-update id, weight, rows), ...]})``: every slot after
    the update is the weighted row-wise sum of those terms (a copy is one term
    of weight 1 over the whole block; an emptied slot has none), before the
    rounding to the storage type.
    """
    kp = np.array(kpool, dtype=np.float64, copy=True)
    vp = np.array(vpool, dtype=np.float64, copy=True)
    ln = np.array(blk_len, copy=True)
    ps = np.array(blk_pos, copy=True)
    kb = np.array(k_bar, dtype=np.float64, copy=True)
    ss = np.array(slot_src, copy=True)
    sw = np.array(slot_w, dtype=np.float64, copy=True)
    B, H = kp.shape[:2]
    info = {}
    for b in range(B):
        for h in range(H):
            items = []
            sinks_in = []
            for s in range(n_sink, P):
                if ss[b, h, s] >= 0:
                    items.append(_Item(s, ss[b, h, s], sw[b, h, s], mem_score[b, h, s], s))
            for c, src in zip(cand_ids, cand_src):
                if src < n_sink:
                    sinks_in.append((int(src), int(c)))
                else:
                    items.append(_Item(c, src, 1.0, mem_score[b, h, c], None))
            order = sorted(items, key=lambda it: (-it.m, it.src))
            n_keep = min(P - n_sink, len(order))
            kept, losers = order[:n_keep], order[n_keep:]

            slot_of = {}
            taken = {it.old_slot for it in kept if it.old_slot is not None}
            free = [s for s in range(n_sink, P) if s not in taken]
            for it in kept:
                if it.old_slot is not None:
                    slot_of[id(it)] = it.old_slot
            for it, s in zip(sorted([it for it in kept if it.old_slot is None],
                                    key=lambda it: it.src), free):
                slot_of[id(it)] = s

            merged_into = {s: [] for s in range(P)}
            target = {}
            if policy == MERGE_MEAN and kept:
                by_slot = sorted(kept, key=lambda it: slot_of[id(it)])
                for j in losers:
                    best, best_dot = None, -math.inf
                    for c in by_slot:
                        d = float(np.dot(kb[b, h, j.phys], kb[b, h, c.phys]))
                        if d > best_dot:
                            best, best_dot = c, d
                    s = slot_of[id(best)]
                    merged_into[s].append(j)
                    target[j.src] = s

            # read every source before any slot is written
            K = {id(it): kp[b, h, it.phys].copy() for it in items}
            V = {id(it): vp[b, h, it.phys].copy() for it in items}
            L = {id(it): int(ln[b, h, it.phys]) for it in items}
            POS = {id(it): int(ps[b, h, it.phys]) for it in items}
            KB = {id(it): kb[b, h, it.phys].copy() for it in items}
            sink_K = {s: (kp[b, h, c].copy(), vp[b, h, c].copy(), int(ln[b, h, c]),
                          int(ps[b, h, c]), kb[b, h, c].copy()) for s, c in sinks_in}

            holder = {slot_of[id(it)]: it for it in kept}
            bs = kp.shape[3]
            # what each slot holds after the update, as (pre-update id, weight,
            # rows) terms of a weighted row-wise mean: the backward of the
            # update distributes a slot's gradient by these terms (NEXT-2)
            compose = {s: [(s, 1.0, bs)] for s in range(n_sink)}
            for s in range(n_sink, P):
                if s not in holder:
                    compose[s] = []
                    ss[b, h, s] = -1
                    sw[b, h, s] = 0.0
                    ln[b, h, s] = 0
                    ps[b, h, s] = 0
                    kb[b, h, s] = 0.0
                    continue
                c = holder[s]
                group = merged_into[s]
                if not group:
                    compose[s] = [(c.phys, 1.0, bs)]
                    kp[b, h, s] = K[id(c)]
                    vp[b, h, s] = V[id(c)]
                    ln[b, h, s] = L[id(c)]
                    kb[b, h, s] = KB[id(c)]
                    sw[b, h, s] = c.w
                else:
                    W = c.w + sum(j.w for j in group)
                    compose[s] = [(c.phys, c.w / W, L[id(c)])] + \
                        [(j.phys, j.w / W, L[id(j)]) for j in group]
                    ksum = c.w * _masked_rows(K[id(c)], L[id(c)])
                    vsum = c.w * _masked_rows(V[id(c)], L[id(c)])
                    for j in group:
                        ksum += j.w * _masked_rows(K[id(j)], L[id(j)])
                        vsum += j.w * _masked_rows(V[id(j)], L[id(j)])
                    n = max([L[id(c)]] + [L[id(j)] for j in group])
                    kp[b, h, s] = round_storage(ksum / W, store)
                    vp[b, h, s] = round_storage(vsum / W, store)
                    ln[b, h, s] = n
                    kb[b, h, s] = kp[b, h, s, :n].sum(axis=0) / n
                    sw[b, h, s] = W
                ss[b, h, s] = c.src
                ps[b, h, s] = POS[id(c)]
            for s, (k_, v_, l_, p_, kb_) in sink_K.items():
                compose[s] = [(dict(sinks_in)[s], 1.0, bs)]
                kp[b, h, s], vp[b, h, s] = k_, v_
                ln[b, h, s], ps[b, h, s], kb[b, h, s] = l_, p_, kb_
                ss[b, h, s] = s
                sw[b, h, s] = 1.0
            info[(b, h)] = dict(kept=[it.src for it in kept], losers=[it.src for it in losers],
                                keys={it.src: it.m for it in items}, target=target,
                                slot={it.src: slot_of[id(it)] for it in kept},
                                compose=compose)
    return kp, vp, ln, ps, kb, ss, sw, info


# ---------------------------------------------------------------------------
# a4/a5  local Top-K selection and the attended-block list
# ---------------------------------------------------------------------------

def select_local(S: np.ndarray, win_ids, k: int, mem_ids: Optional[np.ndarray],
                 blk_len: np.ndarray, mask: int = MASK_CHUNK, q_pos0: int = 0,
                 blk_pos: Optional[np.ndarray] = None, bs: int = 0, Tq: int = 0,
                 q_chunk: int = 0):
    """Per query block: Top-K window blocks by block score, united with the memory.

    Inside the sliding window only the K most relevant blocks of each query
    are attended (gist.science/es, section 2 "Arquitectura Propuesta", item
    "Ventana Local"); attention is dense over the persistent memory (section 2
    PBSA, item "Atención Híbrida").

    Readings taken:
      R7   the window list is given by the caller (current chunk included).
      R8   chunk mask: every window block is allowed.  Token mask: a block is
           allowed for query block i when its first token is not after the
           last query token of block i.
      R10  ranking key (score descending, physical id ascending); blocks of
           length 0 are never candidates; if K >= #allowed all are taken.
      R12  the attended list is the union of the memory ids that hold a block
           (length > 0) and the local selection, ascending, without duplicates.

    S: [B,H,nQB,NB] scores indexed by physical block id; mem_ids: [B,H,n_mem]
    physical ids (-1 = none) or None.  Returns a list of lists A[b][h][i]."""
    B, H, nQB, _ = S.shape
    blocks = query_blocks(Tq, bs, q_chunk) if mask == MASK_TOKEN else None
    out = []
    for b in range(B):
        ob = []
        for h in range(H):
            oh = []
            mem = []
            if mem_ids is not None:
                mem = [int(m) for m in mem_ids[b, h] if m >= 0 and blk_len[b, h, m] > 0]
            for i in range(nQB):
                cands = []
                for j in win_ids:
                    j = int(j)
                    if blk_len[b, h, j] <= 0:
                        continue
                    if mask == MASK_TOKEN:
                        last_q = q_pos0 + blocks[i][0] + blocks[i][1] - 1
                        if blk_pos[b, h, j] > last_q:
                            continue
                    cands.append(j)
                order = sorted(cands, key=lambda j: (-S[b, h, i, j], j))
                local = order[:min(k, len(order))]
                oh.append(sorted(set(mem) | set(local)))
            ob.append(oh)
        out.append(ob)
    return out


def frame_groups(T_c: int, bs: int, frame_tokens: int):
    """The frame of each block of a chunk (R20): block j (rows [j*bs, ...) of the
    chunk) belongs to the frame its first row falls in, frame_tokens rows per
    frame.  Returns a list over the chunk's blocks."""
    return [(r0 // frame_tokens) for r0, _ in chunk_blocks(T_c, bs)]


def _frame_scores(cands, s_row, lens):
    """R20: {frame: sum_j len_j s_j / sum_j len_j} over the (block, frame) pairs."""
    num, den = {}, {}
    for j, g in cands:
        num[g] = num.get(g, 0.0) + float(lens[j]) * float(s_row[j])
        den[g] = den.get(g, 0.0) + float(lens[j])
    return {g: num[g] / den[g] for g in num}


def select_hier(S: np.ndarray, win_ids, win_frame, F: int, k: int,
                mem_ids: Optional[np.ndarray], blk_len: np.ndarray, mask: int = MASK_CHUNK,
                q_pos0: int = 0, blk_pos: Optional[np.ndarray] = None, bs: int = 0,
                Tq: int = 0, q_chunk: int = 0):
    """Two-level local selection, frame then block, the alternative router of
    the "next" rows (Light Forcing, gist.science/it, section 2.2 "Attenzione
    Sparsa Gerarchica (HSA)": query and key tokens are mean-pooled per block
    and per frame; each query block first keeps a few relevant historical
    frames by their frame-level keys, then the critical blocks inside those
    frames by their block-level keys; attention runs over the kept blocks).

    Readings taken:
      R20  a frame of the window is the group of window blocks that start in it
           (``win_frame[e]`` is the frame of window entry e, any integer label);
           its pooled key is the mean of its blocks' valid tokens, so its score
           for query block i is the length-weighted mean of those blocks'
           scores: sum_j len_j S_ij / sum_j len_j, over the blocks that are
           candidates for i (length > 0 and, with the token mask, allowed);
      R21  the F frames of highest score are kept (ties: lower frame label);
           the local set is the Top-K blocks of the kept frames by S (ties:
           lower id), all of them if fewer; the list is the union with the
           memory as in ``select_local``.
    With F at least the number of frames this is ``select_local``.

    Shapes and the other arguments as ``select_local``.  Returns A[b][h][i]."""
    B, H, nQB, _ = S.shape
    blocks = query_blocks(Tq, bs, q_chunk) if mask == MASK_TOKEN else None
    out = []
    for b in range(B):
        ob = []
        for h in range(H):
            oh = []
            mem = []
            if mem_ids is not None:
                mem = [int(m) for m in mem_ids[b, h] if m >= 0 and blk_len[b, h, m] > 0]
            for i in range(nQB):
                cands = []
                for j, g in zip(win_ids, win_frame):
                    j = int(j)
                    if blk_len[b, h, j] <= 0:
                        continue
                    if mask == MASK_TOKEN:
                        last_q = q_pos0 + blocks[i][0] + blocks[i][1] - 1
                        if blk_pos[b, h, j] > last_q:
                            continue
                    cands.append((j, int(g)))
                fs = _frame_scores(cands, S[b, h, i], blk_len[b, h])
                frames = sorted(fs, key=lambda g: (-fs[g], g))[:max(F, 0)]
                kept = set(frames)
                order = sorted([j for j, g in cands if g in kept], key=lambda j: (-S[b, h, i, j], j))
                local = order[:min(k, len(order))]
                oh.append(sorted(set(mem) | set(local)))
            ob.append(oh)
        out.append(ob)
    return out


def lists_to_arrays(A, Amax: int):
    """Pack attended lists into idx [B,H,nQB,Amax] (padding -1) and cnt [B,H,nQB]."""
    B, H, nQB = len(A), len(A[0]), len(A[0][0])
    idx = np.full((B, H, nQB, Amax), -1, dtype=np.int32)
    cnt = np.zeros((B, H, nQB), dtype=np.int32)
    for b in range(B):
        for h in range(H):
            for i in range(nQB):
                a = A[b][h][i]
                if len(a) > Amax:
                    raise ValueError("attended list longer than Amax")
                idx[b, h, i, :len(a)] = a
                cnt[b, h, i] = len(a)
    return idx, cnt


# ---------------------------------------------------------------------------
# a6  hybrid (persistent + local) block-sparse attention, forward
# ---------------------------------------------------------------------------

def _gather_keys(kpool, vpool, blk_len, blk_pos, b, h, ids):
    ks, vs, pos = [], [], []
    for j in ids:
        n = int(blk_len[b, h, j])
        ks.append(kpool[b, h, j, :n].astype(np.float64))
        vs.append(vpool[b, h, j, :n].astype(np.float64))
        p0 = int(blk_pos[b, h, j]) if blk_pos is not None else 0
        pos.append(p0 + np.arange(n))
    D = kpool.shape[-1]
    if not ks:
        return np.zeros((0, D)), np.zeros((0, D)), np.zeros(0, dtype=np.int64)
    return np.concatenate(ks), np.concatenate(vs), np.concatenate(pos)


def _logits(qi, kc, scale, mask, q_rows_pos, k_pos):
    s = scale * (qi @ kc.T)
    if mask == MASK_TOKEN:
        s = np.where(k_pos[None, :] > q_rows_pos[:, None], -np.inf, s)
    return s


def _softmax_rows(s):
    """Row-wise softmax of logits s [n, keys] and its log-normaliser.

    A row whose logits are all -inf (no visible key) gets P = 0, LSE = -inf."""
    has = np.isfinite(s).any(axis=1)
    mx = np.where(has, np.max(np.where(np.isfinite(s), s, -np.inf), axis=1, initial=-np.inf), 0.0)
    mx = np.where(has, mx, 0.0)
    e = np.exp(s - mx[:, None])
    z = e.sum(axis=1)
    P = np.where(has[:, None], e / np.where(has, z, 1.0)[:, None], 0.0)
    lse = np.where(has, mx + np.log(np.where(has, z, 1.0)), -np.inf)
    return P, lse


def attention_fwd(q, kpool, vpool, blk_len, blk_pos, idx, cnt, scale: float,
                  mask: int = MASK_CHUNK, q_pos0: int = 0, q_chunk: int = 0):
    """One softmax over the union of the attended blocks of each query block (R12).

    O_r = sum_c softmax_c(scale * <Q_r, K_c>) V_c over the valid tokens c of
    the blocks idx[b,h,i,:cnt] (token mask: only c with position <= the query
    position).  LSE_r = log sum_c exp(scale * <Q_r, K_c>) (natural log).
    A row with no visible key gets O = 0 and LSE = -inf.

    q: [B,H,Tq,D]; kpool/vpool [B,H,NB,bs,D]; idx [B,H,nQB,Amax]; cnt [B,H,nQB]."""
    B, H, Tq, D = q.shape
    bs = kpool.shape[3]
    O = np.zeros((B, H, Tq, D))
    LSE = np.full((B, H, Tq), -np.inf)
    for b in range(B):
        for h in range(H):
            for i, (r0, n) in enumerate(query_blocks(Tq, bs, q_chunk)):
                ids = [int(x) for x in idx[b, h, i, :cnt[b, h, i]]]
                kc, vc, kpos = _gather_keys(kpool, vpool, blk_len, blk_pos, b, h, ids)
                if kc.shape[0] == 0:
                    continue
                qi = q[b, h, r0:r0 + n].astype(np.float64)
                s = _logits(qi, kc, scale, mask, q_pos0 + r0 + np.arange(n), kpos)
                P, lse = _softmax_rows(s)
                O[b, h, r0:r0 + n] = P @ vc
                LSE[b, h, r0:r0 + n] = lse
    return O, LSE


# ---------------------------------------------------------------------------
# a7  backward
# ---------------------------------------------------------------------------

def attention_bwd(q, kpool, vpool, blk_len, blk_pos, idx, cnt, dO, scale: float,
                  mask: int = MASK_CHUNK, q_pos0: int = 0, q_chunk: int = 0):
    """Gradients of ``attention_fwd`` w.r.t. Q, the key pool and the value pool.

    The attended lists are constants (R13: no gradient through selection).
    For each query block with P = softmax(scale * Q K^T) over its gathered
    keys: dV += P^T dO, dP = dO V^T, dS = P * (dP - rowsum(P * dP)),
    dQ = scale * dS K, dK += scale * dS^T Q; key/value gradients are added back
    to the block rows they were gathered from."""
    B, H, Tq, D = q.shape
    bs = kpool.shape[3]
    dq = np.zeros((B, H, Tq, D))
    dk = np.zeros(kpool.shape)
    dv = np.zeros(vpool.shape)
    for b in range(B):
        for h in range(H):
            for i, (r0, n) in enumerate(query_blocks(Tq, bs, q_chunk)):
                ids = [int(x) for x in idx[b, h, i, :cnt[b, h, i]]]
                kc, vc, kpos = _gather_keys(kpool, vpool, blk_len, blk_pos, b, h, ids)
                if kc.shape[0] == 0:
                    continue
                qi = q[b, h, r0:r0 + n].astype(np.float64)
                doi = dO[b, h, r0:r0 + n].astype(np.float64)
                s = _logits(qi, kc, scale, mask, q_pos0 + r0 + np.arange(n), kpos)
                Pm, _ = _softmax_rows(s)
                dvc = Pm.T @ doi
                dP = doi @ vc.T
                dS = Pm * (dP - (Pm * dP).sum(axis=1, keepdims=True))
                dq[b, h, r0:r0 + n] = scale * (dS @ kc)
                dkc = scale * (dS.T @ qi)
                off = 0
                for j in ids:
                    m = int(blk_len[b, h, j])
                    dk[b, h, j, :m] += dkc[off:off + m]
                    dv[b, h, j, :m] += dvc[off:off + m]
                    off += m
    return dq, dk, dv


# ---------------------------------------------------------------------------
# NEXT-2  the recurrent trainable path: gradients through the memory update
# ---------------------------------------------------------------------------

def update_memory_vjp(dk_after, dv_after, info, P: int):
    """Backward of ``update_memory`` for the key and value rows.

    Sparse Forcing trains with the dynamically updated cache, and its memory
    learns to compress, keep and refresh persistent blocks (gist.science/es,
    section 2 "Entrenamiento"; the abstract on the shd-paper.top page), so the
    loss reaches a block's keys and values also through the slots it was
    copied or merged into.  Every slot after the update is a weighted row-wise
    sum of pre-update blocks (``info[(b,h)]["compose"]``, R5: rows past a
    block's length count as zero; the rounding to storage is taken as the
    identity), so the vector-Jacobian product is that sum transposed:

        d(pre id j)[r] += weight * d(slot s)[r]   for r < rows, every term (j,
        weight, rows) of slot s;

    blocks that are not slots keep their own gradient (the update reads them
    only), and a pre-update slot gets only what reaches it through the terms.
    The selection and merge decisions are constants (R13).

    dk_after / dv_after: [B,H,NB,bs,D] gradients w.r.t. the pool after the
    update.  Returns the gradients w.r.t. the pool before it."""
    dk = np.array(dk_after, dtype=np.float64, copy=True)
    dv = np.array(dv_after, dtype=np.float64, copy=True)
    dk[:, :, :P] = 0.0
    dv[:, :, :P] = 0.0
    for (b, h), inf in info.items():
        for s, terms in inf["compose"].items():
            for j, wgt, n in terms:
                dk[b, h, j, :n] += wgt * dk_after[b, h, s, :n]
                dv[b, h, j, :n] += wgt * dv_after[b, h, s, :n]
    return dk, dv


def rollout_bwd(steps, P: int, place, W: int, T_c: int, scale: float, mask: int = MASK_CHUNK):
    """Gradients of a rollout's loss sum_t <O_t, dO_t> w.r.t. every chunk's
    queries, keys and values, through the attention of each step and through
    the persistent memory (the recurrent trainable path).

    ``steps[t]`` holds what step t of the forward used: q [B,H,T_c,D], the
    pool after its memory update (kp, vp, bl, bp), its lists (idx, cnt), the
    update's ``info`` (None if no update ran) and dO.  Going back in time, the
    gradient of the slots after update t is what attention t gives them plus
    what the later steps pass back to the slots before update t+1; the
    update's backward (``update_memory_vjp``) then hands the slots' gradient
    to the blocks they came from.  Before update t the ring holds chunks
    t-W .. t (``place``); a ring block's gradient belongs to the chunk in it.

    Returns (dq, dk, dv): lists over t of [B,H,T_c,D] (dq for step t's
    queries; dk, dv for chunk t's keys and values)."""
    T = len(steps)
    B, H, NB, bs, D = steps[0]["kp"].shape
    Gk = np.zeros((B, H, P, bs, D))
    Gv = np.zeros((B, H, P, bs, D))
    dq = [None] * T
    dkc = [np.zeros((B, H, T_c, D)) for _ in range(T)]
    dvc = [np.zeros((B, H, T_c, D)) for _ in range(T)]
    for t in reversed(range(T)):
        st = steps[t]
        dq[t], dk, dv = attention_bwd(st["q"], st["kp"], st["vp"], st["bl"], st["bp"],
                                      st["idx"], st["cnt"], st["dO"], scale, mask, t * T_c)
        if P:
            dk[:, :, :P] += Gk
            dv[:, :, :P] += Gv
        if st["info"] is not None:
            dk, dv = update_memory_vjp(dk, dv, st["info"], P)
        if P:
            Gk, Gv = dk[:, :, :P].copy(), dv[:, :, :P].copy()
        for c in range(max(0, t - W), t + 1):
            for pid, (r0, n) in zip(place.chunk_ids(c), place.blocks):
                dkc[c][:, :, r0:r0 + n] += dk[:, :, pid, :n]
                dvc[c][:, :, r0:r0 + n] += dv[:, :, pid, :n]
    return dq, dkc, dvc


# ---------------------------------------------------------------------------
# the chunk step: the local window, the blocks leaving it, and where blocks sit
# ---------------------------------------------------------------------------

def window_chunks(t: int, W: int):
    """The chunks of the local window L_t while chunk t is generated (R7): the
    W most recent chunks, chunk t itself included; fewer while the rollout is
    shorter than W chunks (Sparse Forcing, gist.science/es, section 2
    "Arquitectura Propuesta", item "Ventana Local")."""
    return [c for c in range(t - W + 1, t + 1) if c >= 0]


def leaving_chunk(t: int, W: int):
    """The chunk that drops out of the local window when chunk t arrives (R14):
    the chunk of L_{t-1} that is not in L_t, or None while the window is still
    filling.  Its blocks are the new candidates of the memory update
    (section 2 "Arquitectura Propuesta", item "Mecanismo de Actualización":
    Top-C retention over the blocks that leave the local window)."""
    if t == 0:
        return None
    gone = set(window_chunks(t - 1, W)) - set(window_chunks(t, W))
    assert len(gone) <= 1
    return gone.pop() if gone else None


def older_chunks(t: int, W: int):
    """Every chunk before chunk t that is not in its window L_t: the chunks a
    snapshot step offers to the persistent memory, and the chunks the
    trainable path's persistent set is chosen from (R13)."""
    win = set(window_chunks(t, W))
    return [c for c in range(t) if c not in win]


class PoolPlacement:
    """Physical ids of the blocks in the pool of one (b, h).

    The library addresses blocks by physical id in a pool [NB, bs, D] per
    (b, h).  The convention below is the one the tests and the engine both
    follow (each side writes it on its own):

    * ids [0, P) are the persistent slots (P = 0: no slots);
    * then positions of nb_c ids each, one chunk per position: chunk t at
      position t when every chunk stays resident (snapshot), or at position
      t mod (W + 1) in a rollout, whose ring is one chunk longer than the
      window so that the chunk leaving the window is still readable while the
      memory update of the step consumes it (R14);
    * block j of chunk t has the global (source) id t * nb_c + j.
    """

    def __init__(self, P: int, T_c: int, bs: int, W: int, n_chunks: int, ring: bool):
        self.P = P
        self.blocks = chunk_blocks(T_c, bs)
        self.nb_c = len(self.blocks)
        self.positions = W + 1 if ring else n_chunks
        self.ring = ring
        self.NB = P + self.positions * self.nb_c

    def chunk_ids(self, t: int):
        pos = t % self.positions if self.ring else t
        assert 0 <= pos < self.positions
        first = self.P + pos * self.nb_c
        return [first + j for j in range(self.nb_c)]

    def global_ids(self, t: int):
        return [t * self.nb_c + j for j in range(self.nb_c)]


class OracleLayer:
    """The oracle's state of one attention layer, advanced chunk by chunk.

    One step of chunk t follows the order taken in R14: the chunk's keys and
    values are written into their blocks, then the blocks are scored, the
    persistent memory is updated with the blocks that leave the window as new
    candidates (a snapshot step offers every chunk older than the window to an
    empty memory), the local Top-K is selected and the chunk's queries attend
    the union of the memory and their local blocks.  Attention takes bf16
    inputs (R17: an fp32 cache is attended through bf16 copies)."""

    def __init__(self, B, H, D, bs, T_c, P, n_sink, W, k, policy, mask, store, n_chunks,
                 ring):
        self.B, self.H, self.D, self.bs, self.T_c = B, H, D, bs, T_c
        self.P, self.n_sink, self.W, self.k = P, n_sink, W, k
        self.policy, self.mask, self.store, self.ring = policy, mask, store, ring
        self.scale = 1.0 / math.sqrt(D)
        self.place = PoolPlacement(P, T_c, bs, W, n_chunks, ring)
        NB = self.place.NB
        self.kp = np.zeros((B, H, NB, bs, D))
        self.vp = np.zeros_like(self.kp)
        self.bl = np.zeros((B, H, NB), dtype=np.int32)
        self.bp = np.zeros((B, H, NB), dtype=np.int32)
        self.kb = np.zeros((B, H, NB, D))
        self.ss = np.full((B, H, P), -1, dtype=np.int64)
        self.sw = np.zeros((B, H, P))

    @classmethod
    def of(cls, w):
        """Build from any object carrying the layer's shape as attributes."""
        return cls(w.B, w.H, w.D, w.bs, w.chunk_tokens, w.P if w.slots_in_pool else 0,
                   w.n_sink, w.W, w.k, w.policy, w.mask, w.dtype, w.n_chunks, w.rollout)

    @property
    def Amax(self):
        return self.P + self.k

    def write_chunk(self, t, k, v):
        """Chunk t's keys and values [B,H,T_c,D] into its blocks; padding rows are zero."""
        for pid, (r0, n) in zip(self.place.chunk_ids(t), self.place.blocks):
            self.kp[:, :, pid] = 0.0
            self.vp[:, :, pid] = 0.0
            self.kp[:, :, pid, :n] = k[:, :, r0:r0 + n]
            self.vp[:, :, pid, :n] = v[:, :, r0:r0 + n]
            self.bl[:, :, pid] = n
            self.bp[:, :, pid] = t * self.T_c + r0

    def window_ids(self, t):
        return [p for c in window_chunks(t, self.W) for p in self.place.chunk_ids(c)]

    def candidates(self, t):
        """(physical ids, global ids) offered to the memory at step t."""
        if self.ring:
            c = leaving_chunk(t, self.W)
            chunks = [] if c is None else [c]
        else:
            chunks = older_chunks(t, self.W)
        return ([p for c in chunks for p in self.place.chunk_ids(c)],
                [g for c in chunks for g in self.place.global_ids(c)])

    def step(self, t, q, pool_ids=None, attend=True):
        """Score -> update -> select -> attend for chunk t (already written).

        pool_ids: the blocks whose pooled keys are (re)computed (default: the
        chunk's own blocks; older pooled keys are kept).  Returns every
        intermediate result."""
        ids = self.place.chunk_ids(t) if pool_ids is None else list(pool_ids)
        q_bar, self.kb, S, m = score_blocks(q, self.kp, self.bl, ids, self.kb, self.scale,
                                            self.bs)
        pre_kb = self.kb.copy()
        ci, cs = self.candidates(t)
        info = None
        if self.P and ci:
            out = update_memory(self.kp, self.vp, self.bl, self.bp, self.kb, self.ss, self.sw,
                                ci, cs, m, self.P, self.n_sink, self.policy, self.store)
            self.kp, self.vp, self.bl, self.bp, self.kb, self.ss, self.sw, info = out
        mem = (np.broadcast_to(np.arange(self.P), (self.B, self.H, self.P))
               if self.P else None)
        A = select_local(S, self.window_ids(t), self.k, mem, self.bl, self.mask,
                         t * self.T_c, self.bp, self.bs, self.T_c)
        idx, cnt = lists_to_arrays(A, self.Amax)
        res = dict(q_bar=q_bar, k_bar=pre_kb, S=S, m=m, info=info, A=A, idx=idx, cnt=cnt,
                   cand_ids=ci, cand_src=cs, win_ids=self.window_ids(t), kpool=self.kp,
                   vpool=self.vp, blk_len=self.bl, blk_pos=self.bp, k_bar2=self.kb,
                   slot_src=self.ss, slot_w=self.sw)
        if attend:
            q16, k16, v16 = round_bf16(q), round_bf16(self.kp), round_bf16(self.vp)
            res["O"], res["lse"] = attention_fwd(q16, k16, v16, self.bl, self.bp, idx, cnt,
                                                 self.scale, self.mask, t * self.T_c)
            res.update(q16=q16, k16=k16, v16=v16)
        return res


def trainable_lists(q, kpool, blk_len, T_c, bs, P, W, k, scale, density=None):
    """Attended lists of the trainable path over a whole sequence of chunks
    (R13): no slots; chunk t's blocks sit at ids t*nb_c .. (t+1)*nb_c - 1 and
    selection is one-shot per query chunk t:

    * density None: the persistent set is the top-P blocks of the chunks older
      than the window by chunk t's memory score, united with the top-k window
      blocks of each query block by block score (the inference rule applied
      with an empty memory refilled for every chunk);
    * density d (R18): the top ceil(d * n) blocks by block score of the n
      chunk-causally allowed blocks (every block of chunks 0..t).

    q: [B,H,n_chunks*T_c,D]; kpool [B,H,n_chunks*nb_c,bs,D].  Returns
    (idx, cnt) with Amax = P + k (density None) or all blocks."""
    B, H = q.shape[:2]
    n_chunks = q.shape[2] // T_c
    place = PoolPlacement(0, T_c, bs, W, n_chunks, ring=False)
    NB = place.NB
    kb = pool_keys(kpool, blk_len, range(NB), np.zeros((B, H, NB, q.shape[3])))
    nb_c = place.nb_c
    A = [[[None] * (n_chunks * nb_c) for _ in range(H)] for _ in range(B)]
    for t in range(n_chunks):
        S = block_scores(pool_queries(q[:, :, t * T_c:(t + 1) * T_c], bs), kb, scale)
        if density is None:
            older = [p for c in older_chunks(t, W) for p in place.chunk_ids(c)]
            mem_ids = np.full((B, H, P), -1, dtype=np.int64)
            if older:
                chosen = select_local(memory_scores(S)[:, :, None, :], older, P, None, blk_len)
                for b in range(B):
                    for h in range(H):
                        mem_ids[b, h, :len(chosen[b][h][0])] = chosen[b][h][0]
            win = [p for c in window_chunks(t, W) for p in place.chunk_ids(c)]
            At = select_local(S, win, k, mem_ids, blk_len)
        else:
            allowed = [p for c in range(t + 1) for p in place.chunk_ids(c)]
            At = select_local(S, allowed, int(math.ceil(density * len(allowed))), None, blk_len)
        for b in range(B):
            for h in range(H):
                for i in range(nb_c):
                    A[b][h][t * nb_c + i] = At[b][h][i]
    return lists_to_arrays(A, P + k if density is None else NB)
