"""Per-layer PBSA state on the device and the chunk step that drives it.

A ``PbsaLayer`` owns the device buffers of one attention layer: the block
pool (persistent slots + window ring or snapshot chunks), its metadata, the
pooled keys, scores, attended lists, outputs and workspace.  ``step`` runs the
hot path of one chunk -- score -> update memory -> select -> attend -- as four
calls into the C ABI; the host side only decides which physical ids are passed
(ring bookkeeping) and never touches tensor data.
"""
from __future__ import annotations

import math

import torch

from . import pbsa as K
from .layout import PoolLayout


def _i32(x, device):
    return torch.as_tensor(x, dtype=torch.int32, device=device).contiguous()


class PbsaLayer:
    """cfg: any object with the layer's shape as attributes -- B, H, D, bs,
    dtype ("bf16" / "f32"), chunk_tokens, P, n_sink, W, k, policy, mask,
    n_chunks (resident chunks of a snapshot, or the rollout's length) and
    rollout (ring of W + 1 chunk positions)."""

    def __init__(self, cfg, device="cuda"):
        self.w = w = cfg
        self.layout = lay = PoolLayout.of(cfg)
        self.dev = torch.device(device)
        B, H, D, bs = w.B, w.H, w.D, w.bs
        self.scale = 1.0 / math.sqrt(D)
        self.tdtype = torch.bfloat16 if w.dtype == "bf16" else torch.float32
        self.d = K.dims(B, H, D, bs, self.scale, self.tdtype)
        self.dbf = K.dims(B, H, D, bs, self.scale, torch.bfloat16)
        self.P = lay.P
        self.NB = lay.NB
        self.nQB = lay.nb_c
        self.Amax = self.P + w.k
        NB, P = self.NB, self.P
        dev = self.dev
        self.kpool = torch.zeros(B, H, NB, bs, D, dtype=self.tdtype, device=dev)
        self.vpool = torch.zeros_like(self.kpool)
        self.blk_len = torch.zeros(B, H, NB, dtype=torch.int32, device=dev)
        self.blk_pos = torch.zeros(B, H, NB, dtype=torch.int32, device=dev)
        self.k_bar = torch.zeros(B, H, NB, D, dtype=torch.float32, device=dev)
        self.slot_src = torch.full((B, H, max(P, 1)), -1, dtype=torch.int32, device=dev)
        self.slot_w = torch.zeros(B, H, max(P, 1), dtype=torch.float32, device=dev)
        self.q = torch.zeros(B, H, w.chunk_tokens, D, dtype=self.tdtype, device=dev)
        self.q_bar = torch.zeros(B, H, self.nQB, D, dtype=torch.float32, device=dev)
        self.scores = torch.zeros(B, H, self.nQB, NB, dtype=torch.float32, device=dev)
        self.mem = torch.zeros(B, H, NB, dtype=torch.float32, device=dev)
        self.idx = torch.full((B, H, self.nQB, self.Amax), -1, dtype=torch.int32, device=dev)
        self.cnt = torch.zeros(B, H, self.nQB, dtype=torch.int32, device=dev)
        self.o = torch.zeros(B, H, w.chunk_tokens, D, dtype=torch.bfloat16, device=dev)
        self.lse = torch.zeros(B, H, w.chunk_tokens, dtype=torch.float32, device=dev)
        self.mem_ids = _i32(torch.arange(P).expand(B, H, P), dev) if P else None
        max_cand = lay.nb_c * (len(lay.older_chunks(w.n_chunks - 1)) if not w.rollout else 1)
        self.max_cand = max(max_cand, 1)
        ws = K.update_memory_workspace(self.d, max(P, 1), self.max_cand)
        self.ws = torch.empty(ws, dtype=torch.uint8, device=dev)
        # the fused routing call's workspace: barrier words (zero) + update plan
        self.rws = torch.zeros(K.route_workspace(self.d, P, self.max_cand), dtype=torch.uint8,
                               device=dev)
        self._ids = {}
        # an empty id list: a score call that pools only the queries
        self.no_ids = torch.zeros(0, dtype=torch.int32, device=dev)
        if self.tdtype != torch.bfloat16:
            # attention runs on bf16 copies of an fp32 cache (R17)
            self.q16 = torch.zeros(B, H, w.chunk_tokens, D, dtype=torch.bfloat16, device=dev)
            self.k16 = torch.zeros(B, H, NB, bs, D, dtype=torch.bfloat16, device=dev)
            self.v16 = torch.zeros_like(self.k16)

    # ------------------------------------------------------------ id lists
    def ids(self, key, values):
        t = self._ids.get(key)
        if t is None:
            t = _i32(list(values), self.dev)
            self._ids[key] = t
        return t

    def chunk_ids(self, t):
        return self.ids(("chunk", self.layout.position(t)), self.layout.chunk_phys_ids(t))

    def window_ids(self, t):
        lay = self.layout
        chunks = lay.window_chunks(t)
        key = ("win",) + tuple(lay.position(c) for c in chunks)
        return self.ids(key, [p for c in chunks for p in lay.chunk_phys_ids(c)])

    def all_ids(self):
        """Every resident chunk block (a snapshot's cache)."""
        lay = self.layout
        return self.ids(("all",), [p for c in range(lay.positions) for p in lay.chunk_phys_ids(c)])

    # ------------------------------------------------------------ state
    def reset_memory(self):
        """Empty persistent memory (snapshot steps start from it)."""
        if self.P:
            self.slot_src.fill_(-1)
            self.slot_w.zero_()
            self.blk_len[:, :, :self.P] = 0
            self.blk_pos[:, :, :self.P] = 0
            self.k_bar[:, :, :self.P] = 0

    def set_chunk_meta(self, t):
        """Lengths and positions of chunk t's blocks (where the ring puts them)."""
        lay = self.layout
        for j, (pid, n) in enumerate(zip(lay.chunk_phys_ids(t), lay.block_lens())):
            self.blk_len[:, :, pid] = n
            self.blk_pos[:, :, pid] = t * lay.chunk_tokens + j * lay.bs

    def write_chunk(self, t, k_chunk, v_chunk):
        """Place a chunk's K/V [B,H,T_c,D] into its blocks (the caller's cache append)."""
        w = self.w
        ids = self.layout.chunk_phys_ids(t)
        lens = self.layout.block_lens()
        for j, pid in enumerate(ids):
            r0 = j * w.bs
            self.kpool[:, :, pid, :lens[j]] = k_chunk[:, :, r0:r0 + lens[j]]
            self.vpool[:, :, pid, :lens[j]] = v_chunk[:, :, r0:r0 + lens[j]]
            if lens[j] < w.bs:
                self.kpool[:, :, pid, lens[j]:] = 0
                self.vpool[:, :, pid, lens[j]:] = 0
        self.set_chunk_meta(t)

    def append(self, t, k_chunk, v_chunk, stream=None):
        """Chunk t's K/V [B,H,T_c,D] into its blocks with their pooled keys in the
        same pass (pbsa_append_chunk); the next score call then pools only the
        queries (``step(t, appended=True)``)."""
        w = self.w
        K.append_chunk(self.d, k_chunk, v_chunk, w.chunk_tokens, t * w.chunk_tokens, self.kpool,
                       self.vpool, self.NB, self.chunk_ids(t), self.blk_len, self.blk_pos,
                       self.k_bar, stream)

    # ------------------------------------------------------------ the hot path
    def score(self, t, pool_ids=None, stream=None):
        w = self.w
        pids = self.chunk_ids(t) if pool_ids is None else pool_ids
        K.score_blocks(self.d, self.q, w.chunk_tokens, self.kpool, self.NB, self.blk_len, pids,
                       pids.numel(), self.q_bar, self.k_bar, self.scores, self.mem, stream)

    def update(self, cand_ids, cand_src, stream=None):
        if self.P == 0 or cand_ids.numel() == 0:
            return
        K.update_memory(self.d, self.kpool, self.vpool, self.NB, self.blk_len, self.blk_pos,
                        self.k_bar, self.P, self.w.n_sink, self.slot_src, self.slot_w, cand_ids,
                        cand_src, cand_ids.numel(), self.mem, self.w.policy, self.ws, stream)

    def select(self, t, stream=None):
        w = self.w
        win = self.window_ids(t)
        K.select_local(self.d, self.scores, self.nQB, self.NB, win, win.numel(), w.k,
                       self.mem_ids, self.P, self.blk_len, w.mask, t * w.chunk_tokens,
                       self.blk_pos, w.chunk_tokens, self.idx, self.cnt, self.Amax, 0, self.nQB,
                       stream)

    def frame_labels(self, t, frame_tokens):
        """Frame of each window entry (window order) for the two-level selection:
        the window's chunks in order, each cut into frames of frame_tokens rows;
        a block belongs to the frame its first row falls in.  Returns (labels on
        the device, number of frames)."""
        lay = self.layout
        chunks = lay.window_chunks(t)
        per = -(-lay.chunk_tokens // frame_tokens)
        labels = [ci * per + (j * lay.bs) // frame_tokens
                  for ci in range(len(chunks)) for j in range(lay.nb_c)]
        return self.ids(("frames", len(chunks), frame_tokens), labels), len(chunks) * per

    def select_hier(self, t, F, frame_tokens, stream=None):
        """The two-level local selection (frames of frame_tokens rows, the best F of
        them, then the top-k blocks inside) united with the memory
        (pbsa_select_hier); writes self.idx / self.cnt like select()."""
        w = self.w
        win = self.window_ids(t)
        labels, n_frames = self.frame_labels(t, frame_tokens)
        K.select_hier(self.d, self.scores, self.nQB, self.NB, win, labels, win.numel(), n_frames,
                      F, w.k, self.mem_ids, self.P, self.blk_len, w.mask, t * w.chunk_tokens,
                      self.blk_pos, w.chunk_tokens, self.idx, self.cnt, self.Amax, 0, self.nQB,
                      stream)

    def attend(self, t, stream=None):
        w = self.w
        if self.tdtype == torch.bfloat16:
            q, kp, vp = self.q, self.kpool, self.vpool
        else:
            self.q16.copy_(self.q)
            self.k16.copy_(self.kpool)
            self.v16.copy_(self.vpool)
            q, kp, vp = self.q16, self.k16, self.v16
        K.attn_fwd(self.dbf, q, w.chunk_tokens, t * w.chunk_tokens, kp, vp, self.NB, self.blk_len,
                   self.blk_pos, self.idx, self.cnt, self.Amax, w.mask, self.o, self.lse, stream)

    def candidates(self, t):
        """Blocks that leave the window when chunk t arrives (rollout) or every
        block older than the window (snapshot)."""
        lay = self.layout
        if lay.rollout:
            c = lay.leaving_chunk(t)
            chunks = [] if c is None else [c]
        else:
            chunks = lay.older_chunks(t)
        key = ("cand",) + tuple(chunks) if not lay.rollout else ("cand", t)
        ci = self.ids(key + ("phys",), [p for c in chunks for p in lay.chunk_phys_ids(c)])
        cs = self.ids(key + ("src",), [g for c in chunks for g in lay.chunk_global_ids(c)])
        return ci, cs

    def route(self, t, stream=None, appended=False):
        """Score -> update -> select for chunk t in one call (pbsa_route_step).
        appended: the chunk's pooled keys were written by append()."""
        w = self.w
        pids = self.chunk_ids(t)
        ci, cs = self.candidates(t)
        win = self.window_ids(t)
        n_cand = ci.numel() if self.P else 0
        K.route_step(self.d, self.rws, stream,
                     q=self.q, Tq=w.chunk_tokens, kpool=self.kpool, vpool=self.vpool, NB=self.NB,
                     blk_len=self.blk_len, blk_pos=self.blk_pos, pool_ids=pids,
                     n_pool=0 if appended else pids.numel(), q_bar=self.q_bar, k_bar=self.k_bar, scores=self.scores,
                     mem_score=self.mem, P=self.P, n_sink=w.n_sink,
                     slot_src=self.slot_src if self.P else None,
                     slot_w=self.slot_w if self.P else None,
                     cand_ids=ci if n_cand else None, cand_src=cs if n_cand else None,
                     n_cand=n_cand, policy=w.policy, win_ids=win, n_win=win.numel(), k=w.k,
                     mem_ids=self.mem_ids, n_mem=self.P, mask=w.mask, q_pos0=t * w.chunk_tokens,
                     idx=self.idx, cnt=self.cnt, Amax=self.Amax)

    def step(self, t, stream=None, fused=False, appended=False):
        """Score -> update -> select -> attend for chunk t (its Q already in self.q,
        its K/V already in the pool).  fused: the first three as one routing call
        (pbsa_route_step); the default is the per-call path, which is the faster
        schedule on the decode and rollout shapes.  appended: the chunk's K/V
        came in through append(), so its pooled keys exist and only the queries
        are pooled."""
        if fused:
            self.route(t, stream=stream, appended=appended)
        else:
            self.score(t, pool_ids=self.no_ids if appended else None, stream=stream)
            ci, cs = self.candidates(t)
            self.update(ci, cs, stream=stream)
            self.select(t, stream=stream)
        self.attend(t, stream=stream)


class PbsaTrain:
    """Device state of the trainable path: a whole sequence of query chunks
    attending its own block-tiled cache (no slots; the persistent set names
    cache blocks in place), with forward and backward through the C ABI.

    Lists are one-shot per query chunk t: the persistent set is the top-P
    blocks older than the window by chunk t's memory score, the local set the
    top-k window blocks per query block (``lists()``), or, for the density
    sweep, the top ceil(d * allowed) of all allowed blocks per query block
    (``lists(density=d)``)."""

    def __init__(self, cfg, device="cuda"):
        self.w = w = cfg
        self.layout = lay = PoolLayout(w.chunk_tokens, w.bs, 0, w.W, w.n_chunks, rollout=False,
                                       slots_in_pool=False)
        dev = torch.device(device)
        self.dev = dev
        B, H, D, bs = w.B, w.H, w.D, w.bs
        self.scale = 1.0 / math.sqrt(D)
        self.T = w.n_chunks * w.chunk_tokens
        self.G = w.n_chunks
        self.nb_c = lay.nb_c
        self.nQB = w.n_chunks * lay.nb_c
        self.NB = lay.NB
        self.d = K.dims(B, H, D, bs, self.scale, torch.bfloat16, q_chunk=w.chunk_tokens)
        self.d1 = K.dims(B, H, D, bs, self.scale, torch.bfloat16)
        self.q = torch.zeros(B, H, self.T, D, dtype=torch.bfloat16, device=dev)
        self.kpool = torch.zeros(B, H, self.NB, bs, D, dtype=torch.bfloat16, device=dev)
        self.vpool = torch.zeros_like(self.kpool)
        self.dO = torch.zeros(B, H, self.T, D, dtype=torch.bfloat16, device=dev)
        self.blk_len = torch.zeros(B, H, self.NB, dtype=torch.int32, device=dev)
        self.blk_pos = torch.zeros(B, H, self.NB, dtype=torch.int32, device=dev)
        self.k_bar = torch.zeros(B, H, self.NB, D, dtype=torch.float32, device=dev)
        self.q_bar = torch.zeros(B, H, self.nQB, D, dtype=torch.float32, device=dev)
        self.scores = torch.zeros(B, H, self.nQB, self.NB, dtype=torch.float32, device=dev)
        self.mem = torch.zeros(B, H, self.G, self.NB, dtype=torch.float32, device=dev)
        self.mem_idx = torch.full((B, H, self.G, w.P), -1, dtype=torch.int32, device=dev)
        self.mem_cnt = torch.zeros(B, H, self.G, dtype=torch.int32, device=dev)
        self.Amax = self.NB                   # room for the dense (density 1) lists
        self.idx = torch.full((B, H, self.nQB, self.Amax), -1, dtype=torch.int32, device=dev)
        self.cnt = torch.zeros(B, H, self.nQB, dtype=torch.int32, device=dev)
        self.o = torch.zeros(B, H, self.T, D, dtype=torch.bfloat16, device=dev)
        self.lse = torch.zeros(B, H, self.T, dtype=torch.float32, device=dev)
        self.dq = torch.zeros(B, H, self.T, D, dtype=torch.float32, device=dev)
        self.dk = torch.zeros(B, H, self.NB, bs, D, dtype=torch.float32, device=dev)
        self.dv = torch.zeros_like(self.dk)
        self.ws = torch.empty(K.attn_bwd_workspace(self.d, self.T, self.NB, self.Amax),
                              dtype=torch.uint8, device=dev)
        self.all_ids = _i32(list(range(self.NB)), dev)
        self._ids = {}

    def ids(self, key, values):
        t = self._ids.get(key)
        if t is None:
            t = _i32(list(values), self.dev)
            self._ids[key] = t
        return t

    def set_meta(self):
        lay = self.layout
        for t in range(self.G):
            for j, (pid, n) in enumerate(zip(lay.chunk_phys_ids(t), lay.block_lens())):
                self.blk_len[:, :, pid] = n
                self.blk_pos[:, :, pid] = t * lay.chunk_tokens + j * lay.bs

    def write_chunk(self, t, k_chunk, v_chunk):
        """Chunk t's K/V [B,H,T_c,D] into its blocks (padding rows zero)."""
        lay = self.layout
        for j, (pid, n) in enumerate(zip(lay.chunk_phys_ids(t), lay.block_lens())):
            r0 = j * lay.bs
            self.kpool[:, :, pid].zero_()
            self.vpool[:, :, pid].zero_()
            self.kpool[:, :, pid, :n] = k_chunk[:, :, r0:r0 + n]
            self.vpool[:, :, pid, :n] = v_chunk[:, :, r0:r0 + n]

    def lists(self, density=None, stream=None):
        w, lay = self.w, self.layout
        nb_c = lay.nb_c
        K.score_blocks(self.d, self.q, self.T, self.kpool, self.NB, self.blk_len, self.all_ids,
                       self.NB, self.q_bar, self.k_bar, self.scores, self.mem, stream)
        for t in range(self.G):
            if density is None:
                older = [p for c in lay.older_chunks(t) for p in lay.chunk_phys_ids(c)]
                if older:
                    o_ids = self.ids(("older", t), older)
                    K.select_local(self.d1, self.mem, 1, self.NB, o_ids, len(older), w.P, None, 0,
                                   self.blk_len, 0, 0, None, w.bs, self.mem_idx, self.mem_cnt,
                                   w.P, t, self.G, stream)
                win = self.ids(("win", t), [p for c in lay.window_chunks(t)
                                            for p in lay.chunk_phys_ids(c)])
                K.select_local(self.d1, self.scores, nb_c, self.NB, win, win.numel(), w.k,
                               self.mem_idx, w.P, self.blk_len, 0, t * w.chunk_tokens,
                               self.blk_pos, w.chunk_tokens, self.idx, self.cnt, self.Amax,
                               t * nb_c, self.nQB, stream, mem_ld=self.G * w.P,
                               mem_offset=t * w.P)
            else:
                allowed = [p for c in range(t + 1) for p in lay.chunk_phys_ids(c)]
                kd = max(1, int(-(-density * len(allowed) // 1)))
                a_ids = self.ids(("allowed", t), allowed)
                K.select_local(self.d1, self.scores, nb_c, self.NB, a_ids, len(allowed), kd,
                               None, 0, self.blk_len, 0, t * w.chunk_tokens, self.blk_pos,
                               w.chunk_tokens, self.idx, self.cnt, self.Amax, t * nb_c,
                               self.nQB, stream)

    def fwd(self, stream=None):
        K.attn_fwd(self.d, self.q, self.T, 0, self.kpool, self.vpool, self.NB, self.blk_len,
                   self.blk_pos, self.idx, self.cnt, self.Amax, self.w.mask, self.o, self.lse,
                   stream)

    def bwd(self, stream=None):
        K.attn_bwd(self.d, self.q, self.T, 0, self.kpool, self.vpool, self.NB, self.blk_len,
                   self.blk_pos, self.idx, self.cnt, self.Amax, self.w.mask, self.o, self.lse,
                   self.dO, self.dq, self.dk, self.dv, self.ws, stream)


class PbsaRolloutTrain:
    """The recurrent trainable path of a rollout (Sparse Forcing trains with
    the dynamically updated cache): the chunk steps of a ``PbsaLayer`` run
    forward with each step recorded -- its queries, the pool after its memory
    update, its lists, outputs and the update's plan -- and then the backward
    of the loss sum_t <O_t, dO_t> back in time: the attention backward of step
    t (pbsa_attn_bwd) gives the gradient of every pool block it read; the slots
    also receive what the later steps pass back; the memory update's backward
    (pbsa_update_memory_bwd) hands the slots' gradient to the blocks they were
    copied or merged from.  A ring block's gradient belongs to the chunk held
    at that ring position.  Selections and merges are constants."""

    def __init__(self, layer: PbsaLayer):
        self.L = L = layer
        w = L.w
        self.steps = []
        self.plan_bytes = K.update_plan_bytes(L.d, L.P, L.max_cand) if L.P else 0
        self.bwd_ws = torch.empty(K.attn_bwd_workspace(L.dbf, w.chunk_tokens, L.NB, L.Amax),
                                  dtype=torch.uint8, device=L.dev)
        self.upd_ws = (torch.empty(K.update_memory_bwd_workspace(L.d, L.P), dtype=torch.uint8,
                                   device=L.dev) if L.P else None)

    def step(self, t, q, k, v, stream=None):
        """Chunk t's Q/K/V [B,H,T_c,D] (the layer's storage type) through
        score -> update -> select -> attend, recorded for the backward."""
        L = self.L
        L.write_chunk(t, k, v)
        L.q.copy_(q)
        L.score(t, stream=stream)
        ci, cs = L.candidates(t)
        L.update(ci, cs, stream=stream)
        L.select(t, stream=stream)
        L.attend(t, stream=stream)
        n_cand = ci.numel() if L.P else 0
        self.steps.append(dict(
            q=L.q.clone(), kpool=L.kpool.clone(), vpool=L.vpool.clone(),
            blk_len=L.blk_len.clone(), blk_pos=L.blk_pos.clone(), idx=L.idx.clone(),
            cnt=L.cnt.clone(), o=L.o.clone(), lse=L.lse.clone(), n_cand=n_cand,
            plan=L.ws[:self.plan_bytes].clone() if n_cand else None))
        return L.o, L.lse

    def backward(self, dOs, stream=None):
        """dOs: dO [B,H,T_c,D] (bf16) of every recorded step.  Returns (dq, dk,
        dv): float32 [B,H,T_c,D] per step (dq) and per chunk (dk, dv)."""
        L, w = self.L, self.L.w
        lay = L.layout
        T, P, Tc = len(self.steps), L.P, w.chunk_tokens
        shape = (w.B, w.H, Tc, w.D)
        f32 = dict(dtype=torch.float32, device=L.dev)
        dq = [torch.empty(shape, **f32) for _ in range(T)]
        dkc = [torch.zeros(shape, **f32) for _ in range(T)]
        dvc = [torch.zeros(shape, **f32) for _ in range(T)]
        dk = torch.empty(w.B, w.H, L.NB, w.bs, w.D, **f32)
        dv = torch.empty_like(dk)
        Gk = Gv = None
        for t in reversed(range(T)):
            r = self.steps[t]
            K.attn_bwd(L.dbf, r["q"], Tc, t * Tc, r["kpool"], r["vpool"], L.NB, r["blk_len"],
                       r["blk_pos"], r["idx"], r["cnt"], L.Amax, w.mask, r["o"], r["lse"],
                       dOs[t], dq[t], dk, dv, self.bwd_ws, stream)
            if P:
                if Gk is not None:
                    dk[:, :, :P] += Gk
                    dv[:, :, :P] += Gv
                if r["plan"] is not None:
                    K.update_memory_bwd(L.d, L.NB, P, r["n_cand"], r["plan"], dk, dv,
                                        self.upd_ws, stream)
                Gk, Gv = dk[:, :, :P].clone(), dv[:, :, :P].clone()
            for c in range(max(0, t - w.W), t + 1):
                ids = torch.as_tensor(lay.chunk_phys_ids(c), dtype=torch.long, device=L.dev)
                # a chunk's blocks tile its rows in order, only the last one partial
                dkc[c] += dk[:, :, ids].reshape(w.B, w.H, -1, w.D)[:, :, :Tc]
                dvc[c] += dv[:, :, ids].reshape(w.B, w.H, -1, w.D)[:, :, :Tc]
        return dq, dkc, dvc
