"""GPU parity of the attention backward (dQ, dK, dV) against the CPU oracle.

The backward takes the forward's O (bf16) and LSE; here both come from the
oracle (O rounded to bf16), so every input of the GPU call is independent of
the CUDA path.  Gradients are compared with the oracle's exact float64
gradients.  Tolerance: the attention bound plus one bf16 ulp (2^-8) of the
gradient's own scale, because the tensor cores take P and dS rounded to bf16
(relative error <= 2^-9 per term) and gradients, unlike O, are not bounded by
the inputs' range:
    max-abs  <= 2e-2 + 2^-8 * max|ref|,   mean-abs <= 2e-3 + 2^-8 * mean|ref|.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
import pbsa_inputs as PI
from block_sparse_attention_39_b200 import pbsa as K
from tests.gpu_util import band_ok, dev_i32, dev_storage, host

pytestmark = pytest.mark.gpu

G_MAX, G_MEAN = 2e-2, 2e-3
ULP = 2.0 ** -8


def grad_ok(got, ref):
    d = np.abs(got - ref)
    mx, mean = float(d.max()), float(d.mean())
    lim_mx = G_MAX + ULP * float(np.abs(ref).max())
    lim_mean = G_MEAN + ULP * float(np.abs(ref).mean())
    return mx <= lim_mx and mean <= lim_mean, (mx, lim_mx, mean, lim_mean)


@pytest.fixture(autouse=True)
def _status_clean():
    assert torch.cuda.is_available()
    K.get_status()
    yield
    assert K.get_status() == 0


def _run_bwd(d, q, kp, vp, bl, bp, idx, cnt, q_pos0, mask, o, lse, dO):
    B, H, Tq, D = q.shape
    NB, bs = kp.shape[2], kp.shape[3]
    Amax = idx.shape[-1]
    ws = torch.empty(K.attn_bwd_workspace(d, Tq, NB, Amax), dtype=torch.uint8, device="cuda")
    dq = torch.full((B, H, Tq, D), 3.0, dtype=torch.float32, device="cuda")
    dk = torch.full((B, H, NB, bs, D), 3.0, dtype=torch.float32, device="cuda")
    dv = torch.full((B, H, NB, bs, D), 3.0, dtype=torch.float32, device="cuda")
    K.attn_bwd(d, dev_storage(q, "bf16"), Tq, q_pos0, dev_storage(kp, "bf16"),
               dev_storage(vp, "bf16"), NB, dev_i32(bl), dev_i32(bp), dev_i32(idx), dev_i32(cnt),
               Amax, mask, dev_storage(o, "bf16"), torch.from_numpy(lse.astype(np.float32)).cuda(),
               dev_storage(dO, "bf16"), dq, dk, dv, ws)
    torch.cuda.synchronize()
    return host(dq), host(dk), host(dv)


def _errs(got, ref, valid_rows_mask=None):
    d = np.abs(got - ref)
    return float(d.max()), float(d.mean())


def _case(seed, B, H, D, bs, Tq, NB, Amax, mask, empty_rows=True):
    r = np.random.default_rng(seed)
    kp = O.round_bf16(r.standard_normal((B, H, NB, bs, D)))
    vp = O.round_bf16(r.standard_normal((B, H, NB, bs, D)))
    q = O.round_bf16(r.standard_normal((B, H, Tq, D)))
    dO = O.round_bf16(r.standard_normal((B, H, Tq, D)))
    bl = r.integers(1, bs + 1, size=(B, H, NB)).astype(np.int32)
    bp = (np.arange(NB) * bs).astype(np.int32)[None, None, :].repeat(B, 0).repeat(H, 1)
    nQB = -(-Tq // bs)
    idx = np.full((B, H, nQB, Amax), -1, dtype=np.int32)
    cnt = np.zeros((B, H, nQB), dtype=np.int32)
    for b in range(B):
        for h in range(H):
            for i in range(nQB):
                n = int(r.integers(0 if empty_rows else 1, Amax + 1))
                idx[b, h, i, :n] = np.sort(r.choice(NB, size=n, replace=False))
                cnt[b, h, i] = n
    q_pos0 = int(bp[0, 0, -1])
    return q, kp, vp, dO, bl, bp, idx, cnt, q_pos0


@pytest.mark.parametrize("D,bs", [(128, 128), (64, 64), (128, 64), (64, 128)])
@pytest.mark.parametrize("Tq", [50, 200, 384])
@pytest.mark.parametrize("mask", [PI.MASK_CHUNK, PI.MASK_TOKEN])
def test_backward_shapes_ragged_and_empty(D, bs, Tq, mask):
    B, H, NB, Amax = 1, 3, 9, 6
    q, kp, vp, dO, bl, bp, idx, cnt, q_pos0 = _case(D + bs + Tq + 31 * mask, B, H, D, bs, Tq, NB,
                                                    Amax, mask)
    scale = 1 / math.sqrt(D)
    o, lse = O.attention_fwd(q, kp, vp, bl, bp, idx, cnt, scale, mask, q_pos0)
    rq, rk, rv = O.attention_bwd(q, kp, vp, bl, bp, idx, cnt, dO, scale, mask, q_pos0)
    d = K.dims(B, H, D, bs, scale, torch.bfloat16)
    gq, gk, gv = _run_bwd(d, q, kp, vp, bl, bp, idx, cnt, q_pos0, mask, O.round_bf16(o), lse, dO)
    for name, g, rf in (("dq", gq, rq), ("dk", gk, rk), ("dv", gv, rv)):
        ok, info = grad_ok(g, rf)
        assert ok, (name, info)


@pytest.mark.parametrize("bs", [64, 128])
@pytest.mark.parametrize("mask", [PI.MASK_CHUNK, PI.MASK_TOKEN])
def test_backward_chunked_query_tiling(bs, mask):
    # 500 query rows in chunks of 200: blocks tile each chunk on its own
    B, H, D, NB, Amax, Tq, qc = 1, 2, 128, 9, 6, 500, 200
    nQB = len(O.query_blocks(Tq, bs, qc))
    q, kp, vp, dO, bl, bp, idx, cnt, q_pos0 = _case(bs + 7 * mask, B, H, D, bs, nQB * bs, NB, Amax,
                                                    mask)
    q, dO = q[:, :, :Tq], dO[:, :, :Tq]
    scale = 1 / math.sqrt(D)
    o, lse = O.attention_fwd(q, kp, vp, bl, bp, idx, cnt, scale, mask, q_pos0, q_chunk=qc)
    rq, rk, rv = O.attention_bwd(q, kp, vp, bl, bp, idx, cnt, dO, scale, mask, q_pos0, q_chunk=qc)
    d = K.dims(B, H, D, bs, scale, torch.bfloat16, q_chunk=qc)
    gq, gk, gv = _run_bwd(d, q, kp, vp, bl, bp, idx, cnt, q_pos0, mask, O.round_bf16(o), lse, dO)
    for name, g, rf in (("dq", gq, rq), ("dk", gk, rk), ("dv", gv, rv)):
        ok, info = grad_ok(g, rf)
        assert ok, (name, info)


def _train_inputs(w):
    """The trainable shape's inputs on the oracle side: the whole sequence's
    queries and a block pool built through the oracle's own placement (no
    slots, chunk t at ids t*nb_c ..)."""
    chunks = [PI.chunk_tensors(w, t) for t in range(w.n_chunks)]
    q = np.concatenate([c[0] for c in chunks], axis=2)
    orc = O.OracleLayer(w.B, w.H, w.D, w.bs, w.chunk_tokens, 0, 0, w.W, w.k, w.policy, w.mask,
                        w.dtype, w.n_chunks, ring=False)
    for t, c in enumerate(chunks):
        orc.write_chunk(t, c[1], c[2])
    return q, orc.kp, orc.vp, orc.bl, orc.bp, chunks


@pytest.mark.slow
@pytest.mark.parametrize("density", [None, 0.05, 0.50])
def test_backward_train_shape_sampled_heads(density):
    """Forward and backward at the trainable shape's full size (B2 H12, 32 760
    tokens, 259 blocks) with the oracle's lists: the one-shot P32 + top-16
    lists, and the density sweep's 5 % and 50 % lists; the oracle checks two
    sampled heads."""
    w = PI.WORKLOADS["train"]
    q, kpool, vpool, blk_len, blk_pos, _ = _train_inputs(w)
    NB = kpool.shape[2]
    scale = 1 / math.sqrt(w.D)
    T = q.shape[2]
    dO = PI.grad_output(w, T)
    idx, cnt = O.trainable_lists(q, kpool, blk_len, w.chunk_tokens, w.bs, w.P, w.W, w.k, scale,
                                 density=density)
    d = K.dims(w.B, w.H, w.D, w.bs, scale, torch.bfloat16, q_chunk=w.chunk_tokens)
    # forward on the GPU with the oracle's lists (O, LSE feed the backward)
    qd, kd, vd = dev_storage(q, "bf16"), dev_storage(kpool, "bf16"), dev_storage(vpool, "bf16")
    o = torch.empty(w.B, w.H, T, w.D, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(w.B, w.H, T, dtype=torch.float32, device="cuda")
    K.attn_fwd(d, qd, T, 0, kd, vd, NB, dev_i32(blk_len), dev_i32(blk_pos), dev_i32(idx),
               dev_i32(cnt), idx.shape[-1], w.mask, o, lse)
    ws = torch.empty(K.attn_bwd_workspace(d, T, NB, idx.shape[-1]), dtype=torch.uint8,
                     device="cuda")
    dq = torch.empty(w.B, w.H, T, w.D, dtype=torch.float32, device="cuda")
    dk = torch.empty(w.B, w.H, NB, w.bs, w.D, dtype=torch.float32, device="cuda")
    dv = torch.empty_like(dk)
    K.attn_bwd(d, qd, T, 0, kd, vd, NB, dev_i32(blk_len), dev_i32(blk_pos), dev_i32(idx),
               dev_i32(cnt), idx.shape[-1], w.mask, o, lse, dev_storage(dO, "bf16"), dq, dk, dv, ws)
    torch.cuda.synchronize()
    for (b, h) in [(0, 0), (1, 11)]:
        sl = (slice(b, b + 1), slice(h, h + 1))
        ro, rl = O.attention_fwd(q[sl], kpool[sl], vpool[sl], blk_len[sl], blk_pos[sl], idx[sl],
                                 cnt[sl], scale, q_chunk=w.chunk_tokens)
        mx, mean = _errs(host(o[sl]), ro)
        assert mx <= 2e-2 and mean <= 2e-3, ("o", mx, mean)
        rq, rk, rv = O.attention_bwd(q[sl], kpool[sl], vpool[sl], blk_len[sl], blk_pos[sl],
                                     idx[sl], cnt[sl], dO[sl], scale, q_chunk=w.chunk_tokens)
        for name, g, rf in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
            ok, info = grad_ok(host(g[sl]), rf)
            assert ok, (name, density, b, h, info)


@pytest.mark.slow
@pytest.mark.parametrize("density", [None, 0.10, 1.0])
def test_train_lists_built_on_gpu_match_oracle(density):
    """The trainable path's lists, built by the library's own score/select calls
    on a pool the engine filled through its own placement (one-shot per query
    chunk, or top fraction of allowed blocks), equal the oracle's up to
    near-tie swaps."""
    from block_sparse_attention_39_b200.engine import PbsaTrain
    w = PI.variant(PI.WORKLOADS["train"], B=1, H=4)
    q, kpool, vpool, blk_len, blk_pos, chunks = _train_inputs(w)
    T = PbsaTrain(w)
    T.q.copy_(dev_storage(q, "bf16"))
    for t, c in enumerate(chunks):
        T.write_chunk(t, dev_storage(c[1], "bf16"), dev_storage(c[2], "bf16"))
    T.set_meta()
    T.lists(density=density)
    torch.cuda.synchronize()
    idx, cnt = host(T.idx), host(T.cnt)
    scale = 1 / math.sqrt(w.D)
    NB = kpool.shape[2]
    place = O.PoolPlacement(0, w.chunk_tokens, w.bs, w.W, w.n_chunks, ring=False)
    nb_c = place.nb_c
    kb = O.pool_keys(kpool, blk_len, range(NB), np.zeros((w.B, w.H, NB, w.D)))
    for t in range(w.n_chunks):
        qt = q[:, :, t * w.chunk_tokens:(t + 1) * w.chunk_tokens]
        S = O.block_scores(O.pool_queries(qt, w.bs), kb, scale)
        m = O.memory_scores(S)
        older = [p for c in O.older_chunks(t, w.W) for p in place.chunk_ids(c)]
        win = [p for c in O.window_chunks(t, w.W) for p in place.chunk_ids(c)]
        allowed = [p for c in range(t + 1) for p in place.chunk_ids(c)]
        for h in range(w.H):
            for i in range(nb_c):
                r = t * nb_c + i
                lst = [int(x) for x in idx[0, h, r, :cnt[0, h, r]]]
                assert lst == sorted(set(lst))
                if density is None:
                    mem = [x for x in lst if x in set(older)]
                    loc = [x for x in lst if x in set(win)]
                    assert len(mem) + len(loc) == len(lst)
                    if older:
                        ok, _ = band_ok(mem, {j: m[0, h, j] for j in older}, min(w.P, len(older)))
                        assert ok, (t, h, i, "memory")
                    ok, _ = band_ok(loc, {j: S[0, h, i, j] for j in win}, min(w.k, len(win)))
                    assert ok, (t, h, i, "local")
                else:
                    kd = int(np.ceil(density * len(allowed)))
                    ok, _ = band_ok(lst, {j: S[0, h, i, j] for j in allowed}, kd)
                    assert ok, (t, h, i)
