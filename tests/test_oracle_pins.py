"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each test checks the oracle against a closed form, a hand-worked example, an
invariant of the method, brute force, or a library routine (torch float64
attention and autograd).  No GPU is used.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O

RNG = np.random.default_rng(1234)


# --------------------------------------------------------------------------
# storage rounding
# --------------------------------------------------------------------------

def test_round_bf16_matches_torch_conversion():
    x = np.concatenate([RNG.standard_normal(20000) * 10.0 ** RNG.integers(-6, 6, 20000),
                        np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 0.0, 1e30])])
    ours = O.round_bf16(x)
    lib = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    # torch converts float64 -> bf16 directly with round-to-nearest-even
    assert np.array_equal(ours, lib)


# --------------------------------------------------------------------------
# a1 pooling
# --------------------------------------------------------------------------

def test_pool_constant_block_is_the_constant():
    q = np.full((1, 1, 7, 4), 3.25)
    qb = O.pool_queries(q, 4)                 # blocks of 4 and 3 rows
    assert qb.shape == (1, 1, 2, 4)
    assert np.all(qb == 3.25)


def test_pool_partial_block_uses_its_length_only():
    # rows r = r * (1,2,3): the mean of rows 0..n-1 is (n-1)/2 * (1,2,3)
    kpool = np.zeros((1, 1, 2, 8, 3))
    for r in range(8):
        kpool[0, 0, :, r] = r * np.array([1.0, 2.0, 3.0])
    kpool[0, 0, 1, 5:] = 1e9                  # garbage past the length of block 1
    blk_len = np.array([[[8, 5]]])
    kb = O.pool_keys(kpool, blk_len, [0, 1], np.zeros((1, 1, 2, 3)))
    assert np.allclose(kb[0, 0, 0], 3.5 * np.array([1, 2, 3]))
    assert np.allclose(kb[0, 0, 1], 2.0 * np.array([1, 2, 3]))


def test_pool_keeps_unlisted_entries_and_zero_length():
    kpool = RNG.standard_normal((1, 2, 3, 4, 5))
    prev = RNG.standard_normal((1, 2, 3, 5))
    blk_len = np.array([[[4, 0, 2], [4, 0, 2]]])
    kb = O.pool_keys(kpool, blk_len, [1, 2], prev)
    assert np.array_equal(kb[:, :, 0], prev[:, :, 0])
    assert np.all(kb[:, :, 1] == 0)


def test_pool_is_linear():
    a, b = RNG.standard_normal((2, 1, 2, 10, 6))
    lhs = O.pool_queries(2.0 * a - 0.5 * b, 4)
    rhs = 2.0 * O.pool_queries(a, 4) - 0.5 * O.pool_queries(b, 4)
    assert np.allclose(lhs, rhs, atol=1e-13)


# --------------------------------------------------------------------------
# a2 scores
# --------------------------------------------------------------------------

def test_scores_on_an_orthogonal_basis():
    D = 8
    qb = np.zeros((1, 1, 3, D))
    kb = np.zeros((1, 1, 4, D))
    for i in range(3):
        qb[0, 0, i, i] = i + 1.0
    for j in range(4):
        kb[0, 0, j, j % 3] = 10.0 * (j + 1)
    S = O.block_scores(qb, kb, 0.5)
    want = np.zeros((3, 4))
    for i in range(3):
        for j in range(4):
            if j % 3 == i:
                want[i, j] = 0.5 * (i + 1) * 10.0 * (j + 1)
    assert np.allclose(S[0, 0], want)
    m = O.memory_scores(S)
    assert np.allclose(m[0, 0], want.sum(axis=0) / 3)


def test_scores_follow_a_permutation_of_blocks():
    qb = RNG.standard_normal((1, 2, 5, 16))
    kb = RNG.standard_normal((1, 2, 9, 16))
    perm = RNG.permutation(9)
    S = O.block_scores(qb, kb, 0.25)
    Sp = O.block_scores(qb, kb[:, :, perm], 0.25)
    assert np.allclose(Sp, S[:, :, :, perm])


# --------------------------------------------------------------------------
# a3 memory update
# --------------------------------------------------------------------------

def _mem_problem(P, n_slots_used, n_cand, bs=4, D=3, seed=0, merge_w=1.0):
    r = np.random.default_rng(seed)
    NB = P + n_cand
    kpool = r.standard_normal((1, 1, NB, bs, D))
    vpool = r.standard_normal((1, 1, NB, bs, D))
    blk_len = np.zeros((1, 1, NB), dtype=np.int64)
    blk_len[0, 0, :n_slots_used] = bs
    blk_len[0, 0, P:] = r.integers(1, bs + 1, n_cand)
    blk_pos = np.arange(NB).reshape(1, 1, NB) * bs
    slot_src = np.full((1, 1, P), -1)
    slot_src[0, 0, :n_slots_used] = 100 + np.arange(n_slots_used)
    slot_w = np.zeros((1, 1, P))
    slot_w[0, 0, :n_slots_used] = merge_w
    kbar = np.zeros((1, 1, NB, D))
    for j in range(NB):
        n = blk_len[0, 0, j]
        if n:
            kbar[0, 0, j] = kpool[0, 0, j, :n].mean(axis=0)
    cand_ids = np.arange(P, NB)
    cand_src = 200 + np.arange(n_cand)
    m = r.standard_normal((1, 1, NB))
    return kpool, vpool, blk_len, blk_pos, kbar, slot_src, slot_w, cand_ids, cand_src, m


def test_update_hand_example_evict():
    # P = 2, empty memory; candidate scores 0.3, 0.1, 0.5, 0.3 for sources 10..13.
    # Kept: 12 (0.5) and 10 (0.3, wins the tie with 13 by lower source id).
    # New blocks fill free slots in ascending source order: 10 -> slot 0, 12 -> slot 1.
    kp, vp, bl, bp, kb, ss, sw, ci, cs, m = _mem_problem(2, 0, 4)
    cs = np.array([10, 11, 12, 13])
    m[0, 0, 2:6] = [0.3, 0.1, 0.5, 0.3]
    out = O.update_memory(kp, vp, bl, bp, kb, ss, sw, ci, cs, m, 2, 0, O.EVICT, "f64")
    nkp, nvp, nbl, nbp, nkb, nss, nsw, info = out
    assert list(nss[0, 0]) == [10, 12]
    assert list(nsw[0, 0]) == [1.0, 1.0]
    assert np.array_equal(nkp[0, 0, 0], kp[0, 0, 2]) and np.array_equal(nkp[0, 0, 1], kp[0, 0, 4])
    assert np.array_equal(nvp[0, 0, 1], vp[0, 0, 4])
    assert nbl[0, 0, 0] == bl[0, 0, 2] and nbp[0, 0, 1] == bp[0, 0, 4]
    assert np.array_equal(nkb[0, 0, 1], kb[0, 0, 4])
    assert sorted(info[(0, 0)]["losers"]) == [11, 13]


def test_update_hand_example_merge():
    # P = 1, D = 2, blocks of 2 rows.  The slot holds block A (weight 1, 2 rows),
    # the leaving block L has 1 row and the lower score, so it is merged into A:
    #   rows: A = [[1, 2], [3, 4]], L = [[5, 6], <pad 9, 9>]
    #   new = (1*A + 1*[[5,6],[0,0]]) / 2 = [[3, 4], [1.5, 2]], length 2, weight 2,
    #   pooled key = mean of the two rows = [2.25, 3].
    kpool = np.zeros((1, 1, 2, 2, 2))
    kpool[0, 0, 0] = [[1, 2], [3, 4]]
    kpool[0, 0, 1] = [[5, 6], [9, 9]]
    vpool = -kpool
    blk_len = np.array([[[2, 1]]])
    blk_pos = np.array([[[0, 100]]])
    kbar = np.array([[[[2.0, 3.0], [5.0, 6.0]]]])
    out = O.update_memory(kpool, vpool, blk_len, blk_pos, kbar, np.array([[[7]]]),
                          np.array([[[1.0]]]), np.array([1]), np.array([8]),
                          np.array([[[0.9, 0.2]]]), 1, 0, O.MERGE_MEAN, "f64")
    nkp, nvp, nbl, nbp, nkb, nss, nsw, info = out
    assert np.allclose(nkp[0, 0, 0], [[3, 4], [1.5, 2]])
    assert np.allclose(nvp[0, 0, 0], [[-3, -4], [-1.5, -2]])
    assert nbl[0, 0, 0] == 2 and nsw[0, 0, 0] == 2.0 and nss[0, 0, 0] == 7
    assert nbp[0, 0, 0] == 0
    assert np.allclose(nkb[0, 0, 0], [2.25, 3.0])


def test_update_merge_target_is_most_similar_slot():
    # two kept slots with orthogonal pooled keys; a loser aligned with slot 1's key
    P, D = 2, 4
    kpool = np.zeros((1, 1, 3, 1, D))
    kpool[0, 0, 0, 0] = [1, 0, 0, 0]
    kpool[0, 0, 1, 0] = [0, 1, 0, 0]
    kpool[0, 0, 2, 0] = [0.1, 0.9, 0, 0]
    kbar = kpool[:, :, :, 0, :].copy()
    out = O.update_memory(kpool, kpool.copy(), np.ones((1, 1, 3), int), np.zeros((1, 1, 3), int),
                          kbar, np.array([[[5, 6]]]), np.ones((1, 1, 2)), np.array([2]),
                          np.array([9]), np.array([[[1.0, 1.0, -1.0]]]), P, 0, O.MERGE_MEAN, "f64")
    info = out[-1][(0, 0)]
    assert info["target"] == {9: 1}
    assert np.allclose(out[0][0, 0, 1, 0], [0.05, 0.95, 0, 0])
    assert np.allclose(out[0][0, 0, 0, 0], [1, 0, 0, 0])


@pytest.mark.parametrize("policy", [O.EVICT, O.MERGE_MEAN])
@pytest.mark.parametrize("seed", range(6))
def test_update_kept_set_dominates_losers_and_budget_holds(policy, seed):
    r = np.random.default_rng(seed)
    P = int(r.integers(1, 6))
    used = int(r.integers(0, P + 1))
    ncand = int(r.integers(0, 9))
    args = _mem_problem(P, used, ncand, seed=seed)
    m = args[-1]
    m[0, 0, :] = np.round(m[0, 0, :], 1)          # force ties
    out = O.update_memory(*args, P, 0, policy, "f64")
    info = out[-1][(0, 0)]
    keys = info["keys"]
    kept, losers = info["kept"], info["losers"]
    assert len(kept) == min(P, used + ncand)
    assert (out[5][0, 0] >= 0).sum() == len(kept) <= P
    for a in kept:                                   # brute-force pairwise dominance
        for b in losers:
            assert (keys[a] > keys[b]) or (keys[a] == keys[b] and a < b)
    assert sorted(int(s) for s in out[5][0, 0] if s >= 0) == sorted(kept)


def test_update_keeps_everything_when_budget_suffices():
    args = _mem_problem(8, 3, 4, seed=3)
    out = O.update_memory(*args, 8, 0, O.EVICT, "f64")
    assert sorted(int(s) for s in out[5][0, 0] if s >= 0) == sorted([100, 101, 102, 200, 201, 202, 203])
    assert out[-1][(0, 0)]["losers"] == []


def test_update_merge_conserves_mass_over_a_rollout():
    """Sum of w_s * (zero-padded slot content) == sum of every block ever admitted."""
    r = np.random.default_rng(7)
    P, bs, D, nc = 3, 4, 5, 3
    slot_src = np.full((1, 1, P), -1)
    slot_w = np.zeros((1, 1, P))
    kpool = np.zeros((1, 1, P + nc, bs, D))
    vpool = np.zeros_like(kpool)
    blk_len = np.zeros((1, 1, P + nc), dtype=np.int64)
    blk_pos = np.zeros((1, 1, P + nc), dtype=np.int64)
    kbar = np.zeros((1, 1, P + nc, D))
    total_k = np.zeros((bs, D))
    total_v = np.zeros((bs, D))
    admitted = 0
    for step in range(6):
        for c in range(nc):
            n = int(r.integers(1, bs + 1))
            kpool[0, 0, P + c] = r.standard_normal((bs, D))
            vpool[0, 0, P + c] = r.standard_normal((bs, D))
            blk_len[0, 0, P + c] = n
            kbar[0, 0, P + c] = kpool[0, 0, P + c, :n].mean(axis=0)
            total_k[:n] += kpool[0, 0, P + c, :n]
            total_v[:n] += vpool[0, 0, P + c, :n]
            admitted += 1
        m = r.standard_normal((1, 1, P + nc))
        out = O.update_memory(kpool, vpool, blk_len, blk_pos, kbar, slot_src, slot_w,
                              np.arange(P, P + nc), 10 * step + np.arange(nc), m, P, 0,
                              O.MERGE_MEAN, "f64")
        kpool, vpool, blk_len, blk_pos, kbar, slot_src, slot_w, _ = out
        assert (slot_src >= 0).sum() <= P
        acc_k = np.zeros((bs, D))
        acc_v = np.zeros((bs, D))
        for s in range(P):
            if slot_src[0, 0, s] >= 0:
                n = blk_len[0, 0, s]
                acc_k[:n] += slot_w[0, 0, s] * kpool[0, 0, s, :n]
                acc_v[:n] += slot_w[0, 0, s] * vpool[0, 0, s, :n]
                assert np.allclose(kbar[0, 0, s], kpool[0, 0, s, :n].mean(axis=0))
        assert np.allclose(acc_k, total_k, atol=1e-12)
        assert np.allclose(acc_v, total_v, atol=1e-12)
        assert slot_w.sum() == admitted


def test_update_sink_slot_is_pinned():
    P, bs, D = 3, 2, 2
    r = np.random.default_rng(5)
    NB = P + 2
    kpool = r.standard_normal((1, 1, NB, bs, D))
    kbar = kpool.mean(axis=3)
    blk_len = np.full((1, 1, NB), bs)
    blk_len[0, 0, :P] = 0
    slot_src = np.full((1, 1, P), -1)
    slot_w = np.zeros((1, 1, P))
    # global block 0 leaves the window: it enters sink slot 0 whatever its score
    m = np.array([[[0, 0, 0, -100.0, 5.0]]])
    out = O.update_memory(kpool, kpool, blk_len, np.zeros_like(blk_len), kbar, slot_src,
                          slot_w, np.array([3, 4]), np.array([0, 1]), m, P, 1, O.MERGE_MEAN, "f64")
    kp, vp, bl, bp, kb, ss, sw, _ = out
    assert ss[0, 0, 0] == 0 and np.array_equal(kp[0, 0, 0], kpool[0, 0, 3])
    assert ss[0, 0, 1] == 1
    # later steps: sink never ranked or merged into, even with the worst score
    kp2 = kp.copy()
    kp2[0, 0, 3:] = r.standard_normal((2, bs, D))
    kb2 = kb.copy()
    kb2[0, 0, 3:] = kp2[0, 0, 3:].mean(axis=1)
    bl2 = bl.copy()
    bl2[0, 0, 3:] = bs
    out2 = O.update_memory(kp2, kp2, bl2, bp, kb2, ss, sw, np.array([3, 4]), np.array([7, 8]),
                           np.array([[[-1e9, 0.0, 0.0, 1.0, 2.0]]]), P, 1, O.MERGE_MEAN, "f64")
    assert out2[5][0, 0, 0] == 0 and np.array_equal(out2[0][0, 0, 0], kpool[0, 0, 3])
    assert out2[6][0, 0, 0] == 1.0


# --------------------------------------------------------------------------
# a4/a5 local selection
# --------------------------------------------------------------------------

def test_select_hand_example():
    # window ids 4..7 with scores 0.2, 0.9, 0.2, -1 for the only query block; k = 2:
    # 5 (0.9) then 4 (0.2, wins the tie with 6 by lower id); memory ids 0, 2 hold blocks,
    # id 1 is an empty slot.
    S = np.zeros((1, 1, 1, 8))
    S[0, 0, 0, 4:8] = [0.2, 0.9, 0.2, -1.0]
    blk_len = np.array([[[5, 0, 5, 0, 5, 5, 5, 5]]])
    A = O.select_local(S, [4, 5, 6, 7], 2, np.array([[[0, 1, 2]]]), blk_len)
    assert A[0][0][0] == [0, 2, 4, 5]


@pytest.mark.parametrize("seed", range(5))
def test_select_dominance_counts_and_order(seed):
    r = np.random.default_rng(seed)
    NB, nQB = 30, 6
    S = np.round(r.standard_normal((1, 2, nQB, NB)), 1)
    blk_len = np.full((1, 2, NB), 3)
    win = list(range(10, 30))
    k = int(r.integers(1, 25))
    mem = np.array([[[0, 1, -1, 3], [2, -1, -1, -1]]])
    A = O.select_local(S, win, k, mem, blk_len)
    for h in range(2):
        m = [x for x in mem[0, h] if x >= 0]
        for i in range(nQB):
            a = A[0][h][i]
            assert a == sorted(set(a))
            local = [j for j in a if j in win]
            assert len(local) == min(k, len(win))
            assert len(a) == len(m) + len(local)
            rest = [j for j in win if j not in local]
            for x in local:
                for y in rest:
                    assert S[0, h, i, x] > S[0, h, i, y] or (S[0, h, i, x] == S[0, h, i, y] and x < y)


def test_select_token_mask_allows_only_started_blocks():
    # query chunk at positions 64..191 (two query blocks of 64); window blocks start at
    # 0, 64, 128: query block 0 (last position 127) may use blocks starting at 0 and 64.
    S = np.zeros((1, 1, 2, 3))
    blk_len = np.full((1, 1, 3), 64)
    blk_pos = np.array([[[0, 64, 128]]])
    A = O.select_local(S, [0, 1, 2], 8, None, blk_len, O.MASK_TOKEN, 64, blk_pos, 64, 128)
    assert A[0][0][0] == [0, 1] and A[0][0][1] == [0, 1, 2]


# --------------------------------------------------------------------------
# a6 attention
# --------------------------------------------------------------------------

def _dense_case(seed, B=1, H=2, NB=5, bs=8, D=16, Tq=20, last_len=5):
    r = np.random.default_rng(seed)
    kpool = r.standard_normal((B, H, NB, bs, D))
    vpool = r.standard_normal((B, H, NB, bs, D))
    blk_len = np.full((B, H, NB), bs)
    blk_len[:, :, -1] = last_len
    blk_pos = np.broadcast_to(np.arange(NB) * bs, (B, H, NB)).copy()
    q = r.standard_normal((B, H, Tq, D))
    return q, kpool, vpool, blk_len, blk_pos


def _flatten_keys(kpool, vpool, blk_len, b, h):
    ks = [kpool[b, h, j, :blk_len[b, h, j]] for j in range(kpool.shape[2])]
    vs = [vpool[b, h, j, :blk_len[b, h, j]] for j in range(kpool.shape[2])]
    return np.concatenate(ks), np.concatenate(vs)


@pytest.mark.parametrize("mask", [O.MASK_CHUNK, O.MASK_TOKEN])
def test_all_blocks_kept_equals_dense_attention(mask):
    q, kp, vp, bl, bp = _dense_case(0)
    B, H, Tq, D = q.shape
    bs = kp.shape[3]
    nQB = -(-Tq // bs)
    NB = kp.shape[2]
    idx = np.broadcast_to(np.arange(NB), (B, H, nQB, NB)).astype(np.int32)
    cnt = np.full((B, H, nQB), NB, dtype=np.int32)
    total = int(bl[0, 0].sum())                       # 37 keys, queries are the last Tq
    q_pos0 = total - Tq
    out, lse = O.attention_fwd(q, kp, vp, bl, bp, idx, cnt, 1 / math.sqrt(D), mask, q_pos0)
    for b in range(B):
        for h in range(H):
            kc, vc = _flatten_keys(kp, vp, bl, b, h)
            qt, kt, vt = (torch.from_numpy(x) for x in (q[b, h], kc, vc))
            am = None
            if mask == O.MASK_TOKEN:
                am = (torch.arange(total)[None, :] <= (q_pos0 + torch.arange(Tq))[:, None])
            ref = torch.nn.functional.scaled_dot_product_attention(
                qt[None], kt[None], vt[None], attn_mask=am, scale=1 / math.sqrt(D))[0]
            assert np.allclose(out[b, h], ref.numpy(), atol=1e-12)
            logits = (qt @ kt.T) / math.sqrt(D)
            if am is not None:
                logits = logits.masked_fill(~am, -math.inf)
            assert np.allclose(lse[b, h], torch.logsumexp(logits, dim=1).numpy(), atol=1e-12)


def test_attention_rows_sum_to_one_and_single_block_textbook():
    q, kp, vp, bl, bp = _dense_case(1, H=1, NB=3)
    D = q.shape[-1]
    sc = 1 / math.sqrt(D)
    nQB = 3
    idx = np.array([[[[2, -1], [0, 2], [1, -1]]]], dtype=np.int32)
    cnt = np.array([[[1, 2, 1]]], dtype=np.int32)
    # V = identity rows -> O rows are the softmax weights themselves
    out, lse = O.attention_fwd(q, kp, vp, bl, bp, idx, cnt, sc)
    for i in range(nQB):
        ids = idx[0, 0, i, :cnt[0, 0, i]]
        kc = np.concatenate([kp[0, 0, j, :bl[0, 0, j]] for j in ids])
        s = sc * q[0, 0, i * 8:i * 8 + 8] @ kc.T
        s = s[: min(8, 20 - i * 8)]
        assert np.allclose(np.exp(s - lse[0, 0, i * 8:i * 8 + len(s), None]).sum(axis=1), 1.0)
    # single block, textbook softmax(q k^T) v written out by hand
    r0 = 16
    kc, vc = kp[0, 0, 1, :bl[0, 0, 1]], vp[0, 0, 1, :bl[0, 0, 1]]
    for r in range(r0, 20):
        w = np.exp(sc * kc @ q[0, 0, r])
        assert np.allclose(out[0, 0, r], (w[:, None] * vc).sum(axis=0) / w.sum())


def test_attention_invariant_to_list_order_and_empty_list():
    q, kp, vp, bl, bp = _dense_case(2, H=1)
    sc = 0.25
    idx = np.array([[[[4, 0, 2], [1, 3, -1], [0, -1, -1]]]], dtype=np.int32)
    cnt = np.array([[[3, 2, 0]]], dtype=np.int32)
    o1, l1 = O.attention_fwd(q, kp, vp, bl, bp, idx, cnt, sc)
    idx2 = np.array([[[[2, 4, 0], [3, 1, -1], [0, -1, -1]]]], dtype=np.int32)
    o2, l2 = O.attention_fwd(q, kp, vp, bl, bp, idx2, cnt, sc)
    assert np.allclose(o1, o2, atol=1e-13) and np.allclose(l1, l2, atol=1e-13)
    assert np.all(o1[0, 0, 16:] == 0) and np.all(np.isneginf(l1[0, 0, 16:]))


# --------------------------------------------------------------------------
# a7 backward
# --------------------------------------------------------------------------

def test_backward_matches_central_differences():
    q, kp, vp, bl, bp = _dense_case(3, H=1, NB=3, bs=4, D=4, Tq=6, last_len=3)
    r = np.random.default_rng(9)
    dO = r.standard_normal(q.shape)
    idx = np.array([[[[0, 2, -1], [1, 2, 0]]]], dtype=np.int32)
    cnt = np.array([[[2, 3]]], dtype=np.int32)
    sc = 0.7

    def loss(q_, kp_, vp_):
        o, _ = O.attention_fwd(q_, kp_, vp_, bl, bp, idx, cnt, sc)
        return float((o * dO).sum())

    dq, dk, dv = O.attention_bwd(q, kp, vp, bl, bp, idx, cnt, dO, sc)
    eps = 1e-6
    for arr, grad in ((q, dq), (kp, dk), (vp, dv)):
        flat = arr.reshape(-1)
        g = grad.reshape(-1)
        for n in range(flat.size):
            old = flat[n]
            flat[n] = old + eps
            lp = loss(q, kp, vp)
            flat[n] = old - eps
            lm = loss(q, kp, vp)
            flat[n] = old
            fd = (lp - lm) / (2 * eps)
            assert abs(fd - g[n]) <= 1e-6 * max(1.0, abs(fd)), (n, fd, g[n])


@pytest.mark.parametrize("mask", [O.MASK_CHUNK, O.MASK_TOKEN])
def test_backward_all_kept_equals_torch_autograd(mask):
    q, kp, vp, bl, bp = _dense_case(4)
    B, H, Tq, D = q.shape
    NB = kp.shape[2]
    nQB = -(-Tq // 8)
    idx = np.broadcast_to(np.arange(NB), (B, H, nQB, NB)).astype(np.int32)
    cnt = np.full((B, H, nQB), NB, dtype=np.int32)
    total = int(bl[0, 0].sum())
    q_pos0 = total - Tq
    dO = np.random.default_rng(11).standard_normal(q.shape)
    sc = 1 / math.sqrt(D)
    dq, dk, dv = O.attention_bwd(q, kp, vp, bl, bp, idx, cnt, dO, sc, mask, q_pos0)
    for b in range(B):
        for h in range(H):
            kc, vc = _flatten_keys(kp, vp, bl, b, h)
            qt = torch.from_numpy(q[b, h].copy()).requires_grad_()
            kt = torch.from_numpy(kc.copy()).requires_grad_()
            vt = torch.from_numpy(vc.copy()).requires_grad_()
            am = None
            if mask == O.MASK_TOKEN:
                am = (torch.arange(total)[None, :] <= (q_pos0 + torch.arange(Tq))[:, None])
            o = torch.nn.functional.scaled_dot_product_attention(qt[None], kt[None], vt[None],
                                                                 attn_mask=am, scale=sc)[0]
            o.backward(torch.from_numpy(dO[b, h]))
            assert np.allclose(dq[b, h], qt.grad.numpy(), atol=1e-11)
            off = 0
            for j in range(NB):
                n = bl[b, h, j]
                assert np.allclose(dk[b, h, j, :n], kt.grad[off:off + n].numpy(), atol=1e-11)
                assert np.allclose(dv[b, h, j, :n], vt.grad[off:off + n].numpy(), atol=1e-11)
                assert np.all(dk[b, h, j, n:] == 0)
                off += n


# --------------------------------------------------------------------------
# block tiling of chunks (R9)
# --------------------------------------------------------------------------

def test_chunk_tiling_of_the_video_chunk():
    # a chunk of 3 latent frames of 1560 tokens in 128-token blocks
    blocks = O.chunk_blocks(4680, 128)
    assert len(blocks) == 37
    assert blocks[:2] == [(0, 128), (128, 128)]
    assert blocks[-1] == (4608, 72)
    assert all(n == 128 for _, n in blocks[:-1])
    assert O.chunk_blocks(5, 64) == [(0, 5)]
    assert O.chunk_blocks(128, 128) == [(0, 128)]
    assert O.chunk_blocks(256, 64) == [(0, 64), (64, 64), (128, 64), (192, 64)]


def test_query_blocks_tile_each_query_chunk_on_its_own():
    # 500 query rows in chunks of 200 rows (the last chunk 100), blocks of 64:
    # no block crosses a chunk boundary, each chunk ends in a short block
    want = [(0, 64), (64, 64), (128, 64), (192, 8),
            (200, 64), (264, 64), (328, 64), (392, 8),
            (400, 64), (464, 36)]
    assert O.query_blocks(500, 64, 200) == want
    assert list(O.query_block_lengths(500, 64, 200)) == [n for _, n in want]
    # one chunk (q_chunk 0) is the plain tiling
    assert O.query_blocks(500, 64) == O.chunk_blocks(500, 64)
    # the trainable shape: 7 chunks of 4680 tokens -> 7 x 37 = 259 blocks
    tb = O.query_blocks(7 * 4680, 128, 4680)
    assert len(tb) == 259
    assert tb[36] == (4608, 72) and tb[37] == (4680, 128) and tb[-1] == (6 * 4680 + 4608, 72)


def test_pooling_follows_the_query_chunk_tiling():
    # rows of value r: each block's mean is the mean of its own row indices
    q = np.arange(500, dtype=np.float64)[None, None, :, None] * np.ones((1, 1, 1, 3))
    qb = O.pool_queries(q, 64, 200)
    for i, (r0, n) in enumerate(O.query_blocks(500, 64, 200)):
        assert np.allclose(qb[0, 0, i], r0 + (n - 1) / 2.0)
    assert np.allclose(qb[0, 0, 3], 195.5)     # rows 192..199 only


# --------------------------------------------------------------------------
# the local window, the chunk leaving it, the pool placement (R7, R14)
# --------------------------------------------------------------------------

def test_window_and_leaving_chunk_by_hand_for_w2():
    # W = 2: the current chunk and the one before it
    table = {0: ([0], None, []), 1: ([0, 1], None, []), 2: ([1, 2], 0, [0]),
             3: ([2, 3], 1, [0, 1]), 4: ([3, 4], 2, [0, 1, 2])}
    for t, (win, gone, older) in table.items():
        assert O.window_chunks(t, 2) == win
        assert O.leaving_chunk(t, 2) == gone
        assert O.older_chunks(t, 2) == older


def test_window_other_sizes_and_every_chunk_leaves_once():
    assert O.window_chunks(5, 1) == [5] and O.leaving_chunk(5, 1) == 4
    assert O.window_chunks(1, 3) == [0, 1] and O.leaving_chunk(2, 3) is None
    assert O.window_chunks(6, 3) == [4, 5, 6] and O.leaving_chunk(6, 3) == 3
    for W in (1, 2, 3, 5):
        left = [O.leaving_chunk(t, W) for t in range(40)]
        left = [c for c in left if c is not None]
        assert left == list(range(40 - W))      # each chunk leaves once, in order
        for t in range(40):
            assert len(O.window_chunks(t, W)) == min(W, t + 1)
            assert sorted(O.older_chunks(t, W) + O.window_chunks(t, W)) == list(range(t + 1))


def test_placement_by_hand_ring_and_snapshot():
    ring = O.PoolPlacement(P=4, T_c=256, bs=64, W=2, n_chunks=9, ring=True)
    assert ring.nb_c == 4 and ring.NB == 4 + 3 * 4
    assert ring.chunk_ids(0) == [4, 5, 6, 7]
    assert ring.chunk_ids(2) == [12, 13, 14, 15]
    assert ring.chunk_ids(3) == [4, 5, 6, 7]
    assert ring.global_ids(3) == [12, 13, 14, 15]
    snap = O.PoolPlacement(P=24, T_c=4680, bs=128, W=2, n_chunks=5, ring=False)
    assert snap.NB == 24 + 5 * 37 and snap.chunk_ids(4)[-1] == snap.NB - 1
    assert snap.chunk_ids(1)[0] == 24 + 37


def test_ring_keeps_the_leaving_chunk_readable():
    # at every step the window chunks and the chunk leaving the window sit at
    # pairwise different ring positions, so the update can still read it
    for W in (1, 2, 4):
        pl = O.PoolPlacement(P=3, T_c=100, bs=64, W=W, n_chunks=0, ring=True)
        for t in range(30):
            live = O.window_chunks(t, W) + [c for c in [O.leaving_chunk(t, W)] if c is not None]
            firsts = [pl.chunk_ids(c)[0] for c in live]
            assert len(set(firsts)) == len(live)
            assert all(f >= pl.P for f in firsts)


# --------------------------------------------------------------------------
# packing of the attended lists
# --------------------------------------------------------------------------

def test_lists_to_arrays_pads_with_minus_one():
    A = [[[[1, 5], [], [2]], [[0, 1, 2], [7], []]]]
    idx, cnt = O.lists_to_arrays(A, 3)
    assert idx.dtype == np.int32 and idx.shape == (1, 2, 3, 3)
    assert idx[0, 0].tolist() == [[1, 5, -1], [-1, -1, -1], [2, -1, -1]]
    assert idx[0, 1].tolist() == [[0, 1, 2], [7, -1, -1], [-1, -1, -1]]
    assert cnt.tolist() == [[[2, 0, 1], [3, 1, 0]]]
    with pytest.raises(ValueError):
        O.lists_to_arrays([[[[1, 2, 3, 4]]]], 3)


# --------------------------------------------------------------------------
# the layer step (R14) and the trainable lists (R13, R18)
# --------------------------------------------------------------------------

def _tiny_layer(P=4, n_sink=0, policy=O.EVICT, W=2, k=2, ring=True, n_chunks=8):
    return O.OracleLayer(1, 2, 8, 4, 10, P, n_sink, W, k, policy, O.MASK_CHUNK, "f64",
                         n_chunks, ring)


def test_rollout_step_admits_only_blocks_that_left_the_window():
    r = np.random.default_rng(3)
    L = _tiny_layer(P=3)
    nb_c = L.place.nb_c                           # 10 tokens in blocks of 4: 3 blocks
    assert nb_c == 3
    for t in range(8):
        q, k, v = (r.standard_normal((1, 2, 10, 8)) for _ in range(3))
        L.write_chunk(t, k, v)
        res = L.step(t, q)
        gone = O.leaving_chunk(t, 2)
        assert res["cand_src"] == ([] if gone is None else list(range(gone * 3, gone * 3 + 3)))
        # every slot holds a block of a chunk that has left the window
        left = {g for c in range(t + 1) if c not in O.window_chunks(t, 2) for g in range(3 * c, 3 * c + 3)}
        for h in range(2):
            held = [int(s) for s in L.ss[0, h] if s >= 0]
            assert set(held) <= left
            assert len(held) == min(3, len(left))
            # the local part of each list is in the window; the rest are slots
            for i in range(nb_c):
                a = res["A"][0][h][i]
                assert [x for x in a if x < 3] == [s for s in range(3) if L.ss[0, h, s] >= 0]
                assert set(x for x in a if x >= 3) <= set(L.window_ids(t))
                assert len([x for x in a if x >= 3]) == min(2, len(L.window_ids(t)))
        # the row positions of the window blocks follow the chunk order
        for c in O.window_chunks(t, 2):
            ids = L.place.chunk_ids(c)
            assert L.bp[0, 0, ids[0]] == 10 * c and L.bl[0, 0, ids[-1]] == 2


def test_snapshot_step_offers_every_older_chunk():
    r = np.random.default_rng(4)
    L = _tiny_layer(P=4, ring=False, n_chunks=4)
    for t in range(4):
        _, k, v = (r.standard_normal((1, 2, 10, 8)) for _ in range(3))
        L.write_chunk(t, k, v)
    q = r.standard_normal((1, 2, 10, 8))
    all_ids = [p for c in range(4) for p in L.place.chunk_ids(c)]
    res = L.step(3, q, pool_ids=all_ids)
    assert res["cand_src"] == list(range(6))      # chunks 0 and 1
    assert res["cand_ids"] == L.place.chunk_ids(0) + L.place.chunk_ids(1)
    assert res["win_ids"] == L.place.chunk_ids(2) + L.place.chunk_ids(3)


def _train_case(seed, n_chunks=4, T_c=10, bs=4, H=2, D=8):
    r = np.random.default_rng(seed)
    q = r.standard_normal((1, H, n_chunks * T_c, D))
    L = O.OracleLayer(1, H, D, bs, T_c, 0, 0, 2, 2, O.EVICT, O.MASK_CHUNK, "f64", n_chunks,
                      ring=False)
    for t in range(n_chunks):
        L.write_chunk(t, r.standard_normal((1, H, T_c, D)), r.standard_normal((1, H, T_c, D)))
    return q, L


def test_trainable_lists_dense_and_budget_invariants():
    q, L = _train_case(5)
    nb_c, sc = L.place.nb_c, L.scale
    # density 1: every chunk-causally allowed block
    idx, cnt = O.trainable_lists(q, L.kp, L.bl, 10, 4, 2, 2, 2, sc, density=1.0)
    for t in range(4):
        allowed = list(range(0, (t + 1) * nb_c))
        for i in range(nb_c):
            r_ = t * nb_c + i
            assert idx[0, 0, r_, :cnt[0, 0, r_]].tolist() == allowed
    # budgets large enough: the one-shot lists are every allowed block too
    idx, cnt = O.trainable_lists(q, L.kp, L.bl, 10, 4, 12, 2, 6, sc)
    for t in range(4):
        assert all(cnt[0, :, t * nb_c + i].tolist() == [(t + 1) * nb_c] * 2 for i in range(nb_c))
    # small budgets: |A_i| = min(P, #older) + min(k, #window) and the persistent
    # part is the exhaustive top-P of the chunk's memory score
    P, k = 2, 2
    idx, cnt = O.trainable_lists(q, L.kp, L.bl, 10, 4, P, 2, k, sc)
    kb = O.pool_keys(L.kp, L.bl, range(L.place.NB), np.zeros((1, 2, L.place.NB, 8)))
    for t in range(4):
        older = [p for c in O.older_chunks(t, 2) for p in L.place.chunk_ids(c)]
        win = [p for c in O.window_chunks(t, 2) for p in L.place.chunk_ids(c)]
        S = O.block_scores(O.pool_queries(q[:, :, 10 * t:10 * t + 10], 4), kb, sc)
        m = S.mean(axis=2)
        for h in range(2):
            top = sorted(older, key=lambda j: (-m[0, h, j], j))[:P]
            for i in range(nb_c):
                a = idx[0, h, t * nb_c + i, :cnt[0, h, t * nb_c + i]].tolist()
                assert len(a) == min(P, len(older)) + min(k, len(win))
                assert sorted(x for x in a if x in older) == sorted(top)
                loc = sorted(win, key=lambda j: (-S[0, h, i, j], j))[:k]
                assert sorted(x for x in a if x in win) == sorted(loc)


def test_trainable_lists_density_counts():
    q, L = _train_case(6)
    nb_c = L.place.nb_c
    for d in (0.05, 0.25, 0.5):
        idx, cnt = O.trainable_lists(q, L.kp, L.bl, 10, 4, 2, 2, 2, L.scale, density=d)
        for t in range(4):
            n = (t + 1) * nb_c
            assert np.all(cnt[0, :, t * nb_c:(t + 1) * nb_c] == math.ceil(d * n))
