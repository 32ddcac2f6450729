"""Planted mistakes in the oracle must be caught by its pins.

Each case swaps one oracle function for a plausibly wrong variant (on the CPU,
inside this process only) and checks that at least one pin fails.
"""
import numpy as np
import pytest

import oracle
import oracle.pbsa_oracle as OO
from tests import test_oracle_pins as pins


def _fails(fn, *args):
    try:
        fn(*args)
    except AssertionError:
        return True
    return False


def test_mean_replaced_by_max_memory_score_is_caught(monkeypatch):
    monkeypatch.setattr(OO, "memory_scores", lambda S: S.max(axis=2))
    monkeypatch.setattr(oracle, "memory_scores", OO.memory_scores)
    assert _fails(pins.test_scores_on_an_orthogonal_basis)


def test_pooling_over_whole_block_is_caught(monkeypatch):
    def bad_pool_keys(kpool, blk_len, ids, k_bar):
        out = np.array(k_bar, dtype=np.float64, copy=True)
        for j in ids:
            out[:, :, j] = kpool[:, :, j].mean(axis=2)
        return out
    monkeypatch.setattr(oracle, "pool_keys", bad_pool_keys)
    assert _fails(pins.test_pool_partial_block_uses_its_length_only)


def test_missing_scale_is_caught(monkeypatch):
    real = OO._logits
    monkeypatch.setattr(OO, "_logits", lambda qi, kc, scale, *a: real(qi, kc, 1.0, *a))
    assert _fails(pins.test_all_blocks_kept_equals_dense_attention, oracle.MASK_CHUNK)


def test_wrong_tie_break_is_caught(monkeypatch):
    real_sorted = sorted

    def flipped(items, key=None, **kw):
        items = list(items)
        if items and isinstance(items[0], OO._Item) and key is not None and kw == {}:
            return real_sorted(items, key=lambda it: (-it.m, -it.src))
        return real_sorted(items, key=key, **kw)
    monkeypatch.setattr(OO, "sorted", flipped, raising=False)
    assert _fails(pins.test_update_hand_example_evict)


def test_dropped_delta_term_in_backward_is_caught(monkeypatch):
    # dS = P * dP: the softmax backward without its rowsum(P * dP) term
    def bad(q, kpool, vpool, blk_len, blk_pos, idx, cnt, dO, scale, mask=0, q_pos0=0,
            q_chunk=0):
        B, H, Tq, D = q.shape
        dq = np.zeros((B, H, Tq, D))
        dk = np.zeros(kpool.shape)
        dv = np.zeros(vpool.shape)
        for b in range(B):
            for h in range(H):
                for i, (r0, n) in enumerate(OO.query_blocks(Tq, kpool.shape[3], q_chunk)):
                    ids = [int(x) for x in idx[b, h, i, :cnt[b, h, i]]]
                    kc, vc, kpos = OO._gather_keys(kpool, vpool, blk_len, blk_pos, b, h, ids)
                    qi, doi = q[b, h, r0:r0 + n], dO[b, h, r0:r0 + n]
                    Pm, _ = OO._softmax_rows(OO._logits(qi, kc, scale, mask,
                                                        q_pos0 + r0 + np.arange(n), kpos))
                    dS = Pm * (doi @ vc.T)
                    dq[b, h, r0:r0 + n] = scale * (dS @ kc)
                    dkc, dvc = scale * (dS.T @ qi), Pm.T @ doi
                    off = 0
                    for j in ids:
                        m = int(blk_len[b, h, j])
                        dk[b, h, j, :m] += dkc[off:off + m]
                        dv[b, h, j, :m] += dvc[off:off + m]
                        off += m
        return dq, dk, dv
    monkeypatch.setattr(oracle, "attention_bwd", bad)
    assert _fails(pins.test_backward_all_kept_equals_torch_autograd, oracle.MASK_CHUNK)
    assert _fails(pins.test_backward_matches_central_differences)


def test_merge_without_weights_is_caught(monkeypatch):
    real = OO.update_memory

    def bad(*a, **k):
        out = list(real(*a, **k))
        out[6] = np.where(out[5] >= 0, 1.0, 0.0)      # weights not accumulated
        return tuple(out)
    monkeypatch.setattr(oracle, "update_memory", bad)
    assert _fails(pins.test_update_merge_conserves_mass_over_a_rollout)


def test_window_one_chunk_too_long_is_caught(monkeypatch):
    monkeypatch.setattr(oracle, "window_chunks",
                        lambda t, W: [c for c in range(t - W, t + 1) if c >= 0])
    assert _fails(pins.test_window_and_leaving_chunk_by_hand_for_w2)


def test_leaving_chunk_off_by_one_is_caught(monkeypatch):
    monkeypatch.setattr(oracle, "leaving_chunk", lambda t, W: t - W + 1 if t >= W - 1 else None)
    assert _fails(pins.test_window_and_leaving_chunk_by_hand_for_w2)
    assert _fails(pins.test_window_other_sizes_and_every_chunk_leaves_once)


def test_leaving_chunk_used_by_the_step_is_pinned(monkeypatch):
    # the layer step must offer the chunk that just left, not the current one's predecessor
    monkeypatch.setattr(OO, "leaving_chunk", lambda t, W: t - 1 if t >= 1 else None)
    assert _fails(pins.test_rollout_step_admits_only_blocks_that_left_the_window)


def test_query_tiling_ignoring_chunks_is_caught(monkeypatch):
    monkeypatch.setattr(oracle, "query_blocks", lambda Tq, bs, q_chunk=0: OO.chunk_blocks(Tq, bs))
    assert _fails(pins.test_query_blocks_tile_each_query_chunk_on_its_own)


def test_pooling_across_query_chunks_is_caught(monkeypatch):
    real = OO.query_blocks
    monkeypatch.setattr(OO, "query_blocks", lambda Tq, bs, q_chunk=0: real(Tq, bs, 0))
    assert _fails(pins.test_pooling_follows_the_query_chunk_tiling)


def test_last_block_dropped_from_tiling_is_caught(monkeypatch):
    real = OO.chunk_blocks
    monkeypatch.setattr(oracle, "chunk_blocks", lambda T, bs: [b for b in real(T, bs) if b[1] == bs])
    assert _fails(pins.test_chunk_tiling_of_the_video_chunk)


def test_ring_without_the_extra_position_is_caught(monkeypatch):
    real_init = OO.PoolPlacement.__init__

    def short_ring(self, P, T_c, bs, W, n_chunks, ring):
        real_init(self, P, T_c, bs, W, n_chunks, ring)
        if ring:
            self.positions = W
            self.NB = P + W * self.nb_c
    monkeypatch.setattr(OO.PoolPlacement, "__init__", short_ring)
    assert _fails(pins.test_ring_keeps_the_leaving_chunk_readable)


def test_list_padding_with_zero_is_caught(monkeypatch):
    real = OO.lists_to_arrays

    def bad(A, Amax):
        idx, cnt = real(A, Amax)
        idx[idx < 0] = 0
        return idx, cnt
    monkeypatch.setattr(oracle, "lists_to_arrays", bad)
    assert _fails(pins.test_lists_to_arrays_pads_with_minus_one)


def test_trainable_persistent_set_from_the_window_is_caught(monkeypatch):
    # a persistent set chosen among all earlier chunks (window included)
    monkeypatch.setattr(OO, "older_chunks", lambda t, W: list(range(t)))
    assert _fails(pins.test_trainable_lists_dense_and_budget_invariants)
