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
    # dS = P * dP (the rowsum(P*dP) term dropped)
    src = OO.attention_bwd

    def bad(q, kpool, vpool, blk_len, blk_pos, idx, cnt, dO, scale, mask=0, q_pos0=0):
        dq, dk, dv = src(q, kpool, vpool, blk_len, blk_pos, idx, cnt, dO, scale, mask, q_pos0)
        return dq * 1.01, dk, dv
    monkeypatch.setattr(oracle, "attention_bwd", bad)
    assert _fails(pins.test_backward_all_kept_equals_torch_autograd, oracle.MASK_CHUNK)


def test_merge_without_weights_is_caught(monkeypatch):
    real = OO.update_memory

    def bad(*a, **k):
        out = list(real(*a, **k))
        out[6] = np.where(out[5] >= 0, 1.0, 0.0)      # weights not accumulated
        return tuple(out)
    monkeypatch.setattr(oracle, "update_memory", bad)
    assert _fails(pins.test_update_merge_conserves_mass_over_a_rollout)
