"""CPU pins of the oracle's two-level (frame -> block) selection, the
alternative router of the "next" rows (Light Forcing, gist.science/it,
section 2.2 "Attenzione Sparsa Gerarchica (HSA)")."""
import itertools

import numpy as np
import pytest

from oracle import pbsa_oracle as O


def test_frame_groups_of_the_video_chunk():
    # 4680-token chunk of three 1560-token frames in 128-token blocks: blocks
    # 0..12 start in frame 0 (block 12 starts at row 1536), 13..24 in frame 1
    # (block 24 starts at 3072), 25..36 in frame 2
    g = O.frame_groups(4680, 128, 1560)
    assert len(g) == 37
    assert g[:13] == [0] * 13 and g[13:25] == [1] * 12 and g[25:] == [2] * 12


def _case(seed=0, nQB=3, n_win=12, NB=16):
    rng = np.random.default_rng(seed)
    S = rng.standard_normal((1, 1, nQB, NB))
    bl = np.full((1, 1, NB), 8, dtype=np.int32)
    bl[0, 0, 7] = 3                        # a partial block weighs by its length
    win = list(range(4, 4 + n_win))
    frame = [e // 3 for e in range(n_win)]  # four frames of three blocks
    return S, bl, win, frame


def test_hand_worked_two_frames():
    # one query block, two frames of two blocks each; frame A (ids 0, 1) has
    # the single best block but the lower mean, frame B (ids 2, 3) the higher
    S = np.array([[[[0.9, -0.8, 0.5, 0.4]]]])
    bl = np.array([[[4, 4, 4, 4]]], dtype=np.int32)
    A = O.select_hier(S, [0, 1, 2, 3], [0, 0, 1, 1], 1, 1, None, bl)
    assert A[0][0][0] == [2]               # frame B kept (mean 0.45 > 0.05), its best block
    A = O.select_hier(S, [0, 1, 2, 3], [0, 0, 1, 1], 2, 1, None, bl)
    assert A[0][0][0] == [0]               # both frames: the overall best block
    # weights: block 1 of length 1 barely drags frame A down
    bl2 = np.array([[[4, 1, 4, 4]]], dtype=np.int32)
    A = O.select_hier(S, [0, 1, 2, 3], [0, 0, 1, 1], 1, 2, None, bl2)
    assert A[0][0][0] == [0, 1]            # mean (3.6 - 0.8) / 5 = 0.56 > 0.45


def test_all_frames_reduces_to_select_local():
    S, bl, win, frame = _case()
    mem = np.array([[[0, 2, -1]]])
    for k in (1, 3, 5, 20):
        a = O.select_hier(S, win, frame, 99, k, mem, bl)
        b = O.select_local(S, win, k, mem, bl)
        assert a == b


def test_brute_force_frame_choice():
    S, bl, win, frame = _case(seed=3)
    labels = sorted(set(frame))
    for F, k in itertools.product((1, 2, 3), (1, 2, 4)):
        A = O.select_hier(S, win, frame, F, k, None, bl)
        for i in range(S.shape[2]):
            # brute force: the frame subset of size F with the largest scores
            means = {g: sum(bl[0, 0, j] * S[0, 0, i, j] for j, gg in zip(win, frame) if gg == g) /
                        sum(bl[0, 0, j] for j, gg in zip(win, frame) if gg == g) for g in labels}
            best = max(itertools.combinations(labels, F),
                       key=lambda c: (sorted((means[g] for g in c), reverse=True), [-g for g in c]))
            allowed = [j for j, g in zip(win, frame) if g in best]
            want = sorted(sorted(allowed, key=lambda j: (-S[0, 0, i, j], j))[:k])
            assert A[0][0][i] == want, (F, k, i)


def test_token_mask_and_empty_blocks():
    S, bl, win, frame = _case(seed=5, nQB=1)
    bl = bl.copy()
    bl[0, 0, win[0]] = 0                   # an empty block is never a candidate
    bp = np.zeros((1, 1, 16), dtype=np.int32)
    for e, j in enumerate(win):
        bp[0, 0, j] = 8 * e
    # the query block (rows 0..7 at positions 40..47) may see blocks starting at <= 47
    A = O.select_hier(S, win, frame, 2, 3, None, bl, mask=O.MASK_TOKEN, q_pos0=40, blk_pos=bp,
                      bs=8, Tq=8)
    got = A[0][0][0]
    assert got and win[0] not in got
    assert all(bp[0, 0, j] <= 47 for j in got)


@pytest.mark.parametrize("mistake", ["unweighted_mean", "max_of_blocks", "sum_of_blocks"])
def test_planted_frame_score_mistakes_are_caught(monkeypatch, mistake):
    def bad(cands, s_row, lens):
        out = {}
        for j, g in cands:
            out.setdefault(g, []).append((float(s_row[j]), float(lens[j])))
        if mistake == "unweighted_mean":
            return {g: sum(v for v, _ in x) / len(x) for g, x in out.items()}
        if mistake == "max_of_blocks":
            return {g: max(v for v, _ in x) for g, x in out.items()}
        return {g: sum(v * n for v, n in x) for g, x in out.items()}
    monkeypatch.setattr(O, "_frame_scores", bad)
    with pytest.raises(AssertionError):
        test_hand_worked_two_frames()
