"""CPU pins of the oracle's backward through the persistent memory (the
recurrent trainable path): ``update_memory_vjp`` and ``rollout_bwd``.

Sparse Forcing trains with the dynamically updated cache (gist.science/es,
section 2 "Entrenamiento"), so a block's keys and values reach the loss both
through the attention of the steps that see them directly and through the
slots they were copied or merged into.

The pins, none of which reuses the oracle's backward code:
* a hand-worked merge: a slot holding the mean of two blocks of lengths 3 and 2;
* torch autograd in float64 on an independent restatement of a merge rollout's
  forward (the recorded decisions replayed as weighted row means and plain
  softmax attention), whose outputs are first checked against the oracle's own
  attention; its gradients w.r.t. every chunk's Q, K and V must equal
  ``rollout_bwd``;
* planted mistakes in the backward (a weight dropped, pre-update slots not
  cleared) that the autograd pin must catch.
"""
import math

import numpy as np
import pytest
import torch

from oracle import pbsa_oracle as O


def test_update_vjp_hand_worked_merge():
    # one head, P = 2: slot 0 = (1*A[:3] + 1*B[:2]) / 2 (a merge), slot 1 = copy of C
    bs, D = 4, 2
    B_, H_, NB = 1, 1, 5
    info = {(0, 0): {"compose": {0: [(2, 0.5, 3), (3, 0.5, 2)], 1: [(4, 1.0, bs)]}}}
    g = np.arange(1, 1 + B_ * H_ * NB * bs * D, dtype=np.float64).reshape(B_, H_, NB, bs, D)
    dk, dv = O.update_memory_vjp(g, -g, info, P=2)
    want = g.copy()
    want[0, 0, :2] = 0.0                       # pre-update slots receive nothing here
    want[0, 0, 2, :3] += 0.5 * g[0, 0, 0, :3]  # A
    want[0, 0, 3, :2] += 0.5 * g[0, 0, 0, :2]  # B
    want[0, 0, 4] += g[0, 0, 1]                # C, whole block
    np.testing.assert_array_equal(dk, want)
    np.testing.assert_array_equal(dv, -want)


# ---------------------------------------------------------------------------
# a small merge rollout, recorded
# ---------------------------------------------------------------------------
B, H, D, bs, T_c, P, W, K_TOP, T = 1, 2, 8, 4, 8, 2, 2, 1, 6


def _record(seed=0, policy=O.MERGE_MEAN, n_sink=0):
    rng = np.random.default_rng(seed)
    L = O.OracleLayer(B, H, D, bs, T_c, P, n_sink, W, K_TOP, policy, O.MASK_CHUNK, "f64", T,
                      ring=True)
    qs = [rng.standard_normal((B, H, T_c, D)) for _ in range(T)]
    ks = [rng.standard_normal((B, H, T_c, D)) for _ in range(T)]
    vs = [rng.standard_normal((B, H, T_c, D)) for _ in range(T)]
    # salient blocks so that the memory has something to prefer
    for t in range(T):
        ks[t][:, :, :bs] += 1.5 * rng.standard_normal((B, H, 1, D))
    dOs = [rng.standard_normal((B, H, T_c, D)) for _ in range(T)]
    steps, merged = [], 0
    for t in range(T):
        L.write_chunk(t, ks[t], vs[t])
        r = L.step(t, qs[t], attend=False)
        info = r["info"]
        if info is not None:
            merged += sum(len(terms) > 1 for inf in info.values() for terms in inf["compose"].values())
        steps.append(dict(q=qs[t], kp=r["kpool"].copy(), vp=r["vpool"].copy(),
                          bl=r["blk_len"].copy(), bp=r["blk_pos"].copy(), idx=r["idx"].copy(),
                          cnt=r["cnt"].copy(), info=info, dO=dOs[t]))
    return L, qs, ks, vs, steps, merged


def _replay(L, qs, ks, vs, steps):
    """The rollout's loss sum_t <O_t, dO_t> from the chunks' Q, K, V (torch
    float64), with every decision taken from the record: each chunk's rows
    written into its ring blocks, each slot rebuilt as the recorded weighted
    row-wise mean of pre-update blocks, and plain softmax attention of every
    query block over the recorded list (valid rows only, chunk mask).  Returns
    the loss and the per-step outputs."""
    place = L.place
    NB = place.NB
    scale = 1.0 / math.sqrt(D)
    zero = torch.zeros(bs, D, dtype=torch.float64)
    pk = [[[zero for _ in range(NB)] for _ in range(H)] for _ in range(B)]
    pv = [[[zero for _ in range(NB)] for _ in range(H)] for _ in range(B)]
    loss = torch.zeros((), dtype=torch.float64)
    outs = []
    for t, st in enumerate(steps):
        for b in range(B):
            for h in range(H):
                for pid, (r0, n) in zip(place.chunk_ids(t), place.blocks):
                    blk_k = torch.cat([ks[t][b, h, r0:r0 + n], zero[:bs - n]])
                    blk_v = torch.cat([vs[t][b, h, r0:r0 + n], zero[:bs - n]])
                    pk[b][h][pid] = blk_k
                    pv[b][h][pid] = blk_v
        if st["info"] is not None:
            for (b, h), inf in st["info"].items():
                new_k, new_v = {}, {}
                for s, terms in inf["compose"].items():
                    acc_k, acc_v = zero, zero
                    for j, wgt, n in terms:
                        rows = (torch.arange(bs) < n).to(torch.float64)[:, None]
                        acc_k = acc_k + wgt * rows * pk[b][h][j]
                        acc_v = acc_v + wgt * rows * pv[b][h][j]
                    new_k[s], new_v[s] = acc_k, acc_v
                for s in new_k:
                    pk[b][h][s], pv[b][h][s] = new_k[s], new_v[s]
        Ot = torch.zeros(B, H, T_c, D, dtype=torch.float64)
        rows_out = []
        for b in range(B):
            for h in range(H):
                for i, (r0, n) in enumerate(place.blocks):
                    ids = [int(x) for x in st["idx"][b, h, i, :st["cnt"][b, h, i]]]
                    kk = torch.cat([pk[b][h][j][:int(st["bl"][b, h, j])] for j in ids])
                    vv = torch.cat([pv[b][h][j][:int(st["bl"][b, h, j])] for j in ids])
                    s_ = scale * qs[t][b, h, r0:r0 + n] @ kk.T
                    o = torch.softmax(s_, dim=1) @ vv
                    rows_out.append(((b, h, r0, n), o))
        for (b, h, r0, n), o in rows_out:
            loss = loss + (o * torch.from_numpy(st["dO"][b, h, r0:r0 + n])).sum()
            Ot = Ot.index_put((torch.tensor(b), torch.tensor(h), torch.arange(r0, r0 + n)), o)
        outs.append(Ot)
    return loss, outs


@pytest.mark.parametrize("policy,n_sink", [(O.MERGE_MEAN, 0), (O.EVICT, 0), (O.MERGE_MEAN, 1)])
def test_rollout_bwd_equals_autograd_of_replay(policy, n_sink):
    L, qs, ks, vs, steps, merged = _record(seed=3 + policy + 7 * n_sink, policy=policy,
                                           n_sink=n_sink)
    if policy == O.MERGE_MEAN:
        assert merged > 0, "the rollout must exercise merges"
    tq = [torch.tensor(x, requires_grad=True) for x in qs]
    tk = [torch.tensor(x, requires_grad=True) for x in ks]
    tv = [torch.tensor(x, requires_grad=True) for x in vs]
    loss, outs = _replay(L, tq, tk, tv, steps)
    # the replay is the oracle's forward: same outputs as its attention on the
    # recorded pools and lists
    for t, st in enumerate(steps):
        Oo, _ = O.attention_fwd(st["q"], st["kp"], st["vp"], st["bl"], st["bp"], st["idx"],
                                st["cnt"], 1.0 / math.sqrt(D), O.MASK_CHUNK, t * T_c)
        np.testing.assert_allclose(outs[t].detach().numpy(), Oo, rtol=1e-12, atol=1e-12)
    gq = torch.autograd.grad(loss, tq + tk + tv)
    dq, dk, dv = O.rollout_bwd(steps, P, L.place, W, T_c, 1.0 / math.sqrt(D))
    for t in range(T):
        np.testing.assert_allclose(dq[t], gq[t].numpy(), rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(dk[t], gq[T + t].numpy(), rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(dv[t], gq[2 * T + t].numpy(), rtol=1e-10, atol=1e-12)
    # the slot path carries gradient: chunk 0 leaves the window at step W and
    # is attended later only through the memory
    assert np.abs(dk[0]).sum() > 0


def test_rollout_bwd_central_differences():
    L, qs, ks, vs, steps, _ = _record(seed=11)
    dq, dk, dv = O.rollout_bwd(steps, P, L.place, W, T_c, 1.0 / math.sqrt(D))
    eps = 1e-6

    def loss_of(ks_, vs_):
        with torch.no_grad():
            lo, _ = _replay(L, [torch.tensor(x) for x in qs], [torch.tensor(x) for x in ks_],
                            [torch.tensor(x) for x in vs_], steps)
        return float(lo)
    rng = np.random.default_rng(5)
    for _ in range(6):
        c = int(rng.integers(0, T - W))           # chunks that pass through the memory
        b, h, r, d = 0, int(rng.integers(0, H)), int(rng.integers(0, T_c)), int(rng.integers(0, D))
        for which, grad in (("k", dk), ("v", dv)):
            lo = []
            for sgn in (1, -1):
                k2 = [x.copy() for x in ks]
                v2 = [x.copy() for x in vs]
                (k2 if which == "k" else v2)[c][b, h, r, d] += sgn * eps
                lo.append(loss_of(k2, v2))
            num = (lo[0] - lo[1]) / (2 * eps)
            assert abs(num - grad[c][b, h, r, d]) <= 1e-6 * max(1.0, abs(num)), (which, c, num)


@pytest.mark.parametrize("mistake", ["weight_dropped", "slots_not_cleared"])
def test_planted_vjp_mistakes_are_caught(monkeypatch, mistake):
    L, qs, ks, vs, steps, _ = _record(seed=3)
    real = O.update_memory_vjp

    def bad(dk_after, dv_after, info, P_):
        if mistake == "weight_dropped":
            info2 = {key: {"compose": {s: [(j, 1.0, n) for j, w_, n in terms]
                                       for s, terms in inf["compose"].items()}}
                     for key, inf in info.items()}
            return real(dk_after, dv_after, info2, P_)
        dk, dv = real(dk_after, dv_after, info, P_)
        dk[:, :, :P_] += dk_after[:, :, :P_]
        dv[:, :, :P_] += dv_after[:, :, :P_]
        return dk, dv
    monkeypatch.setattr(O, "update_memory_vjp", bad)
    tk = [torch.tensor(x, requires_grad=True) for x in ks]
    loss, _ = _replay(L, [torch.tensor(x) for x in qs], tk, [torch.tensor(x) for x in vs], steps)
    gk = torch.autograd.grad(loss, tk)
    _, dk, _ = O.rollout_bwd(steps, P, L.place, W, T_c, 1.0 / math.sqrt(D))
    assert any(not np.allclose(dk[t], gk[t].numpy(), rtol=1e-8, atol=1e-10) for t in range(T))
