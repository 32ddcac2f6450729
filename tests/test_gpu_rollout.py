"""GPU parity of the chunk-by-chunk rollout (score -> memory update -> select ->
attend) against the CPU oracle, at the rollout workloads' full head count and
chunk size.

Each step the GPU state is re-seeded from the oracle's state after the
previous step, so one near-tie cannot make the two recurrences drift apart;
the step's outputs are then compared.  Kept sets follow the near-tie rule
(ids within 1e-4 of the threshold may swap); slot rows must match exactly for
copies and to one bf16 ulp for merged slots (the GPU averages in fp32, the
oracle in fp64, and both round once to bf16); attention is checked with the
oracle's lists on sampled steps (max-abs <= 2e-2, mean-abs <= 2e-3).
A free-running GPU rollout checks the invariants over all steps.
"""
import numpy as np
import pytest
import torch

import oracle as O
import pbsa_inputs as PI
from block_sparse_attention_39_b200 import pbsa as K
from block_sparse_attention_39_b200.engine import PbsaLayer
from tests.gpu_util import ATT_MAX, ATT_MEAN, attn_errors, band_ok, dev_i32, dev_storage, host

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _status_clean():
    assert torch.cuda.is_available()
    K.get_status()
    yield
    assert K.get_status() == 0


def _seed_gpu(L, orc, w):
    """The GPU layer's whole state set to the oracle's (the re-seeding)."""
    L.kpool.copy_(dev_storage(orc.kp, w.dtype))
    L.vpool.copy_(dev_storage(orc.vp, w.dtype))
    L.blk_len.copy_(dev_i32(orc.bl))
    L.blk_pos.copy_(dev_i32(orc.bp))
    L.k_bar.copy_(torch.from_numpy(orc.kb.astype(np.float32)).cuda())
    L.slot_src.copy_(dev_i32(orc.ss))
    L.slot_w.copy_(torch.from_numpy(orc.sw.astype(np.float32)).cuda())


def _compare_memory(L, orc, w, info, merged_tol):
    src, sw = host(L.slot_src), host(L.slot_w)
    kp, vp, bl, kb = host(L.kpool), host(L.vpool), host(L.blk_len), host(L.k_bar)
    exact = 0
    for b in range(w.B):
        for h in range(w.H):
            inf = info[(b, h)]
            for s in range(w.n_sink):                   # sinks: pinned, never ranked
                assert src[b, h, s] == orc.ss[b, h, s]
                if orc.ss[b, h, s] >= 0:
                    np.testing.assert_array_equal(kp[b, h, s], orc.kp[b, h, s])
                    np.testing.assert_array_equal(vp[b, h, s], orc.vp[b, h, s])
            got = [int(x) for x in src[b, h, w.n_sink:] if x >= 0]
            ok, same = band_ok(got, inf["keys"], len(inf["kept"]))
            assert ok, (b, h, sorted(got), sorted(inf["kept"]))
            assert len(got) <= w.P
            if not same:
                continue
            exact += 1
            assert np.array_equal(src[b, h], orc.ss[b, h])
            assert np.array_equal(bl[b, h, :w.P], orc.bl[b, h, :w.P])
            np.testing.assert_allclose(sw[b, h], orc.sw[b, h], rtol=0, atol=0)
            for s in range(w.P):
                if src[b, h, s] < 0:
                    continue
                if orc.sw[b, h, s] == 1.0:      # a copy: exact
                    np.testing.assert_array_equal(kp[b, h, s], orc.kp[b, h, s])
                    np.testing.assert_array_equal(vp[b, h, s], orc.vp[b, h, s])
                    np.testing.assert_allclose(kb[b, h, s], orc.kb[b, h, s], rtol=1e-5, atol=1e-6)
                else:
                    # a merge: rows to one bf16 ulp; the pooled key is their mean,
                    # so it may differ by about one ulp of the rows / sqrt(len)
                    np.testing.assert_allclose(kp[b, h, s], orc.kp[b, h, s], rtol=merged_tol, atol=1e-6)
                    np.testing.assert_allclose(vp[b, h, s], orc.vp[b, h, s], rtol=merged_tol, atol=1e-6)
                    np.testing.assert_allclose(kb[b, h, s], orc.kb[b, h, s], rtol=0, atol=2e-3)
    return exact


def _run_rollout(w, steps, attn_steps, fused=False):
    """Every step: the GPU state is re-seeded from the oracle's state after the
    previous step, then each side writes chunk t through its own placement
    (the engine's ``write_chunk``, the oracle's ``OracleLayer.write_chunk``)
    and runs score -> update -> select (per call, or as one fused routing
    call); the step's results are compared."""
    orc = O.OracleLayer.of(w)
    L = PbsaLayer(w)
    merged_seen = 0
    for t in range(steps):
        q, k, v = PI.chunk_tensors(w, t)
        _seed_gpu(L, orc, w)                    # state after step t-1
        orc.write_chunk(t, k, v)
        L.write_chunk(t, dev_storage(k, w.dtype), dev_storage(v, w.dtype))
        L.q.copy_(dev_storage(q, w.dtype))
        ref = orc.step(t, q, attend=False)
        if fused:
            L.route(t)
        else:
            L.score(t)
            ci, cs = L.candidates(t)
            L.update(ci, cs)
            L.select(t)
        torch.cuda.synchronize()
        ids = orc.place.chunk_ids(t)
        np.testing.assert_allclose(host(L.scores)[:, :, :, ids], ref["S"][:, :, :, ids],
                                   rtol=1e-4, atol=1e-6)
        if ref["info"] is not None:
            exact = _compare_memory(L, orc, w, ref["info"], merged_tol=2.0 ** -7)
            assert exact >= w.B * w.H // 2, "too many near-tie differences"
            merged_seen += int((orc.sw > 1).sum())
        # local selection: band rule against the oracle's scores
        idx, cnt = host(L.idx), host(L.cnt)
        src = host(L.slot_src)
        win = ref["win_ids"]
        qb = O.query_blocks(w.chunk_tokens, w.bs)
        for b in range(w.B):
            for h in range(w.H):
                slots = [s for s in range(w.P) if src[b, h, s] >= 0]
                for i in range(L.nQB):
                    lst = [int(x) for x in idx[b, h, i, :cnt[b, h, i]]]
                    assert lst == sorted(set(lst))
                    assert [x for x in lst if x < w.P] == slots
                    # token mask: only blocks that start at or before the block's last query
                    last_q = t * w.chunk_tokens + qb[i][0] + qb[i][1] - 1
                    cands = [j for j in win
                             if w.mask == PI.MASK_CHUNK or orc.bp[b, h, j] <= last_q]
                    keys = {j: ref["S"][b, h, i, j] for j in cands}
                    ok, _ = band_ok([x for x in lst if x >= w.P], keys, min(w.k, len(cands)))
                    assert ok, (t, b, h, i)
        if t in attn_steps:
            # attention on the oracle's post-update pool with the oracle's lists
            dbf = K.dims(w.B, w.H, w.D, w.bs, orc.scale, torch.bfloat16)
            o = torch.zeros(w.B, w.H, w.chunk_tokens, w.D, dtype=torch.bfloat16, device="cuda")
            lse = torch.zeros(w.B, w.H, w.chunk_tokens, dtype=torch.float32, device="cuda")
            K.attn_fwd(dbf, dev_storage(q, "bf16"), w.chunk_tokens, t * w.chunk_tokens,
                       dev_storage(orc.kp, "bf16"), dev_storage(orc.vp, "bf16"), orc.place.NB,
                       dev_i32(orc.bl), dev_i32(orc.bp), dev_i32(ref["idx"]), dev_i32(ref["cnt"]),
                       ref["idx"].shape[-1], w.mask, o, lse)
            torch.cuda.synchronize()
            ro, rl = O.attention_fwd(O.round_bf16(q), O.round_bf16(orc.kp), O.round_bf16(orc.vp),
                                     orc.bl, orc.bp, ref["idx"], ref["cnt"], orc.scale, w.mask,
                                     t * w.chunk_tokens)
            mx, mean = attn_errors(host(o), ro)
            assert mx <= ATT_MAX and mean <= ATT_MEAN, (t, mx, mean)
    return merged_seen


@pytest.mark.slow
def test_rollout20s_merge_memory_reseeded():
    w = PI.WORKLOADS["rollout20s"]
    merged = _run_rollout(w, steps=12, attn_steps={6, 11})
    assert merged > 0, "the merge policy never merged a block"


@pytest.mark.slow
def test_rollout1min_one_layer_evict_reseeded():
    w = PI.WORKLOADS["rollout1min"]
    _run_rollout(w, steps=8, attn_steps={7})


@pytest.mark.parametrize("fused", [False, True])
def test_free_running_rollout_invariants(fused):
    # all 27 steps of the 20-second rollout on the GPU alone, through the
    # per-call path and through the fused routing call: budget, list
    # structure and weights stay consistent at every step
    w = PI.WORKLOADS["rollout20s"]
    L = PbsaLayer(w)
    nb_c = len(O.chunk_blocks(w.chunk_tokens, w.bs))
    admitted = 0
    for t in range(w.n_chunks):
        q, k, v = PI.chunk_tensors(w, t)
        L.write_chunk(t, torch.from_numpy(k).cuda().bfloat16(), torch.from_numpy(v).cuda().bfloat16())
        L.q.copy_(dev_storage(q, w.dtype))
        L.step(t, fused=fused)
        torch.cuda.synchronize()
        if O.leaving_chunk(t, w.W) is not None:
            admitted += nb_c
        src, sw, bl = host(L.slot_src), host(L.slot_w), host(L.blk_len)
        cnt, idx = host(L.cnt), host(L.idx)
        for b in range(w.B):
            for h in range(w.H):
                valid = src[b, h] >= 0
                assert valid.sum() == min(w.P, admitted)
                assert np.all(bl[b, h, :w.P][valid] > 0) and np.all(bl[b, h, :w.P][~valid] == 0)
                # every admitted block is in exactly one slot's weight (merge policy)
                assert abs(sw[b, h].sum() - admitted) < 1e-3
                assert np.all(cnt[b, h] == valid.sum() + min(w.k, len(O.window_chunks(t, w.W)) * nb_c))
        o = host(L.o)
        assert np.isfinite(o).all()


@pytest.mark.parametrize("policy", [PI.POLICY_EVICT, PI.POLICY_MERGE_MEAN])
@pytest.mark.parametrize("fused", [False, True])
def test_rollout_with_a_sink_slot(policy, fused):
    # one pinned sink slot (block 0 of the rollout): block 0 leaves the window
    # at step 2 and must land in slot 0 and stay there, never ranked out nor
    # merged into, through both the per-call and the fused routing path
    w = PI.variant(PI.WORKLOADS["tiny"], n_sink=1, policy=policy, rollout=True, n_chunks=7,
                   seed=11)
    _run_rollout(w, steps=7, attn_steps={2, 6}, fused=fused)


def test_rollout_reseeded_with_token_mask_and_fp32():
    # the tiny fp32 shape as a rollout under the token-causal mask
    w = PI.variant(PI.WORKLOADS["tiny"], mask=PI.MASK_TOKEN, rollout=True, n_chunks=6, seed=12)
    _run_rollout(w, steps=6, attn_steps={3, 5})
