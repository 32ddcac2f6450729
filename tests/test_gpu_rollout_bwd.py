"""GPU parity of the recurrent trainable path: the backward of a rollout
through attention and the persistent memory (pbsa_update_memory_bwd) against
the oracle's ``update_memory_vjp`` and ``rollout_bwd``.

A small bf16 merge rollout (2 heads of 64, 64-token blocks, 4-block chunks,
4 slots, 6 steps) runs free on the GPU and on the oracle; its decisions (kept
slots, lists) must agree at every step, and then:
* the memory update's backward on one step with a random incoming gradient
  equals the oracle's transposed weighted means (fp32 against fp64);
* every step's dQ and every chunk's dK, dV of the loss sum_t <O_t, dO_t>
  equal the oracle's within the gradient rule of the other backward tests
  (max-abs <= 2e-2 + 2^-8 max|ref|, mean-abs <= 2e-3 + 2^-8 mean|ref|).
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
import pbsa_inputs as PI
from block_sparse_attention_39_b200 import pbsa as K
from block_sparse_attention_39_b200.engine import PbsaLayer, PbsaRolloutTrain
from tests.gpu_util import dev_storage, host

pytestmark = pytest.mark.gpu

W_ROLL = PI.variant(PI.WORKLOADS["rollout20s"], name="rollout_bwd_small", B=1, H=2, D=64, bs=64,
                    chunk_tokens=256, P=4, k=2, n_chunks=6, salient_frac=0.25, redraw_every=2,
                    seed=21)


@pytest.fixture(autouse=True)
def _status_clean():
    assert torch.cuda.is_available()
    K.get_status()
    yield
    assert K.get_status() == 0


def _grad_ok(got, ref, what):
    d = np.abs(got - ref)
    mx_lim = 2e-2 + 2.0 ** -8 * np.abs(ref).max()
    mean_lim = 2e-3 + 2.0 ** -8 * np.abs(ref).mean()
    assert d.max() <= mx_lim and d.mean() <= mean_lim, (what, d.max(), mx_lim, d.mean(), mean_lim)


def _run_both(w):
    L = PbsaLayer(w)
    tr = PbsaRolloutTrain(L)
    orc = O.OracleLayer.of(w)
    steps, dOs = [], []
    merges = 0
    for t in range(w.n_chunks):
        q, k, v = PI.chunk_tensors(w, t)
        dO = O.round_bf16(PI.normal((w.B, w.H, w.chunk_tokens, w.D), w.seed, "dO", 0, t))
        tr.step(t, dev_storage(q, w.dtype), dev_storage(k, w.dtype), dev_storage(v, w.dtype))
        orc.write_chunk(t, k, v)
        r = orc.step(t, q)
        torch.cuda.synchronize()
        # the two recurrences take the same decisions at every step
        np.testing.assert_array_equal(host(L.slot_src), r["slot_src"], err_msg=f"step {t}")
        np.testing.assert_array_equal(host(L.cnt), r["cnt"], err_msg=f"step {t}")
        np.testing.assert_array_equal(host(L.idx), r["idx"], err_msg=f"step {t}")
        if r["info"] is not None:
            merges += sum(len(terms) > 1 for inf in r["info"].values()
                          for terms in inf["compose"].values())
        steps.append(dict(q=r["q16"], kp=r["kpool"].copy(), vp=r["vpool"].copy(),
                          bl=r["blk_len"].copy(), bp=r["blk_pos"].copy(), idx=r["idx"].copy(),
                          cnt=r["cnt"].copy(), info=r["info"], dO=dO))
        dOs.append(dev_storage(dO, "bf16"))
    return L, tr, orc, steps, dOs, merges


def test_update_memory_bwd_matches_oracle_vjp():
    w = W_ROLL
    L, tr, orc, steps, _, merges = _run_both(w)
    assert merges > 0
    rng = np.random.default_rng(0)
    checked = 0
    for t, st in enumerate(steps):
        rec = tr.steps[t]
        if rec["plan"] is None:
            continue
        g_k = rng.standard_normal((w.B, w.H, L.NB, w.bs, w.D)).astype(np.float32)
        g_v = rng.standard_normal((w.B, w.H, L.NB, w.bs, w.D)).astype(np.float32)
        dk = torch.from_numpy(g_k).cuda()
        dv = torch.from_numpy(g_v).cuda()
        K.update_memory_bwd(L.d, L.NB, L.P, rec["n_cand"], rec["plan"], dk, dv, tr.upd_ws)
        want_k, want_v = O.update_memory_vjp(g_k.astype(np.float64), g_v.astype(np.float64),
                                             st["info"], L.P)
        np.testing.assert_allclose(host(dk), want_k, rtol=1e-5, atol=1e-5)
        np.testing.assert_allclose(host(dv), want_v, rtol=1e-5, atol=1e-5)
        checked += 1
    assert checked >= 2


def test_rollout_backward_matches_oracle():
    w = W_ROLL
    L, tr, orc, steps, dOs, merges = _run_both(w)
    assert merges > 0
    dq, dk, dv = tr.backward(dOs)
    rq, rk, rv = O.rollout_bwd(steps, L.P, orc.place, w.W, w.chunk_tokens, 1.0 / math.sqrt(w.D),
                               w.mask)
    for t in range(w.n_chunks):
        _grad_ok(host(dq[t]), rq[t], ("dq", t))
        _grad_ok(host(dk[t]), rk[t], ("dk", t))
        _grad_ok(host(dv[t]), rv[t], ("dv", t))
    # the memory path matters: the first chunk is attended through the slots
    # long after it left the window, so the backward without the slot path
    # (attention gradients of the steps that saw it directly) differs
    direct = [O.attention_bwd(st["q"], st["kp"], st["vp"], st["bl"], st["bp"], st["idx"],
                              st["cnt"], st["dO"], 1.0 / math.sqrt(w.D), w.mask,
                              t * w.chunk_tokens)[1] for t, st in enumerate(steps[:w.W])]
    ids0 = orc.place.chunk_ids(0)
    direct_k0 = sum(d[:, :, ids0] for d in direct)
    slot_part = np.abs(rk[0] - direct_k0.reshape(w.B, w.H, -1, w.D)[:, :, :w.chunk_tokens]).max()
    assert slot_part > 1e-3
