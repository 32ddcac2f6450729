"""GPU parity of the KV append with fused block compression (pbsa_append_chunk).

The rows must land in their pool blocks bit-exactly (a copy), the padding rows
of a partial block must be zero, every other block and its metadata must be
left alone, and the pooled keys must equal the oracle's block means to fp32
rounding.  They must also be bit-identical to the pooled keys that
pbsa_score_blocks computes for the same blocks, since the chunk step skips the
key pooling after an append.  Two layers run the whole 20-second rollout side
by side, one fed through write_chunk and one through append, and their outputs
must stay identical.
"""
import math
import zlib

import numpy as np
import pytest
import torch

import oracle as O
import pbsa_inputs as PI
from block_sparse_attention_39_b200 import pbsa as K
from block_sparse_attention_39_b200.engine import PbsaLayer
from tests.gpu_util import dev_i32, dev_storage, host

pytestmark = pytest.mark.gpu

ERR_ARG = -1


@pytest.fixture(autouse=True)
def _status_clean():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    K.get_status()
    yield
    assert K.get_status() == 0, "a kernel reported a device-side error"


# (B, H, D, bs, dtype, Tc, NB): several tiles, a ragged last block, a chunk
# shorter than one block, one full block, the decode chunk (4680 = 36*128 + 72)
CASES = {
    "ragged_bf16": (1, 2, 128, 128, "bf16", 300, 8),
    "f32_d64": (2, 3, 64, 64, "f32", 1000, 20),
    "short": (1, 1, 128, 64, "bf16", 5, 3),
    "one_full": (1, 2, 64, 128, "bf16", 128, 2),
    "f32_d128_bs128": (1, 2, 128, 128, "f32", 700, 9),
    "decode_chunk": (1, 12, 128, 128, "bf16", 4680, 48),
}


def _make(key):
    B, H, D, bs, dt, Tc, NB = CASES[key]
    r = np.random.default_rng(zlib.crc32(key.encode()))
    nb = -(-Tc // bs)
    ids = r.permutation(NB)[:nb].astype(np.int32)
    k = O.round_storage(r.standard_normal((B, H, Tc, D)), dt)
    v = O.round_storage(r.standard_normal((B, H, Tc, D)), dt)
    kp0 = O.round_storage(r.standard_normal((B, H, NB, bs, D)) + 5.0, dt)
    vp0 = O.round_storage(r.standard_normal((B, H, NB, bs, D)) - 5.0, dt)
    bl0 = r.integers(1, bs + 1, (B, H, NB)).astype(np.int32)
    bp0 = r.integers(0, 10 ** 6, (B, H, NB)).astype(np.int32)
    kb0 = r.standard_normal((B, H, NB, D))
    return dict(B=B, H=H, D=D, bs=bs, dt=dt, Tc=Tc, NB=NB, nb=nb, ids=ids, k=k, v=v, kp0=kp0,
                vp0=vp0, bl0=bl0, bp0=bp0, kb0=kb0, pos0=int(r.integers(0, 10 ** 5)))


def _expected(c):
    """The pool after the append, placed by hand; pooled keys from the oracle."""
    kp, vp = c["kp0"].copy(), c["vp0"].copy()
    bl, bp = c["bl0"].copy(), c["bp0"].copy()
    bs = c["bs"]
    for j, pid in enumerate(c["ids"]):
        n = min(bs, c["Tc"] - j * bs)
        kp[:, :, pid] = 0.0
        vp[:, :, pid] = 0.0
        kp[:, :, pid, :n] = c["k"][:, :, j * bs:j * bs + n]
        vp[:, :, pid, :n] = c["v"][:, :, j * bs:j * bs + n]
        bl[:, :, pid] = n
        bp[:, :, pid] = c["pos0"] + j * bs
    kb = O.pool_keys(kp, bl, c["ids"], c["kb0"].copy())
    return kp, vp, bl, bp, kb


def _run(c, ids=None):
    tdt = torch.bfloat16 if c["dt"] == "bf16" else torch.float32
    d = K.dims(c["B"], c["H"], c["D"], c["bs"], 1 / math.sqrt(c["D"]), tdt)
    kp, vp = dev_storage(c["kp0"], c["dt"]), dev_storage(c["vp0"], c["dt"])
    bl, bp = dev_i32(c["bl0"]), dev_i32(c["bp0"])
    kb = torch.from_numpy(c["kb0"].astype(np.float32)).cuda()
    K.append_chunk(d, dev_storage(c["k"], c["dt"]), dev_storage(c["v"], c["dt"]), c["Tc"],
                   c["pos0"], kp, vp, c["NB"], dev_i32(c["ids"] if ids is None else ids), bl, bp,
                   kb)
    torch.cuda.synchronize()
    return d, kp, vp, bl, bp, kb


@pytest.mark.parametrize("key", list(CASES))
def test_append_matches_oracle(key):
    c = _make(key)
    d, kp, vp, bl, bp, kb = _run(c)
    ekp, evp, ebl, ebp, ekb = _expected(c)
    # rows, padding and untouched blocks: exact
    np.testing.assert_array_equal(host(kp), ekp)
    np.testing.assert_array_equal(host(vp), evp)
    np.testing.assert_array_equal(host(bl), ebl)
    np.testing.assert_array_equal(host(bp), ebp)
    gkb = host(kb)
    ids = c["ids"]
    others = np.setdiff1d(np.arange(c["NB"]), ids)
    np.testing.assert_array_equal(gkb[:, :, others], c["kb0"][:, :, others].astype(np.float32))
    np.testing.assert_allclose(gkb[:, :, ids], ekb[:, :, ids], rtol=1e-5, atol=1e-6)

    # the same blocks pooled by pbsa_score_blocks give the same bits
    kb2 = torch.zeros_like(kb)
    Tq = c["bs"]
    q = torch.zeros(c["B"], c["H"], Tq, c["D"], dtype=kp.dtype, device="cuda")
    q_bar = torch.zeros(c["B"], c["H"], 1, c["D"], dtype=torch.float32, device="cuda")
    scores = torch.zeros(c["B"], c["H"], 1, c["NB"], dtype=torch.float32, device="cuda")
    mem = torch.zeros(c["B"], c["H"], c["NB"], dtype=torch.float32, device="cuda")
    K.score_blocks(d, q, Tq, kp, c["NB"], bl, dev_i32(ids), len(ids), q_bar, kb2, scores, mem)
    torch.cuda.synchronize()
    assert torch.equal(kb2[:, :, torch.from_numpy(ids).long().cuda()],
                       kb[:, :, torch.from_numpy(ids).long().cuda()])


def test_append_bad_id_sets_status_and_skips_block():
    c = _make("ragged_bf16")
    ids = c["ids"].copy()
    ids[1] = c["NB"]                                  # outside the pool
    K.get_status()
    _, kp, vp, bl, bp, kb = _run(c, ids=ids)
    assert K.get_status() == ERR_ARG
    # blocks 0 and 2 of the chunk are written as usual; block 1 nowhere
    kp_h, bl_h = host(kp), host(bl)
    bs = c["bs"]
    for j in (0, 2):
        pid = ids[j]
        n = min(bs, c["Tc"] - j * bs)
        np.testing.assert_array_equal(kp_h[:, :, pid, :n], c["k"][:, :, j * bs:j * bs + n])
        assert np.all(bl_h[:, :, pid] == n)
    untouched = np.setdiff1d(np.arange(c["NB"]), ids[[0, 2]])
    np.testing.assert_array_equal(kp_h[:, :, untouched], c["kp0"][:, :, untouched])
    np.testing.assert_array_equal(bl_h[:, :, untouched], c["bl0"][:, :, untouched])


@pytest.mark.parametrize("fused", [False, True])
def test_rollout_through_append_is_identical(fused):
    # every step of the 20-second rollout: one layer fed by write_chunk (the
    # chunk's keys pooled inside the score call), one by append (pooled while
    # written); same bits everywhere
    w = PI.WORKLOADS["rollout20s"]
    La, Lb = PbsaLayer(w), PbsaLayer(w)
    for t in range(w.n_chunks):
        q, k, v = PI.chunk_tensors(w, t)
        kd = torch.from_numpy(k).cuda().bfloat16()
        vd = torch.from_numpy(v).cuda().bfloat16()
        qd = dev_storage(q, w.dtype)
        La.write_chunk(t, kd, vd)
        Lb.append(t, kd, vd)
        La.q.copy_(qd)
        Lb.q.copy_(qd)
        La.step(t, fused=fused)
        Lb.step(t, fused=fused, appended=True)
        torch.cuda.synchronize()
        for name in ("kpool", "vpool", "blk_len", "blk_pos", "k_bar", "slot_src", "slot_w",
                     "scores", "idx", "cnt", "o", "lse"):
            assert torch.equal(getattr(La, name), getattr(Lb, name)), (t, name)
