"""GPU parity of pbsa_score_blocks on the shapes the decode snapshots do not
reach: queries of several chunks (a memory score per chunk), chunks that span
score tiles, one query block per chunk, a single chunk longer than a tile,
key-block counts that are not tile multiples, empty key blocks, fp32 and bf16,
D = 64 and 128; calls with thousands of score tiles, whose bits must equal
those of a single head scored alone.

The oracle pools and scores as written (fp64), and its memory score of chunk g
is the mean of S over the chunk's query blocks.  Tolerances as in the other
scoring tests: pooled means rtol 1e-5, scores and memory scores rtol 1e-4.
"""
import math
import zlib

import numpy as np
import pytest
import torch

import oracle as O
from block_sparse_attention_39_b200 import pbsa as K
from tests.gpu_util import dev_i32, dev_storage, host

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _status_clean():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    K.get_status()
    yield
    assert K.get_status() == 0, "a kernel reported a device-side error"


# (B, H, D, bs, dtype, Tq, q_chunk, NB, n_pool)
CASES = {
    # three 4680-token chunks of 37 blocks: chunks start inside score tiles
    "chunks37_bf16": (1, 2, 128, 128, "bf16", 3 * 4680, 4680, 150, 150),
    # chunks of 200 rows tiled into 64 + 64 + 64 + 8: four blocks per chunk
    "chunks4_f32_d64": (2, 3, 64, 64, "f32", 1000, 200, 70, 70),
    # one query block per chunk (q_chunk = bs): a memory score per block
    "chunk_per_block": (1, 1, 128, 64, "bf16", 2100, 64, 33, 33),
    # one chunk of 70 query blocks: longer than a tile
    "one_long_chunk_f32": (1, 1, 128, 128, "f32", 128 * 70, 0, 40, 40),
    # few blocks; only some key blocks re-pooled, the others keep their k_bar
    "small_partial_pool": (1, 2, 64, 128, "bf16", 300, 0, 5, 3),
    # 259 x 259 blocks per head over 12 heads (2700 score tiles, ragged last
    # row and column tiles), chunks of 37 blocks
    "large_d128_bf16": (1, 12, 128, 64, "bf16", 64 * 259 - 5, 64 * 37, 259, 259),
    # 128 x 330 blocks per head over 25 heads, one chunk spanning every row
    # tile; some blocks not re-pooled
    "large_d64_f32": (1, 25, 64, 64, "f32", 64 * 128, 0, 330, 200),
}


def _case(key):
    B, H, D, bs, dt, Tq, qc, NB, n_pool = CASES[key]
    r = np.random.default_rng(zlib.crc32(key.encode()))
    q = O.round_storage(r.standard_normal((B, H, Tq, D)), dt)
    kp = O.round_storage(r.standard_normal((B, H, NB, bs, D)), dt)
    bl = r.integers(0, bs + 1, (B, H, NB)).astype(np.int32)
    bl[..., 0] = 0                                   # an empty block pools to zero
    ids = np.sort(r.permutation(NB)[:n_pool]).astype(np.int32)
    kb0 = r.standard_normal((B, H, NB, D)).astype(np.float32).astype(np.float64)
    return dict(B=B, H=H, D=D, bs=bs, dt=dt, Tq=Tq, qc=qc, NB=NB, q=q, kp=kp, bl=bl, ids=ids,
                kb0=kb0)


def _oracle(c, scale):
    qb, kb, S, _ = O.score_blocks(c["q"], c["kp"], c["bl"], c["ids"], c["kb0"], scale, c["bs"],
                                  c["qc"])
    qc = c["qc"] if c["qc"] > 0 else c["Tq"]
    per_group = -(-qc // c["bs"])
    groups = -(-c["Tq"] // qc)
    nQB = S.shape[2]
    m = np.stack([O.memory_scores(S[:, :, g * per_group:min(nQB, (g + 1) * per_group)])
                  for g in range(groups)], axis=2)
    return qb, kb, S, m


@pytest.mark.parametrize("key", list(CASES))
def test_score_blocks_shapes_match_oracle(key):
    c = _case(key)
    scale = 1 / math.sqrt(c["D"])
    qb, kb, S, m = _oracle(c, scale)
    B, H, D, NB = c["B"], c["H"], c["D"], c["NB"]
    nQB, G = S.shape[2], m.shape[2]
    tdt = torch.bfloat16 if c["dt"] == "bf16" else torch.float32
    d = K.dims(B, H, D, c["bs"], scale, tdt, q_chunk=c["qc"])
    q_bar = torch.zeros(B, H, nQB, D, dtype=torch.float32, device="cuda")
    k_bar = torch.from_numpy(c["kb0"].astype(np.float32)).cuda()
    scores = torch.zeros(B, H, nQB, NB, dtype=torch.float32, device="cuda")
    mem = torch.zeros(B, H, G, NB, dtype=torch.float32, device="cuda")
    K.score_blocks(d, dev_storage(c["q"], c["dt"]), c["Tq"], dev_storage(c["kp"], c["dt"]), NB,
                   dev_i32(c["bl"]), dev_i32(c["ids"]), len(c["ids"]), q_bar, k_bar, scores, mem)
    torch.cuda.synchronize()
    np.testing.assert_allclose(host(q_bar), qb, rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(host(k_bar), kb, rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(host(scores), S, rtol=1e-4, atol=1e-6)
    np.testing.assert_allclose(host(mem), m, rtol=1e-4, atol=1e-6)


def test_large_call_gives_the_single_head_bits():
    # head (0, 3) of the large case scored alone: every score and memory
    # score of the twelve-head call must be the same fp32 number (no result
    # depends on the grid or on other heads)
    c = _case("large_d128_bf16")
    scale = 1 / math.sqrt(c["D"])
    B, H, D, NB, bs, Tq, qc = c["B"], c["H"], c["D"], c["NB"], c["bs"], c["Tq"], c["qc"]
    nQB = -(-Tq // bs)
    G = -(-Tq // qc)
    outs = []
    for hs in (slice(0, H), slice(3, 4)):
        h = hs.stop - hs.start
        d = K.dims(B, h, D, bs, scale, torch.bfloat16, q_chunk=qc)
        q_bar = torch.zeros(B, h, nQB, D, dtype=torch.float32, device="cuda")
        k_bar = torch.from_numpy(c["kb0"][:, hs].astype(np.float32)).cuda()
        scores = torch.zeros(B, h, nQB, NB, dtype=torch.float32, device="cuda")
        mem = torch.zeros(B, h, G, NB, dtype=torch.float32, device="cuda")
        K.score_blocks(d, dev_storage(np.ascontiguousarray(c["q"][:, hs]), "bf16"), Tq,
                       dev_storage(np.ascontiguousarray(c["kp"][:, hs]), "bf16"), NB,
                       dev_i32(np.ascontiguousarray(c["bl"][:, hs])), dev_i32(c["ids"]),
                       len(c["ids"]), q_bar, k_bar, scores, mem)
        torch.cuda.synchronize()
        outs.append((scores, mem))
    (s_all, m_all), (s_one, m_one) = outs
    assert torch.equal(s_all[:, 3:4], s_one)
    assert torch.equal(m_all[:, 3:4], m_one)
