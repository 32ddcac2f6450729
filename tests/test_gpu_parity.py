"""GPU parity of every step of the CUDA path against the CPU oracle.

All calls go through the C ABI (ctypes binding).  Inputs are the seeded
workloads of ``pbsa_inputs``; the oracle runs on the same values.
Tolerances: index sets bit-exact except ids within 1e-4 of the selection
threshold (which may swap); pooled keys / scores to fp32 rounding; attention
max-abs <= 2e-2 and mean-abs <= 2e-3 (bf16 inputs, fp32 accumulation).
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
import pbsa_inputs as PI
from block_sparse_attention_39_b200 import pbsa as K
from block_sparse_attention_39_b200.engine import PbsaLayer
from tests.gpu_util import (ATT_MAX, ATT_MEAN, attn_errors, band_ok, check_step_attention,
                            dev_i32, dev_storage, host, load_snapshot, oracle_snapshot_step)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _status_clean():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    K.get_status()
    yield
    assert K.get_status() == 0, "a kernel reported a device-side error"


def _snapshot_case(name, **kw):
    w = PI.variant(PI.WORKLOADS[name], **kw) if kw else PI.WORKLOADS[name]
    chunks = PI.snapshot_chunks(w)
    return w, chunks, oracle_snapshot_step(w, chunks)


CASES = {
    "tiny": dict(),
    "tiny_allkept": dict(P=8, k=8),
    "tiny_token": dict(mask=PI.MASK_TOKEN),
    # one sink slot (block 0, pinned), both policies
    "tiny_sink": dict(n_sink=1),
    "tiny_sink_merge": dict(n_sink=1, policy=PI.POLICY_MERGE_MEAN),
    "decode": dict(),
}
_cache = {}


def case(key):
    if key not in _cache:
        name = "decode" if key == "decode" else "tiny"
        _cache[key] = _snapshot_case(name, **CASES[key])
    return _cache[key]


def _run_gpu_step(w, chunks):
    L = PbsaLayer(w)
    load_snapshot(L, w, chunks)
    t = w.n_chunks - 1
    L.score(t, pool_ids=L.all_ids())
    torch.cuda.synchronize()
    pre = dict(q_bar=host(L.q_bar), k_bar=host(L.k_bar), S=host(L.scores), m=host(L.mem))
    ci, cs = L.candidates(t)
    L.update(ci, cs)
    L.select(t)
    L.attend(t)
    torch.cuda.synchronize()
    return L, pre


@pytest.mark.parametrize("key", list(CASES))
def test_score_blocks_match_oracle(key):
    w, chunks, ref = case(key)
    _, pre = _run_gpu_step(w, chunks)
    np.testing.assert_allclose(pre["q_bar"], ref["q_bar"], rtol=1e-5, atol=1e-6)
    ids = ref["all_ids"]
    np.testing.assert_allclose(pre["k_bar"][:, :, ids], ref["k_bar"][:, :, ids], rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(pre["S"][:, :, :, ids], ref["S"][:, :, :, ids], rtol=1e-4, atol=1e-6)
    np.testing.assert_allclose(pre["m"][:, :, ids], ref["m"][:, :, ids], rtol=1e-4, atol=1e-6)


@pytest.mark.parametrize("key", list(CASES))
def test_update_memory_matches_oracle(key):
    w, chunks, ref = case(key)
    L, _ = _run_gpu_step(w, chunks)
    src = host(L.slot_src)
    kp, vp, bl = host(L.kpool), host(L.vpool), host(L.blk_len)
    kbar = host(L.k_bar)
    exact = 0
    for b in range(w.B):
        for h in range(w.H):
            info = ref["info"][(b, h)]
            # sink slots hold their own block, never ranked
            for s in range(w.n_sink):
                assert src[b, h, s] == ref["slot_src"][b, h, s] == s
                np.testing.assert_array_equal(kp[b, h, s], ref["kpool"][b, h, s])
            got = [int(x) for x in src[b, h, w.n_sink:] if x >= 0]
            ok, same = band_ok(got, info["keys"], len(info["kept"]))
            assert ok, (b, h, sorted(got), sorted(info["kept"]))
            if not same:
                continue
            exact += 1
            for s in range(w.P):
                assert src[b, h, s] == ref["slot_src"][b, h, s]
                if src[b, h, s] < 0:
                    continue
                assert bl[b, h, s] == ref["blk_len"][b, h, s]
                if ref["slot_w"][b, h, s] == 1.0:
                    # a copied block: exact
                    np.testing.assert_array_equal(kp[b, h, s], ref["kpool"][b, h, s])
                    np.testing.assert_array_equal(vp[b, h, s], ref["vpool"][b, h, s])
                    np.testing.assert_allclose(kbar[b, h, s], ref["k_bar2"][b, h, s], rtol=1e-5,
                                               atol=1e-6)
                else:
                    # a merged slot: the GPU averages in fp32, the oracle in fp64, both
                    # round once to storage, so rows may differ by one storage ulp
                    ulp = 2.0 ** -7 if w.dtype == "bf16" else 2.0 ** -22
                    np.testing.assert_allclose(kp[b, h, s], ref["kpool"][b, h, s], rtol=ulp,
                                               atol=1e-6)
                    np.testing.assert_allclose(vp[b, h, s], ref["vpool"][b, h, s], rtol=ulp,
                                               atol=1e-6)
                    np.testing.assert_allclose(kbar[b, h, s], ref["k_bar2"][b, h, s], rtol=0,
                                               atol=2e-3)
    assert exact >= (w.B * w.H + 1) // 2, "too many near-tie differences"


@pytest.mark.parametrize("key", list(CASES))
def test_select_local_matches_oracle(key):
    w, chunks, ref = case(key)
    L, _ = _run_gpu_step(w, chunks)
    idx, cnt = host(L.idx), host(L.cnt)
    src = host(L.slot_src)
    S = ref["S"]
    lens = O.query_block_lengths(w.chunk_tokens, w.bs)
    for b in range(w.B):
        for h in range(w.H):
            slots = [s for s in range(w.P) if src[b, h, s] >= 0]
            for i in range(L.nQB):
                lst = [int(x) for x in idx[b, h, i, :cnt[b, h, i]]]
                assert lst == sorted(set(lst)), "list must be ascending without duplicates"
                assert all(x == -1 for x in idx[b, h, i, cnt[b, h, i]:])
                assert [x for x in lst if x < w.P] == slots
                local = [x for x in lst if x >= w.P]
                cands = [int(j) for j in ref["win_ids"]
                         if w.mask == PI.MASK_CHUNK or
                         ref["blk_pos"][b, h, j] <= ref["q_pos0"] + i * w.bs + lens[i] - 1]
                keys = {j: S[b, h, i, j] for j in cands}
                ok, _ = band_ok(local, keys, min(w.k, len(cands)))
                assert ok, (b, h, i, local)


@pytest.mark.parametrize("key", list(CASES))
def test_attention_forward_with_oracle_lists(key):
    w, chunks, ref = case(key)
    dbf = K.dims(w.B, w.H, w.D, w.bs, 1 / math.sqrt(w.D), torch.bfloat16)
    q = dev_storage(ref["q16"], "bf16")
    kp = dev_storage(ref["k16"], "bf16")
    vp = dev_storage(ref["v16"], "bf16")
    o = torch.zeros(w.B, w.H, w.chunk_tokens, w.D, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(w.B, w.H, w.chunk_tokens, dtype=torch.float32, device="cuda")
    amax = ref["idx"].shape[-1]
    K.attn_fwd(dbf, q, w.chunk_tokens, ref["q_pos0"], kp, vp, ref["orc"].place.NB, dev_i32(ref["blk_len"]),
               dev_i32(ref["blk_pos"]), dev_i32(ref["idx"]), dev_i32(ref["cnt"]), amax, w.mask, o,
               lse)
    torch.cuda.synchronize()
    mx, mean = attn_errors(host(o), ref["O"])
    assert mx <= ATT_MAX and mean <= ATT_MEAN, (mx, mean)
    np.testing.assert_allclose(host(lse), ref["lse"], atol=2e-3, rtol=0)


def test_all_kept_equals_dense_attention():
    # every cache block is attended: the PBSA output must equal dense attention
    # of the query chunk over the whole cache, built here from the chunk tensors
    # themselves (no pool, no placement)
    w, chunks, ref = case("tiny_allkept")
    assert all(int(c) == 16 for c in ref["cnt"].reshape(-1))
    L, _ = _run_gpu_step(w, chunks)
    q16 = O.round_bf16(chunks[w.n_chunks - 1][0])
    kc = O.round_bf16(np.concatenate([chunks[t][1] for t in range(w.n_chunks)], axis=2))
    vc = O.round_bf16(np.concatenate([chunks[t][2] for t in range(w.n_chunks)], axis=2))
    assert kc.shape[2] == 1024
    dense = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q16), torch.from_numpy(kc), torch.from_numpy(vc),
        scale=1 / math.sqrt(w.D)).numpy()
    mx, mean = attn_errors(host(L.o), dense)
    assert mx <= ATT_MAX and mean <= ATT_MEAN, (mx, mean)


@pytest.mark.parametrize("key", list(CASES))
def test_full_step_output(key):
    w, chunks, ref = case(key)
    L, _ = _run_gpu_step(w, chunks)
    check_step_attention(L, w, ref, chunks[w.n_chunks - 1][0])


# ---------------------------------------------------------------- edge cases

def _random_attention_case(seed, B, H, D, bs, Tq, NB, Amax, mask, empty_rows=True):
    r = np.random.default_rng(seed)
    kp = O.round_bf16(r.standard_normal((B, H, NB, bs, D)))
    vp = O.round_bf16(r.standard_normal((B, H, NB, bs, D)))
    q = O.round_bf16(r.standard_normal((B, H, Tq, D)))
    bl = r.integers(1, bs + 1, size=(B, H, NB)).astype(np.int32)
    bp = (np.arange(NB) * bs).astype(np.int32)[None, None, :].repeat(B, 0).repeat(H, 1)
    nQB = -(-Tq // bs)
    idx = np.full((B, H, nQB, Amax), -1, dtype=np.int32)
    cnt = np.zeros((B, H, nQB), dtype=np.int32)
    for b in range(B):
        for h in range(H):
            for i in range(nQB):
                n = int(r.integers(0 if empty_rows else 1, Amax + 1))
                ids = np.sort(r.choice(NB, size=n, replace=False))
                idx[b, h, i, :n] = ids
                cnt[b, h, i] = n
    q_pos0 = int(bp[0, 0, -1])            # queries sit at the end of the pool (token mask)
    return q, kp, vp, bl, bp, idx, cnt, q_pos0


@pytest.mark.parametrize("D,bs", [(128, 128), (64, 64), (128, 64), (64, 128)])
@pytest.mark.parametrize("Tq", [50, 200, 384])
@pytest.mark.parametrize("mask", [PI.MASK_CHUNK, PI.MASK_TOKEN])
def test_attention_shapes_ragged_and_empty(D, bs, Tq, mask):
    B, H, NB, Amax = 1, 3, 9, 6
    q, kp, vp, bl, bp, idx, cnt, q_pos0 = _random_attention_case(D * 7 + bs + Tq + mask, B, H, D,
                                                                 bs, Tq, NB, Amax, mask)
    scale = 1 / math.sqrt(D)
    ref_o, ref_l = O.attention_fwd(q, kp, vp, bl, bp, idx, cnt, scale, mask, q_pos0)
    d = K.dims(B, H, D, bs, scale, torch.bfloat16)
    o = torch.full((B, H, Tq, D), 7.0, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(B, H, Tq, dtype=torch.float32, device="cuda")
    K.attn_fwd(d, dev_storage(q, "bf16"), Tq, q_pos0, dev_storage(kp, "bf16"),
               dev_storage(vp, "bf16"), NB, dev_i32(bl), dev_i32(bp), dev_i32(idx), dev_i32(cnt),
               Amax, mask, o, lse)
    torch.cuda.synchronize()
    mx, mean = attn_errors(host(o), ref_o)
    assert mx <= ATT_MAX and mean <= ATT_MEAN, (mx, mean)
    gl = host(lse)
    assert np.array_equal(np.isneginf(gl), np.isneginf(ref_l))
    fin = np.isfinite(ref_l)
    np.testing.assert_allclose(gl[fin], ref_l[fin], atol=2e-3, rtol=0)


@pytest.mark.parametrize("bs", [64, 128])
@pytest.mark.parametrize("mask", [PI.MASK_CHUNK, PI.MASK_TOKEN])
def test_attention_chunked_query_tiling(bs, mask):
    # 500 query rows in chunks of 200 (last chunk 100): blocks tile each chunk
    B, H, D, NB, Amax, Tq, qc = 1, 2, 128, 9, 6, 500, 200
    nQB = len(O.query_blocks(Tq, bs, qc))
    q, kp, vp, bl, bp, idx, cnt, q_pos0 = _random_attention_case(bs + mask, B, H, D, bs, nQB * bs,
                                                                 NB, Amax, mask)
    q = q[:, :, :Tq]
    scale = 1 / math.sqrt(D)
    ref_o, ref_l = O.attention_fwd(q, kp, vp, bl, bp, idx, cnt, scale, mask, q_pos0, q_chunk=qc)
    d = K.dims(B, H, D, bs, scale, torch.bfloat16, q_chunk=qc)
    o = torch.zeros(B, H, Tq, D, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(B, H, Tq, dtype=torch.float32, device="cuda")
    K.attn_fwd(d, dev_storage(q, "bf16"), Tq, q_pos0, dev_storage(kp, "bf16"),
               dev_storage(vp, "bf16"), NB, dev_i32(bl), dev_i32(bp), dev_i32(idx), dev_i32(cnt),
               Amax, mask, o, lse)
    torch.cuda.synchronize()
    mx, mean = attn_errors(host(o), ref_o)
    assert mx <= ATT_MAX and mean <= ATT_MEAN, (mx, mean)
    fin = np.isfinite(ref_l)
    np.testing.assert_allclose(host(lse)[fin], ref_l[fin], atol=2e-3, rtol=0)


def test_attention_long_lists_near_capacity():
    # 120 attended blocks per query block (longer than any workload's list)
    B, H, D, bs, Tq, NB, Amax = 1, 2, 128, 128, 256, 130, 120
    q, kp, vp, bl, bp, idx, cnt, q_pos0 = _random_attention_case(5, B, H, D, bs, Tq, NB, Amax,
                                                                 PI.MASK_CHUNK, empty_rows=False)
    cnt[:] = Amax
    for b in range(B):
        for h in range(H):
            for i in range(idx.shape[2]):
                idx[b, h, i] = np.sort(np.random.default_rng(i + 10 * h).choice(NB, Amax, replace=False))
    scale = 1 / math.sqrt(D)
    ref_o, _ = O.attention_fwd(q, kp, vp, bl, bp, idx, cnt, scale)
    d = K.dims(B, H, D, bs, scale, torch.bfloat16)
    o = torch.zeros(B, H, Tq, D, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(B, H, Tq, dtype=torch.float32, device="cuda")
    K.attn_fwd(d, dev_storage(q, "bf16"), Tq, 0, dev_storage(kp, "bf16"), dev_storage(vp, "bf16"),
               NB, dev_i32(bl), dev_i32(bp), dev_i32(idx), dev_i32(cnt), Amax, PI.MASK_CHUNK, o, lse)
    torch.cuda.synchronize()
    mx, mean = attn_errors(host(o), ref_o)
    assert mx <= ATT_MAX and mean <= ATT_MEAN, (mx, mean)
