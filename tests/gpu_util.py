"""Helpers shared by the GPU parity tests: moving seeded inputs to the device,
the oracle pipeline of one step, and the near-tie comparison rule."""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle as O
import pbsa_inputs as PI

TIE = 1e-4          # scores closer than this to the selection threshold may swap
ATT_MAX = 2e-2      # attention: max-abs error (bf16 inputs, fp32 accumulation)
ATT_MEAN = 2e-3     # attention: mean-abs error


def dev_storage(x: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()
    return t.to(torch.bfloat16) if dtype == "bf16" else t


def dev_i32(x) -> torch.Tensor:
    return torch.as_tensor(np.ascontiguousarray(x), dtype=torch.int32).cuda()


def host(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64) if t.is_floating_point() \
        else t.detach().cpu().numpy()


def snapshot_case(w):
    """A snapshot step's inputs: every chunk of the cache as seeded tensors
    (``{t: (q or None, k, v)}``) and the current chunk's index."""
    return PI.snapshot_chunks(w), w.n_chunks - 1


def load_snapshot(layer, w, chunks):
    """The GPU side of a snapshot: every chunk written through the engine's own
    placement, the current chunk's queries, an empty memory."""
    for t, (_, k, v) in chunks.items():
        layer.write_chunk(t, dev_storage(k, w.dtype), dev_storage(v, w.dtype))
    layer.q.copy_(dev_storage(chunks[w.n_chunks - 1][0], w.dtype))
    layer.reset_memory()


def band_ok(chosen, keys: dict, n_take: int, tie=TIE):
    """The chosen id set is the oracle's top-n_take under key (score desc, id asc),
    except that ids whose score is within `tie` of the threshold may swap."""
    order = sorted(keys, key=lambda j: (-keys[j], j))
    want = set(order[:n_take])
    chosen = set(chosen)
    if chosen == want:
        return True, True
    if len(chosen) != len(want) or not chosen <= set(keys):
        return False, False
    tau = keys[order[n_take - 1]]
    must = {j for j in keys if keys[j] > tau + tie}
    never = {j for j in keys if keys[j] < tau - tie}
    return (must <= chosen and not (chosen & never)), False


def oracle_snapshot_step(w, chunks):
    """The oracle's score -> update -> select -> attend on a snapshot: its own
    layer state, every chunk written through its own placement, every
    resident block pooled, the memory empty."""
    orc = O.OracleLayer.of(w)
    for t, (_, k, v) in chunks.items():
        orc.write_chunk(t, k, v)
    t_cur = w.n_chunks - 1
    all_ids = [p for c in range(w.n_chunks) for p in orc.place.chunk_ids(c)]
    ref = orc.step(t_cur, chunks[t_cur][0], pool_ids=all_ids)
    ref.update(orc=orc, all_ids=all_ids, q_pos0=t_cur * w.chunk_tokens,
               new_ids=orc.place.chunk_ids(t_cur))
    return ref


def attn_errors(o_gpu: np.ndarray, o_ref: np.ndarray, rows=None):
    d = np.abs(o_gpu - o_ref)
    if rows is not None:
        d = d[rows]
    return float(d.max()), float(d.mean())


def check_step_attention(L, w, ref, q):
    """The attention of a whole GPU step, checked without depending on near-tie
    luck: the GPU's O and LSE against the oracle's attention over the GPU's own
    lists and its own post-update pool (both read back), and, when the GPU's
    lists and kept slots equal the oracle's, against the oracle's own step."""
    idx, cnt = host(L.idx), host(L.cnt)
    q16 = O.round_bf16(q)
    own_o, own_l = O.attention_fwd(q16, O.round_bf16(host(L.kpool)), O.round_bf16(host(L.vpool)),
                                   host(L.blk_len), host(L.blk_pos), idx, cnt, 1 / math.sqrt(w.D),
                                   w.mask, ref["q_pos0"])
    mx, mean = attn_errors(host(L.o), own_o)
    assert mx <= ATT_MAX and mean <= ATT_MEAN, ("own lists", mx, mean)
    np.testing.assert_allclose(host(L.lse), own_l, atol=2e-3, rtol=0)
    same = (np.array_equal(cnt, ref["cnt"]) and np.array_equal(idx, ref["idx"]) and
            np.array_equal(host(L.slot_src), ref["slot_src"]))
    if same:
        mx, mean = attn_errors(host(L.o), ref["O"])
        assert mx <= ATT_MAX and mean <= ATT_MEAN, ("oracle step", mx, mean)
        np.testing.assert_allclose(host(L.lse), ref["lse"], atol=2e-3, rtol=0)
    return same
