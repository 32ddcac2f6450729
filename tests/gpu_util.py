"""Helpers shared by the GPU parity tests: moving seeded inputs to the device,
the oracle pipeline of one step, and the near-tie comparison rule."""
from __future__ import annotations

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


def load_layer(layer, snap, w):
    layer.kpool.copy_(dev_storage(snap["kpool"], w.dtype))
    layer.vpool.copy_(dev_storage(snap["vpool"], w.dtype))
    layer.blk_len.copy_(dev_i32(snap["blk_len"]))
    layer.blk_pos.copy_(dev_i32(snap["blk_pos"]))
    layer.q.copy_(dev_storage(snap["q"], w.dtype))
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


def oracle_snapshot_step(w, snap):
    """The oracle's score -> update -> select -> attend on a snapshot input."""
    kp = snap["kpool"].astype(np.float64)
    vp = snap["vpool"].astype(np.float64)
    kb0 = np.zeros((w.B, w.H, w.NB_phys, w.D))
    qb, kb, S, m = O.score_blocks(snap["q"], kp, snap["blk_len"], snap["all_ids"], kb0, w.scale,
                                  w.bs)
    up = O.update_memory(kp, vp, snap["blk_len"], snap["blk_pos"], kb, snap["slot_src"],
                         snap["slot_w"], snap["cand_ids"], snap["cand_src"], m, w.P, w.n_sink,
                         w.policy, w.dtype)
    kp2, vp2, bl2, bp2, kb2, ss2, sw2, info = up
    A = O.select_local(S, snap["win_ids"], w.k, PI.mem_ids_all_slots(w), bl2, w.mask,
                       snap["q_pos0"], bp2, w.bs, w.chunk_tokens)
    idx, cnt = O.lists_to_arrays(A, PI.amax(w))
    q16, k16, v16 = O.round_bf16(snap["q"]), O.round_bf16(kp2), O.round_bf16(vp2)
    out, lse = O.attention_fwd(q16, k16, v16, bl2, bp2, idx, cnt, w.scale, w.mask, snap["q_pos0"])
    return dict(q_bar=qb, k_bar=kb, S=S, m=m, kpool=kp2, vpool=vp2, blk_len=bl2, blk_pos=bp2,
                k_bar2=kb2, slot_src=ss2, slot_w=sw2, info=info, A=A, idx=idx, cnt=cnt, O=out,
                lse=lse, q16=q16, k16=k16, v16=v16)


def attn_errors(o_gpu: np.ndarray, o_ref: np.ndarray, rows=None):
    d = np.abs(o_gpu - o_ref)
    if rows is not None:
        d = d[rows]
    return float(d.max()), float(d.mean())
