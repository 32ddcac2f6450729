"""Python binding of the PBSA C ABI: same names as ``include/pbsa.h``.

Argument marshalling only -- every step runs in the CUDA kernels of
``libpbsa.so``.  Tensors are torch CUDA tensors owned by the caller; torch is
used for device memory and streams.  A non-zero status raises ``PbsaError``.
"""
from __future__ import annotations

import ctypes
from typing import Optional

import torch

from ._lib import ROUTE_FIELDS, PbsaDims, PbsaRouteArgs, lib

BF16, FP32 = 0, 1
EVICT, MERGE_MEAN = 0, 1
MASK_CHUNK, MASK_TOKEN = 0, 1

STATUS_NAMES = {0: "OK", -1: "ERR_ARG", -2: "ERR_SHAPE", -3: "ERR_ALIGN", -4: "ERR_DTYPE",
                -5: "ERR_CUDA", -6: "ERR_TIMEOUT", -7: "ERR_WORKSPACE"}


class PbsaError(RuntimeError):
    def __init__(self, fn: str, code: int, msg: str):
        super().__init__(f"{fn} failed: {STATUS_NAMES.get(code, code)} ({msg})")
        self.code = code


def dims(B: int, H: int, D: int, bs: int, scale: float, dtype, q_chunk: int = 0) -> PbsaDims:
    """q_chunk: query rows per chunk, each chunk tiled into blocks on its own
    (0: the whole query is one chunk)."""
    if isinstance(dtype, torch.dtype):
        dtype = BF16 if dtype == torch.bfloat16 else FP32
    return PbsaDims(B, H, D, bs, float(scale), int(dtype), int(q_chunk))


def _p(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("PBSA tensors must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("PBSA tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _s(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        stream = stream.cuda_stream
    return ctypes.c_void_p(int(stream))


def _check(fn: str, rc: int):
    if rc != 0:
        raise PbsaError(fn, rc, lib().pbsa_last_error().decode())


def score_blocks(d: PbsaDims, q, Tq, kpool, NB, blk_len, pool_ids, n_pool, q_bar, k_bar, scores,
                 mem_score, stream=None):
    _check("pbsa_score_blocks", lib().pbsa_score_blocks(
        ctypes.byref(d), _p(q), Tq, _p(kpool), NB, _p(blk_len), _p(pool_ids), n_pool, _p(q_bar),
        _p(k_bar), _p(scores), _p(mem_score), _s(stream)))


def append_chunk(d: PbsaDims, k, v, Tc, pos0, kpool, vpool, NB, blk_ids, blk_len, blk_pos, k_bar,
                 stream=None):
    _check("pbsa_append_chunk", lib().pbsa_append_chunk(
        ctypes.byref(d), _p(k), _p(v), Tc, pos0, _p(kpool), _p(vpool), NB, _p(blk_ids),
        _p(blk_len), _p(blk_pos), _p(k_bar), _s(stream)))


def update_memory_workspace(d: PbsaDims, P: int, n_cand: int) -> int:
    return int(lib().pbsa_update_memory_workspace(ctypes.byref(d), P, n_cand))


def update_memory(d: PbsaDims, kpool, vpool, NB, blk_len, blk_pos, k_bar, P, n_sink, slot_src,
                  slot_w, cand_ids, cand_src, n_cand, mem_score, policy, workspace, stream=None):
    _check("pbsa_update_memory", lib().pbsa_update_memory(
        ctypes.byref(d), _p(kpool), _p(vpool), NB, _p(blk_len), _p(blk_pos), _p(k_bar), P, n_sink,
        _p(slot_src), _p(slot_w), _p(cand_ids), _p(cand_src), n_cand, _p(mem_score), policy,
        _p(workspace), workspace.numel() * workspace.element_size(), _s(stream)))


def update_plan_bytes(d: PbsaDims, P: int, n_cand: int) -> int:
    """Bytes at the head of the update workspace that hold the step's plan
    (what pbsa_update_memory_bwd reads)."""
    return int(lib().pbsa_update_plan_bytes(ctypes.byref(d), P, n_cand))


def update_memory_bwd_workspace(d: PbsaDims, P: int) -> int:
    return int(lib().pbsa_update_memory_bwd_workspace(ctypes.byref(d), P))


def update_memory_bwd(d: PbsaDims, NB, P, n_cand, plan, dk, dv, workspace, stream=None):
    """pbsa_update_memory_bwd: dk / dv (float, pool-shaped) go from the gradient
    w.r.t. the pool after the update to the gradient w.r.t. the pool before it."""
    _check("pbsa_update_memory_bwd", lib().pbsa_update_memory_bwd(
        ctypes.byref(d), NB, P, n_cand, _p(plan), _p(dk), _p(dv), _p(workspace),
        workspace.numel() * workspace.element_size(), _s(stream)))


def select_local(d: PbsaDims, scores, nQB, NB, win_ids, n_win, k, mem_ids, n_mem, blk_len, mask,
                 q_pos0, blk_pos, Tq, idx, cnt, Amax, qb_offset=0, nQB_total=None, stream=None,
                 mem_ld=0, mem_offset=0):
    """mem_ids may be a view into a larger int32 tensor: row (b,h) starts at
    mem_offset + (b*H+h)*mem_ld elements of mem_ids' storage."""
    mp = None
    if mem_ids is not None:
        if not mem_ids.is_cuda:
            raise ValueError("PBSA tensors must live on a CUDA device")
        mp = ctypes.c_void_p(mem_ids.data_ptr() + 4 * mem_offset)
    _check("pbsa_select_local", lib().pbsa_select_local(
        ctypes.byref(d), _p(scores), nQB, NB, _p(win_ids), n_win, k, mp, n_mem, mem_ld,
        _p(blk_len), mask, q_pos0, _p(blk_pos), Tq, _p(idx), _p(cnt), Amax, qb_offset,
        nQB if nQB_total is None else nQB_total, _s(stream)))


def select_hier(d: PbsaDims, scores, nQB, NB, win_ids, win_frame, n_win, n_frames, F, k, mem_ids,
                n_mem, blk_len, mask, q_pos0, blk_pos, Tq, idx, cnt, Amax, qb_offset=0,
                nQB_total=None, stream=None, mem_ld=0):
    """pbsa_select_hier: frame -> block local selection united with the memory."""
    _check("pbsa_select_hier", lib().pbsa_select_hier(
        ctypes.byref(d), _p(scores), nQB, NB, _p(win_ids), _p(win_frame), n_win, n_frames, F, k,
        _p(mem_ids), n_mem, mem_ld, _p(blk_len), mask, q_pos0, _p(blk_pos), Tq, _p(idx),
        _p(cnt), Amax, qb_offset, nQB if nQB_total is None else nQB_total, _s(stream)))


def route_workspace(d: PbsaDims, P: int, n_cand: int) -> int:
    return int(lib().pbsa_route_workspace(ctypes.byref(d), P, n_cand))


def route_step(d: PbsaDims, workspace, stream=None, **fields):
    """pbsa_route_step: score -> update -> select in one call.  `fields` are the
    members of pbsa_route_args (tensors for pointers, ints otherwise); members
    not given are NULL / 0.  The first 256 bytes of `workspace` must be zero
    before the first call (torch.zeros does it)."""
    args = PbsaRouteArgs()
    names = {n for n, _ in ROUTE_FIELDS}
    for name, val in fields.items():
        if name not in names:
            raise TypeError(f"pbsa_route_args has no member {name!r}")
        if isinstance(val, torch.Tensor):
            setattr(args, name, _p(val))
        elif val is None:
            setattr(args, name, None)
        else:
            setattr(args, name, int(val))
    _check("pbsa_route_step", lib().pbsa_route_step(
        ctypes.byref(d), ctypes.byref(args), _p(workspace),
        workspace.numel() * workspace.element_size(), _s(stream)))


def attn_fwd(d: PbsaDims, q, Tq, q_pos0, kpool, vpool, NB, blk_len, blk_pos, idx, cnt, Amax, mask,
             o, lse, stream=None):
    _check("pbsa_attn_fwd", lib().pbsa_attn_fwd(
        ctypes.byref(d), _p(q), Tq, q_pos0, _p(kpool), _p(vpool), NB, _p(blk_len), _p(blk_pos),
        _p(idx), _p(cnt), Amax, mask, _p(o), _p(lse), _s(stream)))


def attn_bwd_workspace(d: PbsaDims, Tq: int, NB: int, Amax: int) -> int:
    return int(lib().pbsa_attn_bwd_workspace(ctypes.byref(d), Tq, NB, Amax))


def attn_bwd(d: PbsaDims, q, Tq, q_pos0, kpool, vpool, NB, blk_len, blk_pos, idx, cnt, Amax, mask,
             o, lse, dO, dq, dk, dv, workspace, stream=None):
    _check("pbsa_attn_bwd", lib().pbsa_attn_bwd(
        ctypes.byref(d), _p(q), Tq, q_pos0, _p(kpool), _p(vpool), NB, _p(blk_len), _p(blk_pos),
        _p(idx), _p(cnt), Amax, mask, _p(o), _p(lse), _p(dO), _p(dq), _p(dk), _p(dv),
        _p(workspace), workspace.numel() * workspace.element_size(), _s(stream)))


def attn_bwd_noalloc(d: PbsaDims, q, Tq, q_pos0, kpool, vpool, NB, blk_len, blk_pos, idx, cnt, Amax,
                     mask, o, lse, dO, dq, dk, dv, stream=None):
    """The backward without a caller workspace: its scratch is a fixed device
    array inside the library (see pbsa_attn_bwd_noalloc in include/pbsa.h)."""
    _check("pbsa_attn_bwd_noalloc", lib().pbsa_attn_bwd_noalloc(
        ctypes.byref(d), _p(q), Tq, q_pos0, _p(kpool), _p(vpool), NB, _p(blk_len), _p(blk_pos),
        _p(idx), _p(cnt), Amax, mask, _p(o), _p(lse), _p(dO), _p(dq), _p(dk), _p(dv), _s(stream)))


def attn_bwd_noalloc_max_scratch() -> int:
    return int(lib().pbsa_attn_bwd_noalloc_max_scratch())


def check_exp2(x, y_poly, y_hw, stream=None):
    """The softmax's FMA-pipe exponent and the special-function unit's, on x."""
    _check("pbsa_check_exp2", lib().pbsa_check_exp2(_p(x), _p(y_poly), _p(y_hw), x.numel(),
                                                     _s(stream)))


def get_status(stream=None) -> int:
    """Synchronise the stream; return and clear the device status word."""
    return int(lib().pbsa_get_status(_s(stream)))


def set_debug(flags: int, wait_limit_ns: int = 0):
    lib().pbsa_set_debug(int(flags), int(wait_limit_ns))


def version() -> str:
    return lib().pbsa_version().decode()
