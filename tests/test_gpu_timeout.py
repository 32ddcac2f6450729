"""Failure detection on the GPU without a GPU fault.

Every wait inside the library's kernels is bounded.  A debug hook
(pbsa_set_debug flag 1) makes the attention forward skip the load of the first
V block, so the MMA warp's wait for it can never succeed: after the (short)
limit the CTA raises its abort flag, drains the copies and MMAs already in
flight, frees its tensor memory and returns, and the device status word holds
PBSA_ERR_TIMEOUT.  The test reads that status through pbsa_get_status and then
checks that the context is still usable: the same call, without the hook,
succeeds and matches the oracle.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
from block_sparse_attention_39_b200 import pbsa as K
from tests.gpu_util import ATT_MAX, ATT_MEAN, attn_errors, dev_i32, dev_storage, host

pytestmark = pytest.mark.gpu

ERR_TIMEOUT = -6


def _case():
    r = np.random.default_rng(11)
    B, H, D, bs, Tq, NB = 1, 1, 128, 128, 256, 4
    q = O.round_bf16(r.standard_normal((B, H, Tq, D)))
    kp = O.round_bf16(r.standard_normal((B, H, NB, bs, D)))
    vp = O.round_bf16(r.standard_normal((B, H, NB, bs, D)))
    bl = np.full((B, H, NB), bs, dtype=np.int32)
    bp = (np.arange(NB) * bs).astype(np.int32)[None, None, :]
    idx = np.array([[[[0, 2], [1, 3]]]], dtype=np.int32)
    cnt = np.array([[[2, 2]]], dtype=np.int32)
    return B, H, D, bs, Tq, NB, q, kp, vp, bl, bp, idx, cnt


def _run(case):
    B, H, D, bs, Tq, NB, q, kp, vp, bl, bp, idx, cnt = case
    d = K.dims(B, H, D, bs, 1 / math.sqrt(D), torch.bfloat16)
    o = torch.zeros(B, H, Tq, D, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(B, H, Tq, dtype=torch.float32, device="cuda")
    K.attn_fwd(d, dev_storage(q, "bf16"), Tq, 0, dev_storage(kp, "bf16"), dev_storage(vp, "bf16"),
               NB, dev_i32(bl), dev_i32(bp), dev_i32(idx), dev_i32(cnt), idx.shape[-1],
               K.MASK_CHUNK, o, lse)
    torch.cuda.synchronize()
    return o, lse


def test_bounded_wait_times_out_and_context_survives():
    case = _case()
    K.get_status()                                   # start from a clear status word
    K.set_debug(1, 20_000_000)                       # skip V(0); 20 ms wait limit
    try:
        _run(case)
        assert K.get_status() == ERR_TIMEOUT
    finally:
        K.set_debug(0, 0)
    # the context is still usable and the same call now gives the right answer
    o, lse = _run(case)
    assert K.get_status() == 0
    B, H, D, bs, Tq, NB, q, kp, vp, bl, bp, idx, cnt = case
    ref_o, ref_l = O.attention_fwd(q, kp, vp, bl, bp, idx, cnt, 1 / math.sqrt(D), K.MASK_CHUNK, 0)
    mx, mean = attn_errors(host(o), ref_o)
    assert mx <= ATT_MAX and mean <= ATT_MEAN, (mx, mean)
    np.testing.assert_allclose(host(lse), ref_l, atol=2e-3, rtol=0)
