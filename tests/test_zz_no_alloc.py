"""The backward entry point that allocates nothing (pbsa_attn_bwd_noalloc).

It is meant for callers that cannot give the library a device buffer -- a host
process that owns all device memory through its own pool, or code that must
never enter the CUDA allocator.  Its scratch is a fixed array of device memory
inside the library, shared by every call.

The GPU test calls it twice in a row through the C ABI, on two different
problems.  Each result must equal, bit for bit, what pbsa_attn_bwd (which
takes a workspace from the caller) gives on the same inputs -- both run the
same kernels, which write dQ, dK and dV without atomics, so any difference
would come from stale contents of the shared scratch -- and must match the
CPU oracle's float64 gradients within the tolerance of the backward tests.
The second call would pick up the first call's leftovers if the shared
scratch were not cleared where it must start at zero.  This file is collected
last so that a run stopping at its first failure has run every other test.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

import oracle as O
import pbsa_inputs as PI
from block_sparse_attention_39_b200 import _lib
from block_sparse_attention_39_b200 import pbsa as K

G_MAX, G_MEAN, ULP = 2e-2, 2e-3, 2.0 ** -8


def _close(got, ref):
    d = np.abs(got - ref)
    return (float(d.max()) <= G_MAX + ULP * float(np.abs(ref).max()) and
            float(d.mean()) <= G_MEAN + ULP * float(np.abs(ref).mean()))


def _problem(seed, B, H, D, bs, Tq, NB, Amax, mask):
    r = np.random.default_rng(seed)
    kp = O.round_bf16(r.standard_normal((B, H, NB, bs, D)))
    vp = O.round_bf16(r.standard_normal((B, H, NB, bs, D)))
    q = O.round_bf16(r.standard_normal((B, H, Tq, D)))
    dO = O.round_bf16(r.standard_normal((B, H, Tq, D)))
    bl = r.integers(1, bs + 1, size=(B, H, NB)).astype(np.int32)
    bp = (np.arange(NB) * bs).astype(np.int32)[None, None, :].repeat(B, 0).repeat(H, 1)
    nQB = -(-Tq // bs)
    idx = np.full((B, H, nQB, Amax), -1, dtype=np.int32)
    cnt = np.zeros((B, H, nQB), dtype=np.int32)
    for b in range(B):
        for h in range(H):
            for i in range(nQB):
                n = int(r.integers(1, Amax + 1))
                idx[b, h, i, :n] = np.sort(r.choice(NB, size=n, replace=False))
                cnt[b, h, i] = n
    q_pos0 = int(bp[0, 0, -1])
    scale = 1 / math.sqrt(D)
    o, lse = O.attention_fwd(q, kp, vp, bl, bp, idx, cnt, scale, mask, q_pos0)
    grads = O.attention_bwd(q, kp, vp, bl, bp, idx, cnt, dO, scale, mask, q_pos0)
    dev = lambda x: torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()
    i32 = lambda x: torch.from_numpy(np.ascontiguousarray(x, dtype=np.int32)).cuda()
    t = dict(q=dev(q).bfloat16(), kp=dev(kp).bfloat16(), vp=dev(vp).bfloat16(),
             o=dev(O.round_bf16(o)).bfloat16(), lse=dev(lse), dO=dev(dO).bfloat16(), bl=i32(bl),
             bp=i32(bp), idx=i32(idx), cnt=i32(cnt))
    d = K.dims(B, H, D, bs, scale, torch.bfloat16)
    return d, t, dict(Tq=Tq, NB=NB, Amax=Amax, mask=mask, q_pos0=q_pos0, B=B, H=H, D=D, bs=bs,
                      oracle=grads)


def _grads(meta):
    B, H, Tq, D, NB, bs = meta["B"], meta["H"], meta["Tq"], meta["D"], meta["NB"], meta["bs"]
    return (torch.full((B, H, Tq, D), 5.0, device="cuda"),
            torch.full((B, H, NB, bs, D), 5.0, device="cuda"),
            torch.full((B, H, NB, bs, D), 5.0, device="cuda"))


def _with_workspace(d, t, m):
    dq, dk, dv = _grads(m)
    ws = torch.empty(K.attn_bwd_workspace(d, m["Tq"], m["NB"], m["Amax"]), dtype=torch.uint8,
                     device="cuda")
    K.attn_bwd(d, t["q"], m["Tq"], m["q_pos0"], t["kp"], t["vp"], m["NB"], t["bl"], t["bp"],
               t["idx"], t["cnt"], m["Amax"], m["mask"], t["o"], t["lse"], t["dO"], dq, dk, dv, ws)
    return dq, dk, dv


def _no_alloc(d, t, m):
    dq, dk, dv = _grads(m)
    K.attn_bwd_noalloc(d, t["q"], m["Tq"], m["q_pos0"], t["kp"], t["vp"], m["NB"], t["bl"],
                       t["bp"], t["idx"], t["cnt"], m["Amax"], m["mask"], t["o"], t["lse"],
                       t["dO"], dq, dk, dv)
    return dq, dk, dv


def test_no_alloc_rejects_problems_beyond_its_scratch():
    # validated on the host before anything touches the device
    lib = _lib.lib()
    cap = K.attn_bwd_noalloc_max_scratch()
    assert cap == 16 << 20
    d = K.dims(1, 64, 128, 128, 0.088, torch.bfloat16)
    Tq, NB, Amax = 65536, 4096, 64
    assert K.attn_bwd_workspace(d, Tq, NB, Amax) > cap
    fake = ctypes.c_void_p(256)
    rc = lib.pbsa_attn_bwd_noalloc(ctypes.byref(d), fake, Tq, 0, fake, fake, NB, fake, fake, fake,
                                   fake, Amax, 0, fake, fake, fake, fake, fake, fake, None)
    assert rc == -7
    assert b"16777216" in lib.pbsa_last_error()


@pytest.mark.gpu
def test_no_alloc_backward_matches_workspace_backward_twice():
    assert torch.cuda.is_available()
    K.get_status()
    # two different problems back to back: the second reuses the shared scratch
    cases = [(1, 2, 2, 128, 128, 384, 9, 6, PI.MASK_TOKEN),
             (2, 1, 3, 64, 64, 200, 7, 5, PI.MASK_CHUNK)]
    for seed, B, H, D, bs, Tq, NB, Amax, mask in cases:
        d, t, m = _problem(seed, B, H, D, bs, Tq, NB, Amax, mask)
        ref = _with_workspace(d, t, m)
        got = _no_alloc(d, t, m)
        torch.cuda.synchronize()
        for name, g, r, o in zip(("dq", "dk", "dv"), got, ref, m["oracle"]):
            assert torch.equal(g, r), (seed, name, float((g - r).abs().max()))
            gh = g.double().cpu().numpy()
            assert _close(gh, o), (seed, name, float(np.abs(gh - o).max()))
    assert K.get_status() == 0
