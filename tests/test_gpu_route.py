"""GPU checks of the fused routing call (pbsa_route_step).

It must give, bit for bit, what the three per-call entry points give when made
in order (pbsa_score_blocks -> pbsa_update_memory -> pbsa_select_local): both
run the same device code, only the schedule differs (one persistent kernel
whose work items wait on per-head counters instead of five launches).  The per-call path is checked
against the oracle in test_gpu_parity.py; the fused path is also checked
against the oracle directly on the decode snapshot.  The barrier words must be
zero again after every call, and the call must work inside a CUDA graph.
"""
import numpy as np
import pytest
import torch

import pbsa_inputs as PI
from block_sparse_attention_39_b200 import pbsa as K
from block_sparse_attention_39_b200.engine import PbsaLayer
from tests.gpu_util import (band_ok, check_step_attention, dev_storage, host, load_snapshot,
                            oracle_snapshot_step)

pytestmark = pytest.mark.gpu

STATE = ["q_bar", "k_bar", "scores", "mem", "kpool", "vpool", "blk_len", "blk_pos", "slot_src",
         "slot_w", "idx", "cnt"]


@pytest.fixture(autouse=True)
def _status_clean():
    assert torch.cuda.is_available()
    K.get_status()
    yield
    assert K.get_status() == 0


def _same_state(La, Lb, where):
    for name in STATE:
        a, b = getattr(La, name), getattr(Lb, name)
        assert torch.equal(a, b), (where, name, (a != b).sum().item())


def _barrier_words_zero(L):
    # the kernel's counters: 4 control words and 5 per-(b,h) counters
    torch.cuda.synchronize()
    n = 4 * (4 + 5 * L.w.B * L.w.H)
    assert int(L.rws[:n].count_nonzero()) == 0


def _snapshot_pair(name):
    w = PI.WORKLOADS[name]
    chunks = PI.snapshot_chunks(w)
    t = w.n_chunks - 1
    layers = []
    for _ in range(2):
        L = PbsaLayer(w)
        load_snapshot(L, w, chunks)
        L.score(t, pool_ids=L.all_ids())        # cached pooled keys
        L.reset_memory()
        layers.append(L)
    torch.cuda.synchronize()
    return w, chunks, t, layers


def _per_call(L, t):
    L.score(t)
    ci, cs = L.candidates(t)
    L.update(ci, cs)
    L.select(t)


@pytest.mark.parametrize("name", ["tiny", "decode"])
def test_route_equals_per_call_on_snapshot(name):
    w, chunks, t, (La, Lb) = _snapshot_pair(name)
    _per_call(La, t)
    Lb.route(t)
    torch.cuda.synchronize()
    _same_state(La, Lb, name)
    _barrier_words_zero(Lb)
    # a second call on the same workspace (barrier words reused)
    Lb.reset_memory()
    La.reset_memory()
    _per_call(La, t)
    Lb.route(t)
    torch.cuda.synchronize()
    _same_state(La, Lb, name + " again")
    _barrier_words_zero(Lb)


@pytest.mark.parametrize("name,steps", [("rollout20s", 9), ("rollout1min", 6)])
def test_route_equals_per_call_over_a_rollout(name, steps):
    # merge policy (rollout20s, P48) and evict with P64 (rollout1min, union of
    # 80 ids): every chunk step through both paths, state compared each step
    w = PI.WORKLOADS[name]
    La, Lb = PbsaLayer(w), PbsaLayer(w)
    merged = 0
    for t in range(steps):
        q, k, v = PI.chunk_tensors(w, t)
        kd, vd = (torch.from_numpy(x).cuda().bfloat16() for x in (k, v))
        for L in (La, Lb):
            L.write_chunk(t, kd, vd)
            L.q.copy_(dev_storage(q, w.dtype))
        _per_call(La, t)
        Lb.route(t)
        torch.cuda.synchronize()
        _same_state(La, Lb, (name, t))
        merged += int((host(Lb.slot_w) > 1).sum())
    _barrier_words_zero(Lb)
    if w.policy == PI.POLICY_MERGE_MEAN:
        assert merged > 0


def test_route_matches_oracle_on_decode_snapshot():
    w, chunks, t, (L, _) = _snapshot_pair("decode")
    ref = oracle_snapshot_step(w, chunks)
    L.route(t)
    L.attend(t)
    torch.cuda.synchronize()
    ids = ref["new_ids"]
    np.testing.assert_allclose(host(L.scores)[..., ids], ref["S"][..., ids], rtol=1e-4, atol=1e-6)
    src = host(L.slot_src)
    for b in range(w.B):
        for h in range(w.H):
            inf = ref["info"][(b, h)]
            ok, _ = band_ok([int(x) for x in src[b, h] if x >= 0], inf["keys"], len(inf["kept"]))
            assert ok, (b, h)
    # attention checked unconditionally: against the oracle over the GPU's own
    # lists and pool, and against the oracle's step when the lists agree
    check_step_attention(L, w, ref, chunks[t][0])


def test_route_inside_a_cuda_graph():
    w, chunks, t, (La, Lb) = _snapshot_pair("decode")
    La.step(t, fused=False)
    s = torch.cuda.Stream()
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        Lb.reset_memory()
        Lb.step(t, fused=True)           # warm-up outside the capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        Lb.reset_memory()
        Lb.step(t, fused=True)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    _same_state(La, Lb, "graph")
    assert torch.equal(La.o, Lb.o) and torch.equal(La.lse, Lb.lse)
    _barrier_words_zero(Lb)


def test_route_wait_times_out_and_context_survives():
    # debug bit 1 withholds head 0's pool completions: its plan, score tiles,
    # lists and slot copies wait on a count that never arrives; with a 20 ms
    # limit the first waiter aborts the kernel, every CTA skips what is left,
    # the status word says PBSA_ERR_TIMEOUT and the counters are zero again;
    # the next call is normal and equals the per-call path
    w, chunks, t, (La, Lb) = _snapshot_pair("decode")
    K.get_status()
    K.set_debug(2, 20_000_000)
    try:
        Lb.route(t)
        assert K.get_status() == -6
    finally:
        K.set_debug(0, 0)
    _barrier_words_zero(Lb)
    Lb.reset_memory()
    _per_call(La, t)
    Lb.route(t)
    torch.cuda.synchronize()
    _same_state(La, Lb, "after a timed-out call")
    _barrier_words_zero(Lb)
