"""Host logic of the multi-GPU bench on CPU: two gloo ranks.

The path shards by (b, h) with no exchange (replicas of the decode problem),
so the only collectives are the timing ones: every rank must see the max of
the ranks' step times, the whole-job throughput counts every rank's work over
that max, and each rank draws its own seeded problem of the same shape.
"""
import os
import socket

import numpy as np
import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import pbsa_inputs as PI


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        step_ms = [0.25, 0.31][rank]
        ms_max = bench.max_over_ranks(step_ms, world)
        bench.barrier(world)
        out[rank] = (ms_max, bench.whole_job_tflops(145.0e9, ms_max, world))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_step():
    ctx = mp.get_context("spawn")
    port = _free_port()
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        res = dict(out)
    assert res[0][0] == res[1][0] == pytest.approx(0.31)
    # weak scaling: 2 ranks x 145 GFLOP over the slowest rank's 0.31 ms
    assert res[0][1] == pytest.approx(2 * 145.0e9 / 0.31e-3 / 1e12)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(0.5, 1) == 0.5
    assert bench.whole_job_tflops(1e12, 1000.0, 1) == pytest.approx(1.0)


def test_each_rank_draws_its_own_problem_of_the_same_shape():
    w0, w1 = bench.rank_workload(0), bench.rank_workload(1)
    assert w0.seed != w1.seed
    for f in ("B", "H", "D", "bs", "chunk_tokens", "n_chunks", "P", "W", "k"):
        assert getattr(w0, f) == getattr(w1, f)
    # the seeded draws differ (checked on a small chunk of each)
    t0 = PI.variant(PI.WORKLOADS["tiny"], seed=w0.seed)
    t1 = PI.variant(PI.WORKLOADS["tiny"], seed=w1.seed)
    q0 = PI.chunk_tensors(t0, 0)[0]
    q1 = PI.chunk_tensors(t1, 0)[0]
    assert q0.shape == q1.shape and not np.array_equal(q0, q1)


# ---------------------------------------------------------------------------
# head-sharded layer: partition, gather, and per-head independence
# ---------------------------------------------------------------------------
from block_sparse_attention_39_b200.shard import gather_heads, head_range  # noqa: E402
import oracle as O  # noqa: E402
import torch  # noqa: E402

# a merge rollout of three heads, split 2 + 1 over two ranks
SHARD_W = PI.variant(PI.WORKLOADS["tiny"], H=3, rollout=True, n_chunks=6, policy=O.MERGE_MEAN)


def test_head_range_covers_every_head_once():
    for H in (1, 2, 3, 5, 12, 13):
        for world in range(1, H + 1):
            got = [head_range(H, world, r) for r in range(world)]
            assert got[0][0] == 0 and got[-1][1] == H
            assert all(a[1] == b[0] for a, b in zip(got, got[1:]))
            sizes = [h1 - h0 for h0, h1 in got]
            assert min(sizes) >= 1 and max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        head_range(2, 3, 0)
    with pytest.raises(ValueError):
        head_range(4, 2, 2)


def _oracle_rollout(w, heads):
    """The oracle's rollout over heads [h0, h1) of w's chunks: (O, idx, slot_src) per step."""
    h0, h1 = heads
    orc = O.OracleLayer.of(PI.variant(w, H=h1 - h0))
    steps = []
    for t in range(w.n_chunks):
        q, k, v = PI.chunk_tensors(w, t)
        orc.write_chunk(t, k[:, h0:h1], v[:, h0:h1])
        res = orc.step(t, q[:, h0:h1])
        steps.append((np.ascontiguousarray(res["O"]), np.ascontiguousarray(res["idx"]),
                      np.ascontiguousarray(res["slot_src"])))
    return steps


def _shard_rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = SHARD_W
        got = []
        for o, idx, ss in _oracle_rollout(w, head_range(w.H, world, rank)):
            got.append(tuple(gather_heads(torch.from_numpy(x), w.H, world).numpy()
                             for x in (o, idx, ss)))
        out[rank] = got
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_of_a_head_sharded_rollout_give_the_whole_layer():
    # every rank runs the oracle's rollout on its own heads only (no exchange
    # during the rollout); one all-gather per step must give each rank the
    # outputs, lists and memory state of the rollout over all heads
    ctx = mp.get_context("spawn")
    port = _free_port()
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_shard_rank_main, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=300)
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        res = dict(out)
    whole = _oracle_rollout(SHARD_W, (0, SHARD_W.H))
    merged = 0
    for t, (o, idx, ss) in enumerate(whole):
        merged += int((ss >= 0).sum())
        for r in range(2):
            go, gidx, gss = res[r][t]
            np.testing.assert_allclose(go, o, rtol=1e-12, atol=1e-13)
            np.testing.assert_array_equal(gidx, idx)
            np.testing.assert_array_equal(gss, ss)
    assert merged > 0, "the rollout must fill its memory"
