"""Head-sharded layers on one GPU: the shards' outputs, concatenated in head
order, are the unsharded layer's, bit for bit, over a merge rollout.

PBSA's state and work are per (batch, head), so a rank that owns heads
[h0, h1) runs exactly the computation of those heads in the whole layer.
The shards here run one after another on the same device (no collective and
no kernel waiting on another); the all-gather itself is covered by the
two-rank gloo test in test_dist_cpu.py.
"""
import pytest
import torch

import pbsa_inputs as PI
from block_sparse_attention_39_b200 import pbsa as K
from block_sparse_attention_39_b200.shard import ShardedLayer, head_range

pytestmark = pytest.mark.gpu

STEPS = 6


@pytest.fixture(autouse=True)
def _status_clean():
    assert torch.cuda.is_available()
    K.get_status()
    yield
    assert K.get_status() == 0


@pytest.mark.parametrize("world", [2, 5])
@pytest.mark.parametrize("fused", [False, True])
def test_shards_give_the_whole_layers_bits(world, fused):
    w = PI.variant(PI.WORKLOADS["rollout20s"], n_chunks=STEPS)
    whole = ShardedLayer(w)                                  # one rank: every head
    shards = [ShardedLayer(w, world, r) for r in range(world)]
    assert [s.h1 - s.h0 for s in shards] == [b - a for a, b in
                                            (head_range(w.H, world, r) for r in range(world))]
    for t in range(STEPS):
        q, k, v = PI.chunk_tensors_device(w, t)
        o = whole.step(t, q, k, v, fused=fused).clone()
        parts = [s.step(t, q, k, v, fused=fused, gather=False).clone() for s in shards]
        torch.cuda.synchronize()
        assert torch.equal(torch.cat(parts, dim=1), o), t
        for name in ("lse", "idx", "cnt", "slot_src", "slot_w", "blk_len", "k_bar"):
            got = torch.cat([getattr(s.layer, name) for s in shards], dim=1)
            assert torch.equal(got, getattr(whole.layer, name)), (t, name)
    # the memory took blocks in: the rollout exercised the update
    assert int((whole.layer.slot_src >= 0).sum()) > 0
