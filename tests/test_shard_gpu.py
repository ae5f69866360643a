"""The (batch, KV-group) split of one forward across ranks, on the GPU.

Each rank's share is an independent forward on views of its contiguous unit
range (no exchange between ranks), so the ranks of a world can run one after
the other on one device.  Reassembled in rank order they must give the
single-call forward bit for bit: a head's arithmetic does not depend on which
other heads share the launch."""
import pytest
import torch

from exact_io_aware_72_b200 import fwd
from exact_io_aware_72_b200.shard import forward_shard, gather_heads, shard_sizes
from harness.inputs import make_qkv

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("shape,mask,window", [
    ((2, 8, 2, 777, 128), "causal", None),           # 4 units: 2 batches x 2 KV groups of 4 heads
    ((1, 16, 16, 1000, 64), "full", None),           # 16 single-head units
    ((1, 32, 8, 2048, 128), "sliding_window", 300),  # 8 KV groups, an SWA-shaped slice
])
@pytest.mark.parametrize("world", [2, 3, 8])
def test_rank_shares_reassemble_to_the_single_forward(cuda_ok, shape, mask, window, world):
    B, Hq, Hkv, N, d = shape
    if B * Hkv < world:
        pytest.skip("fewer units than ranks")
    q, k, v = (t.cuda() for t in make_qkv(B, Hq, Hkv, N, d, 50 + world, device="cpu"))
    ref_out, ref_lse = fwd(q, k, v, mask=mask, window=window)
    parts = []
    for rank in range(world):
        out, lse, (u0, u1) = forward_shard(q, k, v, world, rank, mask=mask, window=window)
        assert out is not None and out.shape[1] == (u1 - u0) * (Hq // Hkv)
        parts.append((out, lse))
    torch.cuda.synchronize()
    out, lse = gather_heads(parts, B, Hq)
    assert sum(shard_sizes(B, Hkv, world)) == B * Hkv
    assert torch.equal(out, ref_out)
    assert torch.equal(lse, ref_lse)
