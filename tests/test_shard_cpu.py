"""The (batch, KV-group) split of the forward across ranks (``shard``), on CPU
gloo ranks: the unit ranges of all ranks cover every (b, h_kv) unit exactly
once (world sizes that divide the units and ones that do not), and the per-rank
slices, each run through an fp64 stand-in of the forward and gathered over
gloo, reassemble to the single-rank result."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from exact_io_aware_72_b200 import shard


def ref_attention(q, k, v, mask="causal", scale=None):
    """fp64 stand-in of the forward on [1, heads, N, d] views (CPU)."""
    q, k, v = (t.double() for t in (q, k, v))
    g = q.shape[1] // k.shape[1]
    k, v = k.repeat_interleave(g, dim=1), v.repeat_interleave(g, dim=1)
    s = (q @ k.transpose(-1, -2)) * (scale or q.shape[-1] ** -0.5)
    if mask == "causal":
        n = s.shape[-1]
        s = s.masked_fill(torch.ones(n, n, dtype=torch.bool).triu(1), float("-inf"))
    lse = torch.logsumexp(s, dim=-1)
    return torch.softmax(s, dim=-1) @ v, lse


@pytest.mark.parametrize("units", [1, 7, 8, 32, 33])
@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_unit_ranges_cover_every_unit_once(units, world):
    seen = []
    for r in range(world):
        a, b = shard.unit_range(units, world, r)
        assert 0 <= a <= b <= units
        seen.extend(range(a, b))
    assert seen == list(range(units))
    sizes = shard.shard_sizes(1, units, world)
    assert sum(sizes) == units and max(sizes) - min(sizes) <= 1


def test_head_shard_views_are_the_units():
    B, Hq, Hkv, N, d = 2, 8, 4, 16, 8
    q = torch.arange(B * Hq * N * d, dtype=torch.float32).reshape(B, Hq, N, d)
    k = torch.arange(B * Hkv * N * d, dtype=torch.float32).reshape(B, Hkv, N, d)
    for world in (1, 3, 8, 9):
        for r in range(world):
            qs, ks, vs, (u0, u1) = shard.head_shard(q, k, k, world, r)
            if u0 == u1:
                assert qs is None
                continue
            for i, u in enumerate(range(u0, u1)):
                b, h = divmod(u, Hkv)
                assert torch.equal(ks[0, i], k[b, h])
                assert torch.equal(qs[0, 2 * i:2 * i + 2], q[b, 2 * h:2 * h + 2])
            assert qs.data_ptr() == q[u0 // Hkv, (u0 % Hkv) * 2].data_ptr()   # a view, not a copy


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, queue):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from harness.inputs import make_qkv
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, Hq, Hkv, N, d = 2, 8, 4, 32, 16
        q, k, v = make_qkv(B, Hq, Hkv, N, d, 7)     # every rank draws the same tensors
        out, lse, (u0, u1) = shard.forward_shard(q, k, v, world, rank, local_attention=ref_attention)
        g = Hq // Hkv
        # gather every rank's slice (padded to the largest slice for all_gather)
        most = max(b - a for a, b in (shard.unit_range(B * Hkv, world, r) for r in range(world)))
        pad_o = torch.zeros(most * g, N, d, dtype=torch.float64)
        pad_l = torch.zeros(most * g, N, dtype=torch.float64)
        if out is not None:
            pad_o[:out.shape[1]] = out[0]
            pad_l[:lse.shape[1]] = lse[0]
        all_o = [torch.zeros_like(pad_o) for _ in range(world)]
        all_l = [torch.zeros_like(pad_l) for _ in range(world)]
        dist.all_gather(all_o, pad_o)
        dist.all_gather(all_l, pad_l)
        if rank == 0:
            parts = []
            for r in range(world):
                a, b = shard.unit_range(B * Hkv, world, r)
                n = (b - a) * g
                parts.append((all_o[r][None, :n], all_l[r][None, :n]) if n else (None, None))
            got_o, got_l = shard.gather_heads(parts, B, Hq)
            ref_o, ref_l = ref_attention(q.reshape(1, B * Hq, N, d), k.reshape(1, B * Hkv, N, d),
                                         v.reshape(1, B * Hkv, N, d))
            err = max(float((got_o - ref_o.reshape(B, Hq, N, d)).abs().max()),
                      float((got_l - ref_l.reshape(B, Hq, N)).abs().max()))
            queue.put(err)
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
@pytest.mark.parametrize("world", [2, 3])
def test_ranks_reassemble_the_single_rank_result(world):
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, queue)) for r in range(world)]
    for p in procs:
        p.start()
    err = queue.get(timeout=150)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert err < 1e-12, err
