"""Ring attention's host logic on CPU: the zigzag layout, the block masks, the
rotation of K/V halves (one process emulating every rank, and real gloo ranks
exchanging halves with send/recv), checked against the fp64 forward oracle on
the whole sequence.  The per-block attention and the merge are plain torch
functions written here (the CUDA kernels run in tests/test_ring_gpu.py)."""
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from exact_io_aware_72_b200 import ring


def cpu_block_attention(q, k, v, mask, scale, window=None, key_offset=0):
    """Plain masked softmax attention of one (query half, key half) block in fp64;
    query row r sits at key position r + key_offset.  Rows that see no key give
    out 0 and lse -inf (what the forward writes for them)."""
    q64, k64, v64 = q.double(), k.double(), v.double()
    g = q.shape[1] // k.shape[1]
    k64 = k64.repeat_interleave(g, dim=1)
    v64 = v64.repeat_interleave(g, dim=1)
    s = (q64 @ k64.transpose(-1, -2)) * scale
    if mask != "full":
        r = torch.arange(s.shape[-2])[:, None] + key_offset
        c = torch.arange(s.shape[-1])[None, :]
        hidden = c > r
        if mask == "sliding_window":
            hidden |= c <= r - window
        s = s.masked_fill(hidden, float("-inf"))
    lse = torch.logsumexp(s, dim=-1)
    p = torch.where(torch.isinf(lse)[..., None], torch.zeros_like(s), torch.exp(s - lse[..., None]))
    return p @ v64, lse


def cpu_merge(acc_o, acc_l, part_o, part_l, first, out):
    """The log-sum-exp merge of two partial results, in fp64."""
    if first:
        acc_o.copy_(part_o)
        acc_l.copy_(part_l)
    else:
        m = torch.maximum(acc_l, part_l)
        empty = torch.isinf(m)                         # neither part saw a key
        m = torch.where(empty, torch.zeros_like(m), m)
        wa, wp = torch.exp(acc_l - m), torch.exp(part_l - m)
        s = torch.where(empty, torch.ones_like(wa), wa + wp)
        acc_o.copy_((wa[..., None] * acc_o + wp[..., None] * part_o) / s[..., None])
        acc_l.copy_(torch.where(empty, torch.full_like(m, float("-inf")), m + torch.log(s)))
    if out is not None:
        out.copy_(acc_o)


def _inputs(B, Hq, Hkv, N, d, seed):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(B, Hq, N, d, generator=g, dtype=torch.float64),
            torch.randn(B, Hkv, N, d, generator=g, dtype=torch.float64),
            torch.randn(B, Hkv, N, d, generator=g, dtype=torch.float64))


@pytest.mark.parametrize("world", [1, 2, 3, 4])
def test_causal_blocks_cover_the_lower_triangle_evenly(world):
    seen = set()
    per_rank = []
    for r in range(world):
        count = 0
        for s in range(world):
            src = (r - s) % world
            for qi in ring.half_ids(world, r):
                for kj in ring.half_ids(world, src):
                    m = ring.block_mask(qi, kj, "causal")
                    if m is not None:
                        assert (qi, kj) not in seen
                        seen.add((qi, kj))
                        assert (m == "causal") == (qi == kj)
                        count += 1 + (m == "full")   # a causal diagonal block is half a full one
        per_rank.append(count)
    assert seen == {(i, j) for i in range(2 * world) for j in range(i + 1)}
    assert len(set(per_rank)) == 1                     # zigzag: equal work on every rank


def test_zigzag_split_and_gather_round_trip():
    x = torch.arange(2 * 3 * 24 * 4).reshape(2, 3, 24, 4)
    for world in (1, 2, 3, 4, 6):
        shares = [ring.zigzag_halves(x, world, r) for r in range(world)]
        assert torch.equal(ring.zigzag_gather(shares), x)
    with pytest.raises(ValueError):
        ring.zigzag_halves(x, 5, 0)


@pytest.mark.parametrize("world", [1, 2, 3, 4])
@pytest.mark.parametrize("mask", ["causal", "full"])
def test_emulated_ring_matches_oracle(world, mask):
    B, Hq, Hkv, N, d = 1, 4, 2, 48, 8
    q, k, v = _inputs(B, Hq, Hkv, N, d, 10 * world)
    scale = 1 / math.sqrt(d)
    out, lse = ring.ring_forward_emulated(q, k, v, world, mask, scale, cpu_block_attention, cpu_merge)
    ref_o, ref_l = oracle.attention(q.numpy(), k.numpy(), v.numpy(), scale, {"full": 0, "causal": 1}[mask])
    assert np.abs(out.numpy() - ref_o).max() < 1e-12
    assert np.abs(lse.numpy() - ref_l).max() < 1e-12


def test_sliding_window_block_mask_is_refused():
    with pytest.raises(ValueError):
        ring.block_mask(1, 0, "sliding_window")
    with pytest.raises(ValueError):
        ring.block_plan(1, 0, "sliding_window", None, 8)


@pytest.mark.parametrize("window", [1, 3, 7, 8, 9, 15, 17, 40, 100])
@pytest.mark.parametrize("world", [1, 2, 3])
def test_window_block_plan_covers_exactly_the_visible_pairs(world, window):
    # A (query half, key half) block is planned iff some query of the first sees
    # some key of the second under the window (i - w < j <= i), and the plan's
    # key offset is the distance between the halves' starts.
    h = 8
    for qi in range(2 * world):
        for kj in range(2 * world):
            visible = any(i - window < j <= i for i in range(qi * h, qi * h + h) for j in range(kj * h, kj * h + h))
            bp = ring.block_plan(qi, kj, "sliding_window", window, h)
            assert (bp is not None) == visible, (qi, kj)
            if bp is not None:
                assert bp == ("sliding_window", (qi - kj) * h)


@pytest.mark.parametrize("world", [1, 2, 3, 4])
@pytest.mark.parametrize("window", [1, 5, 6, 11, 13, 30, 100])
def test_emulated_ring_with_a_window_matches_oracle(world, window):
    B, Hq, Hkv, N, d = 1, 4, 2, 48, 8
    q, k, v = _inputs(B, Hq, Hkv, N, d, 20 * world + window)
    scale = 1 / math.sqrt(d)
    out, lse = ring.ring_forward_emulated(q, k, v, world, "sliding_window", scale, cpu_block_attention, cpu_merge,
                                          window=window)
    ref_o, ref_l = oracle.attention(q.numpy(), k.numpy(), v.numpy(), scale, 2, window)
    assert np.abs(out.numpy() - ref_o).max() < 1e-12
    assert np.abs(lse.numpy() - ref_l).max() < 1e-12


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


WINDOW = 11  # the gloo ring's sliding window (halves of 8 positions: one and two halves back)


def _ring_worker(rank, world, port, mask, queue):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q, k, v = _inputs(1, 4, 2, 8 * world, 8, 77)
        qh, kh, vh = (ring.zigzag_halves(t, world, rank) for t in (q, k, v))
        outs, lses = ring.ring_forward(torch.stack(qh), torch.stack(kh), torch.stack(vh), mask, 1 / math.sqrt(8),
                                       None, cpu_block_attention, cpu_merge,
                                       window=WINDOW if mask == "sliding_window" else None)
        queue.put((rank, outs[0].numpy(), outs[1].numpy(), lses[0].numpy(), lses[1].numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
@pytest.mark.parametrize("world,mask", [(2, "causal"), (3, "causal"), (4, "causal"), (3, "full"),
                                        (2, "sliding_window"), (3, "sliding_window")])
def test_gloo_ranks_exchange_halves(world, mask):
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ring_worker, args=(r, world, port, mask, queue)) for r in range(world)]
    for p in procs:
        p.start()
    got = sorted((queue.get(timeout=150) for _ in procs), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    out = ring.zigzag_gather([(torch.from_numpy(g[1]), torch.from_numpy(g[2])) for g in got]).numpy()
    lse = ring.zigzag_gather([(torch.from_numpy(g[3]), torch.from_numpy(g[4])) for g in got]).numpy()
    q, k, v = _inputs(1, 4, 2, 8 * world, 8, 77)
    ref_o, ref_l = oracle.attention(q.numpy(), k.numpy(), v.numpy(), 1 / math.sqrt(8),
                                    {"full": 0, "causal": 1, "sliding_window": 2}[mask],
                                    WINDOW if mask == "sliding_window" else None)
    assert np.abs(out - ref_o).max() < 1e-12
    assert np.abs(lse - ref_l).max() < 1e-12
