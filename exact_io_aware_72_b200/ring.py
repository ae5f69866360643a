"""Ring attention: exact attention over a sequence spread across ranks.

"Attention Mechanism Variants Beyond Self-Attention" (tempatgunting.com,
section "Ring Attention for Very Long Sequences"): each GPU holds a chunk of
the sequence and key/value blocks rotate around a ring of GPUs, so a sequence
longer than one GPU can hold is processed by all of them together.

Layout: the sequence of N positions is cut into 2R halves of N/(2R); rank r
holds halves r and 2R-1-r of q, k and v (a zigzag, so that under a causal mask
every rank has the same number of visible blocks).  In R steps each rank sees
the K/V halves of every rank: at step s it works on those of rank (r - s) mod
R while sending the halves it holds to rank r+1 and receiving the next ones
from rank r-1 (NCCL send/recv into local buffers, overlapped with the work).
For each (query half i, key half j) block the sm_100a forward kernel computes
a partial result with the block's own mask -- causal: every key of half j < i
is visible ("full"), j == i is the causal diagonal, j > i is skipped; full:
every block; sliding window w: the block of key half j < i is a window whose
queries sit (i - j) * h positions after its keys (the forward's ``key_offset``),
skipped when no row reaches back into it -- written in fp32, and
``attn_merge`` folds it into an fp32 accumulator by its log-sum-exp; only the
final merged rows are rounded to bf16.  The merged rows equal the exact
attention of the whole sequence ("Efficient attention: long context and
sub-quadratic variants", stanleyjacob.dev, section "Sliding-window and local
attention", for the window: query i sees keys i - w < j <= i).

Only the data movement and the loop live here; every arithmetic step runs in
the library's CUDA kernels (``fwd`` and ``merge``).  ``local_attention`` and
``merge`` can be replaced (tests run the ring logic on CPU ranks that way).
"""
from __future__ import annotations

from typing import Callable, List, Optional, Sequence, Tuple

import torch


def half_ids(world: int, rank: int) -> Tuple[int, int]:
    """Global indices of the two sequence halves a rank holds."""
    return rank, 2 * world - 1 - rank


def zigzag_halves(x: torch.Tensor, world: int, rank: int, dim: int = 2) -> Tuple[torch.Tensor, torch.Tensor]:
    """This rank's two halves of ``x`` along the sequence dimension (contiguous copies)."""
    n = x.shape[dim]
    if n % (2 * world) != 0:
        raise ValueError(f"sequence length {n} is not a multiple of 2 x {world} ranks")
    h = n // (2 * world)
    a, b = half_ids(world, rank)
    return x.narrow(dim, a * h, h).contiguous(), x.narrow(dim, b * h, h).contiguous()


def zigzag_gather(halves: Sequence[Tuple[torch.Tensor, torch.Tensor]], dim: int = 2) -> torch.Tensor:
    """Reassemble the full sequence from every rank's (half r, half 2R-1-r)."""
    world = len(halves)
    order = [None] * (2 * world)
    for r, (a, b) in enumerate(halves):
        i, j = half_ids(world, r)
        order[i], order[j] = a, b
    return torch.cat(order, dim=dim)


def block_mask(qi: int, kj: int, mask: str) -> Optional[str]:
    """Mask of the (query half qi, key half kj) block, or None when no key of it is visible."""
    if mask == "full":
        return "full"
    if mask != "causal":
        raise ValueError("block_mask takes the full and causal masks (block_plan also windows)")
    if kj < qi:
        return "full"
    if kj == qi:
        return "causal"
    return None


def block_plan(qi: int, kj: int, mask: str, window: Optional[int] = None, half: Optional[int] = None
               ) -> Optional[Tuple[str, int]]:
    """(mask, key offset) of the (query half qi, key half kj) block, or None when no
    key of it is visible.  Halves hold ``half`` positions; with a sliding window the
    block's query row r sits at key position r + (qi - kj) * half."""
    if mask != "sliding_window":
        m = block_mask(qi, kj, mask)
        return None if m is None else (m, 0)
    if window is None or window < 1 or half is None or half < 1:
        raise ValueError("a sliding window needs window >= 1 and the half length")
    if kj > qi:
        return None
    offset = (qi - kj) * half
    if offset > half + window - 2:        # even row 0's window starts after the block's last key
        return None
    return "sliding_window", offset


def _default_local(q, k, v, mask, scale, window=None, key_offset=0):
    # Block results stay fp32 (unrounded) until the last merge rounds out to bf16 once.
    from .attn import fwd
    return fwd(q, k, v, scale=scale, mask=mask, window=window, key_offset=key_offset, out_fp32=True)


def _default_merge(acc_o, acc_l, part_o, part_l, first, out):
    from .attn import merge
    merge(acc_o, acc_l, part_o, part_l, first=first, out=out)


def rank_forward(rank: int, world: int, q_halves: Sequence[torch.Tensor],
                 kv_at_step: Callable[[int], Tuple[Sequence[torch.Tensor], Sequence[torch.Tensor]]],
                 mask: str = "causal", scale: Optional[float] = None,
                 local_attention: Callable = _default_local, merge: Callable = _default_merge,
                 window: Optional[int] = None) -> Tuple[List[torch.Tensor], List[torch.Tensor]]:
    """One rank's share of ring attention.  ``kv_at_step(s)`` returns the K and V
    halves of rank (rank - s) mod world (waiting for them to arrive if needed).
    Returns ([out_a, out_b] bf16, [lse_a, lse_b] fp32) for the rank's two query halves."""
    qids = half_ids(world, rank)
    half = q_halves[0].shape[-2]
    # Which blocks each query half takes, in step order, so the last one can also write bf16 out.
    plan = [[] for _ in range(2)]
    for s in range(world):
        kids = half_ids(world, (rank - s) % world)
        for a in range(2):
            for b in range(2):
                bp = block_plan(qids[a], kids[b], mask, window, half)
                if bp is not None:
                    plan[a].append((s, b) + bp)
    # The accumulator is fp32 (or the inputs' dtype when that is wider); out has the inputs' dtype.
    acc_t = torch.float32 if q_halves[0].element_size() < 4 else q_halves[0].dtype
    acc_o = [torch.empty(q.shape, dtype=acc_t, device=q.device) for q in q_halves]
    acc_l = [torch.empty(q.shape[:-1], dtype=acc_t, device=q.device) for q in q_halves]
    outs = [torch.empty(q.shape, dtype=q.dtype, device=q.device) for q in q_halves]
    done = [0, 0]
    for s in range(world):
        k_h, v_h = kv_at_step(s)
        for a in range(2):
            for (step, b, m, offset) in plan[a]:
                if step != s:
                    continue
                if m == "sliding_window":
                    o, lse = local_attention(q_halves[a], k_h[b], v_h[b], m, scale, window=window,
                                             key_offset=offset)
                else:
                    o, lse = local_attention(q_halves[a], k_h[b], v_h[b], m, scale)
                last = done[a] == len(plan[a]) - 1
                merge(acc_o[a], acc_l[a], o, lse, done[a] == 0, outs[a] if last else None)
                done[a] += 1
    return outs, acc_l


def ring_forward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, mask: str = "causal",
                 scale: Optional[float] = None, group=None, local_attention: Callable = _default_local,
                 merge: Callable = _default_merge, window: Optional[int] = None
                 ) -> Tuple[List[torch.Tensor], List[torch.Tensor]]:
    """Ring attention across the ranks of ``group`` (torch.distributed, NCCL for
    CUDA tensors).  q, k, v are this rank's zigzag halves stacked on a leading
    axis of 2: q [2, B, Hq, h, d], k and v [2, B, Hkv, h, d] (see
    ``zigzag_halves``).  Returns this rank's ([out_a, out_b], [lse_a, lse_b])."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    nxt = dist.get_global_rank(group, (rank + 1) % world) if group is not None else (rank + 1) % world
    prv = dist.get_global_rank(group, (rank - 1) % world) if group is not None else (rank - 1) % world
    cur = [k.contiguous(), v.contiguous()]
    spare = [torch.empty_like(cur[0]), torch.empty_like(cur[1])]
    pending = []

    def kv_at_step(s):
        nonlocal cur, spare, pending
        if s > 0:
            for r in pending:
                r.wait()
            cur, spare = spare, cur
            pending = []
        if s < world - 1 and world > 1:
            # Send what this step works on to the next rank while receiving the
            # next step's halves from the previous one; grouped so that no rank
            # waits on a send before its receive is posted.
            ops = [dist.P2POp(dist.isend, t, nxt, group) for t in cur] + \
                  [dist.P2POp(dist.irecv, t, prv, group) for t in spare]
            pending = dist.batch_isend_irecv(ops)
        return (cur[0][0], cur[0][1]), (cur[1][0], cur[1][1])

    outs, lses = rank_forward(rank, world, (q[0], q[1]), kv_at_step, mask, scale, local_attention, merge, window)
    for r in pending:
        r.wait()
    return outs, lses


def emulate_shares(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, world: int):
    """Every rank's zigzag halves of full [B, H, N, d] tensors: [(q_halves, k_halves, v_halves)] by rank."""
    return [(zigzag_halves(q, world, r), zigzag_halves(k, world, r), zigzag_halves(v, world, r))
            for r in range(world)]


def run_emulated(shares, mask: str = "causal", scale: Optional[float] = None,
                 local_attention: Callable = _default_local, merge: Callable = _default_merge,
                 window: Optional[int] = None):
    """All ranks of the ring one after the other in this process (the K/V halves a
    rank would receive are taken from the other ranks' shares directly).
    Returns every rank's ((out_a, out_b), (lse_a, lse_b))."""
    world = len(shares)
    results = []
    for r in range(world):
        def kv_at_step(s, r=r):
            src = (r - s) % world
            return shares[src][1], shares[src][2]
        o, l = rank_forward(r, world, shares[r][0], kv_at_step, mask, scale, local_attention, merge, window)
        results.append(((o[0], o[1]), (l[0], l[1])))
    return results


def ring_forward_emulated(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, world: int, mask: str = "causal",
                          scale: Optional[float] = None, local_attention: Callable = _default_local,
                          merge: Callable = _default_merge, window: Optional[int] = None
                          ) -> Tuple[torch.Tensor, torch.Tensor]:
    """Ring attention of ``world`` ranks emulated in this process on full [B, H, N, d]
    tensors; returns the reassembled (out, lse)."""
    res = run_emulated(emulate_shares(q, k, v, world), mask, scale, local_attention, merge, window)
    return zigzag_gather([r[0] for r in res]), zigzag_gather([r[1] for r in res])
