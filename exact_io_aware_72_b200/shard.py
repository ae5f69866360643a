"""Splitting one forward across ranks by (batch, KV-group) units.

The forward's units are the (b, h_kv) pairs: a KV head with the Hq/Hkv query
heads that read it ("Attention Mechanism Variants Beyond Self-Attention",
tempatgunting.com, section "Multi-Query and Grouped-Query Attention": query
heads share a key/value head, repeat_interleave on the head axis).  A unit's q,
k, v, out and lse are its own, so units on different GPUs need no exchange:
rank r of R takes the contiguous unit range [U r / R, U (r + 1) / R) of the
U = B * Hkv units.  With the [B, H, N, d] layouts such a range is one
contiguous block of every tensor, so each rank runs a single forward on
views of it (B = 1, Hkv = units, Hq = units * Hq / Hkv).  Only host-side
indexing lives here; the forward itself is the library's ``fwd``.
"""
from __future__ import annotations

from typing import Callable, List, Optional, Sequence, Tuple

import torch


def unit_range(units: int, world: int, rank: int) -> Tuple[int, int]:
    """Contiguous [start, stop) of the ``units`` units that ``rank`` of ``world`` takes."""
    if world < 1 or not 0 <= rank < world or units < 0:
        raise ValueError("bad world, rank or unit count")
    return units * rank // world, units * (rank + 1) // world


def head_shard(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, world: int, rank: int):
    """This rank's views of q [B,Hq,N,d], k, v [B,Hkv,N,d]: (q_s, k_s, v_s, (u0, u1)),
    each a [1, heads, N, d] view of its units (None when the rank has no unit)."""
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    if Hq % Hkv != 0 or tuple(k.shape) != (B, Hkv, N, d) or tuple(v.shape) != tuple(k.shape):
        raise ValueError("q, k, v shapes disagree")
    g = Hq // Hkv
    u0, u1 = unit_range(B * Hkv, world, rank)
    if u1 == u0:
        return None, None, None, (u0, u1)
    n = u1 - u0
    qs = q.reshape(B * Hkv, g, N, d)[u0:u1].reshape(1, n * g, N, d)
    ks = k.reshape(B * Hkv, N, d)[u0:u1].reshape(1, n, N, d)
    vs = v.reshape(B * Hkv, N, d)[u0:u1].reshape(1, n, N, d)
    return qs, ks, vs, (u0, u1)


def forward_shard(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, world: int, rank: int,
                  local_attention: Optional[Callable] = None, **kwargs):
    """Run this rank's units: (out_s [1, heads, N, d], lse_s [1, heads, N], (u0, u1)),
    or (None, None, range) for a rank without units.  ``local_attention(q, k, v,
    **kwargs)`` defaults to the library's forward."""
    qs, ks, vs, rng = head_shard(q, k, v, world, rank)
    if qs is None:
        return None, None, rng
    if local_attention is None:
        from .attn import fwd as local_attention
    out, lse = local_attention(qs, ks, vs, **kwargs)
    return out, lse, rng


def gather_heads(parts: Sequence[Tuple[Optional[torch.Tensor], Optional[torch.Tensor]]], B: int, Hq: int
                 ) -> Tuple[torch.Tensor, torch.Tensor]:
    """Reassemble out [B,Hq,N,d] and lse [B,Hq,N] from every rank's (out_s, lse_s), rank order."""
    outs = [o for o, _ in parts if o is not None]
    lses = [l for _, l in parts if l is not None]
    out = torch.cat([o.reshape(-1, *o.shape[2:]) for o in outs], dim=0)
    lse = torch.cat([l.reshape(-1, l.shape[-1]) for l in lses], dim=0)
    return out.reshape(B, Hq, *out.shape[1:]), lse.reshape(B, Hq, -1)


def shard_sizes(B: int, Hkv: int, world: int) -> List[int]:
    """Units per rank (for reporting)."""
    return [b - a for a, b in (unit_range(B * Hkv, world, r) for r in range(world))]
