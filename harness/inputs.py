"""Seeded synthetic inputs for the exact attention forward.

This module only draws random tensors and picks row samples; it holds none of
the attention arithmetic, so both the CUDA path's tests/bench and the fp64
oracle can take their inputs from it without sharing any method code.

Workloads (shapes, masks, value distributions) are the five attention-forward
workloads of the exact-attention pages' long-context discussion:

* ``tiny``  : B=1, Hq=Hkv=2, N=256, d=64, causal (every row checked)
* ``dense`` : B=2, Hq=Hkv=32, N=8192, d=128, causal, with 5% of key rows x4
              ("sharp" rows that force online-softmax rescaling)
* ``gqa``   : B=1, Hq=64, Hkv=8, N=16384, d=128, causal
* ``swa``   : B=1, Hq=32, Hkv=8, N=131072, d=128, sliding window w=4096
* ``long``  : B=1, Hq=Hkv=32, N=131072, d=128, causal

Draw recipe (fixed so every consumer sees the same tensors for a seed): a
``torch.Generator`` on the target device seeded with the workload's seed draws
q, k, v in that order as fp32 N(0,1) of shape [B,H,N,d]; for ``sharp`` it then
draws one uniform per key row [B,Hkv,N] and multiplies the rows with u < 0.05
by 4 (exact in bf16); each tensor is then rounded to bf16 (round to nearest
even, torch's cast).  CPU and CUDA generators give different streams for the
same seed; every comparison uses one set of tensors for both sides.
"""
from __future__ import annotations

from dataclasses import dataclass, asdict
from typing import Optional

import numpy as np
import torch

MASK_NAMES = {"full": 0, "causal": 1, "sliding_window": 2}


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    N: int
    d: int
    mask: str
    window: Optional[int]
    seed: int
    sharp: bool = False

    @property
    def mask_kind(self) -> int:
        return MASK_NAMES[self.mask]

    @property
    def scale(self) -> float:
        return 1.0 / float(np.sqrt(self.d))

    def as_dict(self) -> dict:
        return asdict(self)


WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 2, 256, 64, "causal", None, 0),
    "dense": Workload("dense", 2, 32, 32, 8192, 128, "causal", None, 1, sharp=True),
    "gqa": Workload("gqa", 1, 64, 8, 16384, 128, "causal", None, 2),
    "swa": Workload("swa", 1, 32, 8, 131072, 128, "sliding_window", 4096, 3),
    "long": Workload("long", 1, 32, 32, 131072, 128, "causal", None, 4),
}


def make_qkv(B, Hq, Hkv, N, d, seed, device="cpu", sharp=False, dtype=torch.bfloat16):
    """Draw q [B,Hq,N,d], k and v [B,Hkv,N,d] (bf16) following the recipe above."""
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    out = []
    for H in (Hq, Hkv, Hkv):
        t = torch.randn((B, H, N, d), generator=gen, device=device, dtype=torch.float32)
        out.append(t)
    q, k, v = out
    if sharp:
        u = torch.rand((B, Hkv, N), generator=gen, device=device, dtype=torch.float32)
        k = torch.where((u < 0.05).unsqueeze(-1), k * 4.0, k)
    return q.to(dtype), k.to(dtype), v.to(dtype)


def make_workload(w: Workload, device="cpu"):
    return make_qkv(w.B, w.Hq, w.Hkv, w.N, w.d, w.seed, device=device, sharp=w.sharp)


def sample_rows(N: int, window: Optional[int], seed: int, count: int = 256) -> np.ndarray:
    """Sorted query-row indices to check on a large workload.

    Always includes rows 0..7, N-8..N-1, the tile edges 127/128/129 and, for a
    window w, rows w-2..w+1; the rest are uniform without replacement.  With
    N <= count every row is returned.
    """
    if N <= count:
        return np.arange(N, dtype=np.int64)
    fixed = set(range(0, 8)) | set(range(N - 8, N)) | {127, 128, 129}
    if window is not None:
        fixed |= {w for w in range(window - 2, window + 2)}
    fixed = {r for r in fixed if 0 <= r < N}
    rng = np.random.default_rng(seed)
    rest = np.setdiff1d(np.arange(N, dtype=np.int64), np.fromiter(fixed, dtype=np.int64))
    extra = rng.choice(rest, size=count - len(fixed), replace=False)
    return np.sort(np.concatenate([np.fromiter(fixed, dtype=np.int64), extra]))


def make_dout(B, Hq, N, d, seed, device="cpu", dtype=torch.bfloat16):
    """Upstream gradient dO [B,Hq,N,d] for the backward: fp32 N(0,1) from a
    generator seeded with ``seed + 7919`` (so it differs from q for the same
    seed), rounded to bf16."""
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed) + 7919)
    return torch.randn((B, Hq, N, d), generator=gen, device=device, dtype=torch.float32).to(dtype)
