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


# ---------------------------------------------------------------- decoding
# Decoding workloads: the new token(s) of each sequence attend to a paged KV
# cache.  Shapes follow the pages' long-context figures (128k context, d=128,
# 32 heads; GQA with 64 query heads over 8 KV heads; a 4096-token window);
# page_size 16 tokens.  Ragged batches draw each sequence length uniformly in
# [L_min, L_max].
@dataclass(frozen=True)
class DecodeWorkload:
    name: str
    B: int
    Hq: int
    Hkv: int
    Nq: int
    d: int
    L_min: int
    L_max: int
    page_size: int
    mask: str
    window: Optional[int]
    seed: int
    rolling: bool = False   # pages wholly before the window are not allocated (table entry -1)

    @property
    def mask_kind(self) -> int:
        return MASK_NAMES[self.mask]

    @property
    def scale(self) -> float:
        return 1.0 / float(np.sqrt(self.d))

    def as_dict(self) -> dict:
        return asdict(self)


DECODE_WORKLOADS = {
    "decode_gqa": DecodeWorkload("decode_gqa", 1, 64, 8, 1, 128, 131072, 131072, 16, "causal", None, 10),
    "decode_mha": DecodeWorkload("decode_mha", 16, 32, 32, 1, 128, 8192, 32768, 16, "causal", None, 11),
    "decode_swa": DecodeWorkload("decode_swa", 32, 32, 8, 1, 128, 65536, 131072, 16, "sliding_window", 4096,
                                 12, rolling=True),
    "decode_spec": DecodeWorkload("decode_spec", 8, 64, 8, 4, 128, 16384, 32768, 64, "causal", None, 13),
}


def make_seq_lens(B: int, L_min: int, L_max: int, seed: int) -> np.ndarray:
    """Sequence lengths: B integers uniform in [L_min, L_max] (numpy generator
    seeded with ``seed``)."""
    rng = np.random.default_rng(int(seed))
    return rng.integers(L_min, L_max + 1, size=B, dtype=np.int64)


def make_paged_kv(B, Hq, Hkv, Nq, d, seq_lens, page_size, seed, device="cpu", keep_from=None,
                  fill=None, extra_pages=0, table_width=None, dtype=torch.bfloat16):
    """Draw a decoding step's inputs with its KV cache in pages.

    Sequence b keeps logical pages ``keep_from[b] // page_size`` ..
    ``(seq_lens[b] - 1) // page_size`` (``keep_from`` defaults to 0); every
    other table entry is -1.  Physical pages are handed out in the order of a
    seeded random permutation, so consecutive logical pages are scattered over
    the pool, and ``extra_pages`` unused pages are added to it.

    Draw order on a ``torch.Generator`` seeded with ``seed``: q [B,Hq,Nq,d],
    k_cache and v_cache [num_pages,Hkv,page_size,d] as fp32 N(0,1) cast to
    bf16, then the page permutation.  With ``fill`` given, every cache slot
    that holds no kept position (slots past the end of a sequence's last page,
    the extra pages) is set to ``fill`` (e.g. NaN to show it is never read).
    Returns a dict of tensors: q, k_cache, v_cache, block_table (int32
    [B, table_width]), seq_lens (int32 [B]).
    """
    seq_lens = np.asarray(seq_lens, dtype=np.int64)
    keep_from = np.zeros(B, dtype=np.int64) if keep_from is None else np.asarray(keep_from, dtype=np.int64)
    first = keep_from // page_size
    last = (seq_lens - 1) // page_size
    counts = last - first + 1
    num_pages = int(counts.sum()) + int(extra_pages)
    width = int(last.max()) + 1 if table_width is None else int(table_width)
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    q = torch.randn((B, Hq, Nq, d), generator=gen, device=device, dtype=torch.float32).to(dtype)
    k_cache = torch.randn((num_pages, Hkv, page_size, d), generator=gen, device=device,
                          dtype=torch.float32).to(dtype)
    v_cache = torch.randn((num_pages, Hkv, page_size, d), generator=gen, device=device,
                          dtype=torch.float32).to(dtype)
    perm = torch.randperm(num_pages, generator=gen, device=device).cpu().numpy()
    table = np.full((B, width), -1, dtype=np.int32)
    used = np.zeros(num_pages, dtype=np.int64)  # kept slots per physical page (fill bookkeeping)
    nxt = 0
    for b in range(B):
        for lp in range(int(first[b]), int(last[b]) + 1):
            phys = int(perm[nxt])
            nxt += 1
            table[b, lp] = phys
            used[phys] = min(page_size, int(seq_lens[b]) - lp * page_size)
    if fill is not None:
        for phys in range(num_pages):
            if used[phys] < page_size:
                k_cache[phys, :, used[phys]:, :] = fill
                v_cache[phys, :, used[phys]:, :] = fill
    return {
        "q": q, "k_cache": k_cache, "v_cache": v_cache,
        "block_table": torch.from_numpy(table).to(device),
        "seq_lens": torch.from_numpy(seq_lens.astype(np.int32)).to(device),
    }


def make_decode_workload(w: DecodeWorkload, device="cpu", fill=None):
    """Inputs of a decoding workload (lengths from ``make_seq_lens`` with the
    workload's seed; for a rolling window the pages before position
    L_b - Nq - w + 1 are not allocated)."""
    lens = make_seq_lens(w.B, w.L_min, w.L_max, w.seed)
    keep = None
    if w.rolling:
        keep = np.maximum(lens - w.Nq - w.window + 1, 0)
    return make_paged_kv(w.B, w.Hq, w.Hkv, w.Nq, w.d, lens, w.page_size, w.seed, device=device,
                         keep_from=keep, fill=fill)


# ---------------------------------------------------------------- FP8 inputs
def quantise_e4m3(t: torch.Tensor):
    """Per-tensor E4M3 quantisation of a float tensor: scale = amax / 448 (the
    largest finite E4M3 magnitude), codes = round-to-nearest E4M3 of t / scale
    (torch's float8_e4m3fn cast).  Returns (uint8 codes, scale as a Python float)."""
    amax = float(t.abs().max())
    scale = amax / 448.0 if amax > 0 else 1.0
    codes = (t.float() / scale).to(torch.float8_e4m3fn).view(torch.uint8)
    return codes, scale


def make_qkv_fp8(B, Hq, Hkv, N, d, seed, device="cpu", sharp=False):
    """FP8 inputs: the bf16 recipe's fp32 draws (same generator, same order,
    same sharp rows), each quantised per tensor with ``quantise_e4m3``.
    Returns ((q8, sq), (k8, sk), (v8, sv))."""
    q, k, v = make_qkv(B, Hq, Hkv, N, d, seed, device=device, sharp=sharp, dtype=torch.float32)
    return quantise_e4m3(q), quantise_e4m3(k), quantise_e4m3(v)
