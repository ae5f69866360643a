"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
and compare with the fp64 oracle on the same seeded bf16 inputs."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from harness.inputs import MASK_NAMES, make_qkv

# Tolerances of the parity bar: bf16 out and fp32 log-sum-exp against fp64.
OUT_MAX_ABS = 1e-2
OUT_REL_L2 = 4e-3
LSE_MAX_ABS = 1e-3


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy()


def bf16_half_ulp(x: np.ndarray) -> np.ndarray:
    """Half a unit in the last place of bf16 (8 significant bits) at |x|: the
    largest error of a correctly rounded bf16 value."""
    ax = np.maximum(np.abs(x), np.finfo(np.float32).tiny)
    return np.exp2(np.floor(np.log2(ax)) - 8.0)


def element_bound(ref_out: np.ndarray) -> np.ndarray:
    """Per-element bound on |out - exact|: the stated 1e-2 wherever a correctly
    rounded bf16 value can meet it (|exact| < 4, where half an ulp is at most
    2^-7), and above that only the extra rounding the bf16 format forces:
    max(1e-2, half_ulp(exact) + 1e-2 - 2^-7)."""
    return np.maximum(OUT_MAX_ABS, bf16_half_ulp(ref_out) + OUT_MAX_ABS - 2.0 ** -7)


def element_bound_p_bf16(ref_out: np.ndarray) -> np.ndarray:
    """Per-element bound of the bf16-P mode (p_bf16, for V beyond the fp16 range):
    max(1e-2, one bf16 ulp of the exact value).  P rounded to 8 significant bits
    moves a row dominated by a few keys by up to about 2^-9 of their spread, on top
    of the output's own rounding; include/attn.h states the mode's precision."""
    return np.maximum(OUT_MAX_ABS, 2.0 * bf16_half_ulp(ref_out))


def compare(out, lse, ref_out, ref_lse, what="", extra=None, bound=element_bound):
    """Parity bar: out rel-L2 <= 4e-3, lse max-abs <= 1e-3, and every element of
    out within ``bound`` (element_bound: the stated 1e-2) of the exact value.
    ``extra`` (same shape as out) is added to the element bound.
    """
    o = out.astype(np.float64)
    err = np.abs(o - ref_out)
    max_abs = float(err.max()) if err.size else 0.0
    bound = bound(ref_out)
    if extra is not None:   # a caller-derived term for roundings the plain forward does not make
        bound = bound + extra
    worst = float((err - bound).max()) if err.size else -1.0
    denom = float(np.linalg.norm(ref_out))
    rel_l2 = float(np.linalg.norm(o - ref_out) / denom) if denom > 0 else float(np.linalg.norm(o - ref_out))
    lse_err = float(np.abs(lse.astype(np.float64) - ref_lse).max()) if lse.size else 0.0
    assert np.isfinite(o).all() and np.isfinite(lse).all(), f"{what}: non-finite output"
    if worst > 0.0:
        iw = np.unravel_index(int(np.argmax(err - bound)), err.shape)
        raise AssertionError(f"{what}: out max-abs {max_abs:.3e} (exceeds its bound by {worst:.3e}; "
                             f"worst element {tuple(int(x) for x in iw)}: got {o[iw]:.6f}, exact {ref_out[iw]:.6f})")
    assert rel_l2 <= OUT_REL_L2, f"{what}: out rel-L2 {rel_l2:.3e}"
    assert lse_err <= LSE_MAX_ABS, f"{what}: lse max-abs {lse_err:.3e}"
    return dict(max_abs=max_abs, rel_l2=rel_l2, lse_max_abs=lse_err)


def run_cuda(q, k, v, mask, window=None, scale=None, p_bf16=False):
    from exact_io_aware_72_b200 import fwd
    out, lse = fwd(q, k, v, scale=scale, mask=mask, window=window, p_bf16=p_bf16)
    torch.cuda.synchronize()
    return out, lse


def check_case(B, Hq, Hkv, N, d, mask, window=None, seed=0, sharp=False, scale=None, p_bf16=False):
    """Whole-tensor parity of one small case (every row checked)."""
    q, k, v = make_qkv(B, Hq, Hkv, N, d, seed, device="cpu", sharp=sharp)
    out, lse = run_cuda(q.cuda(), k.cuda(), v.cuda(), mask, window, scale, p_bf16)
    ref_out, ref_lse = oracle.attention(to_np(q), to_np(k), to_np(v), scale, MASK_NAMES[mask], window)
    return compare(to_np(out), to_np(lse), ref_out, ref_lse, f"{(B, Hq, Hkv, N, d, mask, window, p_bf16)}",
                   bound=element_bound_p_bf16 if p_bf16 else element_bound)


def check_sampled(q, k, v, out, lse, rows, mask, window=None, scale=None, heads=None):
    """Parity on sampled query rows of a large case (tensors on the GPU)."""
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    g = Hq // Hkv
    heads = range(Hq) if heads is None else heads
    rows_t = torch.as_tensor(rows, device=q.device)
    stats = []
    for b in range(B):
        for h in heads:
            hk = h // g
            qh = to_np(q[b:b + 1, h:h + 1])
            kh = to_np(k[b:b + 1, hk:hk + 1])
            vh = to_np(v[b:b + 1, hk:hk + 1])
            ro, rl = oracle.attention(qh, kh, vh, scale, MASK_NAMES[mask], window, rows=rows)
            go = to_np(out[b, h].index_select(0, rows_t))[None, None]
            gl = to_np(lse[b, h].index_select(0, rows_t))[None, None]
            stats.append(compare(go, gl, ro, rl, f"b={b} h={h}"))
    return stats
