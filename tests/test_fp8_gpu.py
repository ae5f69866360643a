"""CUDA FP8 (E4M3) forward (through the C ABI) against the fp64 FP8 oracle.

Bound, derived from the kernel's roundings (E4M3 inputs are taken exactly,
their products are exact in fp32): P is rounded to E4M3 (round to nearest,
relative error <= 2^-4) before the product with V and O is normalised by the
fp32 sum of the unrounded p, so |O err| <= 2^-4 * sum_j p_j |v_j| / l =
2^-4 * A with A the oracle's attention of |v|; plus one bf16 rounding of O
(2^-9 relative, taken as 2^-8) and an absolute 2e-4 for the fp32 sums and the
flush of weights below 2^-17 of the row max. The log-sum-exp comes from the
fp32 sum of the unrounded p: the bf16 forward's 1e-3 bound.
"""
import numpy as np
import pytest
import torch

from harness.inputs import MASK_NAMES, make_qkv_fp8
from oracle import attention_fp8 as O8
from tests.parity import to_np

pytestmark = pytest.mark.gpu


def run_fp8(qkv, mask, window=None, scale=None, grid_ctas=0):
    from exact_io_aware_72_b200 import fwd_fp8
    (q8, sq), (k8, sk), (v8, sv) = qkv
    out, lse = fwd_fp8(q8, k8, v8, sq, sk, sv, scale=scale, mask=mask, window=window, grid_ctas=grid_ctas)
    torch.cuda.synchronize()
    return out, lse


def check_fp8(B, Hq, Hkv, N, mask, window=None, seed=0, sharp=False, scale=None, rows=None):
    cpu = make_qkv_fp8(B, Hq, Hkv, N, 128, seed, device="cpu", sharp=sharp)
    gpu = tuple((c.cuda(), s) for c, s in cpu)
    out, lse = run_fp8(gpu, mask, window, scale)
    (q8, sq), (k8, sk), (v8, sv) = ((c.numpy(), s) for c, s in cpu)
    kind = MASK_NAMES[mask]
    ref_o, ref_l = O8.attention_fp8(q8, k8, v8, sq, sk, sv, scale, kind, window, rows=rows)
    # attention of |v| (the same weights): bounds what the rounding of P can move
    abs_o, _ = O8.attention_fp8(q8, k8, v8 & np.uint8(0x7F), sq, sk, sv, scale, kind, window, rows=rows)
    o = to_np(out).astype(np.float64)
    if rows is not None:
        o = o[:, :, rows]
        got_l = to_np(lse)[:, :, rows]
    else:
        got_l = to_np(lse)
    err = np.abs(o - ref_o)
    bound = 2.0 ** -4 * abs_o + 2.0 ** -8 * np.abs(ref_o) + 2e-4
    what = f"{(B, Hq, Hkv, N, mask, window, sharp, scale)}"
    assert np.isfinite(o).all() and np.isfinite(got_l).all(), what
    worst = float((err / bound).max())
    assert worst <= 1.0, f"{what}: error reaches {worst:.2f} of the bound (max-abs {err.max():.3e})"
    lse_err = float(np.abs(got_l - ref_l).max())
    assert lse_err <= 1e-3, f"{what}: lse max-abs {lse_err:.3e}"
    rel = float(np.linalg.norm(o - ref_o) / np.linalg.norm(ref_o))
    return dict(worst=worst, rel_l2=rel, max_abs=float(err.max()), lse=lse_err)


@pytest.mark.parametrize("N", [1, 17, 128, 129, 300, 1000])
@pytest.mark.parametrize("mask", ["full", "causal"])
def test_ragged_lengths(cuda_ok, N, mask):
    check_fp8(1, 2, 2, N, mask, seed=N)


@pytest.mark.parametrize("w", [1, 2, 127, 129, 300])
def test_sliding_window(cuda_ok, w):
    check_fp8(1, 2, 1, 700, "sliding_window", window=w, seed=w)


@pytest.mark.parametrize("shape", [(2, 8, 2, 300), (1, 8, 1, 257), (1, 6, 2, 200), (2, 3, 3, 130)])
def test_head_sharing(cuda_ok, shape):
    B, Hq, Hkv, N = shape
    check_fp8(B, Hq, Hkv, N, "causal", seed=sum(shape))


def test_sharp_rows_scale_and_long_rows(cuda_ok):
    # sharp rows (5 % of keys x4) move the running max often: the E4M3 P
    # rescale threshold is half a power of two
    check_fp8(1, 2, 2, 2048, "causal", seed=3, sharp=True)
    check_fp8(1, 2, 1, 1500, "full", seed=4, scale=0.3)


def test_window_ge_n_is_causal_bitwise(cuda_ok):
    gpu = tuple((c.cuda(), s) for c, s in make_qkv_fp8(1, 4, 2, 333, 128, 9))
    ref = run_fp8(gpu, "causal")
    for w in (333, 10 ** 6):
        got = run_fp8(gpu, "sliding_window", w)
        assert torch.equal(got[0], ref[0]) and torch.equal(got[1], ref[1])


def test_repeatable_and_grid_independent(cuda_ok):
    gpu = tuple((c.cuda(), s) for c, s in make_qkv_fp8(2, 4, 2, 640, 128, 11))
    ref = run_fp8(gpu, "causal")
    for grid in (0, 1, 7):
        got = run_fp8(gpu, "causal", grid_ctas=grid)
        assert torch.equal(got[0], ref[0]) and torch.equal(got[1], ref[1])


def test_dense_shape_sampled_rows(cuda_ok):
    # the dense prefill workload's shape (B=2, 32 heads, N=8192) on 96 sampled rows of 2 heads
    from harness.inputs import sample_rows
    rows = sample_rows(8192, None, 101, count=96)
    cpu = make_qkv_fp8(2, 32, 32, 8192, 128, 1, device="cpu", sharp=True)
    gpu = tuple((c.cuda(), s) for c, s in cpu)
    out, lse = run_fp8(gpu, "causal")
    for b, h in ((0, 0), (1, 31)):
        sub = tuple((c[b:b + 1, h:h + 1].numpy(), s) for c, s in cpu)
        (q8, sq), (k8, sk), (v8, sv) = sub
        ref_o, ref_l = O8.attention_fp8(q8, k8, v8, sq, sk, sv, None, 1, None, rows=rows)
        abs_o, _ = O8.attention_fp8(q8, k8, v8 & np.uint8(0x7F), sq, sk, sv, None, 1, None, rows=rows)
        o = to_np(out[b:b + 1, h:h + 1])[:, :, rows].astype(np.float64)
        bound = 2.0 ** -4 * abs_o + 2.0 ** -8 * np.abs(ref_o) + 2e-4
        assert (np.abs(o - ref_o) <= bound).all()
        assert np.abs(to_np(lse[b:b + 1, h:h + 1])[:, :, rows] - ref_l).max() <= 1e-3
