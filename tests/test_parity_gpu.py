"""CUDA path (through the C ABI) against the fp64 oracle, element by element."""
import numpy as np
import pytest
import torch

from harness.inputs import make_qkv
from tests.parity import check_case, run_cuda, to_np

pytestmark = pytest.mark.gpu


def test_tiny_workload_every_row(cuda_ok):
    # B=1, Hq=Hkv=2, N=256, d=64, causal, seed 0: every row against the oracle.
    check_case(1, 2, 2, 256, 64, "causal", seed=0)


@pytest.mark.parametrize("N", [1, 17, 127, 128, 129, 255, 600, 640, 1000])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("mask", ["full", "causal"])
def test_ragged_lengths(cuda_ok, N, d, mask):
    check_case(1, 2, 2, N, d, mask, seed=N + d)


@pytest.mark.parametrize("N,d", [(640, 64), (600, 64), (600, 128), (300, 64)])
def test_repeated_launches_identical(cuda_ok, N, d):
    # An odd number of 128-row blocks leaves one work item with an idle second
    # tile; its MMA warp runs ahead of the busy one.  Every launch must give
    # the same bits (and match the oracle), not only the first.
    q, k, v = (t.cuda() for t in make_qkv(1, 2, 2, N, d, 6))
    o0, l0 = run_cuda(q, k, v, "causal", scale=0.3)
    for _ in range(12):
        o1, l1 = run_cuda(q, k, v, "causal", scale=0.3)
        assert torch.equal(o0, o1) and torch.equal(l0, l1)
    check_case(1, 2, 2, N, d, "causal", seed=6, scale=0.3)


@pytest.mark.parametrize("w", [1, 2, 127, 128, 129, 999, 1000, 1001])
@pytest.mark.parametrize("d", [64, 128])
def test_sliding_window_edges(cuda_ok, w, d):
    check_case(1, 4, 2, 1000, d, "sliding_window", window=w, seed=w)


@pytest.mark.parametrize("shape", [
    (2, 8, 8, 300), (2, 8, 4, 300), (1, 8, 2, 300), (1, 8, 1, 300),   # MHA, g=2, g=4, MQA
    (1, 6, 2, 300), (1, 3, 3, 300), (1, 3, 1, 200), (3, 2, 1, 257),   # odd groups, odd heads, B>1
])
@pytest.mark.parametrize("mask,window", [("causal", None), ("full", None), ("sliding_window", 100)])
def test_head_sharing(cuda_ok, shape, mask, window):
    B, Hq, Hkv, N = shape
    check_case(B, Hq, Hkv, N, 128, mask, window, seed=sum(shape))


def test_sharp_rows_rescale(cuda_ok):
    # 5% of keys x4 (the dense workload's recipe) forces online rescaling.
    check_case(1, 4, 4, 2048, 128, "causal", seed=11, sharp=True)
    check_case(1, 4, 2, 1500, 64, "sliding_window", window=700, seed=12, sharp=True)


def test_multi_tile_full_mask(cuda_ok):
    check_case(1, 2, 1, 2304, 128, "full", seed=13)


def test_nondefault_scale(cuda_ok):
    check_case(1, 2, 2, 300, 128, "causal", seed=14, scale=0.37)
    check_case(1, 2, 2, 300, 64, "full", seed=15, scale=0.02)


# ------------------------------------------------------------------ metamorphic
def test_gqa_equals_repeated_mha_bitwise(cuda_ok):
    q, k, v = (t.cuda() for t in make_qkv(2, 8, 2, 700, 128, 21))
    for mask, w in (("causal", None), ("full", None), ("sliding_window", 200)):
        o1, l1 = run_cuda(q, k, v, mask, w)
        o2, l2 = run_cuda(q, k.repeat_interleave(4, dim=1).contiguous(), v.repeat_interleave(4, dim=1).contiguous(),
                          mask, w)
        assert torch.equal(o1, o2) and torch.equal(l1, l2), mask


def test_window_ge_N_is_causal_bitwise(cuda_ok):
    q, k, v = (t.cuda() for t in make_qkv(1, 4, 2, 777, 128, 22))
    oc, lc = run_cuda(q, k, v, "causal")
    for w in (777, 778, 10 ** 6):
        ow, lw = run_cuda(q, k, v, "sliding_window", w)
        assert torch.equal(oc, ow) and torch.equal(lc, lw)


def test_causal_row0_and_window1_return_v(cuda_ok):
    q, k, v = (t.cuda() for t in make_qkv(2, 4, 2, 513, 128, 23))
    oc, _ = run_cuda(q, k, v, "causal")
    assert torch.equal(oc[:, :, 0], v.repeat_interleave(2, dim=1)[:, :, 0])
    o1, l1 = run_cuda(q, k, v, "sliding_window", 1)
    assert torch.equal(o1, v.repeat_interleave(2, dim=1))
    s_ii = (q.float() * k.repeat_interleave(2, dim=1).float()).sum(-1) / np.sqrt(128)
    assert float((l1 - s_ii).abs().max()) < 1e-3


def test_full_mask_key_permutation(cuda_ok):
    q, k, v = (t.cuda() for t in make_qkv(1, 2, 2, 640, 128, 24))
    perm = torch.randperm(640, generator=torch.Generator().manual_seed(0)).cuda()
    o1, l1 = run_cuda(q, k, v, "full")
    o2, l2 = run_cuda(q, k[:, :, perm].contiguous(), v[:, :, perm].contiguous(), "full")
    assert float((o1.float() - o2.float()).abs().max()) < 1e-2
    assert float((l1 - l2).abs().max()) < 1e-3


def test_outputs_fully_overwritten(cuda_ok):
    from exact_io_aware_72_b200 import fwd
    q, k, v = (t.cuda() for t in make_qkv(1, 2, 2, 300, 64, 25))
    out = torch.full_like(q, float("nan"))
    lse = torch.full((1, 2, 300), float("nan"), device="cuda")
    fwd(q, k, v, mask="causal", out=out, lse=lse)
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()


def test_out_16_byte_aligned_matches_32_byte_aligned_bitwise(cuda_ok):
    # Rows of out are written with 32-byte stores when out is 32-byte aligned
    # and with 16-byte stores otherwise; both paths must give the same bits.
    from exact_io_aware_72_b200 import fwd
    q, k, v = (t.cuda() for t in make_qkv(1, 4, 2, 333, 128, 26))
    o_ref, l_ref = run_cuda(q, k, v, "causal")
    buf = torch.empty(q.numel() + 8, dtype=q.dtype, device=q.device)
    out = buf[8:].view(q.shape)  # 16 bytes past a 256-byte boundary
    assert out.data_ptr() % 32 == 16
    lse = torch.empty_like(l_ref)
    fwd(q, k, v, mask="causal", out=out, lse=lse)
    torch.cuda.synchronize()
    assert torch.equal(out, o_ref) and torch.equal(lse, l_ref)


@pytest.mark.parametrize("shape", [(64, 2, 1, 64, 128), (33, 3, 3, 129, 64), (1, 96, 8, 200, 128)])
def test_many_small_heads_and_sequences(cuda_ok, shape):
    # far more work items than SMs, each tiny: the static schedule's tail split
    B, Hq, Hkv, N, d = shape
    check_case(B, Hq, Hkv, N, d, "causal", seed=B + Hq + N)


def test_grid_sizes_give_identical_bits(cuda_ok):
    from exact_io_aware_72_b200 import fwd
    q, k, v = (t.cuda() for t in make_qkv(2, 8, 2, 1000, 128, 21))
    ref = fwd(q, k, v)
    for grid in (1, 5, 37, 148):
        got = fwd(q, k, v, grid_ctas=grid)
        assert torch.equal(got[0], ref[0]) and torch.equal(got[1], ref[1])
