"""CUDA backward (through the C ABI) against the fp64 backward oracle, element
by element within the bound derived in tests/parity_bwd.py."""
import pytest
import torch

from harness.inputs import make_dout, make_qkv
from tests.parity_bwd import check_bwd_case, run_cuda_bwd

pytestmark = pytest.mark.gpu


def test_tiny_workload(cuda_ok):
    check_bwd_case(1, 2, 2, 256, 64, "causal", seed=0)


@pytest.mark.parametrize("N", [1, 17, 128, 129, 300])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("mask", ["full", "causal"])
def test_ragged_lengths(cuda_ok, N, d, mask):
    check_bwd_case(1, 2, 2, N, d, mask, seed=N + d)


@pytest.mark.parametrize("w", [1, 2, 127, 129, 300])
@pytest.mark.parametrize("d", [64, 128])
def test_sliding_window(cuda_ok, w, d):
    check_bwd_case(1, 2, 1, 700, d, "sliding_window", window=w, seed=w)


@pytest.mark.parametrize("shape", [(2, 8, 2, 300), (1, 8, 1, 257), (1, 6, 2, 200), (2, 3, 3, 130)])
@pytest.mark.parametrize("mask,window", [("causal", None), ("full", None), ("sliding_window", 90)])
def test_head_sharing(cuda_ok, shape, mask, window):
    B, Hq, Hkv, N = shape
    check_bwd_case(B, Hq, Hkv, N, 128, mask, window, seed=sum(shape))


def test_multi_tile_and_scale(cuda_ok):
    check_bwd_case(1, 2, 1, 1024, 128, "causal", seed=5, sharp=True)
    check_bwd_case(1, 2, 2, 600, 64, "full", seed=6, scale=0.3)


def test_window_ge_N_is_causal_bitwise(cuda_ok):
    q, k, v = (t.cuda() for t in make_qkv(1, 4, 2, 333, 128, 9))
    do = make_dout(1, 4, 333, 128, 9).cuda()
    ref = run_cuda_bwd(q, k, v, do, "causal")
    for w in (333, 10 ** 6):
        got = run_cuda_bwd(q, k, v, do, "sliding_window", w)
        for a, b in zip(got, ref):
            assert torch.equal(a, b)


def test_outputs_fully_overwritten(cuda_ok):
    from exact_io_aware_72_b200 import bwd, fwd
    q, k, v = (t.cuda() for t in make_qkv(1, 2, 1, 200, 64, 10))
    do = make_dout(1, 2, 200, 64, 10).cuda()
    out, lse = fwd(q, k, v)
    dq = torch.full_like(q, float("nan"))
    dk = torch.full_like(k, float("nan"))
    dv = torch.full_like(v, float("nan"))
    bwd(q, k, v, out, lse, do, dq=dq, dk=dk, dv=dv)
    torch.cuda.synchronize()
    assert all(torch.isfinite(t.float()).all() for t in (dq, dk, dv))
