"""Host-buffer forward (attn_fwd_host / attn_fwd_fp8_host through the C ABI):
the job cut into chunks of (batch, key/value head) units, uploads, kernels and
downloads overlapped on three streams.  Each chunk is the same kernel on a
contiguous range of heads, so the host results must equal the device call's
bit for bit, for every chunk count (one, ragged, one unit each, more chunks
than units) and for pinned and pageable host memory; one case also goes
against the fp64 oracle directly."""
import pytest
import torch

import oracle
from harness.inputs import MASK_NAMES, make_qkv, make_qkv_fp8
from tests.parity import compare, to_np

pytestmark = pytest.mark.gpu


def _device_result(q, k, v, mask, window, scale):
    from exact_io_aware_72_b200 import fwd
    out, lse = fwd(q.cuda(), k.cuda(), v.cuda(), scale=scale, mask=mask, window=window)
    torch.cuda.synchronize()
    return out.cpu(), lse.cpu()


@pytest.mark.parametrize("shape", [(2, 4, 2, 300, 64), (3, 6, 3, 257, 128), (1, 8, 8, 640, 128),
                                   (2, 8, 1, 129, 64)])
@pytest.mark.parametrize("chunks", [0, 1, 3, 1000])
@pytest.mark.parametrize("pinned", [True, False])
def test_host_forward_equals_device_forward(cuda_ok, shape, chunks, pinned):
    from exact_io_aware_72_b200 import fwd_host
    B, Hq, Hkv, N, d = shape
    q, k, v = make_qkv(B, Hq, Hkv, N, d, seed=sum(shape) + chunks)
    ref_o, ref_l = _device_result(q, k, v, "causal", None, None)
    if pinned:
        q, k, v = q.pin_memory(), k.pin_memory(), v.pin_memory()
    out, lse = fwd_host(q, k, v, mask="causal", chunks=chunks)
    assert not out.is_cuda and out.is_pinned() == pinned
    assert torch.equal(out, ref_o) and torch.equal(lse, ref_l)


@pytest.mark.parametrize("mask,window", [("full", None), ("sliding_window", 100), ("sliding_window", 5000)])
def test_host_forward_masks(cuda_ok, mask, window):
    from exact_io_aware_72_b200 import fwd_host
    q, k, v = make_qkv(2, 4, 2, 1000, 128, seed=41)
    ref_o, ref_l = _device_result(q, k, v, mask, window, 0.07)
    out, lse = fwd_host(q.pin_memory(), k.pin_memory(), v.pin_memory(), scale=0.07, mask=mask, window=window,
                        chunks=3)
    assert torch.equal(out, ref_o) and torch.equal(lse, ref_l)


def test_host_forward_against_oracle(cuda_ok):
    from exact_io_aware_72_b200 import fwd_host
    q, k, v = make_qkv(2, 4, 2, 700, 64, seed=42, sharp=True)
    out, lse = fwd_host(q.pin_memory(), k.pin_memory(), v.pin_memory(), mask="sliding_window", window=300, chunks=3)
    ref_o, ref_l = oracle.attention(to_np(q), to_np(k), to_np(v), None, MASK_NAMES["sliding_window"], 300)
    compare(to_np(out), to_np(lse), ref_o, ref_l, "host forward")


def test_host_forward_waits_for_earlier_work_on_the_stream(cuda_ok):
    # The caller's staging buffers are still being written by earlier work on the
    # stream (a long fill); the uploads must not start before that work ends.
    from exact_io_aware_72_b200 import fwd_host
    B, Hq, Hkv, N, d = 2, 4, 4, 2048, 128
    q, k, v = make_qkv(B, Hq, Hkv, N, d, seed=43)
    ref_o, ref_l = _device_result(q, k, v, "causal", None, None)
    stream = torch.cuda.Stream()
    staging = (torch.empty(q.shape, dtype=q.dtype, device="cuda"), torch.empty(k.shape, dtype=k.dtype, device="cuda"),
               torch.empty(v.shape, dtype=v.dtype, device="cuda"), torch.empty(q.shape, dtype=q.dtype, device="cuda"),
               torch.empty((B, Hq, N), dtype=torch.float32, device="cuda"))
    big = torch.empty(1 << 28, dtype=torch.float32, device="cuda")
    torch.cuda.synchronize()
    hq, hk, hv = q.pin_memory(), k.pin_memory(), v.pin_memory()
    for _ in range(3):
        with torch.cuda.stream(stream):
            for _ in range(16):
                big.fill_(1.0)                      # ~16 GB of writes ahead of the fills below
            for t in staging[:3]:
                t.fill_(float("nan"))
        out, lse = fwd_host(hq, hk, hv, mask="causal", chunks=4, staging=staging, stream=stream)
        assert torch.equal(out, ref_o) and torch.equal(lse, ref_l)


def test_host_forward_reuses_given_outputs(cuda_ok):
    from exact_io_aware_72_b200 import fwd_host
    q, k, v = make_qkv(1, 4, 2, 384, 64, seed=44)
    ref_o, ref_l = _device_result(q, k, v, "causal", None, None)
    out = torch.full(q.shape, float("nan"), dtype=torch.bfloat16).pin_memory()
    lse = torch.full(q.shape[:-1], float("nan"), dtype=torch.float32).pin_memory()
    o, l = fwd_host(q.pin_memory(), k.pin_memory(), v.pin_memory(), out=out, lse=lse)
    assert o.data_ptr() == out.data_ptr() and l.data_ptr() == lse.data_ptr()
    assert torch.equal(out, ref_o) and torch.equal(lse, ref_l)


@pytest.mark.parametrize("chunks", [0, 2, 5])
def test_fp8_host_forward_equals_device_forward(cuda_ok, chunks):
    from exact_io_aware_72_b200 import fwd_fp8, fwd_fp8_host
    (q8, sq), (k8, sk), (v8, sv) = make_qkv_fp8(2, 8, 2, 600, 128, seed=45 + chunks)
    ro, rl = fwd_fp8(q8.cuda(), k8.cuda(), v8.cuda(), sq, sk, sv, mask="causal")
    torch.cuda.synchronize()
    out, lse = fwd_fp8_host(q8.pin_memory(), k8.pin_memory(), v8.pin_memory(), sq, sk, sv, mask="causal",
                            chunks=chunks)
    assert torch.equal(out, ro.cpu()) and torch.equal(lse, rl.cpu())


def test_host_forward_rejects_device_tensors(cuda_ok):
    from exact_io_aware_72_b200 import fwd_host
    q, k, v = make_qkv(1, 2, 2, 128, 64, seed=46)
    with pytest.raises(ValueError):
        fwd_host(q.cuda(), k, v)
