"""Ring attention's CUDA steps on one GPU: every rank of the ring runs in turn in
this process (no rank waits on another), each block through the forward kernel
and each partial result through the attn_merge kernel; the reassembled output
is checked against the fp64 forward oracle on the whole sequence, at the
forward's parity bar (each partial out is rounded to bf16 once more before the
fp32 merge, well inside that bar)."""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_72_b200 import merge, ring
from harness.inputs import make_qkv
from tests.parity import compare, to_np

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("world", [1, 2, 4, 8])
@pytest.mark.parametrize("mask", ["causal", "full"])
def test_emulated_ring_matches_oracle(cuda_ok, world, mask):
    q, k, v = make_qkv(1, 4, 2, 2048, 128, world)
    out, lse = ring.ring_forward_emulated(q.cuda(), k.cuda(), v.cuda(), world, mask)
    torch.cuda.synchronize()
    ref_o, ref_l = oracle.attention(to_np(q), to_np(k), to_np(v), None, {"full": 0, "causal": 1}[mask])
    compare(to_np(out), to_np(lse), ref_o, ref_l, f"ring world {world} {mask}")


def test_emulated_ring_head_dim_64_and_mqa(cuda_ok):
    q, k, v = make_qkv(2, 6, 1, 768, 64, 5)
    out, lse = ring.ring_forward_emulated(q.cuda(), k.cuda(), v.cuda(), 3, "causal")
    torch.cuda.synchronize()
    ref_o, ref_l = oracle.attention(to_np(q), to_np(k), to_np(v), None, 1)
    compare(to_np(out), to_np(lse), ref_o, ref_l, "ring world 3 d 64 mqa")


def test_merge_kernel_modes(cuda_ok):
    g = torch.Generator(device="cuda").manual_seed(3)
    rows, d = 1000, 128
    acc = torch.randn(rows, d, device="cuda", generator=g)
    acc_l = torch.randn(rows, device="cuda", generator=g)
    part = torch.randn(rows, d, device="cuda", generator=g).to(torch.bfloat16)
    part_l = torch.randn(rows, device="cuda", generator=g)
    part_l[:10] = float("-inf")          # rows where the partial saw no key
    a0, l0 = acc.clone(), acc_l.clone()
    out = torch.empty(rows, d, dtype=torch.bfloat16, device="cuda")
    merge(acc, acc_l, part, part_l, out=out)
    m = torch.maximum(l0, part_l)
    wa, wp = torch.exp(l0 - m), torch.exp(part_l - m)
    ref = (wa[:, None] * a0 + wp[:, None] * part.float()) / (wa + wp)[:, None]
    assert torch.allclose(acc, ref, rtol=1e-5, atol=1e-6)
    assert torch.allclose(acc_l, m + torch.log(wa + wp), rtol=0, atol=1e-5)
    assert torch.equal(acc[:10], a0[:10]) and torch.equal(acc_l[:10], l0[:10])
    assert torch.equal(out, acc.to(torch.bfloat16))
    merge(acc, acc_l, part, part_l, first=True, out=part)   # out may be the partial itself
    assert torch.equal(acc, part.float()) and torch.equal(acc_l, part_l)
