"""Ring attention's CUDA steps on one GPU: every rank of the ring runs in turn in
this process (no rank waits on another), each block through the forward kernel
and each partial result through the attn_merge kernel; the reassembled output
is checked against the fp64 forward oracle on the whole sequence at the
forward's own parity bar.  Block partials are the forward's fp32 out, so the
only bf16 rounding is the final merged row's."""
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


def test_fp32_out_is_the_bf16_out_unrounded(cuda_ok):
    # out_fp32 writes O / l before the one rounding the bf16 output makes: rounding
    # it to bf16 must give the bf16 call's bits, and lse is the same.
    from exact_io_aware_72_b200 import fwd
    for shape, mask, window in (((1, 4, 2, 1000, 128), "causal", None), ((2, 2, 2, 300, 64), "full", None),
                                ((1, 8, 2, 700, 128), "sliding_window", 100)):
        B, Hq, Hkv, N, d = shape
        q, k, v = (t.cuda() for t in make_qkv(B, Hq, Hkv, N, d, N))
        o16, l16 = fwd(q, k, v, mask=mask, window=window)
        o32, l32 = fwd(q, k, v, mask=mask, window=window, out_fp32=True)
        torch.cuda.synchronize()
        assert o32.dtype == torch.float32
        assert torch.equal(o32.to(torch.bfloat16), o16) and torch.equal(l32, l16)
        ref_o, ref_l = oracle.attention(to_np(q), to_np(k), to_np(v), None, {"full": 0, "causal": 1,
                                        "sliding_window": 2}[mask], window)
        # unrounded: well inside the bar (no output rounding)
        assert float(np.abs(o32.double().cpu().numpy() - ref_o).max()) < 2e-3


def test_merge_fp32_partials(cuda_ok):
    g = torch.Generator(device="cuda").manual_seed(4)
    rows, d = 700, 64
    acc = torch.randn(rows, d, device="cuda", generator=g)
    acc_l = torch.randn(rows, device="cuda", generator=g)
    part = torch.randn(rows, d, device="cuda", generator=g)
    part_l = torch.randn(rows, device="cuda", generator=g)
    a0, l0 = acc.clone(), acc_l.clone()
    out = torch.empty(rows, d, dtype=torch.bfloat16, device="cuda")
    merge(acc, acc_l, part, part_l, out=out)
    m = torch.maximum(l0, part_l)
    wa, wp = torch.exp(l0 - m), torch.exp(part_l - m)
    ref = (wa[:, None] * a0 + wp[:, None] * part) / (wa + wp)[:, None]
    assert torch.allclose(acc, ref, rtol=1e-5, atol=1e-6)
    assert torch.equal(out, acc.to(torch.bfloat16))
    merge(acc, acc_l, part, part_l, first=True)
    assert torch.equal(acc, part) and torch.equal(acc_l, part_l)


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


# Block partials are the forward's fp32 out (no bf16 rounding before the merge),
# so the merged rows are held to the forward's own bar.


@pytest.mark.parametrize("name,world,heads", [("dense", 8, None), ("long", 8, [(0, 0), (0, 17), (0, 31)])])
def test_emulated_ring_full_size_sampled_rows(cuda_ok, name, world, heads):
    # The ring benchmark's configuration (same inputs, 8 ranks emulated in turn):
    # the reassembled rows against the oracle on 256 seeded rows per head.
    from harness.inputs import MASK_NAMES, WORKLOADS, make_workload, sample_rows
    w = WORKLOADS[name]
    q, k, v = make_workload(w, device="cuda")
    out, lse = ring.ring_forward_emulated(q, k, v, world, w.mask, w.scale)
    torch.cuda.synchronize()
    rows = sample_rows(w.N, w.window, w.seed + 100)
    rows_t = torch.as_tensor(rows, device=q.device)
    g = w.Hq // w.Hkv
    heads = heads or [(b, h) for b in range(w.B) for h in range(w.Hq)]
    kind = MASK_NAMES[w.mask]
    worst = {}
    for b, h in heads:
        qh, kh, vh = to_np(q[b:b + 1, h:h + 1]), to_np(k[b:b + 1, h // g:h // g + 1]), to_np(v[b:b + 1, h // g:h // g + 1])
        ro, rl = oracle.attention(qh, kh, vh, w.scale, kind, w.window, rows=rows)
        go = to_np(out[b:b + 1, h:h + 1].index_select(2, rows_t))
        gl = to_np(lse[b:b + 1, h:h + 1].index_select(2, rows_t))
        st = compare(go, gl, ro, rl, f"ring {name} b={b} h={h}")
        worst = {key: max(worst.get(key, 0.0), val) for key, val in st.items()}
    print(f"\nring {name} x{world}: out max-abs {worst['max_abs']:.3e}  rel-L2 {worst['rel_l2']:.3e}  "
          f"lse max-abs {worst['lse_max_abs']:.3e}  ({len(rows)} rows x {len(heads)} heads)")
    del q, k, v, out, lse
    torch.cuda.empty_cache()


def test_emulated_ring_replays_from_a_cuda_graph(cuda_ok):
    # The benchmark times the emulated ring step as a CUDA graph replay: the
    # captured launches must give the eager step's bits, replay after replay.
    q, k, v = (t.cuda() for t in make_qkv(1, 4, 2, 1024, 128, 21))
    shares = ring.emulate_shares(q, k, v, 4)
    eager = ring.run_emulated(shares, "causal")
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        captured = ring.run_emulated(shares, "causal")
    for _ in range(3):
        for t in (x for res in captured for pair in res for x in pair):
            t.fill_(float("nan"))
        graph.replay()
        torch.cuda.synchronize()
        for (eo, el), (co, cl) in zip(eager, captured):
            for a, b in zip(eo + el, co + cl):
                assert torch.equal(a, b)


@pytest.mark.parametrize("world,window", [(2, 1), (2, 300), (2, 512), (4, 100), (4, 256), (4, 700), (8, 129),
                                          (8, 1000), (4, 2048)])
def test_emulated_ring_with_a_window_matches_oracle(cuda_ok, world, window):
    # Blocks against earlier key halves are windows with a key offset (the forward's
    # key_offset); blocks no row reaches are skipped.  Whole sequence against the oracle.
    q, k, v = make_qkv(1, 4, 2, 2048, 128, world + window)
    out, lse = ring.ring_forward_emulated(q.cuda(), k.cuda(), v.cuda(), world, "sliding_window", window=window)
    torch.cuda.synchronize()
    ref_o, ref_l = oracle.attention(to_np(q), to_np(k), to_np(v), None, 2, window)
    compare(to_np(out), to_np(lse), ref_o, ref_l, f"ring world {world} window {window}")


def test_key_offset_identities(cuda_ok):
    from exact_io_aware_72_b200 import fwd
    q, k, v = (t.cuda() for t in make_qkv(1, 4, 2, 700, 128, 77))
    for mask, window in (("causal", None), ("sliding_window", 150)):
        a = fwd(q, k, v, mask=mask, window=window)
        b = fwd(q, k, v, mask=mask, window=window, key_offset=0)
        assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
    # every key is at or before every query: causal equals full
    full = fwd(q, k, v, mask="full")
    for off in (700, 701, 5000):
        c = fwd(q, k, v, mask="causal", key_offset=off)
        assert torch.equal(c[0], full[0]) and torch.equal(c[1], full[1])
    # a window that reaches the whole block from every row is full too
    c = fwd(q, k, v, mask="sliding_window", window=1400, key_offset=700)
    assert torch.equal(c[0], full[0]) and torch.equal(c[1], full[1])
    # rows whose window starts after the last key see nothing: out 0, lse -inf
    off, w = 900, 400
    o, l = fwd(q, k, v, mask="sliding_window", window=w, key_offset=off)
    torch.cuda.synchronize()
    rows = torch.arange(700, device="cuda")
    empty = rows + off - w + 1 > 699
    assert empty.any() and (~empty).any()
    assert torch.all(o[:, :, empty] == 0) and torch.all(torch.isneginf(l[:, :, empty]))
    assert torch.isfinite(l[:, :, ~empty]).all()
