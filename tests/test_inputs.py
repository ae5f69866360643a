"""The seeded input generators (CPU only): the paged KV cache's table and fill,
and the per-tensor E4M3 quantisation of the FP8 inputs."""
import numpy as np
import torch

from harness.inputs import (DECODE_WORKLOADS, make_paged_kv, make_qkv_fp8, make_seq_lens, quantise_e4m3)
from oracle import attention_fp8 as O8


def test_paged_cache_table_is_a_permutation_of_the_kept_pages():
    lens = [37, 5, 64, 1]
    keep = [20, 0, 33, 0]
    d = make_paged_kv(4, 4, 2, 1, 8, lens, 16, 3, keep_from=keep, fill=float("nan"), extra_pages=2)
    table = d["block_table"].numpy()
    used = table[table >= 0]
    assert len(set(used.tolist())) == len(used)                     # no page shared by two slots
    n_pages = d["k_cache"].shape[0]
    assert n_pages == len(used) + 2 and used.max() < n_pages
    for b, (L, k0) in enumerate(zip(lens, keep)):
        row = table[b]
        kept = [lp for lp in range(len(row)) if row[lp] >= 0]
        assert kept == list(range(k0 // 16, (L - 1) // 16 + 1))     # exactly the pages holding keep..L-1
    # unused slots hold the fill: the tail of each last page and the extra pages
    kc = d["k_cache"].float()
    for b, L in enumerate(lens):
        last = table[b][(L - 1) // 16]
        tail = kc[last, :, (L - 1) % 16 + 1:]
        assert torch.isnan(tail).all() and not torch.isnan(kc[last, :, :(L - 1) % 16 + 1]).any()
    spare = sorted(set(range(n_pages)) - set(used.tolist()))
    assert torch.isnan(kc[spare]).all()


def test_paged_cache_is_reproducible_and_seed_dependent():
    a = make_paged_kv(2, 2, 1, 1, 8, [40, 9], 16, 7)
    b = make_paged_kv(2, 2, 1, 1, 8, [40, 9], 16, 7)
    c = make_paged_kv(2, 2, 1, 1, 8, [40, 9], 16, 8)
    assert all(torch.equal(a[k], b[k]) for k in a)
    assert not torch.equal(a["k_cache"], c["k_cache"])


def test_decode_workloads_lengths_and_rolling_buffer():
    for w in DECODE_WORKLOADS.values():
        lens = make_seq_lens(w.B, w.L_min, w.L_max, w.seed)
        assert lens.min() >= w.L_min and lens.max() <= w.L_max and len(lens) == w.B
        assert w.Hq % w.Hkv == 0 and w.Nq <= w.L_min
    w = DECODE_WORKLOADS["decode_swa"]
    assert w.rolling and w.mask == "sliding_window"


def test_e4m3_quantisation_round_trip():
    g = torch.Generator().manual_seed(0)
    t = torch.randn(4, 64, generator=g) * 3.0
    codes, scale = quantise_e4m3(t)
    assert codes.dtype == torch.uint8
    back = O8.dequantise(codes.numpy(), scale)
    x = t.double().numpy()
    assert abs(scale - float(t.abs().max()) / 448.0) < 1e-12
    assert np.nanmax(np.abs(back)) <= float(t.abs().max()) * (1 + 2 ** -4)   # the largest maps to <= 448
    # round to nearest: within half an E4M3 step (2^-4 relative) of t, or of the subnormal spacing
    err = np.abs(back - x)
    assert (err <= np.maximum(2.0 ** -4 * np.abs(x), 2.0 ** -10 * scale) + 1e-12).all()


def test_fp8_inputs_follow_the_bf16_draws():
    (q8, sq), (k8, sk), (v8, sv) = make_qkv_fp8(1, 2, 2, 16, 128, 5)
    assert q8.shape == (1, 2, 16, 128) and k8.shape == v8.shape == (1, 2, 16, 128)
    assert min(sq, sk, sv) > 0
    (q8b, _), _, _ = make_qkv_fp8(1, 2, 2, 16, 128, 5)
    assert torch.equal(q8, q8b)
