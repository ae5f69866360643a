"""CUDA paged-KV decoding (through the C ABI) against the fp64 decoding oracle,
element by element at the forward's parity bar."""
import numpy as np
import pytest
import torch

from harness.inputs import DECODE_WORKLOADS, make_decode_workload, make_paged_kv
from tests.parity import compare, to_np
from tests.parity_decode import DECODE_BOUND, check_decode_case, oracle_for, run_decode

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("mask", ["causal", "full"])
@pytest.mark.parametrize("group", [1, 4, 8])
def test_single_token_ragged_batch(cuda_ok, d, mask, group):
    lens = [1, 2, 127, 128, 129, 1000, 3000]
    check_decode_case(len(lens), 2 * group, 2, 1, d, lens, 16, mask, seed=d + group)


@pytest.mark.parametrize("page_size", [16, 32, 64, 128, 256])
@pytest.mark.parametrize("splits", [1, 3, None])
def test_page_sizes_and_splits(cuda_ok, page_size, splits):
    lens = [5, 300, 777, 2049]
    check_decode_case(len(lens), 8, 2, 1, 128, lens, page_size, "causal", seed=page_size, num_splits=splits)


@pytest.mark.parametrize("Nq,group", [(2, 8), (4, 8), (7, 8), (3, 1), (16, 8), (8, 16), (8, 32), (5, 30), (1, 32)])
@pytest.mark.parametrize("splits", [1, 3])
def test_multi_token_steps(cuda_ok, Nq, group, splits):
    # rows per (b, KV head) = group * Nq: 16, 32, 56, 3, 128, 128, 256 (two row chunks), 150, 32
    lens = [Nq, Nq + 1, 200, 1500]
    check_decode_case(len(lens), group, 1, Nq, 128, lens, 64, "causal", seed=Nq * 100 + group, num_splits=splits)


@pytest.mark.parametrize("rows", [8, 32, 64, 128])
def test_splits_of_whole_tiles(cuda_ok, rows):
    # every split but the last covers only whole, unmasked tiles: the item
    # epilogue must still wait for all of its P V products
    for L in (1024, 1500, 4096):
        check_decode_case(1, rows, 1, 1, 128, [L], 64, "causal", seed=L + rows, num_splits=L // 256)


@pytest.mark.parametrize("window", [1, 5, 100, 127, 128, 129, 4096])
@pytest.mark.parametrize("Nq", [1, 3])
def test_sliding_window_rolling_buffer(cuda_ok, window, Nq):
    # pages wholly before the oldest visible key are not allocated (table -1)
    lens = [Nq, 130, 1000, 5000]
    check_decode_case(len(lens), 8, 2, Nq, 128, lens, 16, "sliding_window", window=window, seed=window + Nq,
                      rolling=True)


def test_window_at_least_the_sequence_is_causal(cuda_ok):
    lens = [40, 700]
    inp = {k: v.cuda() for k, v in make_paged_kv(2, 8, 2, 2, 128, lens, 32, 77).items()}
    ref = run_decode(inp, "causal")
    for w in (700, 10 ** 6):
        got = run_decode(inp, "sliding_window", w)
        assert torch.equal(got[0], ref[0]) and torch.equal(got[1], ref[1])


@pytest.mark.parametrize("splits", [2, 7, 16, 40])
def test_more_splits_than_tiles(cuda_ok, splits):
    # some splits of the short sequences get no tile at all
    check_decode_case(3, 8, 2, 1, 64, [1, 300, 2000], 16, "causal", seed=splits, num_splits=splits)


@pytest.mark.parametrize("grid", [1, 3, 7])
def test_few_ctas_walk_many_items(cuda_ok, grid):
    lens = [2, 129, 600, 2500, 33, 1024]
    check_decode_case(len(lens), 16, 4, 2, 128, lens, 16, "causal", seed=grid, num_splits=3, grid_ctas=grid)
    check_decode_case(len(lens), 4, 4, 1, 64, lens, 64, "sliding_window", window=200, seed=grid, num_splits=2,
                      grid_ctas=grid, rolling=True)


def test_scale_and_large_scores(cuda_ok):
    # big logits force the lazy running-max rescale of O
    check_decode_case(2, 8, 1, 2, 128, [900, 4000], 16, "causal", seed=3, scale=0.6)
    check_decode_case(2, 8, 8, 1, 64, [900, 4000], 32, "full", seed=4, scale=1.5, num_splits=5)


def test_outputs_fully_overwritten_and_repeatable(cuda_ok):
    lens = [300, 1900, 64]
    inp = {k: v.cuda() for k, v in make_paged_kv(3, 16, 2, 2, 128, lens, 16, 5).items()}
    out = torch.full_like(inp["q"], float("nan"))
    lse = torch.full((3, 16, 2), float("nan"), device="cuda")
    o1, l1 = run_decode(inp, "causal", num_splits=4, out=out, lse=lse)
    assert torch.isfinite(o1.float()).all() and torch.isfinite(l1).all()
    for _ in range(3):
        o2, l2 = run_decode(inp, "causal", num_splits=4)
        assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_bad_sequence_length_is_reported(cuda_ok):
    from exact_io_aware_72_b200 import decode_debug_error
    lens = [100, 50, 400]
    inp = {k: v.cuda() for k, v in make_paged_kv(3, 8, 2, 2, 64, lens, 16, 6).items()}
    ref_o, ref_l = oracle_for({k: v.cpu() for k, v in inp.items()}, "causal", seqs=[0, 2])
    for bad in (1, 10 ** 6):   # fewer keys than new tokens; beyond the page table
        inp["seq_lens"][1] = bad
        for splits in (1, 3):
            out, lse = run_decode(inp, "causal", num_splits=splits)
            st, code = decode_debug_error()
            assert st == 1 and (code >> 20) == 1 and (code & 0xFFFFF) == 1
            assert torch.all(out[1] == 0) and torch.all(torch.isneginf(lse[1]))
            compare(to_np(out[[0, 2]]), to_np(lse[[0, 2]]), ref_o, ref_l, "good sequences", bound=DECODE_BOUND)


def test_missing_page_is_reported(cuda_ok):
    from exact_io_aware_72_b200 import decode_debug_error
    inp = {k: v.cuda() for k, v in make_paged_kv(2, 8, 2, 1, 64, [100, 300], 16, 7).items()}
    inp["block_table"][1, 3] = -1          # a page the step needs
    run_decode(inp, "causal", num_splits=1)
    st, code = decode_debug_error()
    assert st == 1 and (code >> 20) == 2 and (code & 0xFFFFF) == 1


# ---------------------------------------------------------------- full sizes
def _check_workload(name, seqs):
    w = DECODE_WORKLOADS[name]
    inp = make_decode_workload(w, device="cuda")
    lens = inp["seq_lens"].cpu().numpy()
    out, lse = run_decode(inp, w.mask, w.window, max_seq_len=int(lens.max()))
    from exact_io_aware_72_b200 import decode_debug_error
    st, code = decode_debug_error()
    assert st == 0, f"device error {code:#x}"
    ref_o, ref_l = oracle_for(inp, w.mask, w.window, seqs=seqs)
    compare(to_np(out[seqs]), to_np(lse[seqs]), ref_o, ref_l, name, bound=DECODE_BOUND)
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()


def test_workload_decode_gqa(cuda_ok):
    _check_workload("decode_gqa", [0])


def test_workload_decode_mha(cuda_ok):
    _check_workload("decode_mha", [0, 7, 15])


def test_workload_decode_swa(cuda_ok):
    _check_workload("decode_swa", [0, 13, 31])


def test_workload_decode_spec(cuda_ok):
    _check_workload("decode_spec", [0, 5])


def test_shared_workspace_counter_returns_to_zero(cuda_ok):
    from exact_io_aware_72_b200 import decode, decode_workspace_bytes
    lens = [3000, 17, 900, 4000, 1]
    inp = {k: v.cuda() for k, v in make_paged_kv(5, 8, 2, 1, 128, lens, 16, 8).items()}
    ref = None
    for splits, grid in ((1, 0), (3, 0), (3, 2), (1, 5)):
        ws = torch.zeros(decode_workspace_bytes(5, 8, 1, 128, splits) // 4, device="cuda")
        for _ in range(4):
            out, lse = decode(inp["q"], inp["k_cache"], inp["v_cache"], inp["block_table"], inp["seq_lens"],
                              num_splits=splits, workspace=ws, grid_ctas=grid)
            torch.cuda.synchronize()
            assert int(ws[:64].view(torch.int32).abs().sum()) == 0     # the work counter is back at zero
            if ref is None:
                ref = oracle_for({k: v.cpu() for k, v in inp.items()}, "causal")
            compare(to_np(out), to_np(lse), ref[0], ref[1], f"splits {splits} grid {grid}", bound=DECODE_BOUND)


@pytest.mark.parametrize("Nq,window", [(3, None), (5, 100), (2, 1)])
def test_head_dim_64_multi_token_and_window(cuda_ok, Nq, window):
    lens = [Nq, 130, 999, 2500]
    mask = "causal" if window is None else "sliding_window"
    check_decode_case(len(lens), 8, 2, Nq, 64, lens, 32, mask, window=window, seed=Nq + 7, num_splits=2,
                      rolling=window is not None)
