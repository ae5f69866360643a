"""attn_decode_static, the decoding step for callers that cannot allocate device
memory (code inside a host program that owns all device memory and hands over
only inputs and outputs).  It keeps its scratch in a fixed array of the library
instead of a caller workspace.  Called through the C ABI, two calls in a row
must each give the result of the workspace entry point, attn_decode, on the
same inputs.  This file is collected last, so a stop at the first failure has
already run every other test."""
import ctypes

import pytest
import torch

from exact_io_aware_72_b200 import attn as A
from harness.inputs import make_paged_kv
from tests.parity import compare, to_np
from tests.parity_decode import DECODE_BOUND, run_decode

pytestmark = pytest.mark.gpu

ATTN_ERR_UNSUPPORTED = 2


def static_call(lib, inp, out, lse, num_splits, mask, window=0):
    B, Hq, Nq, d = inp["q"].shape
    num_pages, Hkv, page_size, _ = inp["k_cache"].shape
    stream = torch.cuda.current_stream().cuda_stream
    return lib.attn_decode_static(inp["q"].data_ptr(), inp["k_cache"].data_ptr(), inp["v_cache"].data_ptr(),
                                  inp["block_table"].data_ptr(), inp["seq_lens"].data_ptr(), out.data_ptr(),
                                  lse.data_ptr(), B, Hq, Hkv, Nq, d, num_pages, page_size,
                                  inp["block_table"].shape[1], num_splits, 1.0 / d ** 0.5, A.MASKS[mask], window,
                                  ctypes.c_void_p(stream))


def test_static_scratch_matches_workspace_entry_point(cuda_ok):
    lib = A.load_library()
    # Two different steps, both with several splits so the partial results live in
    # the scratch array; the second call follows the first with no synchronisation.
    cases = [
        dict(args=(4, 16, 2, 2, 128, [5, 300, 1000, 3000], 16, 31), splits=3, mask="causal", window=None),
        dict(args=(3, 8, 8, 1, 64, [2049, 17, 640], 64, 32), splits=5, mask="sliding_window", window=500),
    ]
    inputs, outs = [], []
    for c in cases:
        inp = {k: v.cuda() for k, v in make_paged_kv(*c["args"], device="cpu").items()}
        out = torch.empty_like(inp["q"])
        lse = torch.empty(inp["q"].shape[:3], dtype=torch.float32, device="cuda")
        st = static_call(lib, inp, out, lse, c["splits"], c["mask"], c["window"] or 0)
        assert st == 0, A.STATUS.get(st, st)
        inputs.append(inp)
        outs.append((out, lse))
    torch.cuda.synchronize()
    for c, inp, (out, lse) in zip(cases, inputs, outs):
        ref_o, ref_l = run_decode(inp, c["mask"], c["window"], num_splits=c["splits"])
        compare(to_np(out), to_np(lse), to_np(ref_o).astype("float64"), to_np(ref_l).astype("float64"),
                f"attn_decode_static {c['args'][:5]}", bound=DECODE_BOUND)
    st, code = A.decode_debug_error()
    assert st == 0, f"device error {code:#x}"


def test_static_scratch_refuses_steps_beyond_its_size(cuda_ok):
    lib = A.load_library()
    B, Hq, Nq, d, splits = 64, 64, 1, 128, 16
    assert A.decode_workspace_bytes(B, Hq, Nq, d, splits) > A.DECODE_STATIC_SCRATCH_BYTES
    inp = {k: v.cuda() for k, v in make_paged_kv(B, Hq, 8, Nq, d, [300] * B, 16, 33, device="cpu").items()}
    out = torch.empty_like(inp["q"])
    lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device="cuda")
    assert static_call(lib, inp, out, lse, splits, "causal") == ATTN_ERR_UNSUPPORTED
    # one split fits: the same step then runs
    assert static_call(lib, inp, out, lse, 1, "causal") == 0
    ref_o, ref_l = run_decode(inp, "causal", num_splits=1)
    compare(to_np(out), to_np(lse), to_np(ref_o).astype("float64"), to_np(ref_l).astype("float64"), "one split",
            bound=DECODE_BOUND)
