"""V values beyond the fp16 range.  The default forward feeds P V to the tensor
core in fp16; a V value of magnitude 2^16 or more is reported as ATTN_ERR_RANGE
by attn_debug_error (the result is then undefined), and the bf16-P option
(p_bf16) computes such inputs at its own documented bound.  Decoding feeds P V
in bf16 and takes any V."""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_72_b200 import attn as A
from harness.inputs import make_paged_kv, make_qkv
from tests.parity import compare, element_bound_p_bf16, to_np
from tests.parity_decode import oracle_for, run_decode

pytestmark = pytest.mark.gpu


def big_v(v, value):
    v = v.clone()
    v[0, 0, 5, 3] = value
    v[0, -1, -1, -1] = -value
    return v


@pytest.mark.parametrize("value", [65536.0, 1.0e6, 3.0e38])
def test_forward_reports_v_out_of_fp16_range(cuda_ok, value):
    q, k, v = make_qkv(1, 4, 2, 300, 128, 41)
    v = big_v(v, value)
    A.debug_error()
    A.fwd(q.cuda(), k.cuda(), v.cuda(), mask="causal")
    st, code = A.debug_error()
    assert st == A.ATTN_ERR_RANGE, (st, hex(code))
    # the largest finite values fp16 holds exactly pass without a report
    q2, k2, v2 = make_qkv(1, 4, 2, 300, 128, 42)
    A.fwd(q2.cuda(), k2.cuda(), big_v(v2, 65280.0).cuda(), mask="causal")
    assert A.debug_error()[0] == 0


def p_rounding_term(q, k, v, mask, window):
    """3 * 2^-8 times the attention of |v| (the same weights): bf16 P moves each
    weight by a relative error within 3/4 of a bf16 ulp (2^-7), and after
    renormalising by the sum of the written values the spread between two
    weights' errors is at most 3 * 2^-8, so out moves by at most that times
    sum_j w_j |v_j|.  A V value of 10^6 makes this term dominate."""
    a, _ = oracle.attention(to_np(q), to_np(k), np.abs(to_np(v)), None, A.MASKS[mask], window)
    return 3.0 * 2.0 ** -8 * a


@pytest.mark.parametrize("mask,window", [("causal", None), ("full", None), ("sliding_window", 77)])
@pytest.mark.parametrize("d", [64, 128])
def test_forward_p_bf16_takes_any_v(cuda_ok, mask, window, d):
    q, k, v = make_qkv(1, 4, 2, 300, d, 43 + d)
    v = big_v(v, 1.0e6)
    A.debug_error()
    out, lse = A.fwd(q.cuda(), k.cuda(), v.cuda(), mask=mask, window=window, p_bf16=True)
    torch.cuda.synchronize()
    assert A.debug_error()[0] == 0
    ref_o, ref_l = oracle.attention(to_np(q), to_np(k), to_np(v), None, A.MASKS[mask], window)
    compare(to_np(out), to_np(lse), ref_o, ref_l, f"p_bf16 {mask} {d}", bound=element_bound_p_bf16,
            extra=p_rounding_term(q, k, v, mask, window))


def test_decode_takes_any_v(cuda_ok):
    # Decoding feeds P V as bf16, so any bf16 V value is taken (no range report).
    inp = make_paged_kv(2, 8, 2, 1, 128, [300, 900], 16, 44, device="cpu")
    inp["v_cache"][0, 1, 3, 7] = 2.0e5
    g = {k: t.cuda() for k, t in inp.items()}
    A.decode_debug_error()
    out, lse = run_decode(g, "causal", num_splits=2)
    assert A.decode_debug_error()[0] == 0
    ref_o, ref_l = oracle_for(inp, "causal")
    compare(to_np(out), to_np(lse), ref_o, ref_l, "decode large v", bound=element_bound_p_bf16)


@pytest.mark.parametrize("N", [1, 129, 1000])
@pytest.mark.parametrize("mask", ["causal", "full"])
def test_forward_p_bf16_parity(cuda_ok, N, mask):
    from tests.parity import check_case
    check_case(1, 4, 2, N, 128, mask, seed=N + 7, p_bf16=True)
    check_case(1, 4, 4, N, 128, mask, seed=N + 8, sharp=True, p_bf16=True)
