"""C-ABI library: loads without a GPU, exports every symbol include/attn.h
declares, and rejects bad arguments on the host before touching the device."""
import ctypes
import os
import re

import pytest

from exact_io_aware_72_b200 import attn as A
from exact_io_aware_72_b200 import build as BLD

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    BLD.build()
    return A.load_library()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "attn.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:int|int64_t|size_t|const char\*)\s+(attn_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_expected_entry_points():
    assert declared_functions() == sorted(A.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for code, name in A.STATUS.items():
        assert lib.attn_status_string(code).decode() == name
    assert lib.attn_status_string(99).decode() == "ATTN_ERR_UNKNOWN"


# Fake, never-dereferenced device addresses: far apart, 256-byte aligned.
Q, K, V, O, L = (0x10000000000 * (i + 1) for i in range(5))


def call(lib, q=Q, k=K, v=V, o=O, l=L, B=1, Hq=2, Hkv=2, N=256, d=64, scale=0.125, mask=1, window=0):
    return lib.attn_fwd(q, k, v, o, l, B, Hq, Hkv, N, d, scale, mask, window, None)


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), 1), (dict(k=None), 1), (dict(v=None), 1), (dict(o=None), 1), (dict(l=None), 1),
    (dict(B=0), 1), (dict(Hq=0), 1), (dict(Hkv=0), 1), (dict(N=0), 1), (dict(B=-3), 1),
    (dict(Hq=6, Hkv=4), 1), (dict(mask=3), 1), (dict(mask=-1), 1),
    (dict(mask=2, window=0), 1), (dict(mask=2, window=-5), 1),
    (dict(scale=0.0), 1), (dict(scale=-0.1), 1), (dict(scale=float("inf")), 1), (dict(scale=float("nan")), 1),
    (dict(d=32), 2), (dict(d=96), 2), (dict(d=256), 2),
    (dict(q=Q + 8), 3), (dict(k=K + 4), 3), (dict(v=V + 2), 3), (dict(o=O + 8), 3), (dict(l=L + 2), 3),
    (dict(o=Q), 1), (dict(o=K + 64), 1), (dict(l=O + 1024), 1), (dict(l=V), 1),
    (dict(N=(1 << 30) + 1), 1),
    # 2^60 rows x d: each factor within its bound, the byte count beyond 63 bits
    (dict(B=1 << 10, Hq=1 << 20, Hkv=1 << 20, N=1 << 30), 1), (dict(B=1, Hq=1 << 30, Hkv=1, N=1 << 30), 1),
])
def test_invalid_arguments_rejected_before_launch(lib, kw, status):
    assert call(lib, **kw) == status


def test_valid_arguments_reach_the_device_check(lib):
    # Everything valid: the next step needs a CUDA device. Without one the call
    # reports a CUDA error (nothing is launched); with one it would launch.
    import torch
    if torch.cuda.is_available():
        pytest.skip("GPU present")
    assert call(lib) == 4
    assert call(lib, mask=2, window=10 ** 9) == 4     # window >= N is accepted (runs as causal)


def _items(B, Hq, Hkv, N, mask, window):
    """Work-item count of the schedule: two 128-row query tiles per item, paired
    as two heads of one KV group when Hq/Hkv is even, else two blocks of a head."""
    g = Hq // Hkv
    mb = -(-N // 128)
    if g % 2 == 0:
        return mb * B * Hq // 2
    return -(-mb // 2) * B * Hq


@pytest.mark.parametrize("shape", [(1, 2, 2, 256), (2, 32, 32, 8192), (1, 64, 8, 16384), (1, 32, 8, 131072),
                                   (1, 32, 32, 131072), (3, 6, 2, 1000), (1, 3, 1, 129), (1, 1, 1, 1)])
def test_work_item_count(lib, shape):
    B, Hq, Hkv, N = shape
    for mask, window in ((0, 0), (1, 0), (2, 4096)):
        assert lib.attn_fwd_num_work_items(B, Hq, Hkv, N, 128, mask, window) == _items(B, Hq, Hkv, N, mask, window)
    assert lib.attn_fwd_num_work_items(1, 2, 2, 64, 96, 1, 0) == -1
    assert lib.attn_fwd_num_work_items(1, 3, 2, 64, 64, 1, 0) == -1


def test_python_binding_validates_without_launching():
    import torch
    with pytest.raises((TypeError, ValueError)):
        A.fwd(torch.zeros(1, 1, 4, 64, dtype=torch.bfloat16), torch.zeros(1, 1, 4, 64, dtype=torch.bfloat16),
              torch.zeros(1, 1, 4, 64, dtype=torch.bfloat16))


# ------------------------------------------------------------------ backward
DO, DQ, DK, DV, WS = (0x10000000000 * (i + 6) for i in range(5))


def call_bwd(lib, q=Q, k=K, v=V, o=O, l=L, do=DO, dq=DQ, dk=DK, dv=DV, ws=WS, ws_bytes=None, B=1, Hq=2, Hkv=2,
             N=256, d=64, scale=0.125, mask=1, window=0):
    if ws_bytes is None:
        ws_bytes = 4 * B * Hq * N
    return lib.attn_bwd(q, k, v, o, l, do, dq, dk, dv, ws, ws_bytes, B, Hq, Hkv, N, d, scale, mask, window, None)


def test_backward_workspace_bytes(lib):
    rows = 2 * 32 * 8192
    assert lib.attn_bwd_workspace_bytes(2, 32, 8192) == 4 * rows + 4 * rows * 128   # D, then the dQ sums
    assert lib.attn_bwd_workspace_bytes(1, 1, 3) == 256 + 4 * 3 * 128                # the sums start 256-aligned
    assert lib.attn_bwd_workspace_bytes(0, 1, 1) == 0 and lib.attn_bwd_workspace_bytes(1, 1, -1) == 0
    assert lib.attn_bwd_workspace_bytes(1 << 30, 1 << 30, 1 << 30) == 0   # beyond 63 bits


@pytest.mark.parametrize("kw,status", [
    (dict(do=None), 1), (dict(dq=None), 1), (dict(dk=None), 1), (dict(dv=None), 1), (dict(ws=None), 1),
    (dict(o=None), 1), (dict(l=None), 1),
    (dict(ws_bytes=4 * 2 * 256 - 4), 1), (dict(B=0), 1), (dict(Hq=6, Hkv=4), 1), (dict(mask=7), 1),
    (dict(mask=2, window=0), 1), (dict(scale=0.0), 1), (dict(scale=float("nan")), 1),
    (dict(d=32), 2), (dict(d=256), 2),
    (dict(do=DO + 8), 3), (dict(dq=DQ + 8), 3), (dict(dk=DK + 4), 3), (dict(dv=DV + 2), 3), (dict(ws=WS + 2), 3),
    (dict(dq=Q), 1), (dict(dk=V + 64), 1), (dict(dv=DO), 1), (dict(ws=L), 1), (dict(dk=DQ + 128), 1),
    (dict(ws=DV + 256), 1),
    (dict(B=1 << 10, Hq=1 << 20, Hkv=1 << 20, N=1 << 30), 1),
])
def test_backward_invalid_arguments_rejected_before_launch(lib, kw, status):
    assert call_bwd(lib, **kw) == status


def test_backward_valid_arguments_reach_the_device_check(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("GPU present")
    assert call_bwd(lib) == 4
    ws = lib.attn_bwd_workspace_bytes(1, 2, 256)
    assert call_bwd(lib, d=128, mask=2, window=10 ** 9, ws_bytes=ws) == 4
    # d = 128 needs the dQ accumulator and a 16-byte aligned workspace
    assert call_bwd(lib, d=128, ws_bytes=ws - 4) == 1
    assert call_bwd(lib, d=128, ws_bytes=ws, ws=WS + 4) == 3


def test_backward_deterministic_option_needs_only_the_row_terms(lib):
    """attn_bwd_ex with bwd_deterministic takes d = 128 down the two-kernel path, whose
    workspace is D alone (4 B Hq N bytes, 4-byte aligned)."""
    import ctypes
    import torch
    if torch.cuda.is_available():
        pytest.skip("GPU present")
    opts = A.FwdOptions(0, 0, 0)
    opts.bwd_deterministic = 1

    def call(ws, ws_bytes, o):
        return lib.attn_bwd_ex(Q, K, V, O, L, DO, DQ, DK, DV, ws, ws_bytes, 1, 2, 2, 256, 128, 0.125, 1, 0, None,
                               ctypes.byref(o) if o is not None else None)
    assert call(WS + 4, 4 * 2 * 256, opts) == 4          # valid: reaches the device check
    assert call(WS + 4, 4 * 2 * 256, None) == 1          # the fused default needs the dQ sums too
    full = lib.attn_bwd_workspace_bytes(1, 2, 256)
    assert call(WS + 4, full, None) == 3                 # ... in a 16-byte aligned workspace
    assert call(WS, full, None) == 4
    assert call(WS, 4 * 2 * 256 - 4, opts) == 1
    # grouped heads take the two-kernel path by default: D alone suffices
    assert lib.attn_bwd_ex(Q, K, V, O, L, DO, DQ, DK, DV, WS + 4, 4 * 4 * 256, 1, 4, 2, 256, 128, 0.125, 1, 0, None,
                           None) == 4


# ------------------------------------------------------------------ decoding
KC, VC, BT, SL, DOUT, DLSE, DWS = (0x10000000000 * (i + 12) for i in range(7))


def call_dec(lib, q=Q, kc=KC, vc=VC, bt=BT, sl=SL, o=DOUT, l=DLSE, ws=DWS, ws_bytes=None, B=2, Hq=8, Hkv=2, Nq=1,
             d=128, num_pages=64, page_size=16, max_pages=32, splits=4, scale=0.088, mask=1, window=0):
    if ws_bytes is None:
        ws_bytes = lib.attn_decode_workspace_bytes(B, Hq, Nq, d, splits)
    return lib.attn_decode(q, kc, vc, bt, sl, o, l, ws, ws_bytes, B, Hq, Hkv, Nq, d, num_pages, page_size,
                           max_pages, splits, scale, mask, window, None)


def test_decode_workspace_bytes(lib):
    rows = 2 * 8 * 3
    assert lib.attn_decode_workspace_bytes(2, 8, 3, 128, 1) == 256          # the work counter only
    lse_part = -(-(rows * 5 * 4) // 256) * 256
    assert lib.attn_decode_workspace_bytes(2, 8, 3, 128, 5) == 256 + lse_part + rows * 5 * 128 * 4
    assert lib.attn_decode_workspace_bytes(2, 8, 3, 96, 5) == 0
    assert lib.attn_decode_workspace_bytes(0, 8, 3, 64, 5) == 0
    assert lib.attn_decode_workspace_bytes(1, 8, 3, 64, 0) == 0


def test_decode_num_splits_without_a_device(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("GPU present: the count depends on its SM count")
    # 148 SMs assumed: one wave of items for small batches, else splits of at most 64 tiles;
    # never fewer than 4 tiles per split
    assert lib.attn_decode_num_splits(1, 64, 8, 1, 131072, 1, 0) == 148 // 8
    assert lib.attn_decode_num_splits(32, 32, 8, 1, 131072, 1, 0) == -(-(1024 + 1) // 64)
    assert lib.attn_decode_num_splits(16, 32, 32, 1, 31004, 1, 0) == 4      # 244 tiles
    assert lib.attn_decode_num_splits(1, 64, 8, 1, 1000, 1, 0) == 2         # (8 + 1) // 4 tiles limit
    assert lib.attn_decode_num_splits(32, 32, 8, 1, 131072, 2, 4096) == 1   # 33-tile windows
    assert lib.attn_decode_num_splits(1, 32, 8, 1, 131072, 2, 4096) == (4096 // 128 + 1) // 4
    assert lib.attn_decode_num_splits(8, 64, 8, 4, 31818, 1, 0) == 148 // 64          # one wave
    assert lib.attn_decode_num_splits(1, 64, 8, 1, 0, 1, 0) == -1
    assert lib.attn_decode_num_splits(1, 6, 4, 1, 100, 1, 0) == -1


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), 1), (dict(kc=None), 1), (dict(vc=None), 1), (dict(bt=None), 1), (dict(sl=None), 1),
    (dict(o=None), 1), (dict(l=None), 1), (dict(ws=None), 1), (dict(ws_bytes=16), 1),
    (dict(splits=1, ws=None), 1), (dict(splits=1, ws_bytes=128), 1),
    (dict(B=0), 1), (dict(Hq=6, Hkv=4), 1), (dict(Nq=0), 1), (dict(num_pages=0), 1), (dict(max_pages=0), 1),
    (dict(splits=0), 1), (dict(splits=5000), 1), (dict(mask=3), 1), (dict(mask=2, window=0), 1),
    (dict(scale=0.0), 1), (dict(scale=float("nan")), 1),
    (dict(d=96), 2), (dict(page_size=8), 2), (dict(page_size=48), 2), (dict(page_size=512), 2),
    (dict(q=Q + 8), 3), (dict(kc=KC + 8), 3), (dict(vc=VC + 4), 3), (dict(o=DOUT + 2), 3), (dict(l=DLSE + 2), 3),
    (dict(bt=BT + 2), 3), (dict(sl=SL + 1), 3), (dict(ws=DWS + 4), 3),
    (dict(o=Q), 1), (dict(l=KC + 64), 1), (dict(ws=BT), 1), (dict(o=SL), 1), (dict(l=DOUT + 256), 1),
    (dict(ws=DLSE), 1),
])
def test_decode_invalid_arguments_rejected_before_launch(lib, kw, status):
    assert call_dec(lib, **kw) == status


def test_decode_valid_arguments_reach_the_device_check(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("GPU present")
    assert call_dec(lib) == 4
    assert call_dec(lib, splits=1) == 4                          # one split: the counter only
    assert call_dec(lib, Nq=40, d=64, page_size=256, mask=2, window=5) == 4


# ------------------------------------------------------------------ FP8 forward
def call_fp8(lib, q=Q, k=K, v=V, o=O, l=L, sq=0.01, sk=0.02, sv=0.03, B=1, Hq=2, Hkv=2, N=256, d=128, scale=0.088,
             mask=1, window=0):
    return lib.attn_fwd_fp8(q, k, v, sq, sk, sv, o, l, B, Hq, Hkv, N, d, scale, mask, window, None)


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), 1), (dict(v=None), 1), (dict(o=None), 1), (dict(sq=0.0), 1), (dict(sk=-1.0), 1),
    (dict(sv=float("inf")), 1), (dict(scale=float("nan")), 1), (dict(Hq=3, Hkv=2), 1), (dict(mask=5), 1),
    (dict(d=64), 2), (dict(d=96), 2), (dict(q=Q + 8), 3), (dict(l=L + 1), 3), (dict(o=K), 1),
])
def test_fp8_invalid_arguments_rejected_before_launch(lib, kw, status):
    assert call_fp8(lib, **kw) == status


def test_fp8_valid_arguments_reach_the_device_check(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("GPU present")
    assert call_fp8(lib) == 4
    assert call_fp8(lib, mask=2, window=7) == 4


# ------------------------------------------------------------------ partial-result merge
A1, A2, P1, P2, MO = (0x10000000000 * (i + 20) for i in range(5))


def call_merge(lib, acc=A1, accl=A2, part=P1, partl=P2, out=MO, rows=100, d=128, mode=1):
    return lib.attn_merge(acc, accl, part, partl, out, rows, d, mode, None)


@pytest.mark.parametrize("kw,status", [
    (dict(acc=None), 1), (dict(accl=None), 1), (dict(part=None), 1), (dict(partl=None), 1),
    (dict(rows=0), 1), (dict(mode=4), 1), (dict(mode=-1), 1), (dict(d=96), 2),
    (dict(mode=3, part=P1 + 8), 3),                     # fp32 partials need 16-byte alignment
    (dict(mode=3, out=P1), 1), (dict(mode=2, out=P1 + 256), 1),  # a bf16 out may not alias fp32 partials
    (dict(acc=A1 + 8), 3), (dict(part=P1 + 4), 3), (dict(out=MO + 2), 3), (dict(accl=A2 + 2), 3),
    (dict(accl=A1 + 64), 1), (dict(part=A1), 1), (dict(out=A2), 1), (dict(out=P2), 1),
])
def test_merge_invalid_arguments_rejected_before_launch(lib, kw, status):
    assert call_merge(lib, **kw) == status


def test_merge_valid_arguments_reach_the_launch(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("GPU present")
    assert call_merge(lib) == 4          # no device: the launch fails
    assert call_merge(lib, out=None, mode=0) == 4
    assert call_merge(lib, out=P1) == 4  # out may alias the partial
    assert call_merge(lib, mode=3) == 4 and call_merge(lib, mode=2, out=None) == 4   # fp32 partials


# ------------------------------------------------------------------ host-buffer forward
HQ, HK, HV, HO, HL = (0x10000000000 * (i + 40) for i in range(5))


def call_host(lib, hq=HQ, hk=HK, hv=HV, ho=HO, hl=HL, q=Q, k=K, v=V, o=O, l=L, B=2, Hq=4, Hkv=2, N=256, d=64,
              scale=0.125, mask=1, window=0, chunks=0, fp8=False, sq=0.01, sk=0.02, sv=0.03):
    if fp8:
        return lib.attn_fwd_fp8_host(hq, hk, hv, sq, sk, sv, ho, hl, q, k, v, o, l, B, Hq, Hkv, N, d, scale, mask,
                                     window, chunks, None)
    return lib.attn_fwd_host(hq, hk, hv, ho, hl, q, k, v, o, l, B, Hq, Hkv, N, d, scale, mask, window, chunks, None)


@pytest.mark.parametrize("kw,status", [
    (dict(hq=None), 1), (dict(hv=None), 1), (dict(ho=None), 1), (dict(hl=None), 1), (dict(q=None), 1),
    (dict(l=None), 1), (dict(B=0), 1), (dict(Hq=3), 1), (dict(mask=4), 1), (dict(mask=2, window=0), 1),
    (dict(scale=0.0), 1), (dict(chunks=-1), 1), (dict(d=96), 2),
    (dict(q=Q + 8), 3), (dict(o=O + 4), 3), (dict(l=L + 2), 3),
    (dict(o=K), 1), (dict(l=O + 64), 1),                        # device outputs overlap
    (dict(ho=HQ + 1024), 1), (dict(hl=HO + 4096), 1), (dict(hl=HV), 1),   # host outputs overlap
    (dict(fp8=True, d=64), 2), (dict(fp8=True, d=128, sq=0.0), 1), (dict(fp8=True, d=128, sv=float("nan")), 1),
    (dict(k=V), 1), (dict(v=K), 1), (dict(k=Q + 1024), 1),       # device staging inputs overlap
])
def test_host_forward_invalid_arguments_rejected_before_enqueueing(lib, kw, status):
    assert call_host(lib, **kw) == status


def test_host_forward_valid_arguments_reach_the_device(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("GPU present")
    assert call_host(lib) == 4                       # no device: the copy streams cannot be made
    assert call_host(lib, hq=HQ + 3, ho=HO + 2) == 4  # host buffers need no alignment
    assert call_host(lib, chunks=100) == 4
    assert call_host(lib, fp8=True, d=128) == 4


def test_host_binding_validates_before_touching_a_device():
    import torch
    bf = dict(dtype=torch.bfloat16)
    q, k = torch.zeros(1, 4, 8, 64, **bf), torch.zeros(1, 2, 8, 64, **bf)
    with pytest.raises(ValueError):                       # v shaped unlike k
        A.fwd_host(q, k, torch.zeros(1, 2, 9, 64, **bf))
    with pytest.raises(ValueError):                       # wrong dtype
        A.fwd_host(q.float(), k, k)
    with pytest.raises(ValueError):                       # not contiguous
        A.fwd_host(q.transpose(2, 3), k, k)
    with pytest.raises(ValueError):                       # unknown mask
        A.fwd_host(q, k, k, mask="banded")
    with pytest.raises(ValueError):                       # outputs of the wrong shape
        A.fwd_host(q, k, k, out=torch.zeros(1, 4, 8, 32, **bf))
    with pytest.raises(ValueError):                       # FP8 codes must be uint8 / float8_e4m3fn
        A.fwd_fp8_host(q, k, k, 1.0, 1.0, 1.0)


def test_host_forward_rejects_sizes_beyond_any_memory(lib):
    # 2^30 rows of 2^20 heads x 128: far beyond any memory; refused before any product overflows
    assert call_host(lib, B=1, Hq=1 << 20, Hkv=1 << 20, N=1 << 30, d=128) == 1
