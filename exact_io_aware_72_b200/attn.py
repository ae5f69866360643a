"""Python binding of the C ABI in include/attn.h (argument marshalling only).

Every step of the forward runs in the sm_100a kernels of ``libattn_b200.so``;
PyTorch only provides device memory and the current stream.  There is no
fallback: if the library is missing or a call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Tuple

import torch

MASKS = {"full": 0, "causal": 1, "sliding_window": 2}
STATUS = {0: "ATTN_OK", 1: "ATTN_ERR_INVALID_ARG", 2: "ATTN_ERR_UNSUPPORTED", 3: "ATTN_ERR_MISALIGNED",
          4: "ATTN_ERR_CUDA", 5: "ATTN_ERR_TIMEOUT", 6: "ATTN_ERR_RANGE"}
ATTN_ERR_TIMEOUT = 5
ATTN_ERR_RANGE = 6
LIB_NAME = "libattn_b200.so"
EXPORTS = ("attn_fwd", "attn_fwd_ex", "attn_status_string", "attn_debug_error", "attn_fwd_num_work_items",
           "attn_bwd", "attn_bwd_ex", "attn_bwd_workspace_bytes", "attn_bwd_debug_error",
           "attn_decode", "attn_decode_ex", "attn_decode_workspace_bytes", "attn_decode_num_splits",
           "attn_decode_debug_error", "attn_fwd_fp8", "attn_fwd_fp8_ex", "attn_merge", "attn_fwd_host",
           "attn_fwd_fp8_host", "attn_decode_static")

_lib = None


class AttnError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {STATUS.get(status, status)}")
        self.status = status


class FwdOptions(ctypes.Structure):
    """attn_fwd_options of include/attn.h."""
    _fields_ = [("wait_timeout_ns", ctypes.c_uint64), ("inject_stall", ctypes.c_int),
                ("grid_ctas", ctypes.c_int), ("item_visits", ctypes.c_void_p), ("p_bf16", ctypes.c_int),
                ("out_fp32", ctypes.c_int), ("key_offset", ctypes.c_int64), ("bwd_deterministic", ctypes.c_int)]


def lib_path() -> str:
    return os.path.join(os.path.dirname(os.path.abspath(__file__)), LIB_NAME)


def load_library():
    """Load libattn_b200.so (built in-tree); raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    path = lib_path()
    if not os.path.exists(path):
        raise RuntimeError(f"{LIB_NAME} is not built; run `python -m exact_io_aware_72_b200.build`")
    lib = ctypes.CDLL(path)
    vp, i64 = ctypes.c_void_p, ctypes.c_int64
    fwd_args = [vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, ctypes.c_float, ctypes.c_int, i64, vp]
    lib.attn_fwd.argtypes = fwd_args
    lib.attn_fwd.restype = ctypes.c_int
    lib.attn_fwd_ex.argtypes = fwd_args + [ctypes.POINTER(FwdOptions)]
    lib.attn_fwd_ex.restype = ctypes.c_int
    f32 = ctypes.c_float
    fp8_args = [vp, vp, vp, f32, f32, f32, vp, vp, i64, i64, i64, i64, i64, f32, ctypes.c_int, i64, vp]
    lib.attn_fwd_fp8.argtypes = fp8_args
    lib.attn_fwd_fp8.restype = ctypes.c_int
    lib.attn_fwd_fp8_ex.argtypes = fp8_args + [ctypes.POINTER(FwdOptions)]
    lib.attn_fwd_fp8_ex.restype = ctypes.c_int
    lib.attn_status_string.argtypes = [ctypes.c_int]
    lib.attn_status_string.restype = ctypes.c_char_p
    lib.attn_debug_error.argtypes = [vp, ctypes.POINTER(ctypes.c_int)]
    lib.attn_debug_error.restype = ctypes.c_int
    lib.attn_fwd_num_work_items.argtypes = [i64, i64, i64, i64, i64, ctypes.c_int, i64]
    lib.attn_fwd_num_work_items.restype = i64
    bwd_args = [vp] * 10 + [ctypes.c_size_t, i64, i64, i64, i64, i64, ctypes.c_float, ctypes.c_int, i64, vp]
    lib.attn_bwd.argtypes = bwd_args
    lib.attn_bwd.restype = ctypes.c_int
    lib.attn_bwd_ex.argtypes = bwd_args + [ctypes.POINTER(FwdOptions)]
    lib.attn_bwd_ex.restype = ctypes.c_int
    lib.attn_bwd_workspace_bytes.argtypes = [i64, i64, i64]
    lib.attn_bwd_workspace_bytes.restype = ctypes.c_size_t
    lib.attn_bwd_debug_error.argtypes = [vp, ctypes.POINTER(ctypes.c_int)]
    lib.attn_bwd_debug_error.restype = ctypes.c_int
    dec_args = [vp] * 8 + [ctypes.c_size_t] + [i64] * 9 + [ctypes.c_float, ctypes.c_int, i64, vp]
    lib.attn_decode.argtypes = dec_args
    lib.attn_decode.restype = ctypes.c_int
    lib.attn_decode_ex.argtypes = dec_args + [ctypes.POINTER(FwdOptions)]
    lib.attn_decode_ex.restype = ctypes.c_int
    lib.attn_decode_workspace_bytes.argtypes = [i64, i64, i64, i64, i64]
    lib.attn_decode_workspace_bytes.restype = ctypes.c_size_t
    lib.attn_decode_num_splits.argtypes = [i64, i64, i64, i64, i64, ctypes.c_int, i64]
    lib.attn_decode_num_splits.restype = i64
    lib.attn_decode_debug_error.argtypes = [vp, ctypes.POINTER(ctypes.c_int)]
    lib.attn_decode_debug_error.restype = ctypes.c_int
    lib.attn_decode_static.argtypes = [vp] * 7 + [i64] * 9 + [ctypes.c_float, ctypes.c_int, i64, vp]
    lib.attn_decode_static.restype = ctypes.c_int
    host_tail = [vp] * 7 + [i64] * 5 + [f32, ctypes.c_int, i64, i64, vp]
    lib.attn_fwd_host.argtypes = [vp, vp, vp] + host_tail
    lib.attn_fwd_host.restype = ctypes.c_int
    lib.attn_fwd_fp8_host.argtypes = [vp, vp, vp, f32, f32, f32] + host_tail
    lib.attn_fwd_fp8_host.restype = ctypes.c_int
    lib.attn_merge.argtypes = [vp, vp, vp, vp, vp, i64, i64, ctypes.c_int, vp]
    lib.attn_merge.restype = ctypes.c_int
    _lib = lib
    return lib


def _check(t: torch.Tensor, name: str, dtype, ndim):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype or t.dim() != ndim or not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA {dtype} tensor with {ndim} dims")


def fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, scale: Optional[float] = None,
        mask: str = "causal", window: Optional[int] = None, out: Optional[torch.Tensor] = None,
        lse: Optional[torch.Tensor] = None, stream: Optional[torch.cuda.Stream] = None,
        wait_timeout_ns: int = 0, inject_stall: bool = False, grid_ctas: int = 0, p_bf16: bool = False,
        item_visits: Optional[torch.Tensor] = None, out_fp32: bool = False, key_offset: int = 0
        ) -> Tuple[torch.Tensor, torch.Tensor]:
    """Exact attention forward: returns (out bf16 [B,Hq,N,d], lse fp32 [B,Hq,N]).

    q: [B,Hq,N,d], k/v: [B,Hkv,N,d], bf16, contiguous, on one CUDA device.
    ``mask`` is "full", "causal" or "sliding_window" (keys i-window < j <= i).
    The launch is asynchronous on ``stream`` (default: the current stream).
    ``p_bf16`` selects bf16 P for V values beyond the fp16 range (see
    include/attn.h); ``item_visits`` (int32 CUDA tensor of num_work_items
    counters) is a test hook counting each work item's visits; ``out_fp32``
    returns out in fp32, unrounded (partial results to merge); ``key_offset``
    places query row i at key position i + key_offset (causal and window masks).
    """
    lib = load_library()
    _check(q, "q", torch.bfloat16, 4)
    _check(k, "k", torch.bfloat16, 4)
    _check(v, "v", torch.bfloat16, 4)
    B, Hq, N, d = q.shape
    Bk, Hkv, Nk, dk = k.shape
    if (Bk, Nk, dk) != (B, N, d) or tuple(v.shape) != tuple(k.shape):
        raise ValueError("q, k, v shapes disagree")
    if mask not in MASKS:
        raise ValueError(f"mask must be one of {sorted(MASKS)}")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out_dtype = torch.float32 if out_fp32 else torch.bfloat16
    if out is None:
        out = torch.empty(q.shape, dtype=out_dtype, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device)
    _check(out, "out", out_dtype, 4)
    _check(lse, "lse", torch.float32, 3)
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    visits = None
    if item_visits is not None:
        if not (item_visits.is_cuda and item_visits.dtype == torch.int32 and item_visits.is_contiguous()):
            raise ValueError("item_visits must be a contiguous int32 CUDA tensor")
        visits = item_visits.data_ptr()
    opts = FwdOptions(int(wait_timeout_ns), 1 if inject_stall else 0, int(grid_ctas), visits, 1 if p_bf16 else 0,
                      1 if out_fp32 else 0, int(key_offset))
    with torch.cuda.device(q.device):
        st = lib.attn_fwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                             B, Hq, Hkv, N, d, float(scale), MASKS[mask],
                             int(window) if window is not None else 0, ctypes.c_void_p(stream.cuda_stream),
                             ctypes.byref(opts))
    if st != 0:
        raise AttnError(st, "attn_fwd")
    return out, lse


def _codes(t: torch.Tensor, name: str) -> torch.Tensor:
    if isinstance(t, torch.Tensor) and t.dtype == torch.float8_e4m3fn:
        t = t.view(torch.uint8)
    _check(t, name, torch.uint8, 4)
    return t


def fwd_fp8(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, q_scale: float, k_scale: float, v_scale: float,
            scale: Optional[float] = None, mask: str = "causal", window: Optional[int] = None,
            out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
            stream: Optional[torch.cuda.Stream] = None, wait_timeout_ns: int = 0, grid_ctas: int = 0
            ) -> Tuple[torch.Tensor, torch.Tensor]:
    """Exact attention forward of E4M3 inputs: q, k, v hold E4M3 codes (uint8 or
    torch.float8_e4m3fn, [B,H,N,128]) whose values are code * q_scale (k_scale,
    v_scale); returns (out bf16 [B,Hq,N,128], lse fp32 [B,Hq,N])."""
    lib = load_library()
    q, k, v = _codes(q, "q"), _codes(k, "k"), _codes(v, "v")
    B, Hq, N, d = q.shape
    Bk, Hkv, Nk, dk = k.shape
    if (Bk, Nk, dk) != (B, N, d) or tuple(v.shape) != tuple(k.shape):
        raise ValueError("q, k, v shapes disagree")
    if mask not in MASKS:
        raise ValueError(f"mask must be one of {sorted(MASKS)}")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((B, Hq, N, d), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device)
    _check(out, "out", torch.bfloat16, 4)
    _check(lse, "lse", torch.float32, 3)
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    opts = FwdOptions(int(wait_timeout_ns), 0, int(grid_ctas))
    with torch.cuda.device(q.device):
        st = lib.attn_fwd_fp8_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), float(q_scale), float(k_scale),
                                 float(v_scale), out.data_ptr(), lse.data_ptr(), B, Hq, Hkv, N, d, float(scale),
                                 MASKS[mask], int(window) if window is not None else 0,
                                 ctypes.c_void_p(stream.cuda_stream), ctypes.byref(opts))
    if st != 0:
        raise AttnError(st, "attn_fwd_fp8")
    return out, lse


def bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: torch.Tensor, lse: torch.Tensor,
        dout: torch.Tensor, scale: Optional[float] = None, mask: str = "causal", window: Optional[int] = None,
        dq: Optional[torch.Tensor] = None, dk: Optional[torch.Tensor] = None, dv: Optional[torch.Tensor] = None,
        workspace: Optional[torch.Tensor] = None, stream: Optional[torch.cuda.Stream] = None,
        wait_timeout_ns: int = 0, grid_ctas: int = 0,
        deterministic: bool = False) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Exact attention backward: returns (dq, dk, dv), the gradients of
    sum(dout * out) for the forward's q, k, v (same scale / mask / window).

    ``out`` and ``lse`` are the forward's outputs for these inputs. The fp32
    workspace (allocated here when not given) holds the row terms
    D = rowsum(dout * out) and, on the fused path (d = 128, Hq == Hkv), the fp32
    sums of dq: ``attn_bwd_workspace_bytes(B, Hq, N)`` bytes there, B*Hq*N floats
    otherwise.  ``deterministic`` takes the two-kernel path there too (dq bitwise
    reproducible; seven matmuls per pair instead of five).
    """
    lib = load_library()
    for t, name in ((q, "q"), (k, "k"), (v, "v"), (out, "out"), (dout, "dout")):
        _check(t, name, torch.bfloat16, 4)
    _check(lse, "lse", torch.float32, 3)
    B, Hq, N, d = q.shape
    Bk, Hkv, Nk, dk_ = k.shape
    if (Bk, Nk, dk_) != (B, N, d) or tuple(v.shape) != tuple(k.shape) or out.shape != q.shape \
            or dout.shape != q.shape or tuple(lse.shape) != (B, Hq, N):
        raise ValueError("q, k, v, out, lse, dout shapes disagree")
    if mask not in MASKS:
        raise ValueError(f"mask must be one of {sorted(MASKS)}")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    for t, name, ref in ((dq, "dq", q), (dk, "dk", k), (dv, "dv", v)):
        _check(t, name, torch.bfloat16, 4)
        if t.shape != ref.shape:
            raise ValueError(f"{name} has the wrong shape")
    fused = d == 128 and Hq == Hkv and not deterministic  # the library's choice of path
    ws_bytes = int(lib.attn_bwd_workspace_bytes(B, Hq, N)) if fused else 4 * B * Hq * N
    if workspace is None:
        workspace = torch.empty(ws_bytes // 4, dtype=torch.float32, device=q.device)
    if not (workspace.is_cuda and workspace.is_contiguous()):
        raise ValueError("workspace must be a contiguous CUDA tensor")
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    opts = FwdOptions(int(wait_timeout_ns), 0, int(grid_ctas))
    opts.bwd_deterministic = int(bool(deterministic))
    with torch.cuda.device(q.device):
        st = lib.attn_bwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                             dout.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), workspace.data_ptr(),
                             workspace.numel() * workspace.element_size(), B, Hq, Hkv, N, d, float(scale),
                             MASKS[mask], int(window) if window is not None else 0,
                             ctypes.c_void_p(stream.cuda_stream), ctypes.byref(opts))
    if st != 0:
        raise AttnError(st, "attn_bwd")
    return dq, dk, dv


def bwd_debug_error(stream: Optional[torch.cuda.Stream] = None, device=None) -> Tuple[int, int]:
    """Synchronise and read/clear the backward kernels' error word: (status, raw code)."""
    lib = load_library()
    if stream is None:
        stream = torch.cuda.current_stream(device)
    code = ctypes.c_int(0)
    with torch.cuda.device(stream.device):
        st = lib.attn_bwd_debug_error(ctypes.c_void_p(stream.cuda_stream), ctypes.byref(code))
    return st, code.value


def decode_num_splits(B, Hq, Hkv, Nq, max_seq_len, mask="causal", window=None) -> int:
    """Suggested split count for a decoding step (host-only; see include/attn.h)."""
    n = int(load_library().attn_decode_num_splits(B, Hq, Hkv, Nq, int(max_seq_len), MASKS[mask],
                                                   int(window) if window is not None else 0))
    if n < 1:
        raise ValueError("invalid decoding sizes")
    return n


def decode_workspace_bytes(B, Hq, Nq, d, num_splits) -> int:
    return int(load_library().attn_decode_workspace_bytes(B, Hq, Nq, d, int(num_splits)))


def decode(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, block_table: torch.Tensor,
           seq_lens: torch.Tensor, max_seq_len: Optional[int] = None, scale: Optional[float] = None,
           mask: str = "causal", window: Optional[int] = None, num_splits: Optional[int] = None,
           out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
           workspace: Optional[torch.Tensor] = None, stream: Optional[torch.cuda.Stream] = None,
           wait_timeout_ns: int = 0, grid_ctas: int = 0) -> Tuple[torch.Tensor, torch.Tensor]:
    """One decoding step against a paged KV cache: returns (out bf16 [B,Hq,Nq,d],
    lse fp32 [B,Hq,Nq]).

    q: [B,Hq,Nq,d] bf16 (the new tokens, the last Nq positions of each
    sequence); k_cache/v_cache: [num_pages,Hkv,page_size,d] bf16;
    block_table: [B,max_pages] int32; seq_lens: [B] int32 cached positions per
    sequence (new tokens included).  ``max_seq_len`` (a host-side upper bound
    of seq_lens, default max_pages*page_size) only picks the default
    ``num_splits``.  The workspace (work counter and the splits' partial
    results) is allocated here, zero-filled, when not given; a caller's own
    workspace must start zeroed and is left with its counter at zero.
    """
    lib = load_library()
    _check(q, "q", torch.bfloat16, 4)
    _check(k_cache, "k_cache", torch.bfloat16, 4)
    _check(v_cache, "v_cache", torch.bfloat16, 4)
    _check(block_table, "block_table", torch.int32, 2)
    _check(seq_lens, "seq_lens", torch.int32, 1)
    B, Hq, Nq, d = q.shape
    num_pages, Hkv, page_size, dk = k_cache.shape
    if dk != d or tuple(v_cache.shape) != tuple(k_cache.shape) or block_table.shape[0] != B \
            or seq_lens.shape[0] != B:
        raise ValueError("q, cache, block_table and seq_lens shapes disagree")
    if mask not in MASKS:
        raise ValueError(f"mask must be one of {sorted(MASKS)}")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    max_pages = block_table.shape[1]
    if max_seq_len is None:
        max_seq_len = max_pages * page_size
    if num_splits is None:
        num_splits = decode_num_splits(B, Hq, Hkv, Nq, max_seq_len, mask, window)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    _check(out, "out", torch.bfloat16, 4)
    _check(lse, "lse", torch.float32, 3)
    ws_bytes = decode_workspace_bytes(B, Hq, Nq, d, num_splits)
    if workspace is None:
        # zero-filled: its first 256 bytes are the work counter, which each call leaves at zero
        workspace = torch.zeros(ws_bytes // 4, dtype=torch.float32, device=q.device)
    if not (workspace.is_cuda and workspace.is_contiguous()):
        raise ValueError("workspace must be a contiguous CUDA tensor")
    ws_ptr, ws_len = workspace.data_ptr(), workspace.numel() * workspace.element_size()
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    opts = FwdOptions(int(wait_timeout_ns), 0, int(grid_ctas), None, 0, 0, 0)
    with torch.cuda.device(q.device):
        st = lib.attn_decode_ex(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), block_table.data_ptr(),
                                seq_lens.data_ptr(), out.data_ptr(), lse.data_ptr(), ws_ptr, ws_len,
                                B, Hq, Hkv, Nq, d, num_pages, page_size, max_pages, int(num_splits),
                                float(scale), MASKS[mask], int(window) if window is not None else 0,
                                ctypes.c_void_p(stream.cuda_stream), ctypes.byref(opts))
    if st != 0:
        raise AttnError(st, "attn_decode")
    return out, lse


# Bytes of the library's own scratch array used by attn_decode_static (include/attn.h).
DECODE_STATIC_SCRATCH_BYTES = 8 * 1024 * 1024


def decode_static(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, block_table: torch.Tensor,
                  seq_lens: torch.Tensor, out: torch.Tensor, lse: torch.Tensor, num_splits: int,
                  scale: Optional[float] = None, mask: str = "causal", window: Optional[int] = None,
                  stream: Optional[torch.cuda.Stream] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """``decode`` through ``attn_decode_static``: the library's fixed scratch array
    instead of a workspace, for callers that hand over only their inputs and
    outputs and cannot allocate device memory.  Nothing is allocated here either:
    ``out`` (bf16 [B,Hq,Nq,d]) and ``lse`` (fp32 [B,Hq,Nq]) are the caller's, and
    ``num_splits`` is explicit (it decides the scratch size, at most
    DECODE_STATIC_SCRATCH_BYTES).  Calls that overlap on the GPU share the array
    and race; keep them on one stream."""
    lib = load_library()
    for t, name, dt, nd in ((q, "q", torch.bfloat16, 4), (k_cache, "k_cache", torch.bfloat16, 4),
                            (v_cache, "v_cache", torch.bfloat16, 4), (block_table, "block_table", torch.int32, 2),
                            (seq_lens, "seq_lens", torch.int32, 1), (out, "out", torch.bfloat16, 4),
                            (lse, "lse", torch.float32, 3)):
        _check(t, name, dt, nd)
    B, Hq, Nq, d = q.shape
    num_pages, Hkv, page_size, dk = k_cache.shape
    if dk != d or tuple(v_cache.shape) != tuple(k_cache.shape) or block_table.shape[0] != B \
            or seq_lens.shape[0] != B or tuple(out.shape) != tuple(q.shape) or tuple(lse.shape) != (B, Hq, Nq):
        raise ValueError("q, cache, block_table, seq_lens, out and lse shapes disagree")
    if mask not in MASKS:
        raise ValueError(f"mask must be one of {sorted(MASKS)}")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    with torch.cuda.device(q.device):
        st = lib.attn_decode_static(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), block_table.data_ptr(),
                                    seq_lens.data_ptr(), out.data_ptr(), lse.data_ptr(), B, Hq, Hkv, Nq, d,
                                    num_pages, page_size, block_table.shape[1], int(num_splits), float(scale),
                                    MASKS[mask], int(window) if window is not None else 0,
                                    ctypes.c_void_p(stream.cuda_stream))
    if st != 0:
        raise AttnError(st, "attn_decode_static")
    return out, lse


def merge(acc_out: torch.Tensor, acc_lse: torch.Tensor, part_out: torch.Tensor, part_lse: torch.Tensor,
          first: bool = False, out: Optional[torch.Tensor] = None, stream: Optional[torch.cuda.Stream] = None):
    """Fold a partial attention result (out bf16 or fp32, lse fp32 of one block of
    keys) into an fp32 accumulator in place (``first``: set it instead); when
    ``out`` (bf16) is given the merged rows are also written there."""
    lib = load_library()
    if not (acc_out.dtype == torch.float32 and acc_lse.dtype == torch.float32 and
            part_out.dtype in (torch.bfloat16, torch.float32) and part_lse.dtype == torch.float32):
        raise ValueError("merge: acc fp32, part_out bf16 or fp32, lse fp32")
    for t, name in ((acc_out, "acc_out"), (acc_lse, "acc_lse"), (part_out, "part_out"), (part_lse, "part_lse")):
        if not (t.is_cuda and t.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
    d = acc_out.shape[-1]
    rows = acc_out.numel() // d
    if part_out.numel() != rows * d or acc_lse.numel() != rows or part_lse.numel() != rows:
        raise ValueError("merge: shapes disagree")
    if out is not None and (out.dtype != torch.bfloat16 or not out.is_contiguous() or out.numel() != rows * d):
        raise ValueError("merge: out must be a contiguous bf16 tensor of the partial's size")
    if stream is None:
        stream = torch.cuda.current_stream(acc_out.device)
    with torch.cuda.device(acc_out.device):
        st = lib.attn_merge(acc_out.data_ptr(), acc_lse.data_ptr(), part_out.data_ptr(), part_lse.data_ptr(),
                            out.data_ptr() if out is not None else None, rows, d,
                            (0 if first else 1) | (2 if part_out.dtype == torch.float32 else 0),
                            ctypes.c_void_p(stream.cuda_stream))
    if st != 0:
        raise AttnError(st, "attn_merge")


def decode_debug_error(stream: Optional[torch.cuda.Stream] = None, device=None) -> Tuple[int, int]:
    """Synchronise and read/clear the decoding kernel's error word: (status, raw code)."""
    lib = load_library()
    if stream is None:
        stream = torch.cuda.current_stream(device)
    code = ctypes.c_int(0)
    with torch.cuda.device(stream.device):
        st = lib.attn_decode_debug_error(ctypes.c_void_p(stream.cuda_stream), ctypes.byref(code))
    return st, code.value


def debug_error(stream: Optional[torch.cuda.Stream] = None, device=None) -> Tuple[int, int]:
    """Synchronise and read/clear the device error word: (status, raw code)."""
    lib = load_library()
    if stream is None:
        stream = torch.cuda.current_stream(device)
    code = ctypes.c_int(0)
    with torch.cuda.device(stream.device):
        st = lib.attn_debug_error(ctypes.c_void_p(stream.cuda_stream), ctypes.byref(code))
    return st, code.value


def _host_tensor(t, name: str, dtype) -> torch.Tensor:
    if isinstance(t, torch.Tensor) and t.dtype == torch.float8_e4m3fn and dtype == torch.uint8:
        t = t.view(torch.uint8)
    if not isinstance(t, torch.Tensor) or t.dtype != dtype or t.dim() != 4 or t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous host {dtype} tensor with 4 dims")
    return t


def _fwd_host(fp8: bool, q, k, v, q_scale, k_scale, v_scale, scale, mask, window, chunks, device, out, lse,
              staging, stream):
    lib = load_library()
    dt = torch.uint8 if fp8 else torch.bfloat16
    q, k, v = _host_tensor(q, "q", dt), _host_tensor(k, "k", dt), _host_tensor(v, "v", dt)
    B, Hq, N, d = q.shape
    Bk, Hkv, Nk, dk = k.shape
    if (Bk, Nk, dk) != (B, N, d) or tuple(v.shape) != tuple(k.shape):
        raise ValueError("q, k, v shapes disagree")
    if mask not in MASKS:
        raise ValueError(f"mask must be one of {sorted(MASKS)}")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    pin = q.is_pinned()
    if out is None:
        out = torch.empty((B, Hq, N, d), dtype=torch.bfloat16, pin_memory=pin)
    if lse is None:
        lse = torch.empty((B, Hq, N), dtype=torch.float32, pin_memory=pin)
    if out.is_cuda or lse.is_cuda or out.dtype != torch.bfloat16 or lse.dtype != torch.float32 or \
            tuple(out.shape) != (B, Hq, N, d) or tuple(lse.shape) != (B, Hq, N) or \
            not out.is_contiguous() or not lse.is_contiguous():
        raise ValueError("out and lse must be contiguous host tensors: bf16 [B,Hq,N,d] and fp32 [B,Hq,N]")
    device = torch.device(device)
    if staging is None:
        staging = (torch.empty(q.shape, dtype=dt, device=device), torch.empty(k.shape, dtype=dt, device=device),
                   torch.empty(k.shape, dtype=dt, device=device),
                   torch.empty(out.shape, dtype=torch.bfloat16, device=device),
                   torch.empty(lse.shape, dtype=torch.float32, device=device))
    sq, sk, sv, so, sl = staging
    for t, ref, name in ((sq, q, "q"), (sk, k, "k"), (sv, v, "v"), (so, out, "out"), (sl, lse, "lse")):
        if not t.is_cuda or t.dtype != ref.dtype or tuple(t.shape) != tuple(ref.shape) or not t.is_contiguous():
            raise ValueError(f"staging buffer for {name} must be a contiguous CUDA tensor like it")
    if stream is None:
        stream = torch.cuda.current_stream(sq.device)
    common = (out.data_ptr(), lse.data_ptr(), sq.data_ptr(), sk.data_ptr(), sv.data_ptr(), so.data_ptr(),
              sl.data_ptr(), B, Hq, Hkv, N, d, float(scale), MASKS[mask],
              int(window) if window is not None else 0, int(chunks), ctypes.c_void_p(stream.cuda_stream))
    with torch.cuda.device(sq.device):
        if fp8:
            st = lib.attn_fwd_fp8_host(q.data_ptr(), k.data_ptr(), v.data_ptr(), float(q_scale), float(k_scale),
                                       float(v_scale), *common)
        else:
            st = lib.attn_fwd_host(q.data_ptr(), k.data_ptr(), v.data_ptr(), *common)
    if st != 0:
        # A failure part way may leave copies in flight that read or write the
        # staging tensors; wait for them (the call keeps `stream` ordered after
        # them) before those tensors can return to the allocator.
        stream.synchronize()
        raise AttnError(st, "attn_fwd_fp8_host" if fp8 else "attn_fwd_host")
    stream.synchronize()
    return out, lse


def fwd_host(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, scale: Optional[float] = None,
             mask: str = "causal", window: Optional[int] = None, chunks: int = 0, device="cuda",
             out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None, staging=None,
             stream: Optional[torch.cuda.Stream] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """The forward on HOST tensors (pinned for overlapped copies), end to end:
    q, k, v go up and out, lse come back in ``chunks`` pieces whose copies
    overlap the kernels (``attn_fwd_host``).  ``staging`` optionally gives the
    device buffers (dq, dk, dv, dout, dlse); returns host (out, lse), complete."""
    return _fwd_host(False, q, k, v, 1.0, 1.0, 1.0, scale, mask, window, chunks, device, out, lse, staging, stream)


def fwd_fp8_host(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, q_scale: float, k_scale: float,
                 v_scale: float, scale: Optional[float] = None, mask: str = "causal", window: Optional[int] = None,
                 chunks: int = 0, device="cuda", out: Optional[torch.Tensor] = None,
                 lse: Optional[torch.Tensor] = None, staging=None, stream: Optional[torch.cuda.Stream] = None
                 ) -> Tuple[torch.Tensor, torch.Tensor]:
    """``fwd_host`` for the E4M3 codes of ``fwd_fp8`` (``attn_fwd_fp8_host``)."""
    return _fwd_host(True, q, k, v, q_scale, k_scale, v_scale, scale, mask, window, chunks, device, out, lse,
                     staging, stream)


def num_work_items(B, Hq, Hkv, N, d, mask="causal", window=None) -> int:
    return int(load_library().attn_fwd_num_work_items(B, Hq, Hkv, N, d, MASKS[mask],
                                                      int(window) if window is not None else 0))
