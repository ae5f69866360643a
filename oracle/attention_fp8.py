"""fp64 CPU oracle for the FP8 (E4M3) attention forward.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import this
module: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg
of ``bench.py`` use it.  It shares no code with the CUDA path.

The FP8 forward takes q, k and v as E4M3 codes with one scale per tensor
(the value of a code is its E4M3 number times the tensor's scale) and returns
the same exact masked softmax attention as the bf16 forward, of the
dequantised tensors ("Efficient attention: long context and sub-quadratic
variants", stanleyjacob.dev, sections "FlashAttention: exact attention,
IO-aware" and "Implementation, twice"; FP8 inputs are a feature of the later
kernels of that line, "Efficient Attention: Flash Attention, Sliding Window,
Sparse", creativeworksofknowledge.com, section "Flash Attention (exact,
memory-efficient)").  So the oracle is: decode the codes exactly into
float64, multiply by the scales, apply the pinned forward definition
(``oracle.attention_fp64.attention``).

E4M3 (the OCP 8-bit format without infinities): bit 7 sign, bits 6..3 the
exponent with bias 7, bits 2..0 the mantissa; exponent 0 encodes subnormals
m/8 * 2^-6; the all-ones exponent with mantissa 7 is NaN (the largest finite
magnitude is 1.75 * 2^8 = 448).

Pins (``tests/test_oracle_fp8.py``): the decoder against torch's
float8_e4m3fn conversion for all 256 codes and against hand-computed values;
the attention on codes that are small integers against the bf16 forward
oracle on the same values; moving a power of two between codes and scales
changes nothing; planted mistakes are caught.
"""
from __future__ import annotations

import numpy as np

from .attention_fp64 import attention

E4M3_MAX = 448.0


def e4m3_to_float(codes) -> np.ndarray:
    """Exact float64 value of every E4M3 code (uint8 array of any shape)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    exp = (c >> 3) & 0xF
    man = c & 0x7
    normal = (1.0 + man / 8.0) * np.exp2(exp - 7.0)
    subnormal = (man / 8.0) * 2.0 ** -6
    val = np.where(exp == 0, subnormal, normal)
    val = np.where((exp == 15) & (man == 7), np.nan, val)
    return sign * val


def dequantise(codes, scale: float) -> np.ndarray:
    """Tensor value of E4M3 codes with a per-tensor scale."""
    return e4m3_to_float(codes) * float(scale)


def attention_fp8(q8, k8, v8, q_scale, k_scale, v_scale, scale=None, mask_kind: int = 1, window=None, rows=None):
    """Exact attention of the dequantised tensors: q8 [B,Hq,N,d], k8/v8
    [B,Hkv,N,d] uint8 E4M3 codes; ``scale`` (default 1/sqrt(d)) multiplies
    the dequantised q.k.  Returns (out, lse) like the bf16 oracle."""
    q = dequantise(q8, q_scale)
    k = dequantise(k8, k_scale)
    v = dequantise(v8, v_scale)
    return attention(q, k, v, scale, mask_kind, window, rows=rows)
