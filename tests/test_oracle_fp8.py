"""The FP8 oracle against facts that do not come from it (CPU only), and
planted mistakes that those pins catch."""
import numpy as np
import pytest
import torch

from oracle import attention_fp64 as F
from oracle import attention_fp8 as O8

FULL, CAUSAL, WINDOW = 0, 1, 2


def pin_decoder_matches_library(mod):
    """All 256 codes against torch's float8_e4m3fn conversion (NaN codes too)."""
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = mod.e4m3_to_float(codes)
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])


def pin_decoder_hand_values(mod):
    """Values computed by hand from the format: 1.0 = 0x38, the largest finite
    magnitude 0x7E = 448, the smallest subnormal 0x01 = 2^-9, the smallest
    normal 0x08 = 2^-6, 0xB8 = -1.0, 0x3C = 1.5, 0x7F and 0xFF are NaN."""
    vals = mod.e4m3_to_float(np.array([0x38, 0x7E, 0x01, 0x08, 0xB8, 0x3C, 0x00, 0x80], dtype=np.uint8))
    assert list(vals) == [1.0, 448.0, 2.0 ** -9, 2.0 ** -6, -1.0, 1.5, 0.0, -0.0]
    assert np.isnan(mod.e4m3_to_float(np.array([0x7F, 0xFF], dtype=np.uint8))).all()


def _int_codes(shape, rng):
    """Codes of the integers -8..8 (exact in E4M3)."""
    vals = rng.integers(-8, 9, size=shape).astype(np.float32)
    return torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy(), vals.astype(np.float64)


def pin_integer_codes_match_forward_oracle(mod):
    """Codes of small integers with scales 1/8: the FP8 oracle equals the
    forward oracle on the same (exactly representable) values, for all masks
    and grouped heads."""
    rng = np.random.default_rng(5)
    for kind, w in ((CAUSAL, None), (FULL, None), (WINDOW, 5)):
        q8, q = _int_codes((1, 4, 19, 8), rng)
        k8, k = _int_codes((1, 2, 19, 8), rng)
        v8, v = _int_codes((1, 2, 19, 8), rng)
        o1, l1 = mod.attention_fp8(q8, k8, v8, 0.125, 0.125, 0.125, None, kind, w)
        o2, l2 = F.attention(q / 8, k / 8, v / 8, None, kind, w)
        assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def pin_power_of_two_between_codes_and_scale(mod):
    """Doubling every code's value (exponent + 1, exact) while halving the
    scale leaves the result bitwise unchanged; the V scale scales out
    linearly and leaves lse alone; the q and k scales multiply the scores."""
    rng = np.random.default_rng(6)
    q8, q = _int_codes((1, 2, 9, 4), rng)
    k8, k = _int_codes((1, 2, 9, 4), rng)
    v8, v = _int_codes((1, 2, 9, 4), rng)
    dbl = lambda x: torch.from_numpy(2 * x.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    o1, l1 = mod.attention_fp8(q8, k8, v8, 0.25, 0.5, 0.75, 0.3, CAUSAL)
    o2, l2 = mod.attention_fp8(dbl(q), k8, dbl(v), 0.125, 0.5, 0.375, 0.3, CAUSAL)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)
    o3, l3 = mod.attention_fp8(q8, k8, v8, 0.25, 0.5, 1.5, 0.3, CAUSAL)
    assert np.allclose(o3, 2 * o1, rtol=1e-15, atol=0) and np.array_equal(l3, l1)
    o4, l4 = mod.attention_fp8(q8, k8, v8, 0.25, 1.0, 0.75, 0.15, CAUSAL)
    assert np.allclose(o4, o1, rtol=1e-14) and np.allclose(l4, l1, rtol=1e-14)


ALL_PINS = (pin_decoder_matches_library, pin_decoder_hand_values, pin_integer_codes_match_forward_oracle,
            pin_power_of_two_between_codes_and_scale)


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(O8)


def _bias8(codes):
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    exp, man = (c >> 3) & 0xF, c & 0x7
    return sign * np.where(exp == 0, man / 8 * 2.0 ** -6, (1 + man / 8) * np.exp2(exp - 8.0))


def _no_subnormal(codes):
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    exp, man = (c >> 3) & 0xF, c & 0x7
    return sign * (1 + man / 8) * np.exp2(exp - 7.0)


_orig = O8.e4m3_to_float


def _nan_saturates(codes):
    val = _orig(codes)
    c = np.asarray(codes, dtype=np.uint8)
    return np.where(np.isnan(val), np.where(c & 0x80, -448.0, 448.0), val)


def _k_takes_v_scale(q8, k8, v8, q_scale, k_scale, v_scale, scale=None, mask_kind=1, window=None, rows=None):
    return F.attention(O8.dequantise(q8, q_scale), O8.dequantise(k8, v_scale), O8.dequantise(v8, v_scale),
                       scale, mask_kind, window, rows=rows)


def _softmax_scale_dropped(q8, k8, v8, q_scale, k_scale, v_scale, scale=None, mask_kind=1, window=None, rows=None):
    return F.attention(O8.dequantise(q8, q_scale), O8.dequantise(k8, k_scale), O8.dequantise(v8, v_scale),
                       None, mask_kind, window, rows=rows)


MUTANTS = {
    "exponent bias 8": ("e4m3_to_float", _bias8),
    "subnormals read as normals": ("e4m3_to_float", _no_subnormal),
    "sign bit dropped": ("e4m3_to_float", lambda c: np.abs(_orig(c))),
    "NaN codes saturate to 448": ("e4m3_to_float", _nan_saturates),
    "scale ignored": ("dequantise", lambda codes, scale: _orig(codes)),
    "k dequantised with the v scale": ("attention_fp8", _k_takes_v_scale),
    "softmax scale dropped": ("attention_fp8", _softmax_scale_dropped),
}


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_planted_mistake_is_caught(mutant, monkeypatch):
    attr, fn = MUTANTS[mutant]
    monkeypatch.setattr(O8, attr, fn)
    caught = False
    for pin in ALL_PINS:
        try:
            pin(O8)
        except (AssertionError, ValueError):
            caught = True
            break
    assert caught, mutant
