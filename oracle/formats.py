"""Exact number-format codecs for the oracle (test infrastructure only).

The pages fix the precision of the path only by name: activations are FP8 and
expert weights FP4, with FP8 x FP4 the one supported combination ("Mega MoE"
wiki, section "어떻게 작동하나"; "DeepSeek Mega MoE / DeepGEMM mega kernel",
"TL;DR" and the "Thông số kỹ thuật" table).  The concrete encodings are the OCP
microscaling ones the layer's configurations name:

* E4M3 ("FP8 E4M3", the finite-only variant): sign, 4 exponent bits with bias 7,
  3 mantissa bits; exponent field 0 holds subnormals m/8 * 2^-6; the code with
  every exponent and mantissa bit set is NaN; no infinities; largest finite 448.
* E2M1 ("FP4"): sign, 2 exponent bits with bias 1, 1 mantissa bit; exponent
  field 0 holds the subnormal m/2; values +-{0, 0.5, 1, 1.5, 2, 3, 4, 6}.
* UE8M0 (the MX block scale): an unsigned 8-bit exponent, value 2^(c - 127);
  code 0xFF is NaN.
* bf16: the top 16 bits of an IEEE binary32.

Decoders build their tables from the field definitions above, value by value.
Encoders pick the nearest representable value with ties to the even code,
which is the IEEE round-to-nearest-even rule.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0


# ----------------------------------------------------------------------------- E4M3

def _e4m3_value(code: int) -> float:
    sign = -1.0 if code & 0x80 else 1.0
    exp = (code >> 3) & 0xF
    man = code & 0x7
    if exp == 0xF and man == 0x7:
        return float("nan")
    if exp == 0:
        return sign * (man / 8.0) * 2.0 ** -6
    return sign * (1.0 + man / 8.0) * 2.0 ** (exp - 7)


E4M3_TABLE = np.array([_e4m3_value(c) for c in range(256)], dtype=np.float64)
# non-negative finite codes 0x00..0x7E in increasing value order
_E4M3_POS = E4M3_TABLE[:0x7F].copy()


def decode_e4m3(codes) -> np.ndarray:
    """uint8 E4M3 codes -> float64 values.  NaN codes raise ValueError."""
    codes = np.asarray(codes, dtype=np.uint8)
    if np.any((codes & 0x7F) == 0x7F):
        raise ValueError("E4M3 NaN code in input")
    return E4M3_TABLE[codes]


def encode_e4m3(values) -> np.ndarray:
    """float64 -> E4M3 codes, round to nearest (ties to even code), saturating at +-448.

    The sign is kept for values that round to zero (so -0.0 and tiny negatives
    give 0x80), as an IEEE conversion does.  NaN input raises ValueError.
    """
    v = np.asarray(values, dtype=np.float64)
    if np.any(np.isnan(v)):
        raise ValueError("NaN cannot be encoded")
    a = np.abs(v)
    # index of the largest representable value <= a
    lo = np.searchsorted(_E4M3_POS, a, side="right") - 1
    lo = np.clip(lo, 0, 0x7E)
    hi = np.minimum(lo + 1, 0x7E)
    d_lo = a - _E4M3_POS[lo]
    d_hi = _E4M3_POS[hi] - a
    take_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0) & (hi != lo))
    code = np.where(take_hi, hi, lo)
    code = np.where(a >= E4M3_MAX, 0x7E, code)          # saturate (satfinite)
    code = code.astype(np.uint8)
    code |= np.where(np.signbit(v), 0x80, 0).astype(np.uint8)
    return code


# ----------------------------------------------------------------------------- E2M1

def _e2m1_value(code: int) -> float:
    sign = -1.0 if code & 0x8 else 1.0
    exp = (code >> 1) & 0x3
    man = code & 0x1
    if exp == 0:
        return sign * man / 2.0
    return sign * (1.0 + man / 2.0) * 2.0 ** (exp - 1)


E2M1_TABLE = np.array([_e2m1_value(c) for c in range(16)], dtype=np.float64)


def decode_e2m1(nibbles) -> np.ndarray:
    """4-bit E2M1 codes (one per uint8) -> float64 values."""
    return E2M1_TABLE[np.asarray(nibbles, dtype=np.uint8) & 0xF]


def unpack_e2m1(packed) -> np.ndarray:
    """Packed MXFP4 rows [..., K/2] bytes -> float64 [..., K] (no scale applied).

    Byte j holds element 2j in its low nibble and element 2j+1 in its high nibble.
    """
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.float64)
    out[..., 0::2] = E2M1_TABLE[p & 0xF]
    out[..., 1::2] = E2M1_TABLE[p >> 4]
    return out


# ----------------------------------------------------------------------------- UE8M0

def decode_ue8m0(codes) -> np.ndarray:
    """UE8M0 codes -> 2^(code - 127) as float64.  Code 0xFF (NaN) raises."""
    c = np.asarray(codes, dtype=np.uint8)
    if np.any(c == 0xFF):
        raise ValueError("UE8M0 NaN code in input")
    return np.ldexp(1.0, c.astype(np.int64) - 127)


def dequant_mxfp4(packed, scales) -> np.ndarray:
    """Packed E2M1 [..., K/2] with UE8M0 scales [..., K/32] -> float64 [..., K]."""
    vals = unpack_e2m1(packed)
    s = decode_ue8m0(scales)
    return vals * np.repeat(s, 32, axis=-1)


# ----------------------------------------------------------------------------- bf16

def bf16_to_f64(bits) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float64, exactly."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def f64_to_bf16(values) -> np.ndarray:
    """float64 -> bf16 bit patterns, one rounding to nearest even (no double rounding).

    bf16 keeps 8 significant bits; below 2^-126 the quantum stays 2^-133.
    Results that round past the largest finite bf16 become infinity.
    """
    v = np.asarray(values, dtype=np.float64)
    if np.any(np.isnan(v)):
        raise ValueError("NaN cannot be encoded")
    a = np.abs(v)
    _, e = np.frexp(a)                       # a = m * 2^e, m in [0.5, 1)
    e = np.maximum(e - 1, -126)              # exponent of the leading bit, clamped to normal range
    quantum_exp = e - 7
    r = np.ldexp(a, -quantum_exp)            # exact
    n = np.rint(r)                           # round half to even
    q = np.ldexp(n, quantum_exp)
    q = np.where(a == 0, 0.0, q)
    with np.errstate(over="ignore"):
        f32 = q.astype(np.float32)           # exact: q has <= 8 significant bits
    bits = (f32.view(np.uint32) >> 16).astype(np.uint16)
    bits |= np.where(np.signbit(v), 0x8000, 0).astype(np.uint16)
    return bits


# ----------------------------------------------------------------------------- pow2 scale

def pow2_exponent(amax, qmax: float = E4M3_MAX, p_min: int = -126) -> np.ndarray:
    """Smallest integer p with amax <= qmax * 2^p; p = 0 when amax == 0; p >= p_min.

    This is the activation scale rule of the layer: the per-block scale is 2^p,
    a power of two, so that x / 2^p is exact and the scale is a UE8M0 value.
    """
    a = np.asarray(amax, dtype=np.float64)
    _, e = np.frexp(a)                       # a < 2^e
    p = e.astype(np.int64) - 8               # qmax*2^(e-8) >= 1.75*2^e > a for qmax = 448
    # step down while the next smaller power still satisfies the bound
    for _ in range(4):
        smaller_ok = a <= qmax * np.ldexp(1.0, p - 1)
        p = np.where(smaller_ok, p - 1, p)
    p = np.where(a == 0, 0, p)
    return np.maximum(p, p_min).astype(np.int64)
