"""Number-format codecs of the oracle (fp64 numpy), written from the format definitions.

* E4M3 (OCP 8-bit floating point, "FN" variant): 1 sign bit, 4 exponent bits with bias 7,
  3 mantissa bits; exponent 0 encodes subnormals m/8 * 2^-6; S.1111.111 is NaN; there is no
  infinity, so the largest finite magnitude is 1.75 * 2^8 = 448.
* E2M1 (OCP MX 4-bit floating point): 1 sign bit, 2 exponent bits with bias 1, 1 mantissa
  bit: magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6}.  Two codes per byte, element 2i in the low
  nibble.
* UE8M0 (OCP MX scale): an unsigned 8-bit exponent, value 2^(b - 127); 0xFF is NaN.
* BF16: the upper half of an IEEE binary32; rounding is to nearest, ties to even.

The source pages name FP8 and FP4 (jiqizhixin, "DeepSeek悄悄更新：Mega MoE、FP4 Indexer来了",
section "Mega MoE 是什么？", the FP8 x FP4 paragraph; youleyou, "DeepSeek 模型更新解读 Tile
Kernels 与 DeepEP V2 新特性", Tile Kernels feature list, quantisation item) without fixing
their encodings; the OCP definitions above are the plain reading.
"""
from __future__ import annotations

import numpy as np


def _e4m3_value(code: int) -> float:
    sign = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return sign * (m / 8.0) * 2.0 ** -6
    return sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)


E4M3_TABLE = np.array([_e4m3_value(c) for c in range(256)], dtype=np.float64)
E4M3_MAX = 448.0
# non-negative finite codes 0x00..0x7E in increasing order of value
_E4M3_POS = E4M3_TABLE[:0x7F]

E2M1_TABLE = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0,
                       -0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0], dtype=np.float64)


def e4m3_decode(codes) -> np.ndarray:
    return E4M3_TABLE[np.asarray(codes, dtype=np.uint8)]


def e4m3_encode(v) -> np.ndarray:
    """Nearest E4M3 code, ties to the even code, magnitudes above 448 saturate to 448.

    The nearest code is found by searching the table of the 127 non-negative finite values,
    so the rule is the definition itself rather than a bit manipulation."""
    v = np.asarray(v, dtype=np.float64)
    a = np.minimum(np.abs(v), E4M3_MAX)
    hi = np.searchsorted(_E4M3_POS, a, side="left")          # _E4M3_POS[hi-1] < a <= _E4M3_POS[hi]
    hi = np.clip(hi, 0, 0x7E)
    lo = np.clip(hi - 1, 0, 0x7E)
    d_lo = a - _E4M3_POS[lo]
    d_hi = _E4M3_POS[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo).astype(np.uint8)
    code = np.where(np.signbit(v), code | 0x80, code).astype(np.uint8)
    return np.where(np.isnan(v), np.uint8(0x7F), code).astype(np.uint8)


def e2m1_decode_packed(packed) -> np.ndarray:
    """[..., C/2] bytes -> [..., C] fp64; element 2i is the low nibble of byte i."""
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.float64)
    out[..., 0::2] = E2M1_TABLE[p & 0xF]
    out[..., 1::2] = E2M1_TABLE[p >> 4]
    return out


def ue8m0_decode(b) -> np.ndarray:
    b = np.asarray(b, dtype=np.int64)
    return np.where(b == 0xFF, np.nan, np.ldexp(1.0, b - 127))


def bf16_bits_to_f64(bits) -> np.ndarray:
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


_BF16_MAX = (2.0 - 2.0 ** -7) * 2.0 ** 127


def round_bf16(v) -> np.ndarray:
    """Round fp64 values to the nearest BF16 value (ties to even), returned as fp64.

    BF16 keeps 8 significant bits; normal numbers are q * 2^(e-8) with q = rint(m * 2^8)
    for v = m * 2^e, 0.5 <= |m| < 1.  Below 2^-126 the spacing is the fixed 2^-133.
    Magnitudes that round above the largest finite BF16 become infinities."""
    v = np.asarray(v, dtype=np.float64)
    m, e = np.frexp(v)
    normal = np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)
    sub = np.ldexp(np.rint(np.ldexp(v, 133)), -133)
    r = np.where(np.abs(v) < 2.0 ** -126, sub, normal)
    r = np.where(np.abs(r) > _BF16_MAX, np.copysign(np.inf, v), r)
    return np.where(np.isfinite(v), r, v)


def round_bf16_bits(v) -> np.ndarray:
    """round_bf16 as raw uint16 bit patterns."""
    r = round_bf16(v).astype(np.float32)           # exact: every BF16 value is a binary32
    return (r.view(np.uint32) >> 16).astype(np.uint16)
