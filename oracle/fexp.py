"""The fp32 exponential and sigmoid that decide the sigmoid router's top-k selection.

A selection decided by floating-point keys is reproduced bit for bit only if both sides
compute the keys with the same correctly-rounded fp32 operations.  The library's exp is not
such an operation, so the key function is defined here from a published method and written
out once for the oracle (below) and once, independently, in the CUDA router.

Method (Cody & Waite, "Software Manual for the Elementary Functions", 1980: additive range
reduction with a two-part ln 2; the reduced argument is then evaluated by its Taylor series):

    x      <- clamp(x, -80, 80)
    n      =  rint(x * log2(e))                   ties to even
    r      =  (x - n * LN2_HI) - n * LN2_LO       LN2_HI has 15 significant bits, so n*LN2_HI is exact
    p(r)   =  1 + r + r^2/2! + ... + r^7/7!       Horner order, highest coefficient first
    exp(x) =  p(r) * 2^n

Every operation is one fp32 multiply or add, rounded to nearest even, never fused.  The
coefficients are the decimal literals below, each rounded to fp32.  With |r| <= ln2/2 the
truncation error is below 1e-8 relative, so the result is within 2 ulp of exp(x).

sigmoid(x) = 1 / (1 + exp(-x)), again as separately rounded fp32 operations.
"""
from __future__ import annotations

import numpy as np

F = np.float32
LOG2E = F("1.44269504088896340736")
LN2_HI = F("0.693145751953125")
LN2_LO = F("1.42860682030941723212e-6")
# Taylor coefficients 1/7! .. 1/2!
C7 = F("1.98412698412698412698e-4")
C6 = F("1.38888888888888888889e-3")
C5 = F("8.33333333333333333333e-3")
C4 = F("4.16666666666666666667e-2")
C3 = F("1.66666666666666666667e-1")
C2 = F("0.5")
ONE = F(1.0)
XMIN, XMAX = F(-80.0), F(80.0)


def exp_f32(x) -> np.ndarray:
    x = np.clip(np.asarray(x, dtype=F), XMIN, XMAX).astype(F)
    n = np.rint(x * LOG2E).astype(F)
    r = (x - n * LN2_HI).astype(F)
    r = (r - n * LN2_LO).astype(F)
    p = np.full_like(r, C7)
    for c in (C6, C5, C4, C3, C2, ONE, ONE):
        p = (p * r).astype(F)
        p = (p + c).astype(F)
    return np.ldexp(p, n.astype(np.int32)).astype(F)


def sigmoid_f32(x) -> np.ndarray:
    x = np.asarray(x, dtype=F)
    e = exp_f32(-x)
    return (ONE / (ONE + e).astype(F)).astype(F)
