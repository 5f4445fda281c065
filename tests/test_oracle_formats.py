"""Pins for the oracle's number-format codecs (CPU only).

Each codec is checked against something other than itself: the values printed in the OCP
format specifications (tests/golden/ocp_format_examples.txt), torch's own float8 / bfloat16
casts (library routines) and brute-force nearest-value search."""
import math
import os

import numpy as np
import pytest
import torch

from oracle import formats as F

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "ocp_format_examples.txt")


def _golden():
    rows = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            fmt, code, val = line.split()
            rows.append((fmt, int(code, 16), float(val)))
    return rows


@pytest.mark.parametrize("fmt,code,val", _golden())
def test_spec_examples(fmt, code, val):
    if fmt == "e4m3":
        got = F.e4m3_decode(np.array([code], np.uint8))[0]
    elif fmt == "e2m1":
        got = F.e2m1_decode_packed(np.array([code], np.uint8))[0]
    else:
        got = F.ue8m0_decode(np.array([code]))[0]
    if math.isnan(val):
        assert math.isnan(got)
    else:
        assert got == val and math.copysign(1, got) == math.copysign(1, val)


def test_e4m3_table_matches_torch_decode():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = F.E4M3_TABLE
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert np.array_equal(ref[~nan], got[~nan])
    assert nan.sum() == 2                          # only S.1111.111


def test_e4m3_encode_matches_torch_cast():
    rng = np.random.default_rng(0)
    v = np.concatenate([rng.standard_normal(20000) * s for s in (1e-3, 0.05, 1, 30, 200)])
    v = np.clip(v, -448, 448).astype(np.float32)          # torch's cast does not saturate
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = F.e4m3_encode(v.astype(np.float64))
    assert np.array_equal(F.e4m3_decode(ref), F.e4m3_decode(got))


def test_e4m3_encode_brute_force_nearest_and_ties():
    finite = np.array([c for c in range(256) if not math.isnan(F.E4M3_TABLE[c])])
    vals = F.E4M3_TABLE[finite]
    rng = np.random.default_rng(1)
    v = rng.uniform(-448, 448, 3000)
    # exact midpoints between neighbouring codes must go to the even code
    pos = np.sort(np.unique(np.abs(vals)))
    mids = (pos[1:] + pos[:-1]) / 2
    for x in np.concatenate([v, mids, -mids]):
        c = int(F.e4m3_encode(np.array([x]))[0])
        err = abs(F.E4M3_TABLE[c] - x)
        best = np.min(np.abs(vals - x))
        assert err == best
    for m in mids:
        c = int(F.e4m3_encode(np.array([m]))[0])
        assert c % 2 == 0


def test_e4m3_saturates():
    got = F.e4m3_encode(np.array([464.0, 1e6, -500.0, 449.0]))
    assert list(got) == [0x7E, 0x7E, 0xFE, 0x7E]
    assert F.e4m3_encode(np.array([np.nan]))[0] == 0x7F


def test_e2m1_all_codes_and_packing():
    mags = [0, 0.5, 1, 1.5, 2, 3, 4, 6]
    for c in range(16):
        v = F.e2m1_decode_packed(np.array([c | (((c + 3) % 16) << 4)], np.uint8))
        want_lo = (-1 if c >= 8 else 1) * mags[c % 8]
        c2 = (c + 3) % 16
        want_hi = (-1 if c2 >= 8 else 1) * mags[c2 % 8]
        assert v[0] == want_lo and v[1] == want_hi     # element 0 is the low nibble


def test_ue8m0_range():
    b = np.arange(255)
    assert np.array_equal(F.ue8m0_decode(b), np.ldexp(1.0, b - 127))


def test_bf16_round_matches_torch_on_fp32_inputs():
    rng = np.random.default_rng(2)
    v = np.concatenate([rng.standard_normal(50000) * s for s in (1e-40, 1e-3, 1, 1e30)])
    v32 = v.astype(np.float32)
    ref = torch.from_numpy(v32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = F.round_bf16_bits(v32.astype(np.float64))
    assert np.array_equal(ref, got)


def test_bf16_round_ties_and_overflow():
    one = 1.0
    assert F.round_bf16(np.array([one + 2 ** -8]))[0] == 1.0                     # tie -> even
    assert F.round_bf16(np.array([one + 3 * 2 ** -8]))[0] == 1.0 + 2 ** -6       # tie -> even
    assert F.round_bf16(np.array([one + 2 ** -8 + 2 ** -30]))[0] == 1.0 + 2 ** -7
    big = (2 - 2 ** -8) * 2.0 ** 127                                           # max + half ulp
    assert np.isinf(F.round_bf16(np.array([big]))[0])
    assert F.round_bf16(np.array([(2 - 2 ** -7) * 2.0 ** 127]))[0] == (2 - 2 ** -7) * 2.0 ** 127
