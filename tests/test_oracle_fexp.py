"""Pins for the oracle's fp32 exponential / sigmoid (CPU only): closed forms and the error
bound against the correctly rounded exponential (fp64 library exp rounded once to fp32)."""
import numpy as np

from oracle.fexp import exp_f32, sigmoid_f32


def _ulp_diff(a, b):
    ia = a.astype(np.float32).view(np.int32).astype(np.int64)
    ib = b.astype(np.float32).view(np.int32).astype(np.int64)
    return np.abs(ia - ib)


def test_exp_within_two_ulp():
    x = np.linspace(-80, 80, 400001).astype(np.float32)
    ref = np.exp(x.astype(np.float64)).astype(np.float32)
    got = exp_f32(x)
    assert got.dtype == np.float32
    assert _ulp_diff(got, ref).max() <= 2


def test_exp_closed_forms():
    assert exp_f32(np.float32([0.0]))[0] == 1.0
    # clamp: far outside the range the value stays finite and positive
    assert np.isfinite(exp_f32(np.float32([1e4]))[0])
    assert exp_f32(np.float32([-1e4]))[0] > 0
    # exp(n ln2) for integer n is within 1 ulp of 2^n
    n = np.arange(-60, 61)
    x = (n * np.log(2.0)).astype(np.float32)
    assert _ulp_diff(exp_f32(x), np.exp(x.astype(np.float64))).max() <= 2


def test_sigmoid_properties():
    assert sigmoid_f32(np.float32([0.0]))[0] == np.float32(0.5)
    x = np.sort(np.random.default_rng(3).standard_normal(100000).astype(np.float32) * 4)
    s = sigmoid_f32(x)
    assert np.all(np.diff(s) >= 0)                                  # monotone
    ref = (1 / (1 + np.exp(-x.astype(np.float64))))
    assert np.max(np.abs(s - ref) / ref) < 4e-7
    assert np.max(np.abs(s + sigmoid_f32(-x) - 1.0)) < 2e-7
