"""Test helpers: move synth inputs between the GPU path and the oracle, compare results."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import synth


class LazyExperts:
    """Per-expert host copies of a device weight tensor, fetched on first use."""

    def __init__(self, t: torch.Tensor | None):
        self.t = t
        self.cache = {}

    def __getitem__(self, e):
        e = int(e)
        if e not in self.cache:
            self.cache[e] = self.t[e].cpu().numpy()
        return self.cache[e]


def _np(t):
    if t is None:
        return None
    if t.dtype == torch.bfloat16:
        return t.cpu().view(torch.int16).numpy().view(np.uint16)
    return t.cpu().numpy()


def oracle_layer(wl: synth.Workload, d: dict, lazy_weights: bool = False) -> oracle.Layer:
    """oracle.Layer over the same input bytes the GPU path received."""
    if lazy_weights:
        w = {n: (None if d[n] is None else LazyExperts(d[n]))
             for n in ("w1", "w1_scales", "w2", "w2_scales")}
        if wl.wt == "bf16":
            for n in ("w1", "w2"):
                w[n] = LazyExperts(d[n].view(torch.int16))
    else:
        w = {n: _np(d[n]) for n in ("w1", "w1_scales", "w2", "w2_scales")}
    return oracle.Layer(act=wl.act, wt=wl.wt, score=wl.score, renorm=wl.renorm, k=wl.k,
                        x=_np(d["x"]), x_scales=_np(d["x_scales"]), logits=_np(d["logits"]),
                        bias=_np(d["bias"]), **w)


def host_values(t: torch.Tensor, scales: torch.Tensor | None, fmt: str) -> np.ndarray:
    """Device tensor in a library format -> fp64 values (via the oracle's decoders)."""
    if fmt == "f32" or t.dtype == torch.float32:
        return t.float().cpu().numpy().astype(np.float64)
    if fmt == "bf16" or t.dtype == torch.bfloat16:
        return oracle.bf16_bits_to_f64(_np(t))
    return oracle.dequant_x(_np(t), _np(scales), "e4m3")


def rms_err(got: np.ndarray, ref: np.ndarray) -> float:
    """max |got - ref| / rms(ref)."""
    rms = float(np.sqrt(np.mean(ref.astype(np.float64) ** 2)))
    return float(np.max(np.abs(got - ref))) / max(rms, 1e-30)


def store_ulp(ref: np.ndarray, fmt: str) -> np.ndarray:
    """One unit in the last place of the storage format at each reference value."""
    a = np.abs(ref)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    mant = {"bf16": 7, "f32": 23}[fmt]
    return np.where(a > 0, np.ldexp(1.0, (e - mant).astype(np.int64)), 0.0)


def combine_allowance(y_slots: np.ndarray, w: np.ndarray, fmt: str) -> np.ndarray:
    """sum_j |w_j| * ulp(y_j): how far out may move when each stored y row the combine sums
    (the oracle's, [n, k, H]) lands one storage ulp away on the other side."""
    return np.einsum("nk,nkh->nh", np.abs(np.asarray(w, np.float64)),
                     store_ulp(np.asarray(y_slots, np.float64), fmt))


def parity_err(got: np.ndarray, ref: np.ndarray, fmt: str, rms: float | None = None,
               allow: np.ndarray | None = None):
    """The layer's tolerance metric on stored outputs.

    Both sides round to the same storage format, but each takes that rounding decision on
    its own unrounded value (fp32 on the GPU, fp64 in the oracle), so one storage ulp of
    difference at each point where both round is a valid outcome, not an error: one ulp of
    the output itself, plus `allow` for roundings upstream of it (combine_allowance for the
    stored y rows).  Returns
      (max(|got - ref| - ulp(ref) - allow, 0) / rms(ref),  ||got - ref||_2 / ||ref||_2)."""
    ref = ref.astype(np.float64)
    if rms is None:
        rms = float(np.sqrt(np.mean(ref ** 2)))
    excess = np.abs(got - ref) - store_ulp(ref, fmt)
    if allow is not None:
        excess = excess - allow
    excess = np.maximum(excess, 0.0)
    rel_l2 = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))
    return float(np.max(excess)) / max(rms, 1e-30), rel_l2


def raw_err(got: np.ndarray, ref: np.ndarray, rms: float | None = None) -> float:
    """The tolerance figure as stated for the layer, with no allowance of any kind:
    max |got - ref| / rms(ref)."""
    ref = np.asarray(ref, np.float64)
    if rms is None:
        rms = float(np.sqrt(np.mean(ref ** 2)))
    return float(np.max(np.abs(np.asarray(got, np.float64) - ref))) / max(rms, 1e-30)


def assert_parity(got, ref, fmt, tol, rms=None, allow=None):
    mx, l2 = parity_err(got, ref, fmt, rms, allow)
    raw = raw_err(got, ref, rms)
    assert mx <= tol and l2 <= tol, (f"max-excess/rms={mx:.3e} rel-L2={l2:.3e} tol={tol} "
                                     f"(raw max|gpu-oracle|/rms(oracle)={raw:.3e})")
    return mx, l2, raw


# Per-operation relative error of an fp32 accumulation: 2^-23 covers round-to-nearest and
# truncation alike, whatever order the tensor cores or the CUDA cores add in.
FP32_ACC_EPS = 2.0 ** -23


def fp32_sum_bound(abs_terms_sum: np.ndarray, K: int) -> np.ndarray:
    """Bound on |fp32 sum - exact sum| of K exactly representable products whose absolute
    values sum to abs_terms_sum (the classic (K - 1) * eps * sum|a_i b_i| bound of recursive
    summation, valid for any association order)."""
    return (K - 1) * FP32_ACC_EPS * abs_terms_sum


def assert_within_bound(got, ref, bound, fmt, what):
    """|got - ref| <= one storage ulp at |ref| + bound, plus the bound itself, element by
    element: got is ref computed in fp32 (error <= bound) and then rounded to `fmt`, while
    ref is rounded from fp64, so the two roundings can fall one ulp apart on top of the
    fp32 error."""
    ref = np.asarray(ref, np.float64)
    lim = store_ulp(np.abs(ref) + bound, fmt) + bound
    d = np.abs(np.asarray(got, np.float64) - ref)
    bad = d > lim
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {d.size} elements beyond the fp32 "
                           f"accumulation bound; worst |d|/lim = {float(np.max(d / np.maximum(lim, 1e-300))):.3f}")


TOL = {"f32": 1e-4, "bf16": 1e-2, "e4m3": 3e-2}


def weights_of(wl, d):
    import moe_expert_layer_prefix_b200 as M
    return M.Weights(wl.act, wl.wt, d["w1"], d["w2"], d["w1_scales"], d["w2_scales"])
