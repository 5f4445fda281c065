"""Seeded synthetic inputs for the fused MoE expert layer.

This package only *draws* inputs.  It holds none of the layer's arithmetic: no routing, no
dispatch, no GEMM, no activation and no requantisation.  The CUDA library's tests and
benchmark and the CPU oracle all consume the bytes it returns, so both sides of every parity
check see identical inputs.

Workloads (shapes and value distributions) follow the five MoE-layer shapes used throughout
the project: a tiny fp32 layer, a Mixtral-shaped BF16 layer, a DeepSeek-V3-shaped FP8 layer, a
decode-shaped FP8 x FP4 layer and a skewed many-expert FP8 x FP4 layer.  No dataset, checkpoint
or trained weight is involved; every tensor is drawn from a seeded torch generator.

Encodings produced here (they are the *inputs'* formats, fixed before the layer runs):

* E4M3 tensors are torch ``float8_e4m3fn`` codes stored as ``uint8``.  The fp32 values are
  divided by a per-block power of two and rounded by torch's own cast; the block exponent is
  drawn at random from a two-value window so that scales differ block to block.
* E2M1 tensors hold two 4-bit codes per byte, element ``2i`` in the low nibble; the block
  exponent (UE8M0, bias 127) is drawn the same way, one per 32 elements along K.
* BF16 tensors are torch's round-to-nearest-even cast of fp32 draws.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch

# seeds, one per drawn tensor
SEED_W1, SEED_W2, SEED_WR = 10, 11, 12
SEED_X, SEED_LOGITS, SEED_BIAS, SEED_ZIPF = 1, 2, 3, 4
SEED_XEXP, SEED_W1EXP, SEED_W2EXP = 5, 6, 7

E4M3_MAX = 448.0
E2M1_MAX = 6.0
# magnitudes of the eight non-negative E2M1 codes 0..7
_E2M1_MAGS = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)


@dataclass(frozen=True)
class Workload:
    """One MoE-layer shape.  act / wt: 'f32' | 'bf16' | 'e4m3' | 'e2m1'."""
    name: str
    T: int
    H: int
    E: int
    k: int
    I: int
    act: str
    wt: str
    score: str              # 'softmax' | 'sigmoid'
    logits: str             # 'router' (x . Wr^T) | 'normal' | 'zipf'
    bias: bool = False      # per-expert selection bias (sigmoid router)
    renorm: bool = True     # renormalise the k gates
    zipf_alpha: float = 1.2

    @property
    def S(self) -> int:
        return self.T * self.k

    def flops(self) -> float:
        """Algorithmic FLOPs of the two expert GEMMs: 2*S*H*2I + 2*S*I*H."""
        return 6.0 * self.S * self.H * self.I

    def scaled(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", 64, 256, 8, 2, 128, "f32", "f32", "softmax", "router"),
    "mixtral_bf16": Workload("mixtral_bf16", 4096, 4096, 8, 2, 14336, "bf16", "bf16",
                             "softmax", "normal"),
    "v3_fp8": Workload("v3_fp8", 8192, 7168, 256, 8, 2048, "e4m3", "e4m3", "sigmoid",
                       "normal", bias=True),
    "decode_fp8_fp4": Workload("decode_fp8_fp4", 128, 7168, 256, 8, 2048, "e4m3", "e2m1",
                               "softmax", "normal"),
    "skewed_fp8_fp4": Workload("skewed_fp8_fp4", 16384, 7168, 1024, 16, 512, "e4m3", "e2m1",
                               "softmax", "zipf"),
}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _randn(shape, g, device) -> torch.Tensor:
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32)


def _block_exponents(shape, e0: int, g, device) -> torch.Tensor:
    """Random block exponents drawn from {e0, e0+1} (int32)."""
    return torch.randint(0, 2, shape, generator=g, device=device, dtype=torch.int32) + e0


def _to_e4m3_codes(v: torch.Tensor) -> torch.Tensor:
    return v.clamp(-E4M3_MAX, E4M3_MAX).to(torch.float8_e4m3fn).view(torch.uint8)


def _to_e2m1_packed(v: torch.Tensor) -> torch.Tensor:
    """Nearest E2M1 code (ties toward the smaller magnitude), two codes per byte."""
    mags = v.abs().clamp(max=E2M1_MAX)
    bounds = torch.tensor([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], device=v.device)
    code = torch.bucketize(mags, bounds, right=False).to(torch.uint8)
    code = code | ((v < 0).to(torch.uint8) << 3)
    lo, hi = code[..., 0::2], code[..., 1::2]
    return lo | (hi << 4)


def _quant_rows_e4m3(w: torch.Tensor, blk_r: int, blk_c: int, e0: int, g, device):
    """w [R, C] fp32 -> (codes u8 [R, C], scales f32 [R/blk_r, C/blk_c])."""
    R, C = w.shape
    ex = _block_exponents((R // blk_r, C // blk_c), e0, g, device)
    full = ex.repeat_interleave(blk_r, 0).repeat_interleave(blk_c, 1)
    codes = _to_e4m3_codes(torch.ldexp(w, -full))
    return codes, torch.ldexp(torch.ones_like(ex, dtype=torch.float32), ex)


def _quant_rows_e2m1(w: torch.Tensor, e0: int, g, device):
    """w [R, C] fp32 -> (packed u8 [R, C/2], UE8M0 u8 [R, C/32])."""
    R, C = w.shape
    ex = _block_exponents((R, C // 32), e0, g, device)
    full = ex.repeat_interleave(32, 1)
    packed = _to_e2m1_packed(torch.ldexp(w, -full))
    return packed, (ex + 127).to(torch.uint8)


def _e0_for(std: float, maxcode: float, nsig: float) -> int:
    return int(math.ceil(math.log2(nsig * std / maxcode)))


def make_weights(wl: Workload, device="cpu"):
    """Expert weights W1 [E, 2I, H] (rows [0,I) gate, [I,2I) up) and W2 [E, H, I].

    Values ~ N(0, 1/fan_in) in fp32, then stored in ``wl.wt``.  Returns a dict with
    w1, w1_scales, w2, w2_scales (scales None for f32/bf16).
    """
    E, H, I = wl.E, wl.H, wl.I
    out = {}
    for name, rows, cols, seed, seed_e in (("w1", 2 * I, H, SEED_W1, SEED_W1EXP),
                                           ("w2", H, I, SEED_W2, SEED_W2EXP)):
        std = 1.0 / math.sqrt(cols)
        g = _gen(seed, device)
        ge = _gen(seed_e, device)
        if wl.wt == "f32":
            out[name] = _randn((E, rows, cols), g, device) * std
            out[name + "_scales"] = None
        elif wl.wt == "bf16":
            w = torch.empty((E, rows, cols), dtype=torch.bfloat16, device=device)
            for e in range(E):
                w[e] = (_randn((rows, cols), g, device) * std).to(torch.bfloat16)
            out[name], out[name + "_scales"] = w, None
        elif wl.wt == "e4m3":
            codes = torch.empty((E, rows, cols), dtype=torch.uint8, device=device)
            sc = torch.empty((E, rows // 128, cols // 128), dtype=torch.float32, device=device)
            e0 = _e0_for(std, E4M3_MAX, 6.0)
            for e in range(E):
                codes[e], sc[e] = _quant_rows_e4m3(_randn((rows, cols), g, device) * std,
                                                   128, 128, e0, ge, device)
            out[name], out[name + "_scales"] = codes, sc
        elif wl.wt == "e2m1":
            packed = torch.empty((E, rows, cols // 2), dtype=torch.uint8, device=device)
            sc = torch.empty((E, rows, cols // 32), dtype=torch.uint8, device=device)
            e0 = _e0_for(std, E2M1_MAX, 4.0)
            for e in range(E):
                packed[e], sc[e] = _quant_rows_e2m1(_randn((rows, cols), g, device) * std,
                                                    e0, ge, device)
            out[name], out[name + "_scales"] = packed, sc
        else:
            raise ValueError(wl.wt)
    return out


def make_activations(wl: Workload, device="cpu", seed_offset: int = 0):
    """x [T, H] in ``wl.act`` (+ x_scales f32 [T, H/128] for E4M3), logits f32 [T, E] and
    bias f32 [E] (or None).  ``seed_offset`` draws a different batch with the same recipe."""
    T, H, E = wl.T, wl.H, wl.E
    g = _gen(SEED_X + 1000 * seed_offset, device)
    z = _randn((T, H), g, device)
    res = {"x_scales": None}
    if wl.act == "f32":
        res["x"] = z
    elif wl.act == "bf16":
        res["x"] = z.to(torch.bfloat16)
    elif wl.act == "e4m3":
        ge = _gen(SEED_XEXP + 1000 * seed_offset, device)
        res["x"], res["x_scales"] = _quant_rows_e4m3(z, 1, 128, _e0_for(1.0, E4M3_MAX, 6.0),
                                                     ge, device)
    else:
        raise ValueError(wl.act)

    gl = _gen(SEED_LOGITS + 1000 * seed_offset, device)
    if wl.logits == "router":
        # logits = x . Wr^T, Wr ~ N(0, 1/H), evaluated in fp64 and rounded to fp32 once
        gr = _gen(SEED_WR, device)
        wr = _randn((E, H), gr, device).double() / math.sqrt(H)
        res["logits"] = (z.double() @ wr.T).float()
    elif wl.logits == "normal":
        res["logits"] = _randn((T, E), gl, device)
    elif wl.logits == "zipf":
        # per-expert popularity offset: log of a Zipf(alpha) popularity over a seeded rank order
        gz = _gen(SEED_ZIPF, device)
        rank = torch.randperm(E, generator=gz, device=device).double() + 1.0
        off = (-wl.zipf_alpha * torch.log(rank)).float()
        res["logits"] = _randn((T, E), gl, device) + off[None, :]
    else:
        raise ValueError(wl.logits)
    if wl.bias:
        gb = _gen(SEED_BIAS, device)
        res["bias"] = _randn((E,), gb, device) * 0.1
    else:
        res["bias"] = None
    return res


def make_inputs(wl: Workload, device="cpu"):
    d = make_activations(wl, device)
    d.update(make_weights(wl, device))
    return d


def to_numpy(d: dict) -> dict:
    """Host numpy copies of every tensor (bf16 -> its raw uint16 bits)."""
    out = {}
    for k, v in d.items():
        if v is None:
            out[k] = None
        elif v.dtype == torch.bfloat16:
            out[k] = v.detach().cpu().view(torch.int16).numpy().view("uint16")
        else:
            out[k] = v.detach().cpu().numpy()
    return out
