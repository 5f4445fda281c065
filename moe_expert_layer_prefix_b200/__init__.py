"""Python binding of libmoe.so, the B200 fused MoE expert layer.

Argument marshalling only: every step of the layer runs in the library's CUDA kernels.
Torch provides device memory and the current stream.  The entry points keep the C names
(moe_route, moe_dispatch, moe_expert_linear1, moe_expert_linear2, moe_fused_ffn,
moe_combine, moe_forward, moe_workspace_size, moe_get_device_error, moe_status_string);
outputs that are not passed in are allocated with torch.empty.

The library must have been built (``python moe_expert_layer_prefix_b200/build.py``);
importing this package without it raises ImportError -- there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe.so")
if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing; build it with "
                      "`python moe_expert_layer_prefix_b200/build.py`")
_lib = ctypes.CDLL(LIB_PATH)

MOE_OK = 0
STATUS = {0: "MOE_OK", -1: "MOE_ERR_INVALID_ARG", -2: "MOE_ERR_UNSUPPORTED",
          -3: "MOE_ERR_MISALIGNED", -4: "MOE_ERR_WORKSPACE", -5: "MOE_ERR_CUDA",
          -6: "MOE_ERR_TIMEOUT", -7: "MOE_ERR_DEVICE"}
DTYPES = {"f32": 0, "bf16": 1, "e4m3": 2, "e2m1": 3}
SCORES = {"softmax": 0, "sigmoid": 1}
OPS = {"dispatch": 1, "linear1": 2, "linear2": 3, "fused_ffn": 4, "forward": 5, "backward": 6}

EXPORTS = ("moe_route", "moe_dispatch", "moe_expert_linear1", "moe_expert_linear2",
           "moe_fused_ffn", "moe_combine", "moe_forward", "moe_workspace_size",
           "moe_get_device_error", "moe_status_string", "moe_launch_count",
           "moe_dispatch_noalloc", "moe_set_gemm_tiles", "moe_dispatch_quant", "moe_route_ex",
           "moe_forward_ex", "moe_transpose_experts", "moe_expert_backward",
           "moe_set_wait_limit", "moe_selftest_wait")

_P, _I, _Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t


class MoeRouterGroups(ctypes.Structure):
    _fields_ = [("n_group", ctypes.c_int), ("topk_group", ctypes.c_int), ("scale", ctypes.c_float)]


class MoeBackwardArgs(ctypes.Structure):
    _fields_ = ([(n, ctypes.c_int) for n in ("T", "H", "E", "k", "I", "score", "renorm")] +
                [("scale", ctypes.c_float)] +
                [(n, _P) for n in ("dout", "logits", "topk_idx", "topk_w", "expert_offsets",
                                   "slot_of", "x_perm", "h", "y", "w1", "w2", "w1_t", "w2_t",
                                   "dx", "dw1", "dw2", "dlogits")])


class MoeWeights(ctypes.Structure):
    _fields_ = [("act", ctypes.c_int), ("wt", ctypes.c_int), ("w1", _P), ("w1_scales", _P),
                ("w2", _P), ("w2_scales", _P), ("scale_fmt", ctypes.c_int)]


SCALE_FMTS = {"pow2": 0, "fp32": 1}


def _sig(name, res, args):
    f = getattr(_lib, name)
    f.restype, f.argtypes = res, args
    return f


_route = _sig("moe_route", _I, [_P, _P, _I, _I, _I, _I, _I, _P, _P, _P])
_route_ex = _sig("moe_route_ex", _I, [_P, _P, _I, _I, _I, _I, _I, ctypes.POINTER(MoeRouterGroups),
                                      _P, _P, _P])
_dispatch = _sig("moe_dispatch", _I, [_P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _Z,
                                      _P])
_linear1 = _sig("moe_expert_linear1", _I, [_P, _P, _P, _I, _I, _I, _I,
                                           ctypes.POINTER(MoeWeights), _P, _P, _P, _Z, _P])
_linear2 = _sig("moe_expert_linear2", _I, [_P, _P, _P, _I, _I, _I, _I,
                                           ctypes.POINTER(MoeWeights), _P, _P, _Z, _P])
_fused_ffn = _sig("moe_fused_ffn", _I, [_P, _P, _P, _I, _I, _I, _I, ctypes.POINTER(MoeWeights),
                                        _P, _P, _Z, _P])
_dispatch_noalloc = _sig("moe_dispatch_noalloc", _I, [_P, _P, _I, _I, _I, _I, _I, _P, _P, _P,
                                                      _P, _P, _P, _P])
_dispatch_quant = _sig("moe_dispatch_quant", _I, [_P, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P,
                                                  _Z, _P])
_combine = _sig("moe_combine", _I, [_P, _I, _P, _P, _I, _I, _I, _P, _I, _P])
_forward = _sig("moe_forward", _I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I,
                                    ctypes.POINTER(MoeWeights), _P, _P, _P, _P, _P, _Z, _P])
_forward_ex = _sig("moe_forward_ex", _I, [_P, _P, _P, _P, _I, _I, ctypes.POINTER(MoeRouterGroups),
                                          _I, _I, _I, _I, _I, ctypes.POINTER(MoeWeights), _P, _P,
                                          _P, _P, _P, _Z, _P])
_transpose = _sig("moe_transpose_experts", _I, [_P, _I, _I, _I, _I, _P, _P])
_backward = _sig("moe_expert_backward", _I, [ctypes.POINTER(MoeBackwardArgs), _P, _Z, _P])
_ws_size = _sig("moe_workspace_size", _Z, [_I, _I, _I, _I, _I, _I, _I, _I])
_get_err = _sig("moe_get_device_error", _I, [_P, ctypes.POINTER(ctypes.c_int)])
_status_string = _sig("moe_status_string", ctypes.c_char_p, [_I])
_launch_count = _sig("moe_launch_count", ctypes.c_uint64, [])
_set_tiles = _sig("moe_set_gemm_tiles", _I, [_I])
_set_wait_limit = _sig("moe_set_wait_limit", _I, [ctypes.c_longlong])
_selftest_wait = _sig("moe_selftest_wait", _I, [_I, _P])


class MoeError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {moe_status_string(status)} ({status})")
        self.status = status


def moe_status_string(status: int) -> str:
    return _status_string(status).decode()


def moe_launch_count() -> int:
    return int(_launch_count())


TILES = {"auto": 0, "single": 1, "pair": 2, "small": 3}


def moe_set_gemm_tiles(mode="auto"):
    """Process-wide tile shape of the expert GEMMs: 'auto', 'single' (128-row tiles, one
    CTA), 'pair' (256-row tiles, 2-CTA cluster) or 'small' (32-row tiles, one CTA)."""
    _check(_set_tiles(TILES[mode] if isinstance(mode, str) else mode), "moe_set_gemm_tiles")


def moe_set_wait_limit(cycles=0):
    """Limit of every bounded wait in the library's kernels on the current device, in SM
    clock cycles (0: the default, about one second)."""
    _check(_set_wait_limit(int(cycles)), "moe_set_wait_limit")


SELFTEST = {"mbarrier": 0, "grid_barrier": 1}


def moe_selftest_wait(kind, stream=None):
    """Launch a kernel whose bounded wait runs out by construction ('mbarrier' or
    'grid_barrier'); read the recorded timeout with moe_get_device_error()."""
    _check(_selftest_wait(SELFTEST[kind], _stream(stream)), "moe_selftest_wait")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(st, what):
    if st != MOE_OK:
        raise MoeError(st, what)


def _act_torch_dtype(act):
    return {"f32": torch.float32, "bf16": torch.bfloat16, "e4m3": torch.uint8}[act]


def moe_workspace_size(op, T, H, E, k, I, act, wt) -> int:
    return int(_ws_size(OPS[op] if isinstance(op, str) else op, T, H, E, k, I, DTYPES[act],
                        DTYPES[wt]))


def moe_get_device_error(stream=None):
    """(status, site) of the calling device's error word (synchronises the stream)."""
    site = ctypes.c_int(0)
    st = _get_err(_stream(stream), ctypes.byref(site))
    return st, site.value


def workspace(nbytes: int, device) -> torch.Tensor:
    """A 256-byte aligned byte buffer (torch's allocator aligns to at least 512 bytes)."""
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


class Weights:
    """Expert weights in the library's layout (see include/moe.h); holds the tensors alive."""

    def __init__(self, act, wt, w1, w2, w1_scales=None, w2_scales=None, scale_fmt="pow2"):
        """scale_fmt: 'pow2' (fp32 block scales that are powers of two: the UE8M0 fast path)
        or 'fp32' (any positive finite fp32 scales; E4M3 weights only)."""
        self.act, self.wt = act, wt
        self.w1, self.w2, self.w1_scales, self.w2_scales = w1, w2, w1_scales, w2_scales
        self.scale_fmt = scale_fmt
        self.E = w1.shape[0]
        self.H = w1.shape[2] * (2 if wt == "e2m1" else 1)
        self.I = w2.shape[2] * (2 if wt == "e2m1" else 1)
        self.c = MoeWeights(DTYPES[act], DTYPES[wt], w1.data_ptr(),
                            None if w1_scales is None else w1_scales.data_ptr(), w2.data_ptr(),
                            None if w2_scales is None else w2_scales.data_ptr(),
                            SCALE_FMTS[scale_fmt])


def _groups(groups):
    """(n_group, topk_group, scale) -> a moe_router_groups the call can point at."""
    n_group, topk_group, scale = groups
    return MoeRouterGroups(int(n_group), int(topk_group), float(scale))


def moe_route(logits, k, score="softmax", bias=None, renorm=True, topk_idx=None, topk_w=None,
              stream=None, groups=None):
    """Top-k routing.  groups=(n_group, topk_group, scale) selects group-limited routing with
    a routed scaling factor (moe_route_ex)."""
    T, E = logits.shape
    if topk_idx is None:
        topk_idx = torch.empty((T, k), dtype=torch.int32, device=logits.device)
    if topk_w is None:
        topk_w = torch.empty((T, k), dtype=torch.float32, device=logits.device)
    if groups is None:
        _check(_route(_ptr(logits), _ptr(bias), T, E, k, SCORES[score], int(renorm),
                      _ptr(topk_idx), _ptr(topk_w), _stream(stream)), "moe_route")
    else:
        g = _groups(groups)
        _check(_route_ex(_ptr(logits), _ptr(bias), T, E, k, SCORES[score], int(renorm),
                         ctypes.byref(g), _ptr(topk_idx), _ptr(topk_w), _stream(stream)),
               "moe_route_ex")
    return topk_idx, topk_w


def moe_dispatch(x, topk_idx, E, act, x_scales=None, ws=None, out=None, stream=None):
    """Returns dict(x_perm, x_perm_scales, expert_offsets, perm_src, slot_of)."""
    T, H = x.shape
    k = topk_idx.shape[1]
    S = T * k
    dev = x.device
    o = out or {}
    x_perm = o.get("x_perm")
    if x_perm is None:
        x_perm = torch.empty((S, H), dtype=x.dtype, device=dev)
    xps = o.get("x_perm_scales")
    if xps is None and act == "e4m3":
        xps = torch.empty((S, H // 128), dtype=torch.float32, device=dev)
    offs = o.get("expert_offsets")
    if offs is None:
        offs = torch.empty(E + 1, dtype=torch.int32, device=dev)
    perm_src = o.get("perm_src")
    if perm_src is None:
        perm_src = torch.empty(S, dtype=torch.int32, device=dev)
    slot_of = o.get("slot_of")
    if slot_of is None:
        slot_of = torch.empty(S, dtype=torch.int32, device=dev)
    need = moe_workspace_size("dispatch", T, H, E, k, 128, act, act if act != "e4m3" else "e4m3")
    if ws is None:
        ws = workspace(need, dev)
    _check(_dispatch(_ptr(x), _ptr(x_scales), DTYPES[act], T, H, E, k, _ptr(topk_idx),
                     _ptr(x_perm), _ptr(xps), _ptr(offs), _ptr(perm_src), _ptr(slot_of),
                     _ptr(ws), ws.numel(), _stream(stream)), "moe_dispatch")
    return dict(x_perm=x_perm, x_perm_scales=xps, expert_offsets=offs, perm_src=perm_src,
                slot_of=slot_of)


def moe_expert_linear1(x_perm, expert_offsets, W: Weights, x_perm_scales=None, h=None,
                       h_scales=None, stream=None):
    S = x_perm.shape[0]
    dev = x_perm.device
    if h is None:
        h = torch.empty((S, W.I), dtype=_act_torch_dtype(W.act), device=dev)
    if h_scales is None and W.act == "e4m3":
        h_scales = torch.empty((S, W.I // 128), dtype=torch.float32, device=dev)
    _check(_linear1(_ptr(x_perm), _ptr(x_perm_scales), _ptr(expert_offsets), S, W.H, W.I, W.E,
                    ctypes.byref(W.c), _ptr(h), _ptr(h_scales), None, 0, _stream(stream)),
           "moe_expert_linear1")
    return h, h_scales


def moe_expert_linear2(h, expert_offsets, W: Weights, h_scales=None, y=None, stream=None):
    S = h.shape[0]
    if y is None:
        y = torch.empty((S, W.H), dtype=torch.float32 if W.act == "f32" else torch.bfloat16,
                        device=h.device)
    _check(_linear2(_ptr(h), _ptr(h_scales), _ptr(expert_offsets), S, W.H, W.I, W.E,
                    ctypes.byref(W.c), _ptr(y), None, 0, _stream(stream)), "moe_expert_linear2")
    return y


def moe_fused_ffn(x_perm, expert_offsets, W: Weights, x_perm_scales=None, y=None, ws=None,
                  k=1, stream=None):
    S = x_perm.shape[0]
    dev = x_perm.device
    if y is None:
        y = torch.empty((S, W.H), dtype=torch.float32 if W.act == "f32" else torch.bfloat16,
                        device=dev)
    need = moe_workspace_size("fused_ffn", S, W.H, W.E, 1, W.I, W.act, W.wt)
    if ws is None:
        ws = workspace(need, dev)
    _check(_fused_ffn(_ptr(x_perm), _ptr(x_perm_scales), _ptr(expert_offsets), S, W.H, W.I, W.E,
                      ctypes.byref(W.c), _ptr(y), _ptr(ws), ws.numel(), _stream(stream)),
           "moe_fused_ffn")
    return y


def moe_combine(y, slot_of, topk_w, out=None, out_dtype=None, stream=None):
    T, k = topk_w.shape
    H = y.shape[1]
    ydt = "f32" if y.dtype == torch.float32 else "bf16"
    odt = out_dtype or ydt
    if out is None:
        out = torch.empty((T, H), dtype=torch.float32 if odt == "f32" else torch.bfloat16,
                          device=y.device)
    _check(_combine(_ptr(y), DTYPES[ydt], _ptr(slot_of), _ptr(topk_w), T, k, H, _ptr(out),
                    DTYPES[odt], _stream(stream)), "moe_combine")
    return out


def moe_forward(x, logits, W: Weights, k, score="softmax", bias=None, renorm=True,
                x_scales=None, out=None, ws=None, topk_idx=None, topk_w=None,
                expert_offsets=None, stream=None, groups=None):
    """The whole layer.  For an E4M3 layer, x is either E4M3 codes with x_scales, or BF16 with
    x_scales=None (quantised by the dispatch).  groups=(n_group, topk_group, scale) routes as
    moe_route does with the same argument (moe_forward_ex)."""
    T, H = x.shape
    E = logits.shape[1]
    dev = x.device
    if out is None:
        out = torch.empty((T, H), dtype=torch.float32 if W.act == "f32" else torch.bfloat16,
                          device=dev)
    need = moe_workspace_size("forward", T, H, E, k, W.I, W.act, W.wt)
    if ws is None:
        ws = workspace(need, dev)
    if groups is None:
        _check(_forward(_ptr(x), _ptr(x_scales), _ptr(logits), _ptr(bias), SCORES[score],
                        int(renorm), T, H, E, k, W.I, ctypes.byref(W.c), _ptr(out),
                        _ptr(topk_idx), _ptr(topk_w), _ptr(expert_offsets), _ptr(ws), ws.numel(),
                        _stream(stream)), "moe_forward")
    else:
        g = _groups(groups)
        _check(_forward_ex(_ptr(x), _ptr(x_scales), _ptr(logits), _ptr(bias), SCORES[score],
                           int(renorm), ctypes.byref(g), T, H, E, k, W.I, ctypes.byref(W.c),
                           _ptr(out), _ptr(topk_idx), _ptr(topk_w), _ptr(expert_offsets),
                           _ptr(ws), ws.numel(), _stream(stream)), "moe_forward_ex")
    return out


def moe_dispatch_quant(x, topk_idx, E, ws=None, out=None, stream=None):
    """Dispatch of BF16 rows x [T, H] into an E4M3 layer, quantising on the way (1x128
    power-of-two scales).  Returns dict(x_perm (E4M3 codes, uint8), x_perm_scales,
    expert_offsets, perm_src, slot_of); tensors given in `out` are written in place."""
    T, H = x.shape
    k = topk_idx.shape[1]
    S = T * k
    dev = x.device
    o = out or {}
    shapes = {"x_perm": ((S, H), torch.uint8), "x_perm_scales": ((S, H // 128), torch.float32),
              "expert_offsets": ((E + 1,), torch.int32), "perm_src": ((S,), torch.int32),
              "slot_of": ((S,), torch.int32)}
    r = {key: (o[key] if o.get(key) is not None else torch.empty(shp, dtype=dt, device=dev))
         for key, (shp, dt) in shapes.items()}
    need = moe_workspace_size("dispatch", T, H, E, k, 128, "e4m3", "e4m3")
    if ws is None:
        ws = workspace(need, dev)
    _check(_dispatch_quant(_ptr(x), T, H, E, k, _ptr(topk_idx), _ptr(r["x_perm"]),
                           _ptr(r["x_perm_scales"]), _ptr(r["expert_offsets"]),
                           _ptr(r["perm_src"]), _ptr(r["slot_of"]), _ptr(ws), ws.numel(),
                           _stream(stream)), "moe_dispatch_quant")
    return r


def moe_dispatch_noalloc(x, topk_idx, E, act, out, x_scales=None, stream=None):
    """moe_dispatch for callers that cannot allocate device memory: the library's built-in
    scratch buffer replaces the workspace.  `out` must hold every output tensor (x_perm,
    x_perm_scales for E4M3, expert_offsets, perm_src, slot_of); nothing is allocated here."""
    T, H = x.shape
    k = topk_idx.shape[1]
    _check(_dispatch_noalloc(_ptr(x), _ptr(x_scales), DTYPES[act], T, H, E, k, _ptr(topk_idx),
                             _ptr(out["x_perm"]), _ptr(out.get("x_perm_scales")),
                             _ptr(out["expert_offsets"]), _ptr(out["perm_src"]),
                             _ptr(out["slot_of"]), _stream(stream)), "moe_dispatch_noalloc")
    return out


_ELEM_DTYPE = {torch.float32: "f32", torch.bfloat16: "bf16", torch.uint8: "e4m3"}


def moe_transpose_experts(src, out=None, stream=None):
    """dst[e] = src[e]^T for a [E, R, C] tensor (fp32, BF16 or one-byte codes)."""
    E, R, C = src.shape
    if out is None:
        out = torch.empty((E, C, R), dtype=src.dtype, device=src.device)
    _check(_transpose(_ptr(src), DTYPES[_ELEM_DTYPE[src.dtype]], E, R, C, _ptr(out),
                      _stream(stream)), "moe_transpose_experts")
    return out


def moe_expert_backward(dout, logits, topk_idx, topk_w, expert_offsets, slot_of, x_perm, h, y,
                        W: Weights, w1_t, w2_t, k, score="softmax", renorm=True, scale=1.0,
                        ws=None, stream=None):
    """Backward of the BF16 layer from the forward's tensors (see include/moe.h); w1_t, w2_t
    are moe_transpose_experts of W.w1, W.w2.  Returns dict(dx, dw1, dw2, dlogits)."""
    T, H = dout.shape
    E = logits.shape[1]
    I = h.shape[1]
    dev = dout.device
    g = dict(dx=torch.empty((T, H), dtype=torch.bfloat16, device=dev),
             dw1=torch.empty((E, 2 * I, H), dtype=torch.float32, device=dev),
             dw2=torch.empty((E, H, I), dtype=torch.float32, device=dev),
             dlogits=torch.empty((T, E), dtype=torch.float32, device=dev))
    a = MoeBackwardArgs(T, H, E, k, I, SCORES[score], int(bool(renorm)), float(scale),
                        _ptr(dout), _ptr(logits), _ptr(topk_idx), _ptr(topk_w),
                        _ptr(expert_offsets), _ptr(slot_of), _ptr(x_perm), _ptr(h), _ptr(y),
                        _ptr(W.w1), _ptr(W.w2), _ptr(w1_t), _ptr(w2_t), _ptr(g["dx"]),
                        _ptr(g["dw1"]), _ptr(g["dw2"]), _ptr(g["dlogits"]))
    need = moe_workspace_size("backward", T, H, E, k, I, "bf16", "bf16")
    if ws is None:
        ws = workspace(need, dev)
    _check(_backward(ctypes.byref(a), _ptr(ws), ws.numel(), _stream(stream)),
           "moe_expert_backward")
    return g

