"""Pins of the backward oracle (oracle.backward) to things other than itself: central finite
differences of the fp64 forward, an independent torch-autograd formulation in fp64, and
closed forms / invariants of the gate functions and SwiGLU."""
import numpy as np
import pytest
import torch

import oracle
from oracle import backward as B


def _instance(seed, T=5, H=6, I=4, E=4, k=2, score="softmax", bias=False):
    """A tiny fp64 layer whose selection keys are at least 1e-3 apart (so that a 1e-6
    perturbation of a logit never changes the selection)."""
    rng = np.random.default_rng(seed)
    while True:
        logits = rng.standard_normal((T, E))
        b = rng.standard_normal(E) * 0.1 if bias else None
        keys = np.asarray(logits, np.float32).astype(np.float64)
        if score == "sigmoid":
            keys = 1.0 / (1.0 + np.exp(-keys)) + (0.0 if b is None else b)
        gaps = np.diff(np.sort(keys, axis=1), axis=1)
        if gaps.min() > 1e-3:
            break
    x = rng.standard_normal((T, H))
    w1 = rng.standard_normal((E, 2 * I, H)) / np.sqrt(H)
    w2 = rng.standard_normal((E, H, I)) / np.sqrt(I)
    dout = rng.standard_normal((T, H))
    return dict(x=x, logits=logits, bias=b, w1=w1, w2=w2, dout=dout, k=k)


def _loss(inst, score, renorm, groups, **over):
    a = {**inst, **over}
    out = B.forward_values(a["x"], a["logits"], a["bias"], a["w1"], a["w2"], a["k"], score,
                           renorm, *groups)
    return float(np.sum(inst["dout"] * out))


CASES = [
    ("softmax", True, (1, 0, 1.0), dict()),
    ("softmax", False, (1, 0, 1.0), dict()),
    ("sigmoid", True, (1, 0, 1.0), dict(bias=True)),
    ("sigmoid", False, (1, 0, 1.0), dict(bias=True)),
    ("sigmoid", True, (4, 2, 2.5), dict(E=8, k=3, bias=True)),   # grouped + scaling factor
    ("softmax", True, (2, 1, 0.5), dict(E=8, k=3)),
    ("softmax", False, (2, 1, 0.5), dict(E=8, k=3)),
    ("sigmoid", False, (1, 0, 1.5), dict(bias=True)),
]


@pytest.mark.parametrize("score,renorm,groups,shape", CASES)
def test_backward_matches_finite_differences(score, renorm, groups, shape):
    inst = _instance(7, score=score, **shape)
    g = B.backward_values(inst["x"], inst["logits"], inst["bias"], inst["w1"], inst["w2"],
                          inst["k"], score, inst["dout"], renorm, *groups)
    rng = np.random.default_rng(1)
    eps = 1e-6
    for name, grad in (("x", g["dx"]), ("w1", g["dw1"]), ("w2", g["dw2"]),
                       ("logits", g["dlogits"])):
        base = inst[name]
        for _ in range(12):
            pos = tuple(int(rng.integers(0, n)) for n in base.shape)
            up, dn = base.copy(), base.copy()
            up[pos] += eps
            dn[pos] -= eps
            fd = (_loss(inst, score, renorm, groups, **{name: up}) -
                  _loss(inst, score, renorm, groups, **{name: dn})) / (2 * eps)
            assert abs(fd - grad[pos]) <= 1e-6 * max(1.0, abs(fd)), (name, pos, fd, grad[pos])


def _torch_layer(inst, score, renorm, idx, scale):
    """The same layer written with torch ops over the fixed selection, for autograd."""
    x = torch.tensor(inst["x"], requires_grad=True)
    l = torch.tensor(inst["logits"], requires_grad=True)
    w1 = torch.tensor(inst["w1"], requires_grad=True)
    w2 = torch.tensor(inst["w2"], requires_grad=True)
    ii = torch.tensor(idx, dtype=torch.long)
    if score == "softmax":
        gates = (torch.softmax(l.gather(1, ii), dim=1) if renorm
                 else torch.softmax(l, dim=1).gather(1, ii))
    else:
        s = torch.sigmoid(l.gather(1, ii))
        gates = s / s.sum(dim=1, keepdim=True) if renorm else s
    gates = gates * scale
    I = inst["w1"].shape[1] // 2
    W1 = w1[ii]                                   # [T, k, 2I, H]
    W2 = w2[ii]                                   # [T, k, H, I]
    gu = torch.einsum("tkoh,th->tko", W1, x)
    h = torch.nn.functional.silu(gu[..., :I]) * gu[..., I:]
    y = torch.einsum("tkhi,tki->tkh", W2, h)
    out = (gates[..., None] * y).sum(dim=1)
    (out * torch.tensor(inst["dout"])).sum().backward()
    return x.grad.numpy(), w1.grad.numpy(), w2.grad.numpy(), l.grad.numpy()


@pytest.mark.parametrize("score,renorm,groups,shape", CASES)
def test_backward_matches_torch_autograd(score, renorm, groups, shape):
    inst = _instance(11, T=9, H=16, I=8, score=score, **shape)
    g = B.backward_values(inst["x"], inst["logits"], inst["bias"], inst["w1"], inst["w2"],
                          inst["k"], score, inst["dout"], renorm, *groups)
    tx, tw1, tw2, tl = _torch_layer(inst, score, renorm, g["topk_idx"], groups[2])
    for mine, ref in ((g["dx"], tx), (g["dw1"], tw1), (g["dw2"], tw2), (g["dlogits"], tl)):
        assert np.allclose(mine, ref, rtol=1e-10, atol=1e-12)
    if g["dbias"] is not None:
        assert not np.any(g["dbias"])


def test_swiglu_grad_closed_forms():
    u = np.array([0.5, -2.0, 3.0])
    dh = np.array([1.0, 0.25, -1.5])
    dg, du = B.swiglu_grad(np.zeros(3), u, dh)           # sigma(0) = 1/2, silu(0) = 0
    assert np.array_equal(dg, dh * u / 2) and np.array_equal(du, np.zeros(3))
    dg, du = B.swiglu_grad(np.full(3, 60.0), u, dh)      # sigma -> 1: silu(g) -> g
    assert np.allclose(dg, dh * u, rtol=1e-15) and np.allclose(du, dh * 60.0, rtol=1e-15)
    dg, du = B.swiglu_grad(np.full(3, -60.0), u, dh)     # sigma -> 0: everything -> 0
    assert np.all(np.abs(dg) < 1e-20) and np.all(np.abs(du) < 1e-20)


@pytest.mark.parametrize("score", ["softmax", "sigmoid"])
def test_renormalised_gates_ignore_a_common_shift(score):
    """Renormalised gates sum to the scaling factor, so adding the same amount to every
    selected gate's gradient leaves the logit gradient unchanged; k = 1 gates are constant."""
    rng = np.random.default_rng(3)
    logits = rng.standard_normal((6, 10))
    idx, _ = oracle.route(logits, None, 4, score, True)
    dw = rng.standard_normal((6, 4))
    a = B.gate_grad(logits, idx, dw, score, True, 1.7)
    b = B.gate_grad(logits, idx, dw + 3.0, score, True, 1.7)
    assert np.allclose(a, b, atol=1e-14)
    idx1, _ = oracle.route(logits, None, 1, score, True)
    assert not np.any(B.gate_grad(logits, idx1, dw[:, :1], score, True))


def test_shared_experts_reduce_to_the_dense_ffn():
    """With every expert holding the same weights and renormalised gates, the layer is the
    dense SwiGLU FFN: no gradient reaches the logits, and dx, the summed dW1, dW2 are the
    dense FFN's gradients (torch autograd of the dense FFN)."""
    inst = _instance(5, T=7, H=12, I=6, E=5, k=3)
    inst["w1"][:] = inst["w1"][0]
    inst["w2"][:] = inst["w2"][0]
    g = B.backward_values(inst["x"], inst["logits"], None, inst["w1"], inst["w2"], 3,
                          "softmax", inst["dout"])
    assert np.all(np.abs(g["dlogits"]) < 1e-12)
    x = torch.tensor(inst["x"], requires_grad=True)
    w1 = torch.tensor(inst["w1"][0], requires_grad=True)
    w2 = torch.tensor(inst["w2"][0], requires_grad=True)
    gu = x @ w1.T
    out = (torch.nn.functional.silu(gu[:, :6]) * gu[:, 6:]) @ w2.T
    (out * torch.tensor(inst["dout"])).sum().backward()
    assert np.allclose(g["dx"], x.grad.numpy(), rtol=1e-10, atol=1e-12)
    assert np.allclose(g["dw1"].sum(0), w1.grad.numpy(), rtol=1e-10, atol=1e-12)
    assert np.allclose(g["dw2"].sum(0), w2.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_unpicked_experts_get_no_gradient():
    inst = _instance(9, T=3, E=8, k=2)
    g = B.backward_values(inst["x"], inst["logits"], None, inst["w1"], inst["w2"], 2,
                          "softmax", inst["dout"])
    picked = np.zeros(8, bool)
    picked[np.unique(g["topk_idx"])] = True
    assert not picked.all()
    assert not np.any(g["dw1"][~picked]) and not np.any(g["dw2"][~picked])
    assert np.all(np.any(g["dw1"][picked].reshape(picked.sum(), -1), axis=1))


def test_forward_exact_is_the_oracle_forward_before_rounding():
    """forward_exact (the function the backward differentiates) and the oracle's forward
    differ only by the fp32 storage of y and out (f32 layer)."""
    rng = np.random.default_rng(2)
    T, H, I, E, k = 16, 128, 128, 6, 2
    L = oracle.Layer("f32", "f32", "softmax", True, k,
                     rng.standard_normal((T, H)).astype(np.float32), None,
                     rng.standard_normal((T, E)).astype(np.float32), None,
                     (rng.standard_normal((E, 2 * I, H)) / np.sqrt(H)).astype(np.float32), None,
                     (rng.standard_normal((E, H, I)) / np.sqrt(I)).astype(np.float32), None)
    a = B.forward_exact(L)
    b = oracle.forward(L)
    assert np.max(np.abs(a - b)) <= 1e-6 * np.sqrt(np.mean(b * b))
    g = B.layer_backward(L, rng.standard_normal((T, H)))
    assert g["dx"].shape == (T, H) and g["dw1"].shape == (E, 2 * I, H)


def _bf16_layer(seed, score="softmax", renorm=True, bias=False, T=40, H=256, E=6, k=2, I=128):
    import synth
    from tests.util import oracle_layer
    wl = synth.WORKLOADS["mixtral_bf16"].scaled(T=T, H=H, E=E, k=k, I=I, score=score,
                                                bias=bias, renorm=renorm)
    d = synth.make_inputs(wl, "cpu")
    L = oracle_layer(wl, d)
    dout = oracle.round_bf16(np.random.default_rng(seed).standard_normal((T, H)))
    return L, dout


@pytest.mark.parametrize("score,renorm,bias", [("softmax", True, False),
                                               ("softmax", False, False),
                                               ("sigmoid", True, True)])
def test_stored_backward_without_rounding_is_the_exact_backward(score, renorm, bias):
    L, dout = _bf16_layer(4, score, renorm, bias)
    a = B.layer_backward_stored(L, dout, store=lambda v: v)
    b = B.layer_backward(L, dout)
    assert np.array_equal(a["topk_idx"], b["topk_idx"])
    for n in ("dx", "dw1", "dw2", "dlogits"):
        # the only difference: the gates stored as fp32
        assert np.allclose(a[n], b[n], rtol=1e-6, atol=1e-6 * np.abs(b[n]).max()), n


def test_stored_backward_is_close_to_the_exact_backward():
    """BF16 storage of the intermediates moves every gradient by well under 1 % (rel-L2)."""
    L, dout = _bf16_layer(5)
    a = B.layer_backward_stored(L, dout)
    b = B.layer_backward(L, dout)
    for n in ("dx", "dw1", "dw2", "dlogits"):
        rel = np.sqrt(np.sum((a[n] - b[n]) ** 2) / np.sum(b[n] ** 2))
        assert 0 < rel < 1e-2, (n, rel)


def test_stored_backward_slots_are_what_the_weight_gradients_sum():
    """The per-slot values the stored backward returns for the GPU tests' rounding allowance
    are the ones its weight gradients were summed from: dW1_e = dG_e^T x_e and
    dW2_e = dy_w,e^T h_e over each expert's rows, every value on the BF16 grid, and dG
    carrying the SwiGLU backward of dh (both halves zero where dh is zero)."""
    L, dout = _bf16_layer(6, E=5)
    r = B.layer_backward_stored(L, dout, return_slots=True)
    s, offs = r["slots"], r["offsets"]
    assert set(s) == {"dG", "x", "dy_w", "h", "dh"}
    for n, v in s.items():
        assert np.array_equal(oracle.round_bf16(v), v), n
    I = s["h"].shape[1]
    for e in range(L.E):
        a, b = int(offs[e]), int(offs[e + 1])
        assert np.allclose(s["dG"][a:b].T @ s["x"][a:b], r["dw1"][e], rtol=0, atol=1e-9)
        assert np.allclose(s["dy_w"][a:b].T @ s["h"][a:b], r["dw2"][e], rtol=0, atol=1e-9)
    zero = s["dh"] == 0
    assert np.all(s["dG"][:, :I][zero] == 0) and np.all(s["dG"][:, I:][zero] == 0)
    # without return_slots the result is the same, minus the slots
    r0 = B.layer_backward_stored(L, dout)
    assert "slots" not in r0
    for n in ("dx", "dw1", "dw2", "dlogits"):
        assert np.array_equal(r0[n], r[n]), n
