"""Pins of the backward-pass oracle (no GPU): central finite differences of
the fixed-selection layer function, and closed forms that a slip in the
router, combine, RMSNorm or output gradients would break."""
from dataclasses import dataclass

import numpy as np
import torch

from oracle import backward_oracle as bo
from oracle.moe_oracle import F64, rms_norm, router_scores, select_experts

torch.manual_seed(0)


@dataclass
class _Dims:
    T: int = 4
    H: int = 8
    L: int = 6
    E: int = 5
    k: int = 2
    I: int = 4
    S: int = 1
    Is: int = 4
    situ_c: float = 10.0
    rms_eps: float = 1e-6


def _weights(d, rng, identical_experts=False):
    def r(*shape, scale=0.5):
        return torch.as_tensor(rng.standard_normal(shape) * scale, dtype=F64)

    w = {"Wr": r(d.E, d.H), "bias": r(d.E, scale=0.05), "Wdown": r(d.L, d.H), "Wup": r(d.H, d.L),
         "gamma": 1.0 + r(d.L, scale=0.1), "Wsg": r(d.S, d.Is, d.H), "Wsv": r(d.S, d.Is, d.H),
         "Wso": r(d.S, d.H, d.Is)}
    if identical_experts:
        g, v, o = r(d.I, d.L), r(d.I, d.L), r(d.L, d.I)
        w["Wg"], w["Wv"], w["Wo"] = (t.expand(d.E, *t.shape).clone() for t in (g, v, o))
    else:
        w["Wg"], w["Wv"], w["Wo"] = r(d.E, d.I, d.L), r(d.E, d.I, d.L), r(d.E, d.L, d.I)
    return w


def _loss(d, w, x, dy, idx):
    return float((bo.layer_forward_fixed(d, w, x, idx)["y"] * dy).sum())


def test_gradients_match_central_differences():
    d = _Dims()
    rng = np.random.default_rng(1)
    w = _weights(d, rng)
    x = torch.as_tensor(rng.standard_normal((d.T, d.H)), dtype=F64)
    dy = torch.as_tensor(rng.standard_normal((d.T, d.H)), dtype=F64)
    g = bo.layer_backward(d, w, x, dy)
    idx = g["idx"]
    h = 1e-6
    for name in ("x",) + bo.PARAMS:
        base = x if name == "x" else w[name]
        grad = g["dx"] if name == "x" else g["d" + name]
        flat = base.reshape(-1)
        for pos in rng.choice(flat.numel(), size=min(6, flat.numel()), replace=False):
            orig = float(flat[pos])
            vals = []
            for sgn in (1.0, -1.0):
                flat[pos] = orig + sgn * h
                vals.append(_loss(d, w, x, dy, idx))
            flat[pos] = orig
            fd = (vals[0] - vals[1]) / (2 * h)
            an = float(grad.reshape(-1)[pos])
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(fd)), (name, int(pos), fd, an)


def test_top1_router_gets_no_gradient():
    """k = 1: p = 1 whatever the scores, so W_r receives nothing."""
    d = _Dims(k=1)
    rng = np.random.default_rng(2)
    w = _weights(d, rng)
    x = torch.as_tensor(rng.standard_normal((d.T, d.H)), dtype=F64)
    g = bo.layer_backward(d, w, x, torch.ones(d.T, d.H, dtype=F64))
    # d(s/s)/ds vanishes up to the rounding of its two terms
    assert g["dWr"].abs().max() < 1e-12 * max(1.0, g["dWg"].abs().max())


def test_identical_experts_give_the_router_no_gradient():
    """All experts equal: u = E(z) for any p with sum p = 1, so dW_r = 0."""
    d = _Dims()
    rng = np.random.default_rng(3)
    w = _weights(d, rng, identical_experts=True)
    x = torch.as_tensor(rng.standard_normal((d.T, d.H)), dtype=F64)
    dy = torch.as_tensor(rng.standard_normal((d.T, d.H)), dtype=F64)
    g = bo.layer_backward(d, w, x, dy)
    assert g["dWr"].abs().max() < 1e-12 * max(1.0, g["dWg"].abs().max())


def test_unselected_experts_get_zero_gradients():
    d = _Dims(E=7, T=2)
    rng = np.random.default_rng(4)
    w = _weights(d, rng)
    x = torch.as_tensor(rng.standard_normal((d.T, d.H)), dtype=F64)
    g = bo.layer_backward(d, w, x, torch.ones(d.T, d.H, dtype=F64))
    used = set(g["idx"].reshape(-1).tolist())
    for e in range(d.E):
        nz = any(torch.count_nonzero(g[n][e]) for n in ("dWg", "dWv", "dWo"))
        assert nz == (e in used)


def test_output_and_gain_gradients_in_closed_form():
    """y = shared(x) + W_up n with n = gamma * u / rms(u): dW_up = dy^T n and
    dgamma = sum_t (W_up^T dy_t) * u_t / rms_t."""
    d = _Dims()
    rng = np.random.default_rng(5)
    w = _weights(d, rng)
    x = torch.as_tensor(rng.standard_normal((d.T, d.H)), dtype=F64)
    dy = torch.as_tensor(rng.standard_normal((d.T, d.H)), dtype=F64)
    g = bo.layer_backward(d, w, x, dy)
    out = bo.layer_forward_fixed(d, w, x, g["idx"])
    u, n = out["u"], out["n"]
    assert torch.allclose(g["dWup"], dy.T @ n, rtol=1e-12, atol=1e-12)
    rms = torch.sqrt((u * u).mean(dim=1, keepdim=True) + d.rms_eps)
    assert torch.allclose(g["dgamma"], ((dy @ w["Wup"]) * u / rms).sum(dim=0), rtol=1e-12, atol=1e-12)
    # the default selection is the forward one
    idx, _, _ = select_experts(router_scores(x, w["Wr"]), w["bias"], d.k)
    assert torch.equal(g["idx"], idx)
    assert torch.allclose(rms_norm(u, w["gamma"], d.rms_eps), n)


def test_gradient_is_linear_in_dy():
    d = _Dims()
    rng = np.random.default_rng(6)
    w = _weights(d, rng)
    x = torch.as_tensor(rng.standard_normal((d.T, d.H)), dtype=F64)
    a = torch.as_tensor(rng.standard_normal((d.T, d.H)), dtype=F64)
    b = torch.as_tensor(rng.standard_normal((d.T, d.H)), dtype=F64)
    ga, gb, gab = (bo.layer_backward(d, w, x, t) for t in (a, b, 2 * a - 3 * b))
    for key in ("dx", "dWr", "dWg", "dWdown"):
        assert torch.allclose(gab[key], 2 * ga[key] - 3 * gb[key], rtol=1e-10, atol=1e-12)


def test_fixed_selection_forward_is_the_pinned_forward():
    """The function the backward oracle differentiates is moe_oracle's layer
    (there with fp32 storage rounding of z, h and n, hence the tolerance)."""
    from oracle.moe_oracle import layer_forward

    @dataclass
    class _Cfg(_Dims):
        act: str = "f32"

    d = _Cfg()
    rng = np.random.default_rng(7)
    w = _weights(d, rng)
    x = torch.as_tensor(rng.standard_normal((d.T, d.H)), dtype=F64)
    ref = layer_forward(d, w, x)
    mine = bo.layer_forward_fixed(d, w, x, ref["idx"])
    scale = ref["y"].abs().max()
    assert torch.allclose(mine["y"], ref["y"], rtol=0, atol=1e-5 * scale)
    assert torch.allclose(mine["p"], ref["p"], rtol=1e-12, atol=0)
