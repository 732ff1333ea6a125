"""moe_layer_backward (the layer's backward pass with the forward's expert
selection held fixed) against the fp64 backward oracle: every gradient (x and
each weight) element by element, on the tiny fp32 layer, the mid bf16 layer
and a slice of the K3 shape (H=7168, L=3584, I=3072, 2 shared experts) with 20
experts."""
import numpy as np
import pytest
import torch

import gen
import sparse_moe_layer_renormalised_b200 as moe
from harness import dims_for, parity
from oracle import backward_oracle as bo
from oracle import inputs as oin

pytestmark = pytest.mark.gpu
F64 = torch.float64
GRADS = ("dx", "dWr", "dWdown", "dWup", "dgamma", "dWg", "dWv", "dWo", "dWsg", "dWsv", "dWso")
# fp32 recomputation and accumulation against the exact fp64 gradient
TOL_GRAD = 1e-3


def _run(cfg, T):
    cfg = cfg.with_(T=T)
    w = gen.device_layer(cfg, "cuda")
    x = w.pop("x")
    layer = moe.MoeLayer(dims_for(cfg), w)
    idx = torch.empty(T, cfg.k, dtype=torch.int32, device="cuda")
    layer.forward(x, aux={"topk_idx": idx})
    dy = torch.randn(T, cfg.H, generator=torch.Generator().manual_seed(T + cfg.E)).to(torch.float32)
    shapes = {"dx": (T, cfg.H), "dWr": (cfg.E, cfg.H), "dWdown": (cfg.L, cfg.H), "dWup": (cfg.H, cfg.L),
              "dgamma": (cfg.L,), "dWg": (cfg.E, cfg.I, cfg.L), "dWv": (cfg.E, cfg.I, cfg.L),
              "dWo": (cfg.E, cfg.L, cfg.I), "dWsg": (cfg.S, cfg.Is, cfg.H), "dWsv": (cfg.S, cfg.Is, cfg.H),
              "dWso": (cfg.S, cfg.H, cfg.Is)}
    grads = {k: torch.full(v, float("nan"), dtype=torch.float32, device="cuda") for k, v in shapes.items()}
    d = dims_for(cfg)
    ws = torch.empty(moe.moe_backward_workspace_size(d), dtype=torch.uint8, device="cuda")
    assert moe.moe_layer_backward(d, layer._w, x, dy.cuda(), idx, moe.make_grads(**grads), ws) == moe.MOE_OK
    torch.cuda.synchronize()
    st, code = moe.moe_device_error()
    assert st == moe.MOE_OK and code == 0, f"device fault {code}"
    wref = oin.all_weights(cfg)
    ref = bo.layer_backward(cfg, wref, oin.x_rows(cfg, np.arange(T)), dy.to(F64), idx.cpu().to(torch.int64))
    out = {}
    scale = float(ref["dx"].pow(2).mean().sqrt())
    for k in GRADS:
        got = grads[k].cpu().to(F64)
        assert torch.isfinite(got).all(), k
        if float(ref[k].pow(2).mean().sqrt()) < 1e-12 * scale:
            # an exactly zero gradient (e.g. the router's when k = 1: p = 1
            # whatever the scores); the oracle's is rounding noise
            out[k] = float(got.abs().max()) / scale
            assert out[k] <= 1e-6, f"{cfg.name} {k}: should vanish, max|d| = {out[k]:.3g} of rms(dx)"
            continue
        out[k] = parity(got, ref[k])
        assert out[k] <= TOL_GRAD, f"{cfg.name} {k}: max|d|/rms = {out[k]:.3g}"
    # experts that no token selected get exactly zero gradients
    used = torch.zeros(cfg.E, dtype=torch.bool)
    used[idx.cpu().long().unique()] = True
    for k in ("dWg", "dWv", "dWo"):
        assert bool((grads[k].cpu()[~used] == 0).all()), k
    print(f"\n[{cfg.name} T={T}] " + " ".join(f"{k}={v:.2e}" for k, v in out.items()))
    return out


def test_backward_tiny_fp32():
    _run(gen.CONFIGS["tiny"], 64)
    _run(gen.CONFIGS["tiny"].with_(gamma="normal", k=1), 37)


def test_backward_mid_bf16():
    _run(gen.CONFIGS["mid"], 48)


@pytest.mark.slow
def test_backward_k3_shape_slice():
    """K3 matrix shapes with 20 routed experts (top-16), 3 tokens: the oracle
    needs every routed weight in fp64, so the expert count is cut."""
    _run(gen.CONFIGS["decode"].with_(E=20), 3)
