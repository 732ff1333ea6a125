"""fp64 CPU oracle of the layer's BACKWARD pass (test infrastructure only).

What it differentiates: the layer function of moe_oracle.layer_forward with
the expert selection held fixed -- the top-k choice is a discrete function of
the biased keys and has no gradient, while the mixture weights
p_j = s_{e_j} / sum_j' s_{e_j'} are differentiable in the router scores s =
Sigmoid(W_r x).  Gradients therefore reach the router through p only, and the
selection bias gets none (it is set by Quantile Balancing, not by gradients).

Sources (web pages; cited by title and section):
[K3-896] "Kimi K3の896エキスパートを「896人の専門家」と呼ぶと何がズレるか、
         ルーターは何を選んでいるのか" (lilting.ch): section
   "K3のエキスパートは896個の小型LLMではない" (the three layer equations) and
   section "ルーターは計算の割当器" (sigmoid router, bias only in the choice,
   mixture weights from the unbiased scores); section "ルーター専用の独立訓練は
   ない": the router is trained with the model, through the language-model
   loss, and only the bias is set by Quantile Balancing.

Readings (listed in the design notes): the gradient is that of the exact
fp64 function -- the device's storage roundings (bf16 z, h, n) are not part
of it -- and it is the vector-Jacobian product with a given upstream
gradient dy = dLoss/dy.

The derivatives come from torch autograd over the same fp64 building blocks
as the forward oracle; tests/test_oracle_backward.py pins them against
central finite differences and closed forms.
"""
from __future__ import annotations

import torch

from .moe_oracle import F64, combine, expert_forward, rms_norm, router_scores, select_experts, shared_experts

__all__ = ["PARAMS", "layer_forward_fixed", "layer_backward"]

# weights that receive gradients (the bias does not)
PARAMS = ("Wr", "Wdown", "Wup", "gamma", "Wg", "Wv", "Wo", "Wsg", "Wsv", "Wso")


def _identity(t):
    return t


def layer_forward_fixed(dims, w: dict, x: torch.Tensor, idx: torch.Tensor) -> dict:
    """Forward pass (fp64, no storage rounding) with the selection idx [T, k]
    given: s = Sigmoid(W_r x); p = s_sel / sum s_sel; z = W_down x;
    u = sum_j p_j E_{e_j}(z); y = shared(x) + W_up RMSNorm(u)."""
    c, eps = dims.situ_c, dims.rms_eps
    s = router_scores(x, w["Wr"])
    s_sel = torch.gather(s, 1, idx)
    p = s_sel / s_sel.sum(dim=1, keepdim=True)
    z = x @ w["Wdown"].T
    T, k = idx.shape
    rows = []
    for j in range(k):
        # slot j of every token, one expert at a time (selection is fixed)
        y_j = torch.zeros(T, w["Wdown"].shape[0], dtype=F64)
        for e in torch.unique(idx[:, j]).tolist():
            t = torch.nonzero(idx[:, j] == e, as_tuple=True)[0]
            y_e = expert_forward(z[t], w["Wg"][e], w["Wv"][e], w["Wo"][e], c, _identity)
            y_j = y_j.index_put((t,), y_e)
        rows.append(y_j)
    y_slots = torch.stack(rows, dim=1)
    u = combine(y_slots, p)
    n = rms_norm(u, w["gamma"], eps)
    y = shared_experts(x, w["Wsg"], w["Wsv"], w["Wso"], c, _identity) + n @ w["Wup"].T
    return {"y": y, "u": u, "n": n, "z": z, "s": s, "p": p}


def layer_backward(dims, w: dict, x: torch.Tensor, dy: torch.Tensor, idx: torch.Tensor | None = None) -> dict:
    """Gradients of sum(y * dy) with respect to x and every weight in PARAMS.

    idx: the fixed selection; by default the forward selection (keys
    s + bias, top k, ties to the lower index).  Returns {"idx", "y",
    "dx", "d<name>" for name in PARAMS}; experts that no token selected get
    zero gradients."""
    x = x.detach().to(F64).clone().requires_grad_(True)
    wp = {}
    for name, t in w.items():
        t = t.detach().to(F64).clone()
        if name in PARAMS:
            t.requires_grad_(True)
        wp[name] = t
    if idx is None:
        with torch.no_grad():
            idx, _, _ = select_experts(router_scores(x, wp["Wr"]), wp["bias"], dims.k)
    out = layer_forward_fixed(dims, wp, x, idx)
    (out["y"] * dy.to(F64)).sum().backward()
    res = {"idx": idx, "y": out["y"].detach(), "dx": x.grad.detach()}
    for name in PARAMS:
        g = wp[name].grad
        res["d" + name] = torch.zeros_like(wp[name]) if g is None else g.detach()
    return res
