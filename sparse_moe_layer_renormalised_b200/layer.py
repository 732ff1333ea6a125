"""A resident Stable LatentMoE layer: device weights plus a workspace, called
through moe_layer_forward.  PyTorch only allocates memory and provides the
stream; every step runs in libmoe_b200.so."""
from __future__ import annotations

from dataclasses import replace

import torch

from ._binding import Dims, check, make_aux, make_weights, moe_layer_forward, moe_workspace_size

_TORCH_DT = {"f32": torch.float32, "bf16": torch.bfloat16}


class MoeLayer:
    """Weights: dict with Wr, bias, Wdown, Wup, gamma, Wg, Wv, Wo, Wsg, Wsv, Wso
    and, for MXFP4 routed weights, Sg, Sv, So (device tensors in the shapes of
    include/moe.h).  max_tokens sizes the
    workspace; each call may use any T <= max_tokens."""

    def __init__(self, dims: Dims, weights: dict, max_tokens: int | None = None):
        self.dims = dims
        self.weights = weights
        self.max_tokens = dims.T if max_tokens is None else max_tokens
        self._w = make_weights(**weights)
        dev = weights["Wr"].device
        nbytes = moe_workspace_size(replace(dims, T=self.max_tokens))
        if nbytes == 0:
            raise ValueError(f"invalid layer dimensions {dims}")
        self.workspace = torch.empty(nbytes, dtype=torch.uint8, device=dev)

    def output(self, T: int) -> torch.Tensor:
        return torch.empty((T, self.dims.H), dtype=_TORCH_DT[self.dims.y_out], device=self.workspace.device)

    def forward(self, x: torch.Tensor, y: torch.Tensor | None = None, aux: dict | None = None, stream=None):
        T = x.shape[0]
        if T > self.max_tokens:
            raise ValueError(f"{T} tokens > workspace capacity {self.max_tokens}")
        if y is None:
            y = self.output(T)
        d = replace(self.dims, T=T)
        a = make_aux(**aux) if aux else None
        check(moe_layer_forward(d, self._w, x, y, a, self.workspace, None, stream))
        return y

    __call__ = forward
