"""A resident Stable LatentMoE layer: device weights plus a workspace, called
through moe_layer_forward.  PyTorch only allocates memory and provides the
stream; every step runs in libmoe_b200.so."""
from __future__ import annotations

from dataclasses import replace

import torch

from ._binding import (BLOCK_SCALED, Dims, check, make_aux, make_weights, moe_layer_forward, moe_mx_tile_scales,
                       moe_mx_tiled_scales_size, moe_workspace_size)

_TORCH_DT = {"f32": torch.float32, "bf16": torch.bfloat16}


def tile_weight_scales(dims: Dims, Sg: torch.Tensor, Sv: torch.Tensor, So: torch.Tensor, stream=None) -> dict:
    """The routed weights' E8M0 scales in the tiled order of the block-scaled
    expert kernels (moe_mx_tile_scales): {"Sgv_tiled", "So_tiled"} uint8 device
    tensors, to pass as weights alongside the codes."""
    st, n_gu, n_dn = moe_mx_tiled_scales_size(dims)
    check(st)
    gu = torch.empty(n_gu, dtype=torch.uint8, device=Sg.device)
    dn = torch.empty(n_dn, dtype=torch.uint8, device=Sg.device)
    check(moe_mx_tile_scales(dims, Sg, Sv, So, gu, dn, stream))
    return {"Sgv_tiled": gu, "So_tiled": dn}


class MoeLayer:
    """Weights: dict with Wr, bias, Wdown, Wup, gamma, Wg, Wv, Wo, Wsg, Wsv, Wso
    and, for MXFP4 routed weights, Sg, Sv, So (device tensors in the shapes of
    include/moe.h).  With routed = "mxfp4_a8" or "mxfp4_a4" (block-scaled
    MXFP4 weights x MXFP8 / MXFP4 inputs) the scales are re-ordered once here by moe_mx_tile_scales into
    Sgv_tiled / So_tiled, which the layer keeps.  max_tokens sizes the
    workspace; each call may use any T <= max_tokens."""

    def __init__(self, dims: Dims, weights: dict, max_tokens: int | None = None):
        self.dims = dims
        self.weights = dict(weights)
        self.max_tokens = dims.T if max_tokens is None else max_tokens
        dev = weights["Wr"].device
        if dims.routed in BLOCK_SCALED and "Sgv_tiled" not in weights:
            self.weights.update(tile_weight_scales(dims, weights["Sg"], weights["Sv"], weights["So"]))
        self._w = make_weights(**self.weights)
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
