"""Oracle-side view of the seeded inputs: the generator's host output converted
to fp64 tensors (test infrastructure only)."""
from __future__ import annotations

import numpy as np
import torch

import gen

from .moe_oracle import F64, bf16_bits_to_f64, f32_to_f64, mxfp4_dequant


def to_f64(a) -> torch.Tensor:
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return bf16_bits_to_f64(a)
    return f32_to_f64(a)


def dense_weights(cfg) -> dict:
    """Router, bias, latent projections, gain and shared experts as fp64."""
    out = {}
    for name in ("Wr", "Wdown", "Wup", "Wsg", "Wsv", "Wso"):
        out[name] = to_f64(gen.host_tensor(cfg, name))
    out["bias"] = f32_to_f64(gen.bias(cfg))
    out["gamma"] = f32_to_f64(gen.gamma(cfg))
    return out


def expert_weights(cfg, e: int):
    """(Wg_e, Wv_e, Wo_e) as fp64; MXFP4 weights are dequantised here from
    the same packed bits the device reads."""
    mats = []
    for name in ("Wg", "Wv", "Wo"):
        a = gen.host_expert(cfg, name, e)
        if isinstance(a, tuple):
            mats.append(mxfp4_dequant(*a))
        else:
            mats.append(to_f64(a))
    return tuple(mats)


def expert_weights_raw(cfg, e: int):
    """(Wg_e, Wv_e, Wo_e) as the generator's host arrays: float32 values, bf16
    bit patterns (uint16) or MXFP4 (codes, scales) pairs.  The C++ oracle
    decodes these bits itself."""
    return tuple(gen.host_expert(cfg, name, e) for name in ("Wg", "Wv", "Wo"))


def all_weights(cfg) -> dict:
    """Every weight as fp64 (small configurations only)."""
    w = dense_weights(cfg)
    per = [expert_weights(cfg, e) for e in range(cfg.E)]
    w["Wg"] = torch.stack([p[0] for p in per])
    w["Wv"] = torch.stack([p[1] for p in per])
    w["Wo"] = torch.stack([p[2] for p in per])
    return w


def x_rows(cfg, rows) -> torch.Tensor:
    return to_f64(gen.host_rows(cfg, "x", np.asarray(rows)))
