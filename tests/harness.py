"""Helpers shared by the GPU parity tests, smoke() and bench.py: device layers
from the seeded generator, oracle references, and the parity metrics."""
from __future__ import annotations

import math
import os

import numpy as np
import torch

import gen
import oracle
import sparse_moe_layer_renormalised_b200 as moe
from oracle import inputs as oin

F64 = torch.float64

# Tolerances (max|y - y_ref| / rms(y_ref)) stated for the layer output.
TOL_BF16 = 1e-2
TOL_MXFP4 = 3e-2
# Block-scaled path, expert GEMMs on the same bf16 input rows: both sides
# quantise identical z rows to identical MXFP8 codes, so the error is that of
# the MXFP4 layer (fp32 accumulation, bf16 h, and an E4M3 code of h flipping
# where h itself differs by a bf16 step); bar 3e-2.
TOL_MXFP4_A8 = 3e-2
# The whole layer on that path: the device's bf16 z (fp32 sum) and the
# oracle's (fp64 sum) differ by one bf16 step in some elements, and h too.
# Where such a step (2^-8 relative) crosses an E4M3 rounding boundary (spaced
# 2^-3 relative), about 1 in 32 of the differing elements, the quantised
# element moves by a whole E4M3 step (1/16 to 1/8 of it).  A few such flips
# per row of z and h change g and y by ~1% of rms, and the largest of some 10^6
# outputs lands near 5 standard deviations: bars 1e-1 on max|d|/rms and 2e-2
# on rms(d)/rms for y and u.
TOL_MXFP4_A8_LAYER = 1e-1
TOL_RMS_A8_LAYER = 2e-2
# All-4-bit path (MXFP4 inputs on kind::mxf4).  The gate/up GEMM multiplies
# identical codes on both sides, so its stored h may differ from the
# oracle's only where fp32 accumulation and the SiTU-GLU evaluation put it on
# the other side of a bf16 rounding point: elementwise, one bf16 step, plus
# 1e-3 of rms(h) where |h| is tiny.  An E2M1 step is 2^-1 to 2^-2 of the
# value (8x an E4M3 step), and a one-step change of a block's largest
# element can move the block's shared scale, re-rounding all 32 codes.  The
# oracle alone, with one in 10^3 elements of h (and of z, for the layer)
# moved by one bf16 step, gives max|d|/rms up to 0.14 and rms(d)/rms up to
# 2.7e-3 for the expert outputs; up to 0.32 and 8.5e-3 for y and 0.39 and
# 1.1e-2 for u at the small layer (three seeds; the device's rate of such
# steps is below 10^-3: the MXFP8 path, with the same h, stays under bars
# that a rate of 10^-3 would exceed).  Bars: expert outputs 0.3 max and 1e-2
# rms; layer 0.5 max and 2e-2 rms.
TOL_H_BLOCK_SCALED = 1e-3
TOL_MXFP4_A4 = 0.3
TOL_RMS_A4 = 1e-2
TOL_MXFP4_A4_LAYER = 0.5
TOL_RMS_A4_LAYER = 2e-2
TOL_F32 = 1e-4
NEAR_TIE = 1e-4  # key margin below which an index-set difference is allowed
# Router scores and mixture weights: fp32 on the device from the same bf16 (or
# fp32) inputs.  The router logits carry the fp32 (tensor-core) accumulation
# error of H products, measured up to ~2e-5 at H = 7168; the score error is
# at most a quarter of that (sigmoid' <= 1/4), and the relative error of a
# mixture weight p_j = s_j / sum s is about (1 - s_j) times the logit error,
# so up to the same ~2e-5.  Bars: 1e-4 of rms(s) for s, 1e-4 relative for p.
TOL_SCORES = 1e-4
TOL_P_REL = 1e-4
TOL_Z_F32 = 1e-5


# Tokens of the K3-size workloads checked against the oracle.
K3_SAMPLE = int(os.environ.get("MOE_K3_SAMPLE", "512"))


def dims_for(cfg, T=None, y_out="f32") -> moe.Dims:
    return moe.Dims(T=cfg.T if T is None else T, H=cfg.H, L=cfg.L, E=cfg.E, k=cfg.k, I=cfg.I, S=cfg.S, Is=cfg.Is,
                    act=cfg.act, routed=cfg.routed, y_out=y_out if cfg.act == "bf16" else "f32",
                    situ_c=cfg.situ_c, rms_eps=cfg.rms_eps)


def make_device_layer(cfg, y_out="f32", max_tokens=None, weights=None):
    """(MoeLayer, input tensors dict) with every input generated on the device."""
    w = gen.device_layer(cfg, "cuda") if weights is None else weights
    layer = moe.MoeLayer(dims_for(cfg, y_out=y_out), {k: v for k, v in w.items() if k != "x"}, max_tokens=max_tokens)
    return layer, w


def run_layer(layer, x, want_aux=True):
    T = x.shape[0]
    d = layer.dims
    dev = x.device
    act_dt = torch.bfloat16 if d.act == "bf16" else torch.float32
    aux = None
    if want_aux:
        aux = {
            "scores": torch.empty(T, d.E, dtype=torch.float32, device=dev),
            "topk_idx": torch.empty(T, d.k, dtype=torch.int32, device=dev),
            "topk_w": torch.empty(T, d.k, dtype=torch.float32, device=dev),
            "expert_offsets": torch.empty(d.E + 1, dtype=torch.int32, device=dev),
            "u": torch.empty(T, d.L, dtype=torch.float32, device=dev),
            "n": torch.empty(T, d.L, dtype=act_dt, device=dev),
            "z": torch.empty(T, d.L, dtype=act_dt, device=dev),
        }
    y = layer.forward(x, aux=aux)
    torch.cuda.synchronize()
    st, code = moe.moe_device_error()
    assert st == moe.MOE_OK and code == 0, f"device fault {code}"
    return y, aux


def parity(a: torch.Tensor, ref: torch.Tensor) -> float:
    a = a.to(F64).cpu()
    ref = ref.to(F64).cpu()
    rms = torch.sqrt((ref * ref).mean()).item()
    return (a - ref).abs().max().item() / rms


_WCACHE: dict = {}


def _dense(cfg):
    key = (cfg.name, cfg.H, cfg.L, cfg.E, cfg.I, cfg.S, cfg.Is, cfg.act, cfg.bias, cfg.gamma, cfg.seed)
    if key not in _WCACHE:
        _WCACHE.clear()
        _WCACHE[key] = oin.dense_weights(cfg)
    return _WCACHE[key]


def small_enough_for_memory(cfg) -> bool:
    return cfg.E * cfg.I * cfg.L * 3 <= 200_000_000


def oracle_forward(cfg, tokens, forced_idx=None) -> dict:
    """Oracle outputs for the given token rows of cfg's synthetic input."""
    tokens = np.asarray(tokens)
    x = oin.x_rows(cfg, tokens)
    if small_enough_for_memory(cfg):
        key = ("all", cfg)
        if key not in _WCACHE:
            _WCACHE.clear()
            _WCACHE[key] = oin.all_weights(cfg)
        return oracle.layer_forward(cfg, _WCACHE[key], x, forced_idx=forced_idx)
    dense = _dense(cfg)
    return oracle.layer_forward_streamed(cfg, dense, x, lambda e: oin.expert_weights_raw(cfg, e), forced_idx=forced_idx)


def rms_parity(a: torch.Tensor, ref: torch.Tensor) -> float:
    a = a.to(F64).cpu()
    ref = ref.to(F64).cpu()
    return float(torch.sqrt(((a - ref) ** 2).mean()) / torch.sqrt((ref * ref).mean()))


def compare_layer(cfg, tokens, y_gpu, aux, tol, ref=None, rms_tol=None) -> dict:
    """Parity of the device layer on the sampled tokens against the oracle.

    Index sets must match except for tokens whose oracle key margin (k-th
    minus (k+1)-th largest key) is below NEAR_TIE; those are counted and
    their outputs are checked against the oracle forced to the device's
    choice.  Returns the metrics; asserts the bars."""
    tokens = np.asarray(tokens)
    ref = oracle_forward(cfg, tokens) if ref is None else ref
    idx_gpu = aux["topk_idx"].cpu().to(torch.int64)[torch.as_tensor(tokens)]
    set_gpu = torch.sort(idx_gpu, dim=1).values
    set_ref = torch.sort(ref["idx"], dim=1).values
    differ = (set_gpu != set_ref).any(dim=1)
    n_diff = int(differ.sum())
    near = ref["margin"] < NEAR_TIE
    assert bool((~differ | near).all()), (
        f"{int((differ & ~near).sum())} tokens choose different experts with margin >= {NEAR_TIE}")
    y_ref = ref["y"].clone()
    u_ref, n_ref = ref["u"].clone(), ref["n"].clone()
    if n_diff:
        forced = ref["idx"].clone()
        forced[differ] = idx_gpu[differ]
        rf = oracle_forward(cfg, tokens, forced_idx=forced)
        y_ref, u_ref, n_ref = rf["y"], rf["u"], rf["n"]
    sel = torch.as_tensor(tokens)
    m = {
        "tokens_checked": len(tokens),
        "index_set_differences": n_diff,
        "near_tie_tokens": int(near.sum()),
        "y": parity(y_gpu.cpu()[sel], y_ref),
        "u": parity(aux["u"].cpu()[sel], u_ref),
        "n": parity(aux["n"].cpu()[sel], n_ref),
    }
    # Router scores s = Sigmoid(W_r x): bf16 operands with fp32 accumulation
    # against the fp64 oracle; the accumulation error is ~1e-7 of rms(s).
    m["scores"] = parity(aux["scores"].cpu()[sel], ref["s"])
    assert m["scores"] <= TOL_SCORES, f"scores: max|d|/rms = {m['scores']:.3g} > {TOL_SCORES}"
    # z = W_down x is stored in the activation type.  bf16: the device's fp32
    # sum and the oracle's fp64 sum round to the same bf16 value or to
    # neighbours, so at most one storage step apart.  fp32: a few fp32 ulps of
    # accumulation-order difference, gated relative to rms(z).
    if cfg.act == "bf16":
        m["z_steps"] = storage_steps(aux["z"].cpu()[sel], ref["z"], cfg.act)
        assert m["z_steps"] <= 1.0 + 1e-6, f"z differs from the oracle by {m['z_steps']:.3g} storage steps"
    else:
        m["z"] = parity(aux["z"].cpu()[sel], ref["z"])
        assert m["z"] <= TOL_Z_F32, f"z: max|d|/rms = {m['z']:.3g} > {TOL_Z_F32}"
    # mixture weights: unbiased scores renormalised over the chosen experts,
    # matched expert by expert (slots of nearly equal keys may swap order)
    p_gpu = aux["topk_w"].cpu().to(F64)[sel]
    assert torch.allclose(p_gpu.sum(dim=1), torch.ones(len(tokens), dtype=F64), atol=1e-5)
    same = ~differ
    if same.any():
        og, oref = torch.argsort(idx_gpu[same], dim=1), torch.argsort(ref["idx"][same], dim=1)
        pg = torch.gather(p_gpu[same], 1, og)
        pr = torch.gather(ref["p"][same], 1, oref)
        m["p_rel"] = ((pg - pr).abs() / pr).max().item()
        assert m["p_rel"] <= TOL_P_REL, f"p: max relative error {m['p_rel']:.3g} > {TOL_P_REL}"
    for key in ("y", "u"):
        assert m[key] <= tol, f"{key}: max|d|/rms = {m[key]:.3g} > {tol}"
    if rms_tol is not None:
        m["y_rms"] = rms_parity(y_gpu.cpu()[sel], y_ref)
        m["u_rms"] = rms_parity(aux["u"].cpu()[sel], u_ref)
        for key in ("y_rms", "u_rms"):
            assert m[key] <= rms_tol, f"{key}: rms(d)/rms = {m[key]:.3g} > {rms_tol}"
    # The RMSNorm step: n must be RMSNorm of the device's own u, rounded to the
    # activation type, to within one rounding step of that type.  (Against the
    # oracle's n, per-token normalisation magnifies u's error in tokens whose
    # u is small, so that comparison is reported, not gated.)
    u_dev = aux["u"].cpu().to(F64)[sel]
    gamma = torch.from_numpy(gen.gamma(cfg)).to(F64)
    n_from_u = oracle.storage_round(cfg.act)(oracle.rms_norm(u_dev, gamma, cfg.rms_eps))
    m["n_steps"] = storage_steps(aux["n"].cpu()[sel], n_from_u, cfg.act)
    assert m["n_steps"] <= 1.0 + 1e-6, f"n differs from RMSNorm(u) by {m['n_steps']:.3g} storage steps"
    return m


def storage_steps(a: torch.Tensor, ref: torch.Tensor, act: str) -> float:
    """Largest |a - ref| in units of the spacing of the storage type at |ref|
    (bf16: 2^-7 |ref| bounds one step; fp32: 2^-23 |ref|), with a floor of
    1e-3 rms(ref) for values near zero."""
    a = a.to(F64)
    ref = ref.to(F64)
    rel = 2.0**-7 if act == "bf16" else 2.0**-23
    rms = torch.sqrt((ref * ref).mean())
    step = torch.clamp(ref.abs() * rel, min=float(1e-3 * rms))
    return float(((a - ref).abs() / step).max())


def moe_inputs_rows(cfg, tokens, device="cuda"):
    """x rows as a device tensor in the activation type (for sub-batch calls)."""
    a = gen.host_rows(cfg, "x", np.asarray(tokens))
    if cfg.act == "bf16":
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(a).to(device)
