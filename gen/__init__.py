"""Seeded synthetic inputs for the Stable LatentMoE layer.

This module is the only code that both the CPU oracle and the CUDA library
see: it makes their inputs and holds none of the layer's arithmetic.  The
host half (C) and the device half (CUDA) produce bit-identical values for the
same (seed, tensor id, element index); see ``csrc/gen_common.h`` for the
generator's definition (Philox-4x32-10 counters, Irwin-Hall normal variates,
OCP MXFP4 quantiser).

Host outputs are numpy arrays: fp32 tensors as float32, bf16 tensors as the
raw uint16 bit patterns, MXFP4 tensors as (packed codes uint8, E8M0 scales
uint8).  Device outputs are torch tensors.
"""
from __future__ import annotations

import ctypes
import os
from functools import lru_cache

import numpy as np

from .configs import CONFIGS, TID, LayerConfig, tensor_dtype, tensor_shape, tensor_std

__all__ = [
    "CONFIGS",
    "TID",
    "LayerConfig",
    "tensor_shape",
    "tensor_std",
    "tensor_dtype",
    "lib",
    "host_tensor",
    "host_rows",
    "host_expert",
    "bias",
    "gamma",
    "sample_tokens",
    "qb_scores",
    "device_layer",
    "philox4x32_10",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoegen.so")


def _nthreads() -> int:
    return max(1, min(64, os.cpu_count() or 1))


@lru_cache(maxsize=1)
def lib() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        from .build import build

        build()
    L = ctypes.CDLL(LIB_PATH)
    u32, u64, f32, vp, i32 = ctypes.c_uint32, ctypes.c_uint64, ctypes.c_float, ctypes.c_void_p, ctypes.c_int
    L.gen_philox4x32_10.argtypes = [vp, vp, vp]
    L.gen_scale.argtypes = [ctypes.c_double]
    L.gen_scale.restype = f32
    L.gen_fill_f32.argtypes = [u32, u32, u64, u64, f32, f32, vp, i32]
    L.gen_fill_bf16.argtypes = [u32, u32, u64, u64, f32, f32, vp, i32]
    L.gen_fill_mxfp4.argtypes = [u32, u32, u64, u64, u64, f32, vp, vp, i32]
    L.gen_fill_u32.argtypes = [u32, u32, u64, u64, vp]
    L.gen_dev_fill_f32.argtypes = [u32, u32, u64, u64, f32, f32, vp, vp]
    L.gen_dev_fill_f32.restype = i32
    L.gen_dev_fill_bf16.argtypes = [u32, u32, u64, u64, f32, f32, vp, vp]
    L.gen_dev_fill_bf16.restype = i32
    L.gen_dev_fill_mxfp4.argtypes = [u32, u32, u64, u64, u64, f32, vp, vp, vp]
    L.gen_dev_fill_mxfp4.restype = i32
    return L


def philox4x32_10(ctr, key) -> tuple[int, int, int, int]:
    c = (ctypes.c_uint32 * 4)(*ctr)
    k = (ctypes.c_uint32 * 2)(*key)
    o = (ctypes.c_uint32 * 4)()
    lib().gen_philox4x32_10(c, k, o)
    return tuple(int(v) for v in o)


def _scale(std: float) -> float:
    return float(lib().gen_scale(float(std)))


def _offset(name: str) -> float:
    return 1.0 if name == "gamma" else 0.0


def fill_host(seed: int, tid: int, start: int, count: int, std: float, offset: float, dtype: str) -> np.ndarray:
    """Elements start..start+count-1 of one generated tensor, as float32 or bf16 bits."""
    if dtype == "f32":
        out = np.empty(count, np.float32)
        lib().gen_fill_f32(seed, tid, start, count, _scale(std), offset, out.ctypes.data, _nthreads())
    elif dtype == "bf16":
        out = np.empty(count, np.uint16)
        lib().gen_fill_bf16(seed, tid, start, count, _scale(std), offset, out.ctypes.data, _nthreads())
    else:
        raise ValueError(dtype)
    return out


def fill_host_mxfp4(seed: int, tid: int, row_start: int, nrows: int, K: int, std: float):
    codes = np.empty((nrows, K // 2), np.uint8)
    scales = np.empty((nrows, K // 32), np.uint8)
    lib().gen_fill_mxfp4(seed, tid, row_start, nrows, K, _scale(std), codes.ctypes.data, scales.ctypes.data,
                         _nthreads())
    return codes, scales


def host_rows(cfg: LayerConfig, name: str, rows) -> np.ndarray:
    """Selected rows (first index) of a 2-D input tensor (x, Wr, Wdown, ...)."""
    shape = tensor_shape(cfg, name)
    assert len(shape) == 2
    ncol = shape[1]
    dt = tensor_dtype(cfg, name)
    out = np.empty((len(rows), ncol), np.float32 if dt == "f32" else np.uint16)
    for i, r in enumerate(rows):
        out[i] = fill_host(cfg.seed, TID[name], int(r) * ncol, ncol, tensor_std(cfg, name), _offset(name), dt)
    return out


def host_tensor(cfg: LayerConfig, name: str) -> np.ndarray:
    """A whole non-routed input tensor on the host (not for the K3 routed weights)."""
    if name == "bias":
        return bias(cfg)
    if name == "gamma":
        return gamma(cfg)
    shape = tensor_shape(cfg, name)
    dt = tensor_dtype(cfg, name)
    if dt == "mxfp4":
        raise ValueError("use host_expert for MXFP4 routed weights")
    n = int(np.prod(shape))
    return fill_host(cfg.seed, TID[name], 0, n, tensor_std(cfg, name), 0.0, dt).reshape(shape)


def host_expert(cfg: LayerConfig, name: str, e: int):
    """Routed-expert weight matrix e of Wg / Wv ([I, L]) or Wo ([L, I]).

    Returns a float32 or uint16 (bf16 bits) array, or for MXFP4 a tuple
    (codes [rows, K/2] uint8, scales [rows, K/32] uint8)."""
    _, R, K = tensor_shape(cfg, name)
    dt = tensor_dtype(cfg, name)
    std = tensor_std(cfg, name)
    if dt == "mxfp4":
        return fill_host_mxfp4(cfg.seed, TID[name], e * R, R, K, std)
    return fill_host(cfg.seed, TID[name], e * R * K, R * K, std, 0.0, dt).reshape(R, K)


def gamma(cfg: LayerConfig) -> np.ndarray:
    """RMSNorm gain: exactly 1 in the measured workloads, 1 + N(0, 0.1) on request."""
    if cfg.gamma == "ones":
        return np.ones(cfg.L, np.float32)
    return fill_host(cfg.seed, TID["gamma"], 0, cfg.L, 0.1, 1.0, "f32")


def u32_words(seed: int, tid: int, start: int, count: int) -> np.ndarray:
    out = np.empty(count, np.uint32)
    lib().gen_fill_u32(seed, tid, start, count, out.ctypes.data)
    return out


def zipf_bias(E: int, k: int, s: float, seed: int) -> np.ndarray:
    """Selection bias that makes expert loads follow Zipf(s) over a seeded
    random permutation of the experts.

    Expert e gets rank r_e (a seeded permutation of 1..E) and a target
    selection probability p_e proportional to r_e^-s, scaled so the p_e sum to
    k and capped at 0.99.  With router logits l ~ N(0, 1) and a common
    selection threshold, expert e is chosen when sigmoid(l_e) + b_e exceeds
    it, so b_e = -sigmoid(Phi^-1(1 - p_e)) up to a constant; the constant is
    fixed by centring b.  This is a generator of inputs only; the realised
    loads are reported by the tests, not assumed."""
    from scipy.special import ndtri

    words = u32_words(seed, TID["zipf_perm"], 0, E).astype(np.int64)
    order = np.lexsort((np.arange(E), words))
    rank = np.empty(E, np.int64)
    rank[order] = np.arange(1, E + 1)
    w = rank.astype(np.float64) ** (-s)
    p = k * w / w.sum()
    for _ in range(1000):
        over = p > 0.99
        if not over.any():
            break
        p[over] = 0.99
        free = ~over
        p[free] *= (k - 0.99 * over.sum()) / p[free].sum()
    q = ndtri(1.0 - p)
    b = -1.0 / (1.0 + np.exp(-q))
    b -= b.mean()
    return b.astype(np.float32)


def bias(cfg: LayerConfig) -> np.ndarray:
    if cfg.bias == "zipf":
        return zipf_bias(cfg.E, cfg.k, cfg.zipf_s, cfg.seed)
    return fill_host(cfg.seed, TID["bias"], 0, cfg.E, cfg.bias_std, 0.0, "f32")


def qb_scores(cfg: LayerConfig) -> np.ndarray:
    """Router-score stand-in [T, E] for the Quantile Balancing step: uniform
    fp32 values in [0, 1) with 24 random bits each (Philox words >> 8, times
    2^-24, exact in fp32)."""
    words = u32_words(cfg.seed, TID["qb_scores"], 0, cfg.T * cfg.E)
    return ((words >> 8).astype(np.float32) * np.float32(2.0 ** -24)).reshape(cfg.T, cfg.E)


def sample_tokens(cfg: LayerConfig, n: int | None = None) -> np.ndarray:
    """Seeded, sorted sample of distinct token indices (all tokens if n >= T)."""
    n = cfg.oracle_tokens if n is None else n
    if n is None or n >= cfg.T:
        return np.arange(cfg.T, dtype=np.int64)
    words = u32_words(cfg.seed, TID["sample"], 0, cfg.T).astype(np.int64)
    order = np.lexsort((np.arange(cfg.T), words))
    return np.sort(order[:n]).astype(np.int64)


# ----------------------------------------------------------------------------------------------
# Device-resident layer inputs (torch tensors), filled by the device half of the generator.
# ----------------------------------------------------------------------------------------------
def _dev_fill(t, cfg: LayerConfig, name: str, start: int = 0):
    import torch

    L = lib()
    stream = torch.cuda.current_stream(t.device).cuda_stream
    std = tensor_std(cfg, name)
    n = t.numel()
    if t.dtype == torch.float32:
        rc = L.gen_dev_fill_f32(cfg.seed, TID[name], start, n, _scale(std), _offset(name), t.data_ptr(), stream)
    elif t.dtype == torch.bfloat16:
        rc = L.gen_dev_fill_bf16(cfg.seed, TID[name], start, n, _scale(std), _offset(name), t.data_ptr(), stream)
    else:
        raise TypeError(t.dtype)
    if rc != 0:
        raise RuntimeError(f"generator launch failed: cuda error {rc}")


def device_layer(cfg: LayerConfig, device="cuda", with_x: bool = True) -> dict:
    """All inputs of one layer, resident on the device."""
    import torch

    dev = torch.device(device)
    tdt = {"f32": torch.float32, "bf16": torch.bfloat16}
    out = {}
    names = ["x", "Wr", "Wdown", "Wup", "Wsg", "Wsv", "Wso"] if with_x else ["Wr", "Wdown", "Wup", "Wsg", "Wsv", "Wso"]
    for name in names:
        t = torch.empty(tensor_shape(cfg, name), dtype=tdt[tensor_dtype(cfg, name)], device=dev)
        _dev_fill(t, cfg, name)
        out[name] = t
    for name in ("Wg", "Wv", "Wo"):
        E, R, K = tensor_shape(cfg, name)
        if tensor_dtype(cfg, name) == "mxfp4":
            codes = torch.empty((E, R, K // 2), dtype=torch.uint8, device=dev)
            scales = torch.empty((E, R, K // 32), dtype=torch.uint8, device=dev)
            stream = torch.cuda.current_stream(dev).cuda_stream
            rc = lib().gen_dev_fill_mxfp4(cfg.seed, TID[name], 0, E * R, K, _scale(tensor_std(cfg, name)),
                                          codes.data_ptr(), scales.data_ptr(), stream)
            if rc != 0:
                raise RuntimeError(f"generator launch failed: cuda error {rc}")
            out[name] = codes
            out[{"Wg": "Sg", "Wv": "Sv", "Wo": "So"}[name]] = scales
        else:
            t = torch.empty((E, R, K), dtype=tdt[tensor_dtype(cfg, name)], device=dev)
            _dev_fill(t, cfg, name)
            out[name] = t
    out["bias"] = torch.from_numpy(bias(cfg)).to(dev)
    out["gamma"] = torch.from_numpy(gamma(cfg)).to(dev)
    return out
