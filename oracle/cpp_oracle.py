"""ctypes binding of the fp64 C++ oracle (``oracle/moe_oracle.cpp``), with the
same functions and signatures as the PyTorch restatement in ``moe_oracle.py``
(test infrastructure only).

Tensors are fp64 torch CPU tensors in and out.  Weight matrices may also be
given as the generator's raw host arrays -- float32, bf16 bit patterns
(uint16) or an MXFP4 (codes, scales) pair -- which the C++ code decodes
itself, so the K3-size weights need no fp64 copy in Python.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

from . import moe_oracle as _py

F64 = torch.float64
_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_oracle.so")

OC_F64, OC_F32, OC_BF16, OC_MXFP4 = 0, 1, 2, 3
ROUND_NONE, ROUND_BF16, ROUND_F32 = 0, 1, 2

__all__ = list(_py.__all__) + ["num_threads"]


class oc_mat(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("type", ctypes.c_int32),
                ("rows", ctypes.c_int64), ("cols", ctypes.c_int64)]


class oc_dims(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("H", ctypes.c_int32), ("L", ctypes.c_int32), ("E", ctypes.c_int32),
                ("k", ctypes.c_int32), ("I", ctypes.c_int32), ("S", ctypes.c_int32), ("Is", ctypes.c_int32),
                ("situ_c", ctypes.c_double), ("rms_eps", ctypes.c_double), ("mode", ctypes.c_int32),
                ("routed_act", ctypes.c_int32)]


class oc_weights(ctypes.Structure):
    _fields_ = [("Wr", oc_mat), ("bias", ctypes.c_void_p), ("Wdown", oc_mat), ("Wup", oc_mat),
                ("gamma", ctypes.c_void_p), ("Wg", oc_mat), ("Wv", oc_mat), ("Wo", oc_mat), ("Wsg", oc_mat),
                ("Wsv", oc_mat), ("Wso", oc_mat)]


class oc_outputs(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("s", "idx", "p", "margin", "z", "u", "n", "y", "y_shared")]


PROVIDER = ctypes.CFUNCTYPE(ctypes.c_int, ctypes.c_void_p, ctypes.c_int32, ctypes.POINTER(oc_mat),
                            ctypes.POINTER(oc_mat), ctypes.POINTER(oc_mat))

_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            from .build import build

            build()
        L = ctypes.CDLL(LIB_PATH)
        vp, i64, i32, f64 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_double
        pm = ctypes.POINTER(oc_mat)
        L.oc_num_threads.restype = ctypes.c_int
        L.oc_bf16_round.argtypes = [vp, i64, vp]
        L.oc_f32_round.argtypes = [vp, i64, vp]
        L.oc_decode.argtypes = [pm, vp]
        L.oc_sigmoid.argtypes = [vp, i64, vp]
        L.oc_situ_glu.argtypes = [vp, vp, i64, f64, vp]
        L.oc_linear.argtypes = [vp, i64, i64, pm, vp]
        L.oc_router_scores.argtypes = [vp, i64, i64, pm, vp]
        L.oc_select.argtypes = [vp, vp, ctypes.c_int, i64, i64, i64, vp, vp, vp]
        L.oc_select_f32.argtypes = [vp, vp, i64, i64, i64, vp, vp]
        L.oc_permute.argtypes = [vp, i64, i64, i64, vp, vp, vp, vp]
        L.oc_permute.restype = ctypes.c_int
        L.oc_expert_forward.argtypes = [vp, i64, i64, pm, pm, pm, f64, i32, i32, vp]
        L.oc_e4m3_decode.argtypes = [vp, i64, vp]
        L.oc_e4m3_encode.argtypes = [vp, i64, vp]
        L.oc_mx8_quantize.argtypes = [vp, i64, i64, vp, vp]
        L.oc_e2m1_encode.argtypes = [vp, i64, vp]
        L.oc_mx4_quantize.argtypes = [vp, i64, i64, vp, vp]
        L.oc_combine.argtypes = [vp, vp, i64, i64, i64, vp]
        L.oc_rms_norm.argtypes = [vp, vp, i64, i64, f64, vp]
        L.oc_shared_experts.argtypes = [vp, i64, i64, i64, i64, pm, pm, pm, f64, i32, vp]
        L.oc_layer_forward.argtypes = [ctypes.POINTER(oc_dims), ctypes.POINTER(oc_weights), vp, vp, PROVIDER, vp,
                                       ctypes.POINTER(oc_outputs)]
        L.oc_layer_forward.restype = ctypes.c_int
        _lib = L
    return _lib


def num_threads() -> int:
    """Worker threads the oracle uses (std::thread::hardware_concurrency, or
    MOE_ORACLE_THREADS)."""
    return int(lib().oc_num_threads())


# ------------------------------------------------------------------------------------ marshalling
def _f64(t) -> torch.Tensor:
    t = torch.as_tensor(t)
    return t.to(F64).contiguous()


def _ptr(t: torch.Tensor) -> int:
    return t.data_ptr()


def _mat(w, keep: list, rows: int | None = None, cols: int | None = None) -> oc_mat:
    """oc_mat view of a weight matrix (torch / numpy values, bf16 bits as
    uint16, or an MXFP4 (codes, scales) pair); arrays are kept alive in keep."""
    if isinstance(w, tuple):
        codes = np.ascontiguousarray(w[0], dtype=np.uint8)
        scales = np.ascontiguousarray(w[1], dtype=np.uint8)
        codes2 = codes.reshape(-1, codes.shape[-1])
        keep += [codes, scales]
        return oc_mat(codes.ctypes.data, scales.ctypes.data, OC_MXFP4, codes2.shape[0], 2 * codes2.shape[1])
    if isinstance(w, np.ndarray):
        a = np.ascontiguousarray(w)
        keep.append(a)
        typ = {np.dtype(np.uint16): OC_BF16, np.dtype(np.float32): OC_F32, np.dtype(np.float64): OC_F64}[a.dtype]
        a2 = a.reshape(-1, a.shape[-1]) if a.ndim > 0 else a.reshape(1, 1)
        return oc_mat(a.ctypes.data, None, typ, a2.shape[0], a2.shape[1])
    t = _f64(w)
    keep.append(t)
    t2 = t.reshape(-1, t.shape[-1])
    return oc_mat(t.data_ptr(), None, OC_F64, t2.shape[0], t2.shape[1])


def _empty_mat() -> oc_mat:
    return oc_mat(None, None, OC_F64, 0, 0)


def _mode_of(rnd) -> int | None:
    if rnd in (bf16_round, _py.bf16_round):
        return ROUND_BF16
    if rnd in (f32_round, _py.f32_round):
        return ROUND_F32
    return None


# ------------------------------------------------------------------------------------ number formats
def bf16_round(t: torch.Tensor) -> torch.Tensor:
    """Round fp64 values to the nearest bfloat16 (ties to even), as fp64."""
    t = _f64(t)
    out = torch.empty_like(t)
    lib().oc_bf16_round(_ptr(t), t.numel(), _ptr(out))
    return out


def f32_round(t: torch.Tensor) -> torch.Tensor:
    t = _f64(t)
    out = torch.empty_like(t)
    lib().oc_f32_round(_ptr(t), t.numel(), _ptr(out))
    return out


def storage_round(act: str):
    return {"bf16": bf16_round, "f32": f32_round}[act]


def _decode(m: oc_mat, keep) -> torch.Tensor:
    out = torch.empty(m.rows, m.cols, dtype=F64)
    lib().oc_decode(ctypes.byref(m), _ptr(out))
    return out


def bf16_bits_to_f64(a) -> torch.Tensor:
    a = np.ascontiguousarray(np.asarray(a))
    assert a.dtype == np.uint16
    keep: list = []
    return _decode(_mat(a, keep), keep).reshape(a.shape)


def f32_to_f64(a) -> torch.Tensor:
    a = np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    keep: list = []
    return _decode(_mat(a, keep), keep).reshape(a.shape)


E2M1_VALUES = _py.E2M1_VALUES
routed_act = _py.routed_act  # a name mapping, no arithmetic


def mxfp4_dequant(codes, scales) -> torch.Tensor:
    """MXFP4 weights -> fp64 [rows, K], decoded by the C++ oracle."""
    keep: list = []
    return _decode(_mat((np.asarray(codes), np.asarray(scales)), keep), keep)


# ------------------------------------------------------------------------------------ router
def sigmoid(t: torch.Tensor) -> torch.Tensor:
    t = _f64(t)
    out = torch.empty_like(t)
    lib().oc_sigmoid(_ptr(t), t.numel(), _ptr(out))
    return out


def router_scores(x: torch.Tensor, Wr) -> torch.Tensor:
    x = _f64(x)
    keep: list = []
    m = _mat(Wr, keep)
    out = torch.empty(x.shape[0], m.rows, dtype=F64)
    lib().oc_router_scores(_ptr(x), x.shape[0], x.shape[1], ctypes.byref(m), _ptr(out))
    return out


def select_experts(s: torch.Tensor, b: torch.Tensor, k: int):
    s, b = _f64(s), _f64(b)
    T, E = s.shape
    idx = torch.empty(T, k, dtype=torch.int64)
    p = torch.empty(T, k, dtype=F64)
    margin = torch.empty(T, dtype=F64)
    lib().oc_select(_ptr(s), _ptr(b), int(b.dim() == 2), T, E, k, _ptr(idx), _ptr(p), _ptr(margin))
    return idx, p, margin


def select_experts_from_f32_scores(s32, b32, k: int):
    s32 = np.ascontiguousarray(np.asarray(s32, dtype=np.float32))
    b32 = np.ascontiguousarray(np.asarray(b32, dtype=np.float32))
    T, E = s32.shape
    idx = torch.empty(T, k, dtype=torch.int64)
    p = torch.empty(T, k, dtype=F64)
    lib().oc_select_f32(s32.ctypes.data, b32.ctypes.data, T, E, k, _ptr(idx), _ptr(p))
    return idx, p


def permute(idx, E: int):
    idx = np.ascontiguousarray(np.asarray(idx), dtype=np.int64)
    T, k = idx.shape
    counts = np.empty(E, np.int64)
    offsets = np.empty(E + 1, np.int64)
    perm_token = np.empty(T * k, np.int64)
    inv_perm = np.empty(T * k, np.int64)
    rc = lib().oc_permute(idx.ctypes.data, T, k, E, counts.ctypes.data, offsets.ctypes.data, perm_token.ctypes.data,
                          inv_perm.ctypes.data)
    if rc != 0:
        raise ValueError("expert index out of range")
    return counts, offsets, perm_token, inv_perm


# ------------------------------------------------------------------------------------ experts
def situ_glu(g: torch.Tensor, v: torch.Tensor, c: float) -> torch.Tensor:
    g, v = torch.broadcast_tensors(_f64(g), _f64(v))
    g, v = g.contiguous(), v.contiguous()
    out = torch.empty_like(g)
    lib().oc_situ_glu(_ptr(g), _ptr(v), g.numel(), float(c), _ptr(out))
    return out


def _linear(a: torch.Tensor, W) -> torch.Tensor:
    a = _f64(a)
    keep: list = []
    m = _mat(W, keep)
    out = torch.empty(a.shape[0], m.rows, dtype=F64)
    lib().oc_linear(_ptr(a), a.shape[0], a.shape[1], ctypes.byref(m), _ptr(out))
    return out


_ACT_CODE = {None: 0, "mxfp8": 1, "mxfp4": 2}


def expert_forward(z_rows: torch.Tensor, Wg, Wv, Wo, c: float, rnd, act: str | None = None):
    """g = W_g z, v = W_v z, h = rnd(SiTU-GLU(g, v)), y = W_o h (fp64); with
    act ("mxfp8" / "mxfp4") the rows of z and of h (after rnd) are first
    replaced by their values in that format."""
    mode = _mode_of(rnd)
    if mode is None:  # a caller-supplied rounding function: the same steps, one call each
        zq = act_round(act, z_rows)
        h = rnd(situ_glu(_linear(zq, Wg), _linear(zq, Wv), c))
        return _linear(act_round(act, h), Wo)
    z = _f64(z_rows)
    keep: list = []
    mg, mv, mo = _mat(Wg, keep), _mat(Wv, keep), _mat(Wo, keep)
    y = torch.empty(z.shape[0], mo.rows, dtype=F64)
    lib().oc_expert_forward(_ptr(z), z.shape[0], z.shape[1], ctypes.byref(mg), ctypes.byref(mv), ctypes.byref(mo),
                            float(c), mode, _ACT_CODE[act], _ptr(y))
    return y


def e4m3_decode(codes) -> torch.Tensor:
    """E4M3 codes (uint8) -> fp64 values (NaN for 0x7F / 0xFF)."""
    c = np.ascontiguousarray(np.asarray(codes, dtype=np.uint8))
    out = torch.empty(c.shape, dtype=F64)
    lib().oc_e4m3_decode(c.ctypes.data, c.size, _ptr(out))
    return out


def e4m3_encode(v) -> np.ndarray:
    """fp64 values -> nearest E4M3 codes (ties to even, saturating to +-448)."""
    v = _f64(v)
    out = np.empty(tuple(v.shape), dtype=np.uint8)
    lib().oc_e4m3_encode(_ptr(v), v.numel(), out.ctypes.data)
    return out


def mx8_quantize(v) -> tuple[np.ndarray, np.ndarray]:
    """Rows of fp64 values [R, K] -> MXFP8 (codes [R, K] uint8, E8M0 scale
    bytes [R, K/32] uint8)."""
    v = _f64(v)
    R, K = v.shape
    codes = np.empty((R, K), dtype=np.uint8)
    scales = np.empty((R, K // 32), dtype=np.uint8)
    lib().oc_mx8_quantize(_ptr(v), R, K, codes.ctypes.data, scales.ctypes.data)
    return codes, scales


def mx8_round(v) -> torch.Tensor:
    """The values of the MXFP8 encoding of rows v [R, K] (fp64)."""
    codes, scales = mx8_quantize(v)
    return mx8_dequant(codes, scales)


def e2m1_encode(v) -> np.ndarray:
    """fp64 values -> nearest E2M1 codes, one per byte (ties to even,
    saturating to +-6)."""
    v = _f64(v)
    out = np.empty(tuple(v.shape), dtype=np.uint8)
    lib().oc_e2m1_encode(_ptr(v), v.numel(), out.ctypes.data)
    return out


def mx4_quantize(v) -> tuple[np.ndarray, np.ndarray]:
    """Rows of fp64 values [R, K] -> MXFP4 (packed codes [R, K/2] uint8, E8M0
    scale bytes [R, K/32] uint8)."""
    v = _f64(v)
    R, K = v.shape
    codes = np.empty((R, K // 2), dtype=np.uint8)
    scales = np.empty((R, K // 32), dtype=np.uint8)
    lib().oc_mx4_quantize(_ptr(v), R, K, codes.ctypes.data, scales.ctypes.data)
    return codes, scales


def mx4_round(v) -> torch.Tensor:
    """The values of the MXFP4 encoding of rows v [R, K] (fp64)."""
    return mxfp4_dequant(*mx4_quantize(v))


def act_round(act: str | None, v) -> torch.Tensor:
    if act is None:
        return v
    return {"mxfp8": mx8_round, "mxfp4": mx4_round}[act](v)


def mx8_dequant(codes, scales) -> torch.Tensor:
    """MXFP8 codes [R, K] and E8M0 scale bytes [R, K/32] -> fp64 values."""
    v = e4m3_decode(codes)
    s = torch.from_numpy(np.ascontiguousarray(np.asarray(scales, dtype=np.int64))).repeat_interleave(32, dim=1)
    f = torch.pow(torch.tensor(2.0, dtype=F64), (s - 127).to(F64))
    return v * torch.where(s == 255, torch.tensor(float("nan"), dtype=F64), f)


def combine(y_slots: torch.Tensor, p: torch.Tensor) -> torch.Tensor:
    y_slots, p = _f64(y_slots), _f64(p)
    T, k, L = y_slots.shape
    u = torch.empty(T, L, dtype=F64)
    lib().oc_combine(_ptr(y_slots), _ptr(p), T, k, L, _ptr(u))
    return u


def rms_norm(u: torch.Tensor, gamma: torch.Tensor, eps: float) -> torch.Tensor:
    u, gamma = _f64(u), _f64(gamma)
    n = torch.empty_like(u)
    lib().oc_rms_norm(_ptr(u), _ptr(gamma), u.shape[0], u.shape[1], float(eps), _ptr(n))
    return n


def shared_experts(x: torch.Tensor, Wsg, Wsv, Wso, c: float, rnd) -> torch.Tensor:
    mode = _mode_of(rnd)
    x = _f64(x)
    S = Wsg.shape[0]
    if mode is None:
        y = torch.zeros(x.shape[0], Wso.shape[1], dtype=F64)
        for i in range(S):
            y = y + expert_forward(x, Wsg[i], Wsv[i], Wso[i], c, rnd)
        return y
    keep: list = []
    Is, H = Wsg.shape[1], Wsg.shape[2]
    mg, mv, mo = _mat(Wsg, keep), _mat(Wsv, keep), _mat(Wso, keep)
    y = torch.empty(x.shape[0], H, dtype=F64)
    lib().oc_shared_experts(_ptr(x), x.shape[0], H, S, Is, ctypes.byref(mg), ctypes.byref(mv), ctypes.byref(mo),
                            float(c), mode, _ptr(y))
    return y


# ------------------------------------------------------------------------------------ the whole layer
def _run_layer(cfg, dense: dict, x: torch.Tensor, routed, forced_idx) -> dict:
    x = _f64(x)
    T = x.shape[0]
    keep: list = []
    mode = {"bf16": ROUND_BF16, "f32": ROUND_F32}[cfg.act]
    d = oc_dims(T, cfg.H, cfg.L, cfg.E, cfg.k, cfg.I, cfg.S, cfg.Is, float(cfg.situ_c), float(cfg.rms_eps), mode,
                _ACT_CODE[routed_act(cfg)])
    bias, gamma = _f64(dense["bias"]), _f64(dense["gamma"])
    keep += [bias, gamma]
    shared = [_mat(dense[n], keep) if cfg.S > 0 else _empty_mat() for n in ("Wsg", "Wsv", "Wso")]
    w = oc_weights(_mat(dense["Wr"], keep), bias.data_ptr(), _mat(dense["Wdown"], keep), _mat(dense["Wup"], keep),
                   gamma.data_ptr(), _empty_mat(), _empty_mat(), _empty_mat(), *shared)
    provider = None
    if callable(routed):
        hold: list = []
        failed: list = []

        def fill(ctx, e, pg, pv, po):
            try:
                hold.clear()
                Wg, Wv, Wo = routed(int(e))
                pg[0], pv[0], po[0] = _mat(Wg, hold), _mat(Wv, hold), _mat(Wo, hold)
                return 0
            except BaseException as exc:  # reported after the C call returns
                failed.append(exc)
                return 1

        provider = PROVIDER(fill)
    else:
        w.Wg, w.Wv, w.Wo = _mat(routed["Wg"], keep), _mat(routed["Wv"], keep), _mat(routed["Wo"], keep)
    out = {"s": torch.empty(T, cfg.E, dtype=F64), "idx": torch.empty(T, cfg.k, dtype=torch.int64),
           "p": torch.empty(T, cfg.k, dtype=F64), "margin": torch.empty(T, dtype=F64),
           "z": torch.empty(T, cfg.L, dtype=F64), "u": torch.empty(T, cfg.L, dtype=F64),
           "n": torch.empty(T, cfg.L, dtype=F64), "y": torch.empty(T, cfg.H, dtype=F64),
           "y_shared": torch.empty(T, cfg.H, dtype=F64)}
    o = oc_outputs(*[out[n].data_ptr() for n in ("s", "idx", "p", "margin", "z", "u", "n", "y", "y_shared")])
    fidx = None
    if forced_idx is not None:
        fidx = torch.as_tensor(np.asarray(forced_idx), dtype=torch.int64).contiguous()
        keep.append(fidx)
    rc = lib().oc_layer_forward(ctypes.byref(d), ctypes.byref(w), x.data_ptr(),
                                fidx.data_ptr() if fidx is not None else None,
                                provider if provider is not None else PROVIDER(), None, ctypes.byref(o))
    if callable(routed) and failed:
        raise failed[0]
    if rc != 0:
        raise ValueError("oracle layer forward failed (expert index out of range)")
    return out


def layer_forward(cfg, w: dict, x: torch.Tensor, forced_idx=None) -> dict:
    """Forward pass for token rows x; w holds every weight (routed ones as
    [E, I, L] / [E, L, I] tensors or raw arrays)."""
    return _run_layer(cfg, w, x, {"Wg": w["Wg"], "Wv": w["Wv"], "Wo": w["Wo"]}, forced_idx)


def layer_forward_streamed(cfg, dense: dict, x: torch.Tensor, expert_weights, forced_idx=None) -> dict:
    """Same computation with the routed weights supplied one expert at a time:
    expert_weights(e) -> (Wg_e [I, L], Wv_e [I, L], Wo_e [L, I]) as fp64
    tensors or the generator's raw host arrays."""
    return _run_layer(cfg, dense, x, expert_weights, forced_idx)
