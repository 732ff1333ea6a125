"""ctypes binding of the C ABI in include/moe.h.

Argument marshalling only: every function forwards to the CUDA library
libmoe_b200.so under the same name and returns its moe_status code.  Tensors
may be passed as torch tensors (their device address is used), raw integer
addresses, or None (NULL).  The library must have been built
(``python -m sparse_moe_layer_renormalised_b200.build``); there is no other
implementation to fall back to.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_CUDA, MOE_ERR_DEVICE = 0, 1, 2, 3, 4
MOE_F32, MOE_BF16, MOE_MXFP4, MOE_MXFP4_A8, MOE_MXFP4_A4 = 0, 1, 2, 3, 4
_DTYPES = {"f32": MOE_F32, "bf16": MOE_BF16, "mxfp4": MOE_MXFP4, "mxfp4_a8": MOE_MXFP4_A8, "mxfp4_a4": MOE_MXFP4_A4}
# routed types whose experts run on the block-scaled MMA (tiled weight scales)
BLOCK_SCALED = ("mxfp4_a8", "mxfp4_a4")

EXPORTED = (
    "moe_workspace_size",
    "moe_router_topk",
    "moe_permute",
    "moe_expert_ffn",
    "moe_combine",
    "moe_layer_forward",
    "moe_status_str",
    "moe_device_error",
    "moe_last_launch_count",
    "moe_permute_noalloc",
    "moe_qb_bias_update",
    "moe_latent_shared",
    "moe_output",
    "moe_expert_ffn_blocks_workspace_size",
    "moe_expert_ffn_blocks",
    "moe_backward_workspace_size",
    "moe_layer_backward",
    "moe_selftest_wait_timeout",
    "moe_mx_tiled_scales_size",
    "moe_mx_tile_scales",
    "moe_mx8_quantize",
    "moe_mx4_quantize",
    "moe_gather_rows",
)

MOE_PERMUTE_NOALLOC_SCRATCH_BYTES = 4 << 20


class moe_dims(ctypes.Structure):
    _fields_ = [
        ("T", ctypes.c_int64),
        ("H", ctypes.c_int32),
        ("L", ctypes.c_int32),
        ("E", ctypes.c_int32),
        ("k", ctypes.c_int32),
        ("I", ctypes.c_int32),
        ("S", ctypes.c_int32),
        ("Is", ctypes.c_int32),
        ("situ_c", ctypes.c_float),
        ("rms_eps", ctypes.c_float),
        ("act", ctypes.c_int),
        ("routed", ctypes.c_int),
        ("y_out", ctypes.c_int),
    ]


_WEIGHT_FIELDS = ("Wr", "bias", "Wdown", "Wup", "gamma", "Wg", "Wv", "Wo", "Sg", "Sv", "So", "Wsg", "Wsv", "Wso",
                  "Sgv_tiled", "So_tiled")
_AUX_FIELDS = ("scores", "topk_idx", "topk_w", "expert_offsets", "u", "n", "z")


class moe_weights(ctypes.Structure):
    _fields_ = [(f, ctypes.c_void_p) for f in _WEIGHT_FIELDS]


MOE_NUM_STAGES = 10
STAGE_NAMES = ("router", "topk", "latent_down", "shared_gate_up", "permute", "gather", "expert_gate_up",
               "expert_down", "combine", "output")


_GRAD_FIELDS = ("dx", "dWr", "dWdown", "dWup", "dgamma", "dWg", "dWv", "dWo", "dWsg", "dWsv", "dWso")


class moe_grads(ctypes.Structure):
    _fields_ = [(f, ctypes.c_void_p) for f in _GRAD_FIELDS]


class moe_aux(ctypes.Structure):
    _fields_ = [(f, ctypes.c_void_p) for f in _AUX_FIELDS] + [("stage_events", ctypes.POINTER(ctypes.c_void_p))]


class MoeLibraryMissing(RuntimeError):
    pass


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded CUDA library; raises MoeLibraryMissing if it was not built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise MoeLibraryMissing(
                f"{LIB_PATH} not found: build it with `python -m sparse_moe_layer_renormalised_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32 = ctypes.c_void_p, ctypes.c_int
        pd, pw, pa = ctypes.POINTER(moe_dims), ctypes.POINTER(moe_weights), ctypes.POINTER(moe_aux)
        L.moe_workspace_size.argtypes = [pd]
        L.moe_workspace_size.restype = ctypes.c_size_t
        L.moe_router_topk.argtypes = [pd, vp, vp, vp, vp, i32, vp, vp, vp]
        L.moe_permute.argtypes = [pd, vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp]
        L.moe_expert_ffn.argtypes = [pd, pw, vp, vp, vp, vp, ctypes.c_size_t, vp]
        L.moe_combine.argtypes = [pd, vp, vp, vp, vp, vp, vp, vp]
        L.moe_layer_forward.argtypes = [pd, pw, vp, vp, pa, vp, ctypes.c_size_t, vp]
        L.moe_status_str.argtypes = [i32]
        L.moe_status_str.restype = ctypes.c_char_p
        L.moe_device_error.argtypes = [ctypes.POINTER(i32), vp]
        L.moe_last_launch_count.argtypes = []
        L.moe_permute_noalloc.argtypes = [pd, vp, vp, vp, vp, vp, vp, vp]
        f32 = ctypes.c_float
        L.moe_qb_bias_update.argtypes = [pd, vp, vp, vp, vp, vp, i32, f32, f32, vp]
        L.moe_latent_shared.argtypes = [pd, pw, vp, vp, vp, vp]
        L.moe_output.argtypes = [pd, pw, vp, vp, vp, vp]
        L.moe_expert_ffn_blocks_workspace_size.argtypes = [pd, ctypes.c_int64, ctypes.c_int32]
        L.moe_expert_ffn_blocks_workspace_size.restype = ctypes.c_size_t
        L.moe_expert_ffn_blocks.argtypes = [pd, pw, vp, ctypes.c_int64, vp, ctypes.c_int32, vp, vp, ctypes.c_size_t,
                                            vp]
        L.moe_selftest_wait_timeout.argtypes = [ctypes.c_int32, vp, vp]
        L.moe_backward_workspace_size.argtypes = [pd]
        L.moe_backward_workspace_size.restype = ctypes.c_size_t
        L.moe_layer_backward.argtypes = [pd, pw, vp, vp, vp, ctypes.POINTER(moe_grads), vp, ctypes.c_size_t, vp]
        L.moe_mx_tiled_scales_size.argtypes = [pd, ctypes.POINTER(ctypes.c_size_t), ctypes.POINTER(ctypes.c_size_t)]
        L.moe_mx_tile_scales.argtypes = [pd, vp, vp, vp, vp, vp, vp]
        L.moe_mx8_quantize.argtypes = [vp, ctypes.c_int64, ctypes.c_int32, vp, vp, vp]
        L.moe_mx4_quantize.argtypes = [vp, ctypes.c_int64, ctypes.c_int32, vp, vp, vp]
        L.moe_gather_rows.argtypes = [vp, ctypes.c_int64, ctypes.c_int64, vp, ctypes.c_int64, vp, vp]
        for f in EXPORTED:
            if f not in ("moe_workspace_size", "moe_status_str", "moe_expert_ffn_blocks_workspace_size",
                         "moe_backward_workspace_size"):
                getattr(L, f).restype = i32
        _lib = L
    return _lib


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is not None:
        return stream if isinstance(stream, int) else stream.cuda_stream
    import torch

    return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None


def _nbytes(t) -> int:
    return t.numel() * t.element_size()


@dataclass
class Dims:
    T: int
    H: int
    L: int
    E: int
    k: int
    I: int
    S: int
    Is: int
    act: str = "bf16"
    routed: str = "bf16"
    y_out: str = "f32"
    situ_c: float = 10.0
    rms_eps: float = 1e-6

    def c(self) -> moe_dims:
        return moe_dims(self.T, self.H, self.L, self.E, self.k, self.I, self.S, self.Is, self.situ_c, self.rms_eps,
                        _DTYPES[self.act], _DTYPES[self.routed], _DTYPES[self.y_out])


def _dims(d) -> moe_dims:
    return d.c() if isinstance(d, Dims) else d


def _keep_alive(struct, tensors: dict):
    """The struct holds device addresses only; it also keeps a reference to
    the tensors behind them, so that a tensor made for the call (e.g.
    make_weights(**tile_weight_scales(...))) is not freed, and its memory
    reused, while the struct is in use."""
    struct._tensors = dict(tensors)
    return struct


def make_weights(**tensors) -> moe_weights:
    """moe_weights from keyword tensors named as the C struct fields."""
    unknown = set(tensors) - set(_WEIGHT_FIELDS)
    if unknown:
        raise KeyError(f"unknown weight fields {sorted(unknown)}")
    return _keep_alive(moe_weights(*[_ptr(tensors.get(f)) for f in _WEIGHT_FIELDS]), tensors)


def make_aux(stage_events=None, **tensors) -> moe_aux:
    """moe_aux from keyword tensors; stage_events: 2 * MOE_NUM_STAGES CUDA
    events (torch.cuda.Event, already recorded once so they exist, or raw
    handles)."""
    unknown = set(tensors) - set(_AUX_FIELDS)
    if unknown:
        raise KeyError(f"unknown aux fields {sorted(unknown)}")
    a = _keep_alive(moe_aux(*[_ptr(tensors.get(f)) for f in _AUX_FIELDS]), tensors)
    if stage_events is not None:
        if len(stage_events) != 2 * MOE_NUM_STAGES:
            raise ValueError("need 2 * MOE_NUM_STAGES events")
        arr = (ctypes.c_void_p * len(stage_events))(
            *[e if isinstance(e, int) else e.cuda_event for e in stage_events])
        a._events_keepalive = arr
        a.stage_events = ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p))
    return a


# ------------------------------------------------------------------------------------ the ABI
def moe_workspace_size(d) -> int:
    return int(lib().moe_workspace_size(ctypes.byref(_dims(d))))


def moe_router_topk(d, x, Wr, bias, scores, from_scores, topk_idx, topk_w, stream=None) -> int:
    return lib().moe_router_topk(ctypes.byref(_dims(d)), _ptr(x), _ptr(Wr), _ptr(bias), _ptr(scores),
                                 int(bool(from_scores)), _ptr(topk_idx), _ptr(topk_w), _stream(stream))


def moe_permute(d, topk_idx, z, expert_offsets, perm_token, inv_perm, z_perm, ws, ws_bytes=None, stream=None) -> int:
    ws_bytes = _nbytes(ws) if ws_bytes is None else ws_bytes
    return lib().moe_permute(ctypes.byref(_dims(d)), _ptr(topk_idx), _ptr(z), _ptr(expert_offsets), _ptr(perm_token),
                             _ptr(inv_perm), _ptr(z_perm), _ptr(ws), ws_bytes, _stream(stream))


def moe_expert_ffn(d, weights: moe_weights, z_perm, expert_offsets, y_perm, ws, ws_bytes=None, stream=None) -> int:
    ws_bytes = _nbytes(ws) if ws_bytes is None else ws_bytes
    return lib().moe_expert_ffn(ctypes.byref(_dims(d)), ctypes.byref(weights), _ptr(z_perm), _ptr(expert_offsets),
                                _ptr(y_perm), _ptr(ws), ws_bytes, _stream(stream))


def moe_combine(d, y_perm, inv_perm, topk_w, gamma, u_out, n_out, stream=None) -> int:
    return lib().moe_combine(ctypes.byref(_dims(d)), _ptr(y_perm), _ptr(inv_perm), _ptr(topk_w), _ptr(gamma),
                             _ptr(u_out), _ptr(n_out), _stream(stream))


def moe_layer_forward(d, weights: moe_weights, x, y, aux: moe_aux | None, ws, ws_bytes=None, stream=None) -> int:
    ws_bytes = _nbytes(ws) if ws_bytes is None else ws_bytes
    return lib().moe_layer_forward(ctypes.byref(_dims(d)), ctypes.byref(weights), _ptr(x), _ptr(y),
                                   ctypes.byref(aux) if aux is not None else None, _ptr(ws), ws_bytes,
                                   _stream(stream))


def moe_permute_noalloc(d, topk_idx, z, expert_offsets, perm_token, inv_perm, z_perm, stream=None) -> int:
    """moe_permute without a workspace, for callers that cannot allocate: its
    scratch is a fixed array inside the library (see include/moe.h)."""
    return lib().moe_permute_noalloc(ctypes.byref(_dims(d)), _ptr(topk_idx), _ptr(z), _ptr(expert_offsets),
                                     _ptr(perm_token), _ptr(inv_perm), _ptr(z_perm), _stream(stream))


def moe_qb_bias_update(d, scores, bias_in, bias_out, quantile_out, hist, nbins: int, lo: float, hi: float,
                       stream=None) -> int:
    """Quantile Balancing bias update from a batch of router scores (see
    include/moe.h); hist is an [E, nbins] uint32 workspace, overwritten."""
    return lib().moe_qb_bias_update(ctypes.byref(_dims(d)), _ptr(scores), _ptr(bias_in), _ptr(bias_out),
                                    _ptr(quantile_out), _ptr(hist), int(nbins), float(lo), float(hi), _stream(stream))


def moe_latent_shared(d, weights: moe_weights, x, z, h_s, stream=None) -> int:
    return lib().moe_latent_shared(ctypes.byref(_dims(d)), ctypes.byref(weights), _ptr(x), _ptr(z), _ptr(h_s),
                                   _stream(stream))


def moe_output(d, weights: moe_weights, h_s, n, y, stream=None) -> int:
    return lib().moe_output(ctypes.byref(_dims(d)), ctypes.byref(weights), _ptr(h_s), _ptr(n), _ptr(y),
                            _stream(stream))


def moe_expert_ffn_blocks_workspace_size(d, n_rows: int, n_blocks: int) -> int:
    return int(lib().moe_expert_ffn_blocks_workspace_size(ctypes.byref(_dims(d)), int(n_rows), int(n_blocks)))


def moe_expert_ffn_blocks(d, weights: moe_weights, x_rows, n_rows: int, block_offsets, n_blocks: int, y_rows, ws,
                          ws_bytes=None, stream=None) -> int:
    ws_bytes = _nbytes(ws) if ws_bytes is None else ws_bytes
    return lib().moe_expert_ffn_blocks(ctypes.byref(_dims(d)), ctypes.byref(weights), _ptr(x_rows), int(n_rows),
                                       _ptr(block_offsets), int(n_blocks), _ptr(y_rows), _ptr(ws), ws_bytes,
                                       _stream(stream))


def make_grads(**tensors) -> moe_grads:
    """moe_grads from keyword tensors named as the C struct fields."""
    unknown = set(tensors) - set(_GRAD_FIELDS)
    if unknown:
        raise KeyError(f"unknown gradient fields {sorted(unknown)}")
    return _keep_alive(moe_grads(*[_ptr(tensors.get(f)) for f in _GRAD_FIELDS]), tensors)


def moe_backward_workspace_size(d) -> int:
    return int(lib().moe_backward_workspace_size(ctypes.byref(_dims(d))))


def moe_layer_backward(d, weights: moe_weights, x, dy, topk_idx, grads: moe_grads, ws, ws_bytes=None,
                       stream=None) -> int:
    """Backward pass with the forward's selection held fixed (see include/moe.h)."""
    ws_bytes = _nbytes(ws) if ws_bytes is None else ws_bytes
    return lib().moe_layer_backward(ctypes.byref(_dims(d)), ctypes.byref(weights), _ptr(x), _ptr(dy), _ptr(topk_idx),
                                    ctypes.byref(grads), _ptr(ws), ws_bytes, _stream(stream))


MOE_FAULT_SELFTEST_WAIT = 9


def moe_mx_tiled_scales_size(d) -> tuple[int, int, int]:
    """(status, gate/up bytes, down bytes) of the tiled weight scales."""
    gu, dn = ctypes.c_size_t(0), ctypes.c_size_t(0)
    st = lib().moe_mx_tiled_scales_size(ctypes.byref(_dims(d)), ctypes.byref(gu), ctypes.byref(dn))
    return st, gu.value, dn.value


def moe_mx_tile_scales(d, Sg, Sv, So, Sgv_tiled, So_tiled, stream=None) -> int:
    return lib().moe_mx_tile_scales(ctypes.byref(_dims(d)), _ptr(Sg), _ptr(Sv), _ptr(So), _ptr(Sgv_tiled),
                                    _ptr(So_tiled), _stream(stream))


def moe_mx8_quantize(x, rows: int, K: int, codes, scales, stream=None) -> int:
    return lib().moe_mx8_quantize(_ptr(x), int(rows), int(K), _ptr(codes), _ptr(scales), _stream(stream))


def moe_mx4_quantize(x, rows: int, K: int, codes, scales, stream=None) -> int:
    return lib().moe_mx4_quantize(_ptr(x), int(rows), int(K), _ptr(codes), _ptr(scales), _stream(stream))


def moe_gather_rows(src, src_rows: int, row_bytes: int, idx, n: int, dst, stream=None) -> int:
    return lib().moe_gather_rows(_ptr(src), int(src_rows), int(row_bytes), _ptr(idx), int(n), _ptr(dst),
                                 _stream(stream))


def moe_selftest_wait_timeout(limit_ms: int, waited_ns, stream=None) -> int:
    """Runs the bounded-wait self-test (see include/moe.h)."""
    return lib().moe_selftest_wait_timeout(int(limit_ms), _ptr(waited_ns), _stream(stream))


def moe_status_str(status: int) -> str:
    return lib().moe_status_str(int(status)).decode()


def moe_device_error(stream=None) -> tuple[int, int]:
    """(status, fault code); synchronises the stream."""
    code = ctypes.c_int(0)
    st = lib().moe_device_error(ctypes.byref(code), _stream(stream))
    return int(st), int(code.value)


def moe_last_launch_count() -> int:
    return int(lib().moe_last_launch_count())


def check(status: int) -> None:
    """Raise RuntimeError for a non-OK status."""
    if status != MOE_OK:
        raise RuntimeError(f"moe call failed: {moe_status_str(status)}")
