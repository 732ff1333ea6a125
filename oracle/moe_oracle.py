"""fp64 CPU oracle of the Stable LatentMoE layer (test infrastructure only).

Sources (web pages; cited by title and section):

[K3-896] "Kimi K3の896エキスパートを「896人の専門家」と呼ぶと何がズレるか、
         ルーターは何を選んでいるのか" (lilting.ch)
   - section "K3のエキスパートは896個の小型LLMではない": the dimension table and
     the three layer equations  z = W_down x ;  u = sum_{i in Top16} p_i E_i(z) ;
     y = E1_shared(x) + E2_shared(x) + W_up RMSNorm(u).
   - section "ルーターは計算の割当器": s = Sigmoid(W_r x); a per-expert balancing
     bias is added to the scores to choose the top 16; the mixture weights are
     the original (unbiased) scores normalised over the chosen experts.
   - section "ルーター専用の独立訓練はない": the bias is frozen at inference.
[K3-2axis] "Kimi K3の二軸スケーリング戦略とは何か" (studioglobal.ai), section
   "Stable LatentMoE：条件付きの大容量を安定させる": inference uses the fixed
   expert bias with ordinary top-k selection.
[K3-report] Kimi K3 tech-report summary (jiwasawa.github.io), section
   "幅のスケーリング：Stable LatentMoE": SiTU-GLU keeps SwiGLU's local
   non-linearity and puts smooth caps on both the linear and the up branch.
[K3-QAT] ai-tech-express.jp article, section "量子化を前提とした学習「MXFP4
   Quantization-Aware Training」": routed weights are served in MXFP4.  The
   pages name no activation format; for the block-scaled variants, whose routed
   experts take MXFP8 or MXFP4 inputs, the reading is OCP MX v1.0's MXFP8
   (E4M3) or MXFP4 (E2M1) with that specification's shared-scale rule.

Readings where the pages are silent (each is also listed in the design notes):
  * SiTU-GLU is taken as  h = sigmoid(g) * c*tanh(g/c) * c*tanh(v/c),  c = 10:
    SwiGLU is silu(g)*v = sigmoid(g)*g*v, and the two soft caps replace the
    linear factor g and the up branch v by c*tanh(./c).
  * The shared experts use the same SiTU-GLU.
  * RMSNorm(u) = gamma * u / sqrt(mean(u^2) + eps), eps = 1e-6, gamma given.
  * Ties in the selection key go to the lower expert index; slots are listed
    in descending key order.
  * Dropless routing (every token gets its k experts).
  * Storage-faithful rounding: where the device path must hold a tensor in the
    activation type (bf16) because it is a tensor-core operand -- z, h, the
    shared h and n -- the oracle rounds its fp64 value to that type (round to
    nearest even); everything else stays fp64.
"""
from __future__ import annotations

import math

import numpy as np
import torch

__all__ = [
    "bf16_round",
    "f32_round",
    "storage_round",
    "bf16_bits_to_f64",
    "f32_to_f64",
    "E2M1_VALUES",
    "mxfp4_dequant",
    "e4m3_decode",
    "e4m3_encode",
    "mx8_quantize",
    "mx8_dequant",
    "mx8_round",
    "e2m1_encode",
    "mx4_quantize",
    "mx4_round",
    "routed_act",
    "act_round",
    "sigmoid",
    "router_scores",
    "select_experts",
    "select_experts_from_f32_scores",
    "permute",
    "situ_glu",
    "expert_forward",
    "combine",
    "rms_norm",
    "shared_experts",
    "layer_forward",
    "layer_forward_streamed",
]

F64 = torch.float64


# ----------------------------------------------------------------------------------------------
# Number formats
# ----------------------------------------------------------------------------------------------
def bf16_round(t: torch.Tensor) -> torch.Tensor:
    """Round fp64 values to the nearest bfloat16 (ties to even), returned as fp64.

    bfloat16 keeps 8 significant bits, i.e. the top 7 of fp64's 52 stored
    mantissa bits; the 45 bits below are rounded away in one step (no
    intermediate fp32 rounding).  Values are assumed finite and inside the
    normal bf16 range."""
    t = t.to(F64).contiguous()
    u = t.view(torch.int64)
    lsb = (u >> 45) & 1
    u = (u + ((1 << 44) - 1) + lsb) & ~((1 << 45) - 1)
    return u.view(F64)


def f32_round(t: torch.Tensor) -> torch.Tensor:
    """Round fp64 values to the nearest fp32, returned as fp64."""
    return t.to(torch.float32).to(F64)


def storage_round(act: str):
    """The rounding applied where the device path stores an activation."""
    return {"bf16": bf16_round, "f32": f32_round}[act]


def bf16_bits_to_f64(a) -> torch.Tensor:
    """Raw bfloat16 bit patterns (uint16) -> fp64 values (exact): the 16 bits
    are the top half of the fp32 with the same value."""
    a = np.ascontiguousarray(np.asarray(a))
    assert a.dtype == np.uint16
    w = torch.from_numpy(a.view(np.int16)).to(torch.int32).bitwise_left_shift(16)
    return w.view(torch.float32).to(F64)


def f32_to_f64(a) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(np.asarray(a, dtype=np.float32))).to(F64)


# E2M1 magnitudes of codes 0..7 (OCP Microscaling Formats v1.0, FP4 E2M1).
E2M1_VALUES = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)


def mxfp4_dequant(codes, scales) -> torch.Tensor:
    """MXFP4 weights -> fp64 [rows, K] ([K3-QAT] names the format; OCP MX v1.0
    fixes it): element k of a row is  E2M1(code_k) * 2^(scale_{k//32} - 127),
    code_k the low nibble of byte k//2 for even k and the high nibble for odd
    k, bit 3 of the code being the sign.  Scale byte 255 is NaN."""
    codes = torch.from_numpy(np.ascontiguousarray(codes)).to(torch.int64)
    scales = torch.from_numpy(np.ascontiguousarray(scales)).to(torch.int64)
    rows, half = codes.shape
    K = 2 * half
    nib = torch.empty(rows, K, dtype=torch.int64)
    nib[:, 0::2] = codes & 0xF
    nib[:, 1::2] = codes >> 4
    table = torch.tensor(E2M1_VALUES, dtype=F64)
    mag = table[nib & 7]
    val = torch.where((nib & 8) != 0, -mag, mag)
    s = scales.repeat_interleave(32, dim=1)
    factor = torch.pow(torch.tensor(2.0, dtype=F64), (s - 127).to(F64))
    factor = torch.where(s == 255, torch.tensor(float("nan"), dtype=F64), factor)
    return val * factor


def e4m3_decode(codes) -> torch.Tensor:
    """OCP FP8 E4M3 codes -> fp64: sign bit 7, exponent bits 6-3 with bias 7,
    mantissa bits 2-0; exponent field 0 is subnormal (m/8 * 2^-6); no
    infinities; S.1111.111 is NaN."""
    c = torch.from_numpy(np.ascontiguousarray(np.asarray(codes, dtype=np.uint8))).to(torch.int64)
    e = (c >> 3) & 15
    m = (c & 7).to(F64)
    two = torch.tensor(2.0, dtype=F64)
    normal = (1.0 + m / 8.0) * torch.pow(two, (e - 7).to(F64))
    sub = (m / 8.0) * torch.pow(two, torch.tensor(-6.0, dtype=F64))
    mag = torch.where(e == 0, sub, normal)
    mag = torch.where((e == 15) & ((c & 7) == 7), torch.tensor(float("nan"), dtype=F64), mag)
    return torch.where((c & 0x80) != 0, -mag, mag)


def e4m3_encode(v) -> np.ndarray:
    """Nearest E4M3 code to each fp64 value, ties to the even code, magnitudes
    beyond 448 (the largest finite E4M3) saturated to 448; -0 keeps its sign.

    Between 2^q and 2^(q+1) the E4M3 numbers are spaced 2^(q-3) (2^-9 below
    2^-6, the subnormal range), so rounding is  round_half_even(a / spacing)
    spacing units."""
    v = torch.as_tensor(v).to(F64)
    neg = torch.signbit(v)
    a = torch.clamp(v.abs(), max=448.0)
    _, ex = torch.frexp(a)                  # a in [2^(ex-1), 2^ex)
    q = torch.clamp(ex.to(torch.int64) - 1, min=-6)
    q = torch.where(a == 0, torch.full_like(q, -6), q)   # zero: the subnormal range
    units = torch.round(torch.ldexp(a, (3 - q).to(torch.int64)))   # half to even
    # units: 0..8 in the subnormal range (8 = the smallest normal, 2^-6); 8..16 else
    carry = units >= 16
    q = torch.where(carry, q + 1, q)
    units = torch.where(carry, units / 2, units)
    sub = (q == -6) & (units < 8)
    exp_field = torch.where(sub, torch.zeros_like(q), q + 7)
    mant = torch.where(sub, units, units - 8).to(torch.int64)
    code = (exp_field << 3) | mant
    code = torch.where(neg, code | 0x80, code)
    return code.to(torch.uint8).numpy()


def mx8_quantize(v) -> tuple[np.ndarray, np.ndarray]:
    """Rows of fp64 values [R, K] (K a multiple of 32) -> OCP MXFP8: per block
    of 32 along K the shared scale 2^s, s = floor(log2(max |v|)) - 8 (8 = the
    largest E4M3 exponent) clamped to the E8M0 range [-127, 127] (an all-zero
    block takes -127), and the E4M3 codes of v / 2^s.  Returns (codes [R, K],
    scale bytes s + 127 [R, K/32]), both uint8."""
    v = torch.as_tensor(v).to(F64)
    R, K = v.shape
    blocks = v.reshape(R, K // 32, 32)
    amax = blocks.abs().amax(dim=2)
    _, ex = torch.frexp(amax)
    s = torch.clamp(ex.to(torch.int64) - 1 - 8, min=-127, max=127)
    s = torch.where(amax == 0, torch.full_like(s, -127), s)
    scaled = torch.ldexp(blocks, (-s)[:, :, None].expand(R, K // 32, 32))
    codes = e4m3_encode(scaled.reshape(R, K))
    return codes, (s + 127).to(torch.uint8).numpy()


def mx8_dequant(codes, scales) -> torch.Tensor:
    """MXFP8 codes [R, K] and scale bytes [R, K/32] -> fp64 values."""
    val = e4m3_decode(codes)
    s = torch.from_numpy(np.ascontiguousarray(np.asarray(scales, dtype=np.int64))).repeat_interleave(32, dim=1)
    factor = torch.pow(torch.tensor(2.0, dtype=F64), (s - 127).to(F64))
    factor = torch.where(s == 255, torch.tensor(float("nan"), dtype=F64), factor)
    return val * factor


def mx8_round(v) -> torch.Tensor:
    """The values the MXFP8 encoding of rows v stands for."""
    return mx8_dequant(*mx8_quantize(v))


def e2m1_encode(v) -> np.ndarray:
    """Nearest E2M1 code (one per byte, 0..15) to each fp64 value, ties to the
    even code, magnitudes beyond 6 (the largest E2M1) saturated to 6; -0 keeps
    its sign.

    The E2M1 numbers are spaced 0.5 below 2 (0.5 is the subnormal) and
    2^(q-1) between 2^q and 2^(q+1) for q = 1, 2, so rounding is
    round_half_even(a / spacing) spacing units."""
    v = torch.as_tensor(v).to(F64)
    neg = torch.signbit(v)
    a = torch.clamp(v.abs(), max=6.0)
    _, ex = torch.frexp(a)                   # a in [2^(ex-1), 2^ex)
    q = torch.clamp(ex.to(torch.int64) - 1, min=0)
    units = torch.round(torch.ldexp(a, (1 - q).to(torch.int64)))   # half to even
    # q = 0: units 0..4 are the codes 0..4 (4 = 2.0); q >= 1: units 2..4, 4 carries
    carry = (q >= 1) & (units >= 4)
    q = torch.where(carry, q + 1, q)
    units = torch.where(carry, units / 2, units).to(torch.int64)
    code = torch.where(q == 0, units, ((q + 1) << 1) | (units - 2))
    code = torch.where(neg, code | 8, code)
    return code.to(torch.uint8).numpy()


def mx4_quantize(v) -> tuple[np.ndarray, np.ndarray]:
    """Rows of fp64 values [R, K] (K a multiple of 32) -> OCP MXFP4: per block
    of 32 along K the shared scale 2^s, s = floor(log2(max |v|)) - 2 (2 = the
    largest E2M1 exponent) clamped to [-127, 127] (an all-zero block takes
    -127), and the E2M1 codes of v / 2^s, two per byte (element 2i in the low
    nibble).  Returns (codes [R, K/2], scale bytes s + 127 [R, K/32])."""
    v = torch.as_tensor(v).to(F64)
    R, K = v.shape
    blocks = v.reshape(R, K // 32, 32)
    amax = blocks.abs().amax(dim=2)
    _, ex = torch.frexp(amax)
    s = torch.clamp(ex.to(torch.int64) - 1 - 2, min=-127, max=127)
    s = torch.where(amax == 0, torch.full_like(s, -127), s)
    scaled = torch.ldexp(blocks, (-s)[:, :, None].expand(R, K // 32, 32))
    nib = e2m1_encode(scaled.reshape(R, K))
    codes = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    return codes, (s + 127).to(torch.uint8).numpy()


def mx4_round(v) -> torch.Tensor:
    """The values the MXFP4 encoding of rows v stands for."""
    return mxfp4_dequant(*mx4_quantize(v))


def routed_act(cfg) -> str | None:
    """The input format of the routed experts' GEMMs: "mxfp8" for the
    block-scaled MXFP4 x MXFP8 variant, "mxfp4" for MXFP4 x MXFP4, else None
    (the stored activations)."""
    return {"mxfp4_a8": "mxfp8", "mxfp4_a4": "mxfp4"}.get(getattr(cfg, "routed", None))


def act_round(act: str | None, v) -> torch.Tensor:
    """Rows v replaced by their values in the activation format act."""
    if act is None:
        return v
    return {"mxfp8": mx8_round, "mxfp4": mx4_round}[act](v)


# ----------------------------------------------------------------------------------------------
# Router: s = Sigmoid(W_r x), bias for selection only, renormalised unbiased scores
# ([K3-896] section "ルーターは計算の割当器"; [K3-2axis] fixed bias + ordinary top-k)
# ----------------------------------------------------------------------------------------------
def sigmoid(t: torch.Tensor) -> torch.Tensor:
    return 1.0 / (1.0 + torch.exp(-t))


def router_scores(x: torch.Tensor, Wr: torch.Tensor) -> torch.Tensor:
    """s[t, e] = sigmoid(sum_h x[t, h] * W_r[e, h]) in fp64."""
    return sigmoid(x.to(F64) @ Wr.to(F64).T)


def _top_k_by_key(key: torch.Tensor, k: int):
    """Indices of the k largest keys per row, largest first, ties to the lower
    index (a stable descending sort keeps equal keys in index order)."""
    sorted_key, order = torch.sort(key, dim=1, descending=True, stable=True)
    return order[:, :k], sorted_key


def select_experts(s: torch.Tensor, b: torch.Tensor, k: int):
    """Selection with the frozen bias: key = s + b (fp64); the top k keys are
    chosen; p_j = s_{e_j} / sum_{j'} s_{e_j'} with the UNBIASED scores.

    b is [E] (one bias for all tokens) or [T, E].
    Returns (idx [T,k] int64, p [T,k] fp64, margin [T] fp64) where margin is
    key_(k) - key_(k+1), the gap between the k-th and (k+1)-th largest key
    (+inf when k == E)."""
    s = s.to(F64)
    b = b.to(F64)
    key = s + (b[None, :] if b.dim() == 1 else b)
    idx, sorted_key = _top_k_by_key(key, k)
    s_sel = torch.gather(s, 1, idx)
    p = s_sel / s_sel.sum(dim=1, keepdim=True)
    if k < key.shape[1]:
        margin = sorted_key[:, k - 1] - sorted_key[:, k]
    else:
        margin = torch.full((key.shape[0],), math.inf, dtype=F64)
    return idx, p, margin


def select_experts_from_f32_scores(s32, b32, k: int):
    """Selection from given fp32 scores, as the device computes it: the key is
    the fp32 sum fl32(s + b); the order rule is that of select_experts.
    p is returned in fp64 from the fp32 scores."""
    s32 = torch.as_tensor(np.asarray(s32, dtype=np.float32))
    b32 = torch.as_tensor(np.asarray(b32, dtype=np.float32))
    key = s32 + b32[None, :]  # fp32 add, round to nearest
    idx, _ = _top_k_by_key(key, k)
    s_sel = torch.gather(s32.to(F64), 1, idx)
    p = s_sel / s_sel.sum(dim=1, keepdim=True)
    return idx, p


def permute(idx, E: int):
    """Expert-contiguous ordering of the (token, slot) pairs.

    Rows of expert e occupy positions offsets[e] .. offsets[e+1]-1, in
    ascending token order.  perm_token[pos] is the token of the pair stored
    at pos; inv_perm[t*k + j] is the position of pair (t, j)."""
    idx = np.asarray(idx)
    T, k = idx.shape
    lists = [[] for _ in range(E)]
    for t in range(T):
        for j in range(k):
            lists[int(idx[t, j])].append((t, j))
    counts = np.array([len(l) for l in lists], dtype=np.int64)
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    perm_token = np.empty(T * k, dtype=np.int64)
    inv_perm = np.empty(T * k, dtype=np.int64)
    pos = 0
    for e in range(E):
        for t, j in lists[e]:
            perm_token[pos] = t
            inv_perm[t * k + j] = pos
            pos += 1
    return counts, offsets, perm_token, inv_perm


# ----------------------------------------------------------------------------------------------
# Experts ([K3-896] section "K3のエキスパートは896個の小型LLMではない"; SiTU-GLU from [K3-report])
# ----------------------------------------------------------------------------------------------
def situ_glu(g: torch.Tensor, v: torch.Tensor, c: float) -> torch.Tensor:
    """SiTU-GLU: sigmoid(g) * (c * tanh(g / c)) * (c * tanh(v / c))."""
    return sigmoid(g) * (c * torch.tanh(g / c)) * (c * torch.tanh(v / c))


def expert_forward(z_rows: torch.Tensor, Wg: torch.Tensor, Wv: torch.Tensor, Wo: torch.Tensor, c: float, rnd,
                   act: str | None = None):
    """One GLU expert on latent rows: g = W_g z, v = W_v z, h = SiTU-GLU(g, v)
    (stored, so rounded by rnd), y = W_o h (fp64, not rounded).  act ("mxfp8"
    or "mxfp4", the block-scaled variants): the rows of z, and of h after rnd,
    are replaced by their values in that format before they enter the
    products."""
    z_rows = act_round(act, z_rows)
    g = z_rows @ Wg.T
    v = z_rows @ Wv.T
    h = rnd(situ_glu(g, v, c))
    h = act_round(act, h)
    return h @ Wo.T


def combine(y_slots: torch.Tensor, p: torch.Tensor) -> torch.Tensor:
    """u = sum_j p_j * y_j over the k slots, added in slot order."""
    T, k, _ = y_slots.shape
    u = torch.zeros(T, y_slots.shape[2], dtype=F64)
    for j in range(k):
        u = u + p[:, j : j + 1] * y_slots[:, j, :]
    return u


def rms_norm(u: torch.Tensor, gamma: torch.Tensor, eps: float) -> torch.Tensor:
    """gamma * u / sqrt(mean(u^2) + eps) over the latent dimension."""
    ms = (u * u).mean(dim=1, keepdim=True)
    return gamma.to(F64)[None, :] * u / torch.sqrt(ms + eps)


def shared_experts(x: torch.Tensor, Wsg, Wsv, Wso, c: float, rnd) -> torch.Tensor:
    """sum_i W_so,i SiTU-GLU(W_sg,i x, W_sv,i x); each h_i is stored (rounded)."""
    y = torch.zeros(x.shape[0], Wso.shape[1], dtype=F64)
    for i in range(Wsg.shape[0]):
        h = rnd(situ_glu(x @ Wsg[i].T, x @ Wsv[i].T, c))
        y = y + h @ Wso[i].T
    return y


# ----------------------------------------------------------------------------------------------
# The whole layer
# ----------------------------------------------------------------------------------------------
def _finish(x, z, idx, p, y_slots, dense, cfg, rnd):
    u = combine(y_slots, p)
    n = rnd(rms_norm(u, dense["gamma"], cfg.rms_eps))
    y_sh = shared_experts(x, dense["Wsg"], dense["Wsv"], dense["Wso"], cfg.situ_c, rnd)
    y = y_sh + n @ dense["Wup"].T
    return {"y": y, "u": u, "n": n, "z": z, "y_shared": y_sh}


def layer_forward(cfg, w: dict, x: torch.Tensor, forced_idx=None) -> dict:
    """Forward pass of the layer for the token rows x (fp64 [T, H]).

    w holds fp64 tensors: Wr [E,H], bias [E], Wdown [L,H], Wup [H,L],
    gamma [L], Wg/Wv [E,I,L], Wo [E,L,I], Wsg/Wsv [S,Is,H], Wso [S,H,Is].
    forced_idx (optional [T,k]) replaces the selected experts (the mixture
    weights are then the unbiased scores renormalised over those experts).

    Steps, in the order the pages give them:
      s = Sigmoid(W_r x); key = s + b; top-k; p = renormalised s   (router)
      z = W_down x                                                  (latent)
      u = sum_j p_j E_{e_j}(z)                                      (routed experts)
      y = E1_shared(x) + E2_shared(x) + W_up RMSNorm(u)             (output)
    """
    rnd = storage_round(cfg.act)
    s = router_scores(x, w["Wr"])
    idx, p, margin = select_experts(s, w["bias"], cfg.k)
    if forced_idx is not None:
        idx = torch.as_tensor(np.asarray(forced_idx), dtype=torch.int64)
        s_sel = torch.gather(s, 1, idx)
        p = s_sel / s_sel.sum(dim=1, keepdim=True)
    z = rnd(x @ w["Wdown"].T)
    T, k = idx.shape
    y_slots = torch.zeros(T, k, cfg.L, dtype=F64)
    for e in torch.unique(idx).tolist():
        t, j = torch.nonzero(idx == e, as_tuple=True)
        y_slots[t, j] = expert_forward(z[t], w["Wg"][e], w["Wv"][e], w["Wo"][e], cfg.situ_c, rnd,
                                       act=routed_act(cfg))
    out = _finish(x, z, idx, p, y_slots, w, cfg, rnd)
    out.update({"s": s, "idx": idx, "p": p, "margin": margin})
    return out


def layer_forward_streamed(cfg, dense: dict, x: torch.Tensor, expert_weights, forced_idx=None) -> dict:
    """Same computation as layer_forward for a sample of token rows, with the
    routed-expert weights supplied one expert at a time:
    expert_weights(e) -> (Wg_e [I,L], Wv_e [I,L], Wo_e [L,I]) fp64.
    Used when all routed weights do not fit in host memory at once."""
    rnd = storage_round(cfg.act)
    s = router_scores(x, dense["Wr"])
    idx, p, margin = select_experts(s, dense["bias"], cfg.k)
    if forced_idx is not None:
        idx = torch.as_tensor(np.asarray(forced_idx), dtype=torch.int64)
        s_sel = torch.gather(s, 1, idx)
        p = s_sel / s_sel.sum(dim=1, keepdim=True)
    z = rnd(x @ dense["Wdown"].T)
    T, k = idx.shape
    y_slots = torch.zeros(T, k, cfg.L, dtype=F64)
    for e in torch.unique(idx).tolist():
        t, j = torch.nonzero(idx == e, as_tuple=True)
        Wg, Wv, Wo = expert_weights(e)
        y_slots[t, j] = expert_forward(z[t], Wg, Wv, Wo, cfg.situ_c, rnd, act=routed_act(cfg))
    out = _finish(x, z, idx, p, y_slots, dense, cfg, rnd)
    out.update({"s": s, "idx": idx, "p": p, "margin": margin})
    return out
