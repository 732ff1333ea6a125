"""Block-scaled routed experts (MXFP4 weights x MXFP8 inputs on tcgen05.mma
kind::mxf8f6f4, and x MXFP4 inputs on kind::mxf4) against the oracle: the
quantisers bit for bit, the weight-scale tiling index by index, the expert
GEMMs and the whole layer to the stated bars.  The oracle quantises the same
bf16 inputs by the same rule (OCP MX v1.0 MXFP8 / MXFP4 with the shared-scale
rule): given the same input rows the gate/up GEMMs multiply the same numbers
on both sides; after that the device's bf16 h (and in the whole layer its z)
can differ from the oracle's by a rounding step, which can flip a code (bars
derived in harness.py)."""
import numpy as np
import pytest
import torch

import gen
import oracle
import sparse_moe_layer_renormalised_b200 as moe
from harness import (TOL_H_BLOCK_SCALED, TOL_MXFP4_A4, TOL_MXFP4_A4_LAYER, TOL_MXFP4_A8, TOL_MXFP4_A8_LAYER,
                     TOL_RMS_A4, TOL_RMS_A4_LAYER, TOL_RMS_A8_LAYER, compare_layer, dims_for, make_device_layer, parity,
                     rms_parity, run_layer)
from oracle import inputs as oin
from sparse_moe_layer_renormalised_b200.layer import tile_weight_scales

pytestmark = pytest.mark.gpu
F64 = torch.float64


def _no_fault():
    st, code = moe.moe_device_error()
    assert st == moe.MOE_OK and code == 0, f"device fault {code}"


def _quantiser_input(rows: int, K: int, seed: int) -> torch.Tensor:
    """bf16 rows whose 32-blocks span many binades, with the quantiser's
    special cases planted: an all-zero block (with a -0), a block whose
    largest value saturates (1.9375 * 2^e -> 496 units -> 448), bf16
    subnormals, and values near the bf16 maximum."""
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(rows, K, generator=g, dtype=torch.float64)
    binade = torch.randint(-30, 30, (rows, K // 32, 1), generator=g).to(F64)
    x = (x.reshape(rows, K // 32, 32) * torch.exp2(binade)).reshape(rows, K)
    x[0, :32] = 0.0
    x[0, 5] = -0.0
    if K >= 64:
        x[0, 32:64] = 0.25
        x[0, 40] = -1.9375
    if K >= 96:
        x[0, 64:96] = torch.linspace(-3e-39, 3e-39, 32, dtype=F64)  # bf16 subnormals
    if rows > 1 and K >= 64:
        x[1, 32:64] = torch.linspace(-3.0e38, 3.0e38, 32, dtype=F64)
    return x.to(torch.bfloat16)


# (device entry, oracle quantiser, code bytes per element) of each input format
_QUANT = {"mxfp8": (moe.moe_mx8_quantize, oracle.mx8_quantize, 1),
          "mxfp4": (moe.moe_mx4_quantize, oracle.mx4_quantize, 2)}


@pytest.mark.parametrize("fmt", ["mxfp8", "mxfp4"])
@pytest.mark.parametrize("rows,K", [(1, 32), (300, 1024), (1000, 3584), (129, 3072)])
def test_mx_quantize_bit_exact(fmt, rows, K):
    entry, ref_q, per = _QUANT[fmt]
    x = _quantiser_input(rows, K, rows + K)
    codes = torch.empty(rows, K // per, dtype=torch.uint8, device="cuda")
    scales = torch.empty(rows, K // 32, dtype=torch.uint8, device="cuda")
    assert entry(x.cuda(), rows, K, codes, scales) == moe.MOE_OK
    torch.cuda.synchronize()
    _no_fault()
    ref_codes, ref_scales = ref_q(x.to(F64))
    got_c, got_s = codes.cpu().numpy(), scales.cpu().numpy()
    assert np.array_equal(got_s, ref_scales), int((got_s != ref_scales).sum())
    assert np.array_equal(got_c, ref_codes), int((got_c != ref_codes).sum())


@pytest.mark.parametrize("fmt", ["mxfp8", "mxfp4"])
def test_mx_quantize_rejects_bad_arguments(fmt):
    entry = _QUANT[fmt][0]
    x = torch.zeros(4, 64, dtype=torch.bfloat16, device="cuda")
    c = torch.empty(4, 64, dtype=torch.uint8, device="cuda")
    s = torch.empty(4, 2, dtype=torch.uint8, device="cuda")
    assert entry(x, 4, 48, c, s) == moe.MOE_ERR_INVALID_ARG  # K not a multiple of 32
    assert entry(None, 4, 64, c, s) == moe.MOE_ERR_INVALID_ARG
    assert entry(x, 0, 64, None, None) == moe.MOE_OK


def test_tile_scales_layout():
    """moe_mx_tile_scales against a host re-indexing of the row-major scales by
    the layout include/moe.h states (atom byte 16*(m%32) + 4*(m/32) + j)."""
    cfg = gen.CONFIGS["mxfp4a8-small"]
    d = dims_for(cfg)
    w = gen.device_layer(cfg, "cuda", with_x=False)
    t = tile_weight_scales(d, w["Sg"], w["Sv"], w["So"])
    torch.cuda.synchronize()
    E, I, L = cfg.E, cfg.I, cfg.L
    Sg, Sv, So = (w[n].cpu().numpy() for n in ("Sg", "Sv", "So"))
    j = np.arange(512)
    m = (j >> 4) + 32 * ((j >> 2) & 3)
    kb = j & 3
    gu = t["Sgv_tiled"].cpu().numpy().reshape(E, I // 128, 2, L // 128, 512)
    e, wt, c, ch, jj = np.meshgrid(np.arange(E), np.arange(I // 128), np.arange(2), np.arange(L // 128), j,
                                   indexing="ij")
    mm = m[jj]
    row = wt * 128 + c * 64 + (mm % 64)
    col = 4 * ch + kb[jj]
    want = np.where(mm < 64, Sg[e, row, col], Sv[e, row, col])
    assert np.array_equal(gu, want)
    dn = t["So_tiled"].cpu().numpy().reshape(E, L // 256, 2, I // 128, 512)
    e, wt, c, ch, jj = np.meshgrid(np.arange(E), np.arange(L // 256), np.arange(2), np.arange(I // 128), j,
                                   indexing="ij")
    assert np.array_equal(dn, So[e, wt * 256 + c * 128 + m[jj], 4 * ch + kb[jj]])


def _routing(T, E, k, skew, seed):
    g = torch.Generator().manual_seed(seed)
    logits = torch.randn(T, E, generator=g)
    if skew:  # a few experts take most tokens (several 240-row tiles each)
        logits = logits + 3.0 * (torch.arange(E, dtype=torch.float32) + 1.0) ** -0.3
    return torch.topk(logits, k, dim=1).indices.to(torch.int32)


@pytest.mark.parametrize("T,skew", [(300, False), (40, False), (1024, True), (1, False)])
def test_expert_ffn_a8(T, skew):
    """Routed experts on the block-scaled path against the oracle, which
    quantises the same bf16 rows (z, then h) and decodes the same weight bits.
    The skewed case gives experts several token tiles; T = 1 a 16-wide MMA."""
    cfg = gen.CONFIGS["mxfp4a8-small"].with_(T=T)
    E, k, L = cfg.E, cfg.k, cfg.L
    d = dims_for(cfg, T=T)
    w = gen.device_layer(cfg, "cuda", with_x=False)
    idx = _routing(T, E, k, skew, 31 + T)
    counts, offsets, _, _ = oracle.permute(idx.numpy(), E)
    R = T * k
    z_perm = torch.randn(R, L, generator=torch.Generator().manual_seed(6)).to(torch.bfloat16)
    y_perm = torch.full((R, L), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.empty(moe.moe_workspace_size(d), dtype=torch.uint8, device="cuda")
    wts = moe.make_weights(Wg=w["Wg"], Wv=w["Wv"], Wo=w["Wo"], **tile_weight_scales(d, w["Sg"], w["Sv"], w["So"]))
    off = torch.as_tensor(offsets, dtype=torch.int32).cuda()
    assert moe.moe_expert_ffn(d, wts, z_perm.cuda(), off, y_perm, ws) == moe.MOE_OK
    torch.cuda.synchronize()
    _no_fault()
    if skew:
        assert int(np.max(counts)) > 2 * 240  # several tiles for the largest expert
    zf = z_perm.to(F64)
    ref = torch.empty(R, L, dtype=F64)
    for e in range(E):
        a, b = offsets[e], offsets[e + 1]
        if a == b:
            continue
        Wg, Wv, Wo = oin.expert_weights(cfg, e)
        ref[a:b] = oracle.expert_forward(zf[a:b], Wg, Wv, Wo, cfg.situ_c, oracle.bf16_round, act="mxfp8")
    assert parity(y_perm.cpu().to(F64), ref) <= TOL_MXFP4_A8


@pytest.mark.parametrize("T,skew", [(300, False), (40, False), (1024, True), (1, False)])
def test_expert_ffn_a4(T, skew):
    """Routed experts on the all-4-bit path (kind::mxf4) against the oracle.
    Both sides quantise the same bf16 z rows to the same MXFP4 codes, so the
    gate/up GEMM multiplies identical numbers: its stored h (read from the
    entry's workspace) is checked elementwise to within a bf16 step.  y then
    takes the derived bars for h's code flips (max and rms)."""
    cfg = gen.CONFIGS["mxfp4a4-small"].with_(T=T)
    E, k, L, I = cfg.E, cfg.k, cfg.L, cfg.I
    d = dims_for(cfg, T=T)
    w = gen.device_layer(cfg, "cuda", with_x=False)
    idx = _routing(T, E, k, skew, 31 + T)
    counts, offsets, _, _ = oracle.permute(idx.numpy(), E)
    R = T * k
    z_perm = torch.randn(R, L, generator=torch.Generator().manual_seed(6)).to(torch.bfloat16)
    y_perm = torch.full((R, L), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.zeros(moe.moe_expert_ffn_blocks_workspace_size(d, R, 1), dtype=torch.uint8, device="cuda")
    wts = moe.make_weights(Wg=w["Wg"], Wv=w["Wv"], Wo=w["Wo"], **tile_weight_scales(d, w["Sg"], w["Sv"], w["So"]))
    off = torch.as_tensor(offsets, dtype=torch.int32).cuda()
    assert moe.moe_expert_ffn_blocks(d, wts, z_perm.cuda(), R, off, 1, y_perm, ws) == moe.MOE_OK
    torch.cuda.synchronize()
    _no_fault()
    if skew:
        assert int(np.max(counts)) > 2 * 208  # several tiles for the largest expert
    h_dev = ws[: R * I * 2].view(torch.bfloat16).view(R, I).cpu().to(F64)
    zf = z_perm.to(F64)
    ref = torch.empty(R, L, dtype=F64)
    h_ref = torch.empty(R, I, dtype=F64)
    for e in range(E):
        a, b = offsets[e], offsets[e + 1]
        if a == b:
            continue
        Wg, Wv, Wo = oin.expert_weights(cfg, e)
        zq = oracle.mx4_round(zf[a:b])
        h_ref[a:b] = oracle.bf16_round(oracle.situ_glu(zq @ Wg.T, zq @ Wv.T, cfg.situ_c))
        ref[a:b] = oracle.expert_forward(zf[a:b], Wg, Wv, Wo, cfg.situ_c, oracle.bf16_round, act="mxfp4")
    step = torch.exp2(torch.frexp(h_ref.abs())[1].to(F64) - 8)  # one bf16 step at |h_ref|
    assert bool(((h_dev - h_ref).abs() <= step + TOL_H_BLOCK_SCALED * h_ref.pow(2).mean().sqrt()).all())
    y = y_perm.cpu().to(F64)
    assert parity(y, ref) <= TOL_MXFP4_A4
    assert rms_parity(y, ref) <= TOL_RMS_A4


def test_a8_layer_all_tokens():
    """The whole layer with block-scaled routed experts, every token against
    the oracle (bars derived in harness.py: the layer's bf16 z and h differ
    from the oracle's by a rounding step, which can flip an E4M3 code)."""
    cfg = gen.CONFIGS["mxfp4a8-small"]
    layer, w = make_device_layer(cfg)
    y, aux = run_layer(layer, w["x"])
    m = compare_layer(cfg, np.arange(cfg.T), y, aux, TOL_MXFP4_A8_LAYER, rms_tol=TOL_RMS_A8_LAYER)
    print(f"\n[mxfp4a8-small] " + " ".join(f"{k}={v:.3g}" if isinstance(v, float) else f"{k}={v}" for k, v in m.items()))


def test_a8_layer_matches_mxfp4_up_to_activation_rounding():
    """Same weights and selection: the block-scaled layer differs from the
    bf16-activation MXFP4 layer by the MXFP8 rounding of the expert inputs,
    a few per cent of rms (the oracle's own distance between the two, about
    4% of rms(y) at this shape), not more."""
    c8 = gen.CONFIGS["mxfp4a8-small"]
    c4 = gen.CONFIGS["mxfp4-small"]
    l8, w = make_device_layer(c8)
    y8, _ = run_layer(l8, w["x"])
    l4 = moe.MoeLayer(dims_for(c4), {k: v for k, v in w.items() if k != "x"})
    y4, _ = run_layer(l4, w["x"])
    d = (y8 - y4).double()
    rel_rms = (d.pow(2).mean().sqrt() / y4.double().pow(2).mean().sqrt()).item()
    assert 1e-3 < rel_rms < 0.1, rel_rms


def test_a4_layer_all_tokens():
    """The whole layer with all-4-bit routed experts, every token against the
    oracle (bars derived in harness.py)."""
    cfg = gen.CONFIGS["mxfp4a4-small"]
    layer, w = make_device_layer(cfg)
    y, aux = run_layer(layer, w["x"])
    m = compare_layer(cfg, np.arange(cfg.T), y, aux, TOL_MXFP4_A4_LAYER, rms_tol=TOL_RMS_A4_LAYER)
    print(f"\n[mxfp4a4-small] " + " ".join(f"{k}={v:.3g}" if isinstance(v, float) else f"{k}={v}" for k, v in m.items()))


def test_a4_layer_matches_mxfp4_up_to_activation_rounding():
    """Same weights and selection: the all-4-bit layer differs from the
    bf16-activation MXFP4 layer by the MXFP4 rounding of the expert inputs
    (the oracle's own distance between the two is 17% of rms(y) at this
    shape), neither much less nor much more."""
    c4a = gen.CONFIGS["mxfp4a4-small"]
    c4 = gen.CONFIGS["mxfp4-small"]
    la, w = make_device_layer(c4a)
    ya, _ = run_layer(la, w["x"])
    l4 = moe.MoeLayer(dims_for(c4), {k: v for k, v in w.items() if k != "x"})
    y4, _ = run_layer(l4, w["x"])
    d = (ya - y4).double()
    rel_rms = (d.pow(2).mean().sqrt() / y4.double().pow(2).mean().sqrt()).item()
    assert 0.08 < rel_rms < 0.35, rel_rms


@pytest.mark.slow
def test_k3_a4_sampled():
    """K3 shape, all-4-bit routed experts at T = 8192, seeded token sample."""
    from harness import K3_SAMPLE

    cfg = gen.CONFIGS["mxfp4-a4"]
    layer, w = make_device_layer(cfg)
    y, aux = run_layer(layer, w["x"])
    tokens = gen.sample_tokens(cfg, min(K3_SAMPLE, cfg.T))
    m = compare_layer(cfg, tokens, y, aux, TOL_MXFP4_A4_LAYER, rms_tol=TOL_RMS_A4_LAYER)
    print(f"\n[mxfp4-a4] " + " ".join(f"{k}={v:.3g}" if isinstance(v, float) else f"{k}={v}" for k, v in m.items()))


@pytest.mark.slow
def test_k3_a8_sampled():
    """K3 shape, block-scaled routed experts at the full T = 8192, seeded sample
    of tokens against the oracle quantising and decoding the same bits."""
    from harness import K3_SAMPLE

    cfg = gen.CONFIGS["mxfp4-a8"]
    layer, w = make_device_layer(cfg)
    y, aux = run_layer(layer, w["x"])
    tokens = gen.sample_tokens(cfg, min(K3_SAMPLE, cfg.T))
    m = compare_layer(cfg, tokens, y, aux, TOL_MXFP4_A8_LAYER, rms_tol=TOL_RMS_A8_LAYER)
    print(f"\n[mxfp4-a8] " + " ".join(f"{k}={v:.3g}" if isinstance(v, float) else f"{k}={v}" for k, v in m.items()))
