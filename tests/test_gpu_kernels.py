"""Parity of each ABI stage against the oracle, element by element, on seeded
inputs that span several tiles and a ragged tail (GPU)."""
import numpy as np
import pytest
import torch

import gen
import oracle
import sparse_moe_layer_renormalised_b200 as moe
from harness import dims_for, parity, storage_steps
from oracle import inputs as oin

pytestmark = pytest.mark.gpu
F64 = torch.float64


def _dims(T, E, k, L=1024, I=768, H=2048, act="bf16"):
    return moe.Dims(T=T, H=H, L=L, E=E, k=k, I=I, S=2, Is=1024, act=act, routed=act)


def _no_fault():
    st, code = moe.moe_device_error()
    assert st == moe.MOE_OK and code == 0, f"device fault {code}"


# ------------------------------------------------------------------------------ top-k
@pytest.mark.parametrize("T,E,k,ties", [(1000, 896, 16, False), (4096, 128, 8, False), (64, 32, 4, False),
                                        (333, 896, 16, True), (1, 1024, 32, False), (77, 40, 32, True),
                                        (129, 5, 5, True)])
def test_topk_bit_exact_from_scores(T, E, k, ties):
    g = torch.Generator().manual_seed(T * 7 + E)
    s = torch.rand(T, E, generator=g, dtype=torch.float32)
    b = (torch.randn(E, generator=g, dtype=torch.float32) * 0.05)
    if ties:  # coarse values: many exactly equal keys (scores kept > 0)
        s = (torch.round(s * 16) + 1) / 17
        b = torch.round(b * 64) / 64
    idx_ref, p_ref = oracle.select_experts_from_f32_scores(s.numpy(), b.numpy(), k)
    d = _dims(T, E, k)
    sd, bd = s.cuda(), b.cuda()
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, k, dtype=torch.float32, device="cuda")
    assert moe.moe_router_topk(d, None, None, bd, sd, 1, idx, w) == moe.MOE_OK
    torch.cuda.synchronize()
    _no_fault()
    assert torch.equal(idx.cpu().to(torch.int64), idx_ref)
    rel = ((w.cpu().to(F64) - p_ref).abs() / p_ref).max().item()
    assert rel <= 1e-6


# ------------------------------------------------------------------------------ permute
def _routing(T, E, k, skew, seed):
    g = torch.Generator().manual_seed(seed)
    logits = torch.randn(T, E, generator=g)
    if skew:  # Zipf-like loads: a few experts take most tokens
        logits = logits + 3.0 * (torch.arange(E, dtype=torch.float32) + 1.0) ** -0.3
    return torch.topk(logits, k, dim=1).indices.to(torch.int32)


@pytest.mark.parametrize("T,E,k,skew", [(4096, 128, 8, False), (1000, 896, 16, True), (300, 32, 4, False),
                                        (1, 64, 8, False), (16384, 896, 16, True)])
def test_permute_exact(T, E, k, skew):
    idx = _routing(T, E, k, skew, T + E)
    counts, offsets, perm_token, inv_perm = oracle.permute(idx.numpy(), E)
    d = _dims(T, E, k, L=256)
    ws = torch.empty(moe.moe_workspace_size(d), dtype=torch.uint8, device="cuda")
    z = torch.randn(T, 256, device="cuda").to(torch.bfloat16)
    off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    pt = torch.empty(T * k, dtype=torch.int32, device="cuda")
    ip = torch.empty(T * k, dtype=torch.int32, device="cuda")
    zp = torch.empty(T * k, 256, dtype=torch.bfloat16, device="cuda")
    assert moe.moe_permute(d, idx.cuda(), z, off, pt, ip, zp, ws) == moe.MOE_OK
    torch.cuda.synchronize()
    _no_fault()
    assert np.array_equal(off.cpu().numpy(), offsets)
    assert np.array_equal(pt.cpu().numpy(), perm_token)
    assert np.array_equal(ip.cpu().numpy(), inv_perm)
    assert torch.equal(zp.cpu(), z.cpu()[torch.as_tensor(perm_token)])


def test_permute_reports_bad_expert_index():
    T, E, k = 64, 32, 4
    idx = _routing(T, E, k, False, 1)
    idx[5, 2] = E + 3  # out of range: recorded, no access outside the buffers
    d = _dims(T, E, k, L=256)
    ws = torch.empty(moe.moe_workspace_size(d), dtype=torch.uint8, device="cuda")
    off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    pt = torch.empty(T * k, dtype=torch.int32, device="cuda")
    ip = torch.empty(T * k, dtype=torch.int32, device="cuda")
    assert moe.moe_permute(d, idx.cuda(), None, off, pt, ip, None, ws) == moe.MOE_OK
    st, code = moe.moe_device_error()
    assert st == moe.MOE_ERR_DEVICE and code == 11
    _no_fault()  # the flag was cleared


# ------------------------------------------------------------------------------ combine
@pytest.mark.parametrize("T,L,k,act", [(700, 1024, 8, "bf16"), (64, 128, 4, "f32"), (129, 3584, 16, "bf16"),
                                       (5, 512, 1, "f32")])
def test_combine_rmsnorm(T, L, k, act):
    E = 64
    g = torch.Generator().manual_seed(L + k)
    idx = _routing(T, E, k, False, T + L)
    _, _, _, inv_perm = oracle.permute(idx.numpy(), E)
    y_perm = torch.randn(T * k, L, generator=g, dtype=torch.float32)
    p = torch.rand(T, k, generator=g, dtype=torch.float32) + 0.1
    p = (p / p.sum(dim=1, keepdim=True)).to(torch.float32)
    gamma = (1.0 + 0.1 * torch.randn(L, generator=g)).to(torch.float32)
    d = moe.Dims(T=T, H=256, L=L, E=E, k=k, I=256, S=0, Is=0, act=act, routed=act)
    act_dt = torch.bfloat16 if act == "bf16" else torch.float32
    u = torch.empty(T, L, dtype=torch.float32, device="cuda")
    n = torch.empty(T, L, dtype=act_dt, device="cuda")
    ipd = torch.as_tensor(inv_perm, dtype=torch.int32).cuda()
    assert moe.moe_combine(d, y_perm.cuda(), ipd, p.cuda(), gamma.cuda(), u, n) == moe.MOE_OK
    torch.cuda.synchronize()
    _no_fault()
    y_slots = y_perm.to(F64)[torch.as_tensor(inv_perm)].reshape(T, k, L)
    u_ref = oracle.combine(y_slots, p.to(F64))
    n_ref = oracle.storage_round(act)(oracle.rms_norm(u_ref, gamma.to(F64), 1e-6))
    assert parity(u.cpu(), u_ref) <= 1e-5
    assert storage_steps(n.cpu(), n_ref, act) <= 1.0 + 1e-6 or parity(n.cpu(), n_ref) <= 1e-5


# ------------------------------------------------------------------------------ experts
@pytest.mark.parametrize("kernel", ["two_tile", "one_tile"])
@pytest.mark.parametrize("T,L", [(512, 1024), (37, 1024), (300, 1152)])
def test_expert_ffn_mid_dims(T, L, kernel, monkeypatch):
    # L = 1024 runs the expert GEMMs on CTA pairs; L = 1152 (not a multiple of
    # 256) on single CTAs, where the down projection's 9 weight tiles leave the
    # last two-tile item with one tile.  MOE_EXPERT_KERNEL picks the bf16
    # expert kernel (one weight tile or two per work item).
    monkeypatch.setenv("MOE_EXPERT_KERNEL", "one" if kernel == "one_tile" else "two")
    cfg = gen.CONFIGS["mid"].with_(L=L)
    E, k, L, I = cfg.E, cfg.k, cfg.L, cfg.I
    d = dims_for(cfg, T=T)
    w = gen.device_layer(cfg.with_(T=T), "cuda", with_x=False)
    idx = _routing(T, E, k, True, 5)
    counts, offsets, perm_token, _ = oracle.permute(idx.numpy(), E)
    R = T * k
    g = torch.Generator().manual_seed(9)
    z_perm = torch.randn(R, L, generator=g).to(torch.bfloat16)
    y_perm = torch.full((R, L), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.empty(moe.moe_workspace_size(d), dtype=torch.uint8, device="cuda")
    wts = moe.make_weights(Wg=w["Wg"], Wv=w["Wv"], Wo=w["Wo"])
    off = torch.as_tensor(offsets, dtype=torch.int32).cuda()
    assert moe.moe_expert_ffn(d, wts, z_perm.cuda(), off, y_perm, ws) == moe.MOE_OK
    torch.cuda.synchronize()
    _no_fault()
    y = y_perm.cpu().to(F64)
    zf = z_perm.to(F64)
    ref = torch.empty(R, L, dtype=F64)
    for e in range(E):
        a, b = offsets[e], offsets[e + 1]
        if a == b:
            continue
        Wg, Wv, Wo = oin.expert_weights(cfg, e)
        ref[a:b] = oracle.expert_forward(zf[a:b], Wg, Wv, Wo, cfg.situ_c, oracle.bf16_round)
    assert parity(y, ref) <= 1e-2


def test_expert_ffn_same_gate_and_up_weights():
    """W_v = W_g (one buffer passed twice): h = SiTU-GLU(g, g)."""
    cfg = gen.CONFIGS["mid"]
    T = 256
    E, k, L, I = cfg.E, cfg.k, cfg.L, cfg.I
    d = dims_for(cfg, T=T)
    w = gen.device_layer(cfg.with_(T=T), "cuda", with_x=False)
    idx = _routing(T, E, k, True, 11)
    _, offsets, _, _ = oracle.permute(idx.numpy(), E)
    R = T * k
    z_perm = torch.randn(R, L, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    y_perm = torch.full((R, L), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.empty(moe.moe_workspace_size(d), dtype=torch.uint8, device="cuda")
    wts = moe.make_weights(Wg=w["Wg"], Wv=w["Wg"], Wo=w["Wo"])
    off = torch.as_tensor(offsets, dtype=torch.int32).cuda()
    assert moe.moe_expert_ffn(d, wts, z_perm.cuda(), off, y_perm, ws) == moe.MOE_OK
    torch.cuda.synchronize()
    _no_fault()
    zf = z_perm.to(F64)
    ref = torch.empty(R, L, dtype=F64)
    for e in range(E):
        a, b = offsets[e], offsets[e + 1]
        if a == b:
            continue
        Wg, _, Wo = oin.expert_weights(cfg, e)
        ref[a:b] = oracle.expert_forward(zf[a:b], Wg, Wg, Wo, cfg.situ_c, oracle.bf16_round)
    assert parity(y_perm.cpu().to(F64), ref) <= 1e-2


@pytest.mark.parametrize("T", [300, 40])
def test_expert_ffn_mxfp4(T):
    """Routed experts with MXFP4 weights against the oracle, which decodes the
    same bits (E2M1 codes x E8M0 scales) to fp64."""
    cfg = gen.CONFIGS["mxfp4-small"].with_(T=T)
    E, k, L, I = cfg.E, cfg.k, cfg.L, cfg.I
    d = dims_for(cfg, T=T)
    w = gen.device_layer(cfg, "cuda", with_x=False)
    idx = _routing(T, E, k, True, 21)
    _, offsets, _, _ = oracle.permute(idx.numpy(), E)
    R = T * k
    z_perm = torch.randn(R, L, generator=torch.Generator().manual_seed(5)).to(torch.bfloat16)
    y_perm = torch.full((R, L), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.empty(moe.moe_workspace_size(d), dtype=torch.uint8, device="cuda")
    wts = moe.make_weights(Wg=w["Wg"], Wv=w["Wv"], Wo=w["Wo"], Sg=w["Sg"], Sv=w["Sv"], So=w["So"])
    off = torch.as_tensor(offsets, dtype=torch.int32).cuda()
    assert moe.moe_expert_ffn(d, wts, z_perm.cuda(), off, y_perm, ws) == moe.MOE_OK
    torch.cuda.synchronize()
    _no_fault()
    zf = z_perm.to(F64)
    ref = torch.empty(R, L, dtype=F64)
    for e in range(E):
        a, b = offsets[e], offsets[e + 1]
        if a == b:
            continue
        Wg, Wv, Wo = oin.expert_weights(cfg, e)
        ref[a:b] = oracle.expert_forward(zf[a:b], Wg, Wv, Wo, cfg.situ_c, oracle.bf16_round)
    assert parity(y_perm.cpu().to(F64), ref) <= 1e-2


# ------------------------------------------------------------------------------ bounded waits
def test_bounded_wait_gives_up_and_reports():
    """A pipeline wait that nothing completes (no copy or MMA in flight) gives
    up after its limit, records its site in the device fault flag, and leaves
    the context usable."""
    waited = torch.zeros(1, dtype=torch.int64, device="cuda")
    assert moe.moe_selftest_wait_timeout(50, waited) == moe.MOE_OK
    st, code = moe.moe_device_error()
    assert st == moe.MOE_ERR_DEVICE and code == moe.MOE_FAULT_SELFTEST_WAIT
    ns = int(waited.item())
    assert 50_000_000 <= ns < 2_000_000_000, ns
    _no_fault()  # the flag was cleared
    assert moe.moe_selftest_wait_timeout(0, waited) == moe.MOE_ERR_INVALID_ARG
    # the context still runs kernels
    test_permute_exact(300, 32, 4, False)
