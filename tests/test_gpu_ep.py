"""Expert-parallel pieces on one GPU: moe_expert_ffn_blocks (the routed experts
over rows received from several ranks, one expert-major block per source)
against the oracle, and the whole expert-parallel layer step (world size 1
over NCCL) against the oracle layer."""
import datetime
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import gen
import oracle
import sparse_moe_layer_renormalised_b200 as moe
from harness import TOL_BF16, TOL_MXFP4_A4, TOL_RMS_A4, dims_for, oracle_forward, parity, rms_parity
from oracle import inputs as oin
from sparse_moe_layer_renormalised_b200 import expert_parallel as ep
from sparse_moe_layer_renormalised_b200.layer import tile_weight_scales

pytestmark = pytest.mark.gpu
F64 = torch.float64


def _no_fault():
    st, code = moe.moe_device_error()
    assert st == moe.MOE_OK and code == 0, f"device fault {code}"


@pytest.mark.parametrize("name,lo,hi", [("mid", 40, 104), ("mxfp4-small", 0, 64), ("mxfp4a8-small", 8, 40),
                                         ("mxfp4a4-small", 8, 40)])
def test_expert_ffn_blocks_three_sources(name, lo, hi):
    """Rows of experts lo..hi-1 from three 'sources' (each expert-major), as
    an expert-parallel rank receives them; every row against the oracle."""
    cfg = gen.CONFIGS[name]
    w = gen.device_layer(cfg.with_(T=64), "cuda", with_x=False)
    E_loc = hi - lo
    rng = np.random.default_rng(3)
    blocks, rows = [], 0
    for src, n_src in enumerate((300, 0, 517)):  # source 1 sends nothing
        e = np.sort(rng.integers(lo, hi, size=n_src))
        counts = np.bincount(e - lo, minlength=E_loc)
        blocks.append(np.concatenate([[0], np.cumsum(counts)]) + rows)
        rows += n_src
    offs = np.stack(blocks).astype(np.int32)
    expert_of_row = np.concatenate([np.repeat(np.arange(lo, hi), np.diff(b)) for b in blocks])
    x = torch.randn(rows, cfg.L, generator=torch.Generator().manual_seed(4)).to(torch.bfloat16)
    mx = cfg.routed in ("mxfp4",) + moe.BLOCK_SCALED
    names = ("Wg", "Wv", "Wo") + (("Sg", "Sv", "So") if mx else ())
    wl = {n: w[n][lo:hi].contiguous() for n in names}
    d = moe.Dims(T=rows, H=cfg.H, L=cfg.L, E=E_loc, k=1, I=cfg.I, S=cfg.S, Is=cfg.Is, act=cfg.act,
                 routed=cfg.routed)
    if cfg.routed in moe.BLOCK_SCALED:
        wl.update(tile_weight_scales(d, wl.pop("Sg"), wl.pop("Sv"), wl.pop("So")))
    ws = torch.empty(moe.moe_expert_ffn_blocks_workspace_size(d, rows, 3), dtype=torch.uint8, device="cuda")
    y = torch.full((rows, cfg.L), float("nan"), dtype=torch.float32, device="cuda")
    assert moe.moe_expert_ffn_blocks(d, moe.make_weights(**wl), x.cuda(), rows, torch.from_numpy(offs).cuda(), 3, y,
                                     ws) == moe.MOE_OK
    torch.cuda.synchronize()
    _no_fault()
    ref = torch.empty(rows, cfg.L, dtype=F64)
    xf = x.to(F64)
    for e in np.unique(expert_of_row):
        r = torch.as_tensor(np.nonzero(expert_of_row == e)[0])
        ref[r] = oracle.expert_forward(xf[r], *oin.expert_weights_raw(cfg, int(e)), cfg.situ_c, oracle.bf16_round,
                                       act=oracle.routed_act(cfg))
    if cfg.routed == "mxfp4_a4":  # h's E2M1 codes can flip (bars derived in harness.py)
        assert parity(y.cpu().to(F64), ref) <= TOL_MXFP4_A4
        assert rms_parity(y.cpu().to(F64), ref) <= TOL_RMS_A4
    else:
        assert parity(y.cpu().to(F64), ref) <= 1e-2


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("balance", [True, False])
def test_expert_parallel_layer_world_one_matches_the_oracle(balance):
    """The expert-parallel step (router, latent + shared, permute, exchange
    plan, all_to_all dispatch, block expert FFN, all_to_all combine,
    combine + RMSNorm, output) on one NCCL rank holding every expert equals
    the oracle layer; the exchanges then move the rows to the same rank (the
    balanced mode's row reordering through moe_gather_rows included)."""
    cfg = gen.CONFIGS["mid"].with_(T=700)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=120))
    try:
        w = gen.device_layer(cfg, "cuda")
        x = w.pop("x")
        layer = ep.ExpertParallelMoeLayer(dims_for(cfg), w, balance=balance)
        y = layer(x)
        torch.cuda.synchronize()
        _no_fault()
        tokens = np.arange(cfg.T)
        ref = oracle_forward(cfg, tokens)
        # the standard layer on the same inputs runs the same kernels on the
        # same tiles: bit-identical output
        std = moe.MoeLayer(dims_for(cfg), w)
        y_std = std.forward(x)
        torch.cuda.synchronize()
        assert torch.equal(y, y_std)
        # against the oracle on the tokens without a near tie in their selection
        keep = torch.as_tensor(ref["margin"] >= 1e-4)
        assert parity(y.cpu()[keep], ref["y"][keep]) <= TOL_BF16
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("n,row_bytes", [(1, 16), (1000, 2048), (777, 7168 * 2)])
def test_gather_rows_bit_exact(n, row_bytes):
    g = torch.Generator().manual_seed(n)
    src_rows = n + 5
    src = torch.randint(0, 256, (src_rows, row_bytes), generator=g, dtype=torch.uint8).cuda()
    idx = torch.randint(0, src_rows, (n,), generator=g, dtype=torch.int32)
    dst = torch.empty(n, row_bytes, dtype=torch.uint8, device="cuda")
    assert moe.moe_gather_rows(src, src_rows, row_bytes, idx.cuda(), n, dst) == moe.MOE_OK
    torch.cuda.synchronize()
    _no_fault()
    assert torch.equal(dst.cpu(), src.cpu()[idx.long()])


def test_gather_rows_reports_a_bad_index():
    """An index outside the source rows is recorded as a device fault (code
    15) and its row is zero-filled; the other rows are copied."""
    src = torch.arange(64 * 4, dtype=torch.float32, device="cuda").reshape(64, 4)
    idx = torch.tensor([3, 64, 5], dtype=torch.int32, device="cuda")
    dst = torch.full((3, 4), -1.0, device="cuda")
    assert moe.moe_gather_rows(src, 64, 16, idx, 3, dst) == moe.MOE_OK
    torch.cuda.synchronize()
    st, code = moe.moe_device_error()
    assert st == moe.MOE_ERR_DEVICE and code == 15
    _no_fault()  # the flag was cleared
    assert torch.equal(dst.cpu(), torch.stack([src[3].cpu(), torch.zeros(4), src[5].cpu()]))
    assert moe.moe_gather_rows(src, 64, 12, idx, 3, dst) == moe.MOE_ERR_INVALID_ARG  # row not 16-byte multiple


@pytest.mark.parametrize("name", ["mid", "mxfp4a4-small"])
def test_expert_ffn_blocks_with_redundant_copies(name):
    """A rank's local expert set as the balanced mode builds it: its own
    experts followed by redundant copies of other ranks' experts (weight
    slices appended behind its own); rows from two sources against the oracle
    under the global expert ids."""
    cfg = gen.CONFIGS[name]
    w = gen.device_layer(cfg.with_(T=64), "cuda", with_x=False)
    own = list(range(8, 20))
    reps = [2, 31, 40]
    local = own + reps
    mx = cfg.routed in ("mxfp4",) + moe.BLOCK_SCALED
    names = ("Wg", "Wv", "Wo") + (("Sg", "Sv", "So") if mx else ())
    sel = torch.tensor(local, device="cuda")
    wl = {n: w[n].index_select(0, sel).contiguous() for n in names}
    d = moe.Dims(T=1, H=cfg.H, L=cfg.L, E=len(local), k=1, I=cfg.I, S=cfg.S, Is=cfg.Is, act=cfg.act,
                 routed=cfg.routed)
    if cfg.routed in moe.BLOCK_SCALED:
        wl.update(tile_weight_scales(d, wl.pop("Sg"), wl.pop("Sv"), wl.pop("So")))
    rng = np.random.default_rng(5)
    blocks, rows, li_of_row = [], 0, []
    for n_src in (211, 96):
        li = np.sort(rng.integers(0, len(local), size=n_src))
        c = np.bincount(li, minlength=len(local))
        blocks.append(np.concatenate([[0], np.cumsum(c)]) + rows)
        li_of_row.append(li)
        rows += n_src
    li_of_row = np.concatenate(li_of_row)
    x = torch.randn(rows, cfg.L, generator=torch.Generator().manual_seed(8)).to(torch.bfloat16 if cfg.act == "bf16"
                                                                                else torch.float32)
    ws = torch.empty(moe.moe_expert_ffn_blocks_workspace_size(d, rows, 2), dtype=torch.uint8, device="cuda")
    y = torch.full((rows, cfg.L), float("nan"), dtype=torch.float32, device="cuda")
    offs = torch.from_numpy(np.stack(blocks).astype(np.int32)).cuda()
    assert moe.moe_expert_ffn_blocks(d, moe.make_weights(**wl), x.cuda(), rows, offs, 2, y, ws) == moe.MOE_OK
    torch.cuda.synchronize()
    _no_fault()
    ref = torch.empty(rows, cfg.L, dtype=F64)
    xf = x.to(F64)
    for li in np.unique(li_of_row):
        r = torch.as_tensor(np.nonzero(li_of_row == li)[0])
        ref[r] = oracle.expert_forward(xf[r], *oin.expert_weights_raw(cfg, local[li]), cfg.situ_c,
                                       oracle.storage_round(cfg.act), act=oracle.routed_act(cfg))
    yd = y.cpu().to(F64)
    if cfg.routed == "mxfp4_a4":
        assert parity(yd, ref) <= TOL_MXFP4_A4 and rms_parity(yd, ref) <= TOL_RMS_A4
    else:
        assert parity(yd, ref) <= 1e-2
