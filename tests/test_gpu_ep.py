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


def test_expert_parallel_layer_world_one_matches_the_oracle():
    """The expert-parallel step (router, latent + shared, permute, exchange
    plan, all_to_all dispatch, block expert FFN, all_to_all combine,
    combine + RMSNorm, output) on one NCCL rank holding every expert equals
    the oracle layer; the exchanges then move the rows to the same rank."""
    cfg = gen.CONFIGS["mid"].with_(T=700)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=120))
    try:
        w = gen.device_layer(cfg, "cuda")
        x = w.pop("x")
        layer = ep.ExpertParallelMoeLayer(dims_for(cfg), w)
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
