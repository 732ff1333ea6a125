"""The Quantile Balancing bias update through moe_qb_bias_update against the
oracle (GPU): the margin histogram bit-exact, the boundaries and the new bias
to fp32 rounding, at the K3 prefill size and at small and ragged shapes."""
import numpy as np
import pytest
import torch

import gen
import sparse_moe_layer_renormalised_b200 as moe
from oracle import qb_oracle as qb

pytestmark = pytest.mark.gpu


def _run(cfg, nb, lo, hi):
    s = gen.qb_scores(cfg)
    b = gen.bias(cfg)
    dev = torch.device("cuda")
    s_d = torch.from_numpy(s).to(dev)
    b_d = torch.from_numpy(b).to(dev)
    out = torch.empty(cfg.E, dtype=torch.float32, device=dev)
    q = torch.empty(cfg.E, dtype=torch.float32, device=dev)
    hist = torch.empty(cfg.E * nb, dtype=torch.int32, device=dev)
    d = moe.Dims(T=cfg.T, H=cfg.H, L=cfg.L, E=cfg.E, k=cfg.k, I=cfg.I, S=cfg.S, Is=cfg.Is)
    assert moe.moe_qb_bias_update(d, s_d, b_d, out, q, hist, nb, lo, hi) == moe.MOE_OK
    torch.cuda.synchronize()
    assert moe.moe_device_error() == (moe.MOE_OK, 0)
    ref = qb.qb_bias_update(s, b, cfg.k, nb, lo, hi)
    counts = hist.view(cfg.E, nb).cpu().numpy().astype(np.int64)
    return ref, counts, q.cpu().numpy().astype(np.float64), out.cpu().numpy().astype(np.float64), b


@pytest.mark.parametrize("name,E,k,T,nb", [("prefill", 896, 16, 16384, 1024), ("mid", 128, 8, 1000, 1024),
                                             ("ragged", 100, 3, 777, 1024), ("fine-bins", 128, 8, 1000, 8192)])
def test_qb_update_matches_oracle(name, E, k, T, nb):
    """Coarse and fine histograms, full and small shapes."""
    cfg = gen.CONFIGS["prefill" if name == "prefill" else "mid"].with_(E=E, k=k, T=T)
    lo, hi = -1.5, 1.5
    ref, counts, q, bias_out, b = _run(cfg, nb, lo, hi)
    # integer work: the histogram is exact
    assert np.array_equal(counts, ref["counts"])
    assert (counts.sum(axis=1) == cfg.T).all()
    # the boundary and the new bias to fp32 rounding of the interpolation
    w = (hi - lo) / nb
    assert np.max(np.abs(q - ref["q"])) <= 1e-5
    assert np.max(np.abs(bias_out - (b.astype(np.float64) - ref["q"]))) <= 2e-5
    # the histogram boundary lies in the c-th margin's bin: within one bin plus
    # half the gap between the c-th and (c+1)-th margins of the exact quantile
    assert np.all(np.abs(q - ref["q_exact"]) <= w + 0.5 * ref["rank_gap"] + 1e-5)


def test_qb_update_balances_a_skewed_batch():
    """After one update on a Zipf-biased batch, re-selecting with the new
    bias moves every expert's load toward the target count."""
    cfg = gen.CONFIGS["prefill-e64"].with_(T=4096)
    nb, lo, hi = 2048, -2.0, 2.0
    ref, counts, q, bias_out, b = _run(cfg, nb, lo, hi)
    s = gen.qb_scores(cfg)
    c = qb.qb_target(cfg.T, cfg.k, cfg.E)
    load0 = qb.qb_margins(s, b, cfg.k)[2].sum(axis=0)
    load1 = qb.qb_margins(s, bias_out.astype(np.float32), cfg.k)[2].sum(axis=0)
    assert np.abs(load1 - c).max() < 0.25 * np.abs(load0 - c).max()
