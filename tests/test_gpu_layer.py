"""The whole layer through moe_layer_forward against the oracle (GPU)."""

import numpy as np
import pytest
import torch

import gen
import sparse_moe_layer_renormalised_b200 as moe
from harness import (K3_SAMPLE, TOL_BF16, TOL_F32, TOL_MXFP4, compare_layer, make_device_layer, moe_inputs_rows, oracle_forward,
                     run_layer)

pytestmark = pytest.mark.gpu


def _report(name, m):
    print(f"\n[{name}] " + " ".join(f"{k}={v:.3g}" if isinstance(v, float) else f"{k}={v}" for k, v in m.items()))


def test_tiny_fp32_all_tokens():
    cfg = gen.CONFIGS["tiny"]
    layer, w = make_device_layer(cfg)
    y, aux = run_layer(layer, w["x"])
    m = compare_layer(cfg, np.arange(cfg.T), y, aux, TOL_F32)
    _report("tiny", m)


def test_tiny_with_gain_and_top1():
    for cfg in (gen.CONFIGS["tiny"].with_(gamma="normal"), gen.CONFIGS["tiny"].with_(k=1)):
        layer, w = make_device_layer(cfg)
        y, aux = run_layer(layer, w["x"])
        compare_layer(cfg, np.arange(cfg.T), y, aux, TOL_F32)


@pytest.fixture(scope="module")
def mid_layer():
    cfg = gen.CONFIGS["mid"]
    layer, w = make_device_layer(cfg)
    yield cfg, layer, w
    del layer, w
    torch.cuda.empty_cache()


def test_mid_all_tokens(mid_layer):
    cfg, layer, w = mid_layer
    y, aux = run_layer(layer, w["x"])
    m = compare_layer(cfg, np.arange(cfg.T), y, aux, TOL_BF16)
    _report("mid", m)
    # the counts of the expert-major order are the histogram of the choices
    off = aux["expert_offsets"].cpu().numpy()
    counts = np.bincount(aux["topk_idx"].cpu().numpy().ravel(), minlength=cfg.E)
    assert np.array_equal(np.diff(off), counts) and off[-1] == cfg.T * cfg.k


def test_mid_deterministic_and_bf16_output(mid_layer):
    cfg, layer, w = mid_layer
    y1 = layer.forward(w["x"]).clone()
    y2 = layer.forward(w["x"]).clone()
    assert torch.equal(y1, y2)
    lb = moe.MoeLayer(moe.Dims(**{**layer.dims.__dict__, "y_out": "bf16"}), layer.weights)
    yb = lb.forward(w["x"])
    assert torch.equal(yb, y1.to(torch.bfloat16))


@pytest.mark.parametrize("T", [1, 127, 1000])
def test_mid_ragged_token_counts(mid_layer, T):
    cfg, layer, w = mid_layer
    tokens = np.arange(T) * 3 % cfg.T
    x = moe_inputs_rows(cfg, tokens)
    y, aux = run_layer(layer, x)
    ref = oracle_forward(cfg, tokens)
    # rows of a sub-batch are independent of the rest of the batch
    m = compare_layer(cfg, np.arange(T), y, aux, TOL_BF16, ref=ref)
    _report(f"mid T={T}", m)


def test_mxfp4_layer_all_tokens():
    """The whole layer with MXFP4 routed weights (bar 3e-2; the oracle decodes
    the same bits, so the error budget is that of the bf16 layer)."""
    cfg = gen.CONFIGS["mxfp4-small"]
    layer, w = make_device_layer(cfg)
    y, aux = run_layer(layer, w["x"])
    m = compare_layer(cfg, np.arange(cfg.T), y, aux, TOL_MXFP4)
    _report("mxfp4-small", m)


def test_zero_tokens_is_a_no_op(mid_layer):
    cfg, layer, w = mid_layer
    y = torch.full((1, cfg.H), 7.0, device="cuda")
    d = moe.Dims(**{**layer.dims.__dict__, "T": 0})
    assert moe.moe_layer_forward(d, layer._w, w["x"], y, None, layer.workspace) == moe.MOE_OK
    torch.cuda.synchronize()
    assert bool((y == 7.0).all())




@pytest.mark.slow
def test_k3_decode_and_prefill_sampled():
    """K3 shape at the full sizes of the decode (T=256, all tokens) and prefill
    (T=16384, Zipf load, seeded token sample) workloads; one set of weights."""
    dec = gen.CONFIGS["decode"]
    pre = gen.CONFIGS["prefill"]
    layer, w = make_device_layer(pre)
    # prefill
    y, aux = run_layer(layer, w["x"])
    counts = np.diff(aux["expert_offsets"].cpu().numpy())
    tokens = gen.sample_tokens(pre, min(K3_SAMPLE, pre.T))
    m = compare_layer(pre, tokens, y, aux, TOL_BF16)
    m["max_expert_rows"] = int(counts.max())
    m["min_expert_rows"] = int(counts.min())
    _report("prefill", m)
    del y, aux
    # decode: first 256 token rows, its own (normal) bias
    layer.weights["bias"].copy_(torch.from_numpy(gen.bias(dec)))
    x = w["x"][: dec.T].contiguous()
    y, aux = run_layer(layer, x)
    tokens = np.arange(min(dec.T, K3_SAMPLE))
    m = compare_layer(dec, tokens, y, aux, TOL_BF16)
    _report("decode", m)


@pytest.mark.slow
def test_k3_mxfp4_sampled():
    """K3 shape with MXFP4 routed weights at the full T = 8192, seeded sample of
    tokens checked against the oracle decoding the same bits."""
    cfg = gen.CONFIGS["mxfp4"]
    layer, w = make_device_layer(cfg)
    y, aux = run_layer(layer, w["x"])
    tokens = gen.sample_tokens(cfg, min(K3_SAMPLE, cfg.T))
    m = compare_layer(cfg, tokens, y, aux, TOL_MXFP4)
    _report("mxfp4", m)
