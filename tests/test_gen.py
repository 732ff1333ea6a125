"""The seeded input generator: published Philox vectors, exact bf16 rounding,
moments, MXFP4 quantiser against the OCP grid."""
import numpy as np
import pytest
import torch

import gen
from conftest import read_golden


def test_philox_known_answers():
    rows = read_golden("philox4x32_10_kat.txt")
    assert len(rows) == 3
    for r in rows:
        v = [int(a, 16) for a in r if a != "->"]
        ctr, key, want = v[0:4], v[4:6], v[6:10]
        assert list(gen.philox4x32_10(ctr, key)) == want


def test_bf16_is_rne_of_f32():
    a = gen.fill_host(0, 1, 12345, 200_000, 1.0, 0.0, "f32")
    b = gen.fill_host(0, 1, 12345, 200_000, 1.0, 0.0, "bf16")
    ref = torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ref, b)


def test_ranges_are_consistent():
    a = gen.fill_host(0, 4, 0, 10_000, 0.3, 0.0, "f32")
    b = gen.fill_host(0, 4, 2_500, 5_000, 0.3, 0.0, "f32")
    assert np.array_equal(a[2_500:7_500], b)
    c = gen.fill_host(1, 4, 0, 100, 0.3, 0.0, "f32")
    assert not np.array_equal(a[:100], c)


def test_normal_moments():
    n = 4_000_000
    a = gen.fill_host(0, 2, 0, n, 0.25, 0.0, "f32").astype(np.float64)
    assert abs(a.mean()) < 5 * 0.25 / np.sqrt(n)
    assert abs(a.std() / 0.25 - 1.0) < 2e-3
    # Irwin-Hall(8) excess kurtosis is -6/(5*8) = -0.15, bounded at sqrt(6)*2 sigma
    kurt = ((a / a.std()) ** 4).mean() - 3.0
    assert abs(kurt + 0.15) < 0.02
    assert np.abs(a).max() <= 0.25 * 2 * np.sqrt(6) * 1.0001


def test_gamma_offset():
    cfg = gen.CONFIGS["tiny"].with_(gamma="normal")
    g = gen.gamma(cfg)
    assert abs(g.mean() - 1.0) < 0.05 and 0.05 < g.std() < 0.15


def _e2m1_table():
    return {int(r[0]): float(r[1]) for r in read_golden("e2m1_ocp_mx.txt")}


def test_mxfp4_quantiser_is_nearest_on_the_grid():
    K = 256
    codes, scales = gen.fill_host_mxfp4(0, 7, 3, 16, K, 0.05)
    vals = gen.fill_host(0, 7, 3 * K, 16 * K, 0.05, 0.0, "f32").reshape(16, K).astype(np.float64)
    tab = _e2m1_table()
    grid = np.array(sorted({abs(v) for v in tab.values()}))
    for r in range(16):
        for b in range(K // 32):
            blk = vals[r, b * 32 : (b + 1) * 32]
            e = int(scales[r, b]) - 127
            amax = np.abs(blk).max()
            assert e == int(np.floor(np.log2(amax))) - 2
            for i in range(32):
                byte = codes[r, (b * 32 + i) // 2]
                code = (byte >> (4 * (i % 2))) & 0xF
                q = blk[i] / 2.0 ** e
                deq = tab[code]
                # nearest grid point (saturating at 6)
                dist = np.abs(grid - min(abs(q), 6.0))
                assert abs(abs(deq) - min(abs(q), 6.0)) <= dist.min() + 1e-12
                if deq != 0:
                    assert np.sign(deq) == np.sign(q)


def test_zipf_bias_is_centred_and_skewed():
    cfg = gen.CONFIGS["prefill"]
    b = gen.bias(cfg)
    assert b.shape == (896,) and abs(float(b.mean())) < 1e-6
    assert b.max() - b.min() > 0.5


def test_sample_tokens():
    cfg = gen.CONFIGS["prefill"]
    s = gen.sample_tokens(cfg)
    assert len(s) == 512 and len(np.unique(s)) == 512 and s.min() >= 0 and s.max() < cfg.T
    assert np.array_equal(s, gen.sample_tokens(cfg))


def test_qb_scores_are_24_bit_uniforms():
    """The Quantile Balancing input: fp32 in [0, 1) on the 2^-24 grid,
    reproducible, and from its own Philox stream (not the x or bias words)."""
    cfg = gen.CONFIGS["mid"].with_(T=512)
    s = gen.qb_scores(cfg)
    assert s.shape == (cfg.T, cfg.E) and s.dtype == np.float32
    assert s.min() >= 0.0 and s.max() < 1.0
    grid = s.astype(np.float64) * 2.0 ** 24
    assert np.array_equal(grid, np.round(grid))
    assert np.array_equal(s, gen.qb_scores(cfg))
    words = gen.u32_words(cfg.seed, gen.TID["qb_scores"], 0, 8)
    assert np.array_equal(s.ravel()[:8], (words >> 8).astype(np.float32) * np.float32(2.0 ** -24))
    # mean and variance of U[0, 1) within 4 standard errors
    n = s.size
    assert abs(s.mean() - 0.5) < 4 * (1 / 12) ** 0.5 / n ** 0.5
    assert abs(s.var() - 1 / 12) < 4 * (1 / 180) ** 0.5 / n ** 0.5
