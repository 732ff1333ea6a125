"""Host logic of bench.py that the reported numbers depend on (no GPU): the
algorithmic work behind the roofline, and the reference arm's JSON line."""
import json
import os
import subprocess
import sys

import numpy as np

import bench
import gen

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _offsets(counts):
    return np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)


def test_gate_up_flops_per_token_at_k3():
    """2 * k * L * 2I flops per token for the routed gate/up GEMMs: 704.6 MFLOP
    at the K3 shape (k = 16, L = 3584, I = 3072), whatever the routing."""
    cfg = gen.CONFIGS["prefill"]
    counts = np.full(cfg.E, cfg.T * cfg.k // cfg.E)
    counts[: cfg.T * cfg.k - counts.sum()] += 1
    w = bench.stage_work(cfg, _offsets(counts), cfg.T)
    assert w["flops"] / cfg.T == 704_643_072
    assert w["touched_experts"] == cfg.E


def test_gate_up_bytes_count_touched_experts_only():
    """Weight bytes only for experts with at least one row; activations are
    the permuted latent rows read (bf16) and h written (bf16)."""
    cfg = gen.CONFIGS["decode"]
    R = cfg.T * cfg.k
    counts = np.zeros(cfg.E, np.int64)
    counts[:10] = R // 10
    counts[0] += R - counts.sum()
    w = bench.stage_work(cfg, _offsets(counts), cfg.T)
    per_expert = 2 * cfg.I * cfg.L * 2  # W_g and W_v rows, bf16
    assert w["touched_experts"] == 10
    assert w["bytes"] == 10 * per_expert + R * cfg.L * 2 + R * cfg.I * 2


def test_mxfp4_weight_bytes_are_4_25_bits_per_element():
    """OCP MXFP4: a 4-bit code per element plus one 8-bit scale per 32."""
    cfg = gen.CONFIGS["mxfp4"]
    counts = np.zeros(cfg.E, np.int64)
    counts[0] = 16
    w = bench.stage_work(cfg, _offsets(counts), 1)
    act = 16 * cfg.L * 2 + 16 * cfg.I * 2
    assert w["bytes"] - act == 2 * cfg.I * cfg.L * (4 + 8 / 32) / 8


def test_reference_arm_prints_one_contract_line():
    """`bench.py --impl reference` runs the oracle on the host and prints one
    JSON line with the contract's keys (tiny layer, one timed step)."""
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--config", "tiny", "--steps", "1",
                        "--warmup", "3", "--cpu-tokens", "8"], cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["steps"] == 1
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0


def test_ep_balance_statistic():
    """The balanced plan's per-rank load on a skewed routing: the static
    partition's largest rank is well above the mean, the balanced plan's at
    most one row above it, and the copies are counted."""
    rng = np.random.default_rng(3)
    E, k, T = 64, 4, 2000
    w = (np.arange(E) + 1.0) ** -1.0
    idx = np.stack([rng.choice(E, size=k, replace=False, p=w / w.sum()) for _ in range(T)])
    st = bench.ep_balance(idx, E, G=8)
    assert st["rows"] == T * k and st["ranks"] == 8
    assert st["static_max_over_mean"] > 1.5                       # the hot experts sit on rank 0
    assert st["balanced_max_over_mean"] <= 1.0 + 8 / (T * k) + 1e-9
    assert st["copies"] >= 1 and st["max_copies_per_rank"] >= 1


def test_routing_of_batch_logic_on_cpu():
    """routing_of_batch's host logic with a stand-in layer that fills the
    same aux outputs as MoeLayer.forward (scores, topk_idx): the near-tie
    count and the choice it returns."""
    import torch

    class FakeLayer:
        def __init__(self, scores, bias, idx):
            self.s, self.idx = scores, idx
            self.weights = {"bias": bias}

        def forward(self, x, aux):
            aux["scores"].copy_(self.s)
            aux["topk_idx"].copy_(self.idx)

    cfg = gen.CONFIGS["tiny"]
    g = torch.Generator().manual_seed(4)
    s = torch.rand(cfg.T, cfg.E, generator=g)
    s[0, :cfg.k + 1] = 0.9                      # token 0: the k-th and (k+1)-th keys tie
    bias = torch.zeros(cfg.E)
    idx = torch.topk(s, cfg.k, dim=1).indices.to(torch.int32)
    n_tie, got = bench.routing_of_batch(FakeLayer(s, bias, idx), torch.zeros(1), cfg)
    assert n_tie >= 1 and got.dtype == np.int64 and np.array_equal(got, idx.numpy())
    st = bench.ep_balance(got, cfg.E)
    assert st["rows"] == cfg.T * cfg.k
