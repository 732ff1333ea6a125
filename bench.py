#!/usr/bin/env python
"""Throughput of the Stable LatentMoE layer forward pass on B200.

One step = one moe_layer_forward over one batch of T synthetic tokens (all
stages: router, top-k, latent projection, shared experts, permute, routed
experts, combine + RMSNorm, output projection).  Default workload: the
K3-shape prefill layer (T=16384, H=7168, L=3584, 896 experts top-16,
I=3072, 2 shared experts, Zipf(0.8) expert load), bf16 with fp32 accumulation.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config prefill|decode|mid|tiny]
  python bench.py --impl reference ...     # the CPU oracle on a bounded sample

With N > 1 (torchrun, one process per GPU) every rank runs an independent
replica of the layer on its own batch (the forward pass has no exchange step);
time is the max over ranks and value counts all ranks' tokens.
Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import gen  # noqa: E402
import sparse_moe_layer_renormalised_b200 as moe  # noqa: E402

METRIC = "MoE-layer tokens/s at K3 shape (bf16, MXFP4); % of tensor/HBM roofline"
STAGE = {n: i for i, n in enumerate(moe.STAGE_NAMES)}


def load_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def dims_for(cfg, y_out: str) -> moe.Dims:
    return moe.Dims(T=cfg.T, H=cfg.H, L=cfg.L, E=cfg.E, k=cfg.k, I=cfg.I, S=cfg.S, Is=cfg.Is, act=cfg.act,
                    routed=cfg.routed, y_out=y_out if cfg.act == "bf16" else "f32", situ_c=cfg.situ_c,
                    rms_eps=cfg.rms_eps)


def workload_name(cfg) -> str:
    load = "Zipf(0.8) expert load" if cfg.bias == "zipf" else "bias N(0,0.05)"
    w = "MXFP4 routed weights" if cfg.routed == "mxfp4" else f"{cfg.act} weights"
    return (f"{cfg.name}: Stable LatentMoE layer T={cfg.T}, H={cfg.H}, L={cfg.L}, E={cfg.E} top-{cfg.k}, "
            f"I={cfg.I}, {cfg.S} shared (Is={cfg.Is}), {w}, {load}")


# ----------------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int):
        self.proc = None
        try:
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            sel = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "100", "-i", sel], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------------- ranks
def max_over_ranks(ms: float, device) -> float:
    """Slowest rank's elapsed time: every rank contributes its device-timed
    milliseconds; all ranks get the maximum (the job's time)."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return ms
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank_step: int, steps: int, world: int, max_ms: float) -> float:
    """Whole-job tokens/s: all ranks' tokens over the slowest rank's time."""
    return tokens_per_rank_step * steps * world / (max_ms / 1e3)


# ----------------------------------------------------------------------------------- roofline
def dominant_stage(cfg) -> str:
    return "expert_gate_up"


def stage_work(cfg, offsets: np.ndarray, T: int) -> dict:
    """Algorithmic work of the routed-expert gate/up launch: flops of the
    selected (token, expert) pairs only; bytes = weights of the touched
    experts + the permuted latent rows read + h written."""
    R = T * cfg.k
    counts = np.diff(offsets)
    touched = int((counts > 0).sum())
    wbytes = 2 * cfg.I * cfg.L * (0.53125 if cfg.routed == "mxfp4" else 2.0)  # MXFP4: 4 bits + E8M0/32
    flops = 2.0 * R * cfg.L * 2 * cfg.I
    bytes_ = touched * wbytes + R * cfg.L * 2 + R * cfg.I * 2
    return {"flops": flops, "bytes": bytes_, "touched_experts": touched}


def measure_qb(cfg, dev, stream, peaks: dict, reps: int = 10) -> dict:
    """The Quantile Balancing bias update (the training-time step beside the
    router) on a [T, E] score batch of this workload's shape, timed on its
    own with CUDA events; L2 is flushed (a 256 MB write) before every call,
    since the scores alone would fit in it.  Not part of the layer step."""
    nb, lo, hi = 1024, -1.5, 1.5
    s = torch.from_numpy(gen.qb_scores(cfg)).to(dev)
    b = torch.from_numpy(gen.bias(cfg)).to(dev)
    out = torch.empty(cfg.E, dtype=torch.float32, device=dev)
    hist = torch.empty(cfg.E * nb, dtype=torch.int32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    d = dims_for(cfg, "f32")

    def call():
        moe.check(moe.moe_qb_bias_update(d, s, b, out, None, hist, nb, lo, hi, stream))

    for _ in range(3):
        call()
    total = 0.0
    for i in range(reps):
        flush.fill_(i & 0xFF)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        call()
        e1.record(stream)
        torch.cuda.synchronize()
        total += e0.elapsed_time(e1)
    ms = total / reps
    # scores read, histogram zeroed and read back, bias in / out
    nbytes = cfg.T * cfg.E * 4 + 2 * cfg.E * nb * 4 + 2 * cfg.E * 4
    achieved = nbytes / (ms / 1e3) / 1e9
    return {"kernel": "qb_zero_kernel + qb_hist_kernel + qb_quantile_kernel", "ms": round(ms, 4), "bound": "hbm",
            "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": round(achieved / peaks["hbm_gbs"], 4), "algorithmic_bytes": nbytes, "bins": nb,
            "scores": f"[{cfg.T}, {cfg.E}] fp32, uniform in [0, 1); target floor(T k / E) = {cfg.T * cfg.k // cfg.E}"}


# ----------------------------------------------------------------------------------- our arm
def run_ours(args, rank, world, local_rank):
    cfg = gen.CONFIGS[args.config]
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    inputs = gen.device_layer(cfg, dev)
    x = inputs.pop("x")
    layer = moe.MoeLayer(dims_for(cfg, args.y_out), inputs)
    y = layer.output(cfg.T)
    stream = torch.cuda.current_stream(dev)
    offsets = torch.empty(cfg.E + 1, dtype=torch.int32, device=dev)

    def events():
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(2 * moe.MOE_NUM_STAGES)]
        for e in evs:
            e.record(stream)  # creates the event handle
        return evs

    # warm-up (not timed)
    for _ in range(args.warmup):
        layer.forward(x, y)
    torch.cuda.synchronize()
    launches_per_step = moe.moe_last_launch_count()

    step_events = [events() for _ in range(args.steps)]
    auxes = [moe.make_aux(stage_events=ev, expert_offsets=offsets) for ev in step_events]
    torch.cuda.synchronize()
    sampler = ClockSampler(local_rank) if rank == 0 else None
    time.sleep(0.3 if sampler else 0.0)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(args.steps):
        moe.check(moe.moe_layer_forward(layer.dims, layer._w, x, y, auxes[i], layer.workspace, None, stream))
    t1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop() if sampler else None
    ms = max_over_ranks(t0.elapsed_time(t1), dev)
    ms_per_step = ms / args.steps

    # per-stage device time inside the timed region
    stage_ms = {n: 0.0 for n in moe.STAGE_NAMES}
    for ev in step_events:
        for i, n in enumerate(moe.STAGE_NAMES):
            stage_ms[n] += ev[2 * i].elapsed_time(ev[2 * i + 1]) / args.steps

    # end to end through the public API: pinned host x -> device, forward, y -> pinned host
    x_host = torch.empty(x.shape, dtype=x.dtype, pin_memory=True)
    x_host.copy_(x)
    y_host = torch.empty(y.shape, dtype=y.dtype, pin_memory=True)
    x_in = torch.empty_like(x)
    for _ in range(max(1, min(args.warmup, 2))):
        x_in.copy_(x_host, non_blocking=True)
        layer.forward(x_in, y)
        y_host.copy_(y, non_blocking=True)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        x_in.copy_(x_host, non_blocking=True)
        layer.forward(x_in, y)
        y_host.copy_(y, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dev)
    if world > 1:
        torch.distributed.barrier()

    st, code = moe.moe_device_error()
    if st != moe.MOE_OK:
        raise RuntimeError(f"device fault {code} during the bench")
    if rank != 0:
        return None

    peaks = load_peaks()
    value = job_throughput(cfg.T, args.steps, world, ms)
    off = offsets.cpu().numpy()
    work = stage_work(cfg, off, cfg.T)
    dom = dominant_stage(cfg)
    dom_ms = stage_ms[dom]
    flops_step = float(cfg.flops_per_token()) * cfg.T
    R = cfg.T * cfg.k
    counts = np.diff(off)
    bound = "tensor" if (work["flops"] / (peaks["bf16_tflops_sustained"] * 1e12)) >= (
        work["bytes"] / (peaks["hbm_gbs"] * 1e9)) else "hbm"
    if bound == "tensor":
        achieved = work["flops"] / (dom_ms / 1e3) / 1e12
        peak = peaks["bf16_tflops_sustained"]
        unit = "TFLOP/s"
    else:
        achieved = work["bytes"] / (dom_ms / 1e3) / 1e9
        peak = peaks["hbm_gbs"]
        unit = "GB/s"
    traffic = None
    prof = os.path.join(ROOT, "profiles", f"traffic_{cfg.name}_{dom}.json")
    if os.path.exists(prof):
        # dram__bytes_read.sum + dram__bytes_write.sum of one launch, from an ncu
        # capture of this workload (see the file for the command and kernel build)
        with open(prof) as f:
            traffic = json.load(f).get("dram_bytes_per_launch")
    out = {
        "metric": METRIC,
        "value": round(value, 1),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": cfg.act,
        "data": "synthetic (seeded Philox inputs, random-init weights of the K3 layer shape)",
        "config": {
            "workload": workload_name(cfg),
            "tokens_per_step_per_gpu": cfg.T,
            "y_dtype": args.y_out,
            "parallelism": f"replicas x{world} (no data-path collective)",
            "l2": "inputs larger than L2 (routed weights %.1f GB, x %.0f MB per step)" % (
                3 * cfg.E * cfg.I * cfg.L * 2 / 1e9, cfg.T * cfg.H * 2 / 1e6),
            "expert_rows_max": int(counts.max()),
            "expert_rows_min": int(counts.min()),
            "touched_experts": work["touched_experts"],
        },
        "tflops": round(flops_step / (ms_per_step / 1e3) / 1e12, 2),
        "stage_ms": {k: round(v, 4) for k, v in stage_ms.items()},
        "roofline": {
            "kernel": f"tc_expert_kernel (2-CTA grouped gate/up + SiTU epilogue) = stage {dom}",
            "bound": bound,
            "achieved": round(achieved, 1),
            "peak": peak,
            "unit": unit,
            "frac": round(achieved / peak, 4),
            "traffic": traffic,
            "peak_source": peaks["source"] + (" sustained bf16" if bound == "tensor" else " HBM copy"),
            "algorithmic": {"flops": work["flops"], "bytes": work["bytes"]},
        },
        "e2e": {
            "value": round(job_throughput(cfg.T, args.steps, world, e2e_ms), 1),
            "unit": "tokens/s",
            "h2d_bytes_per_step": x.numel() * x.element_size(),
            "d2h_bytes_per_step": y.numel() * y.element_size(),
        },
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }
    out["qb_update"] = measure_qb(cfg, dev, stream, peaks)
    if world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(cfg, args.cpu_tokens, seed_offset=0)
    return out


# ----------------------------------------------------------------------------------- the oracle
def cpu_baseline(cfg, n_tokens: int, seed_offset: int = 0, dense=None) -> dict:
    """The fp64 CPU oracle on a bounded sample of the workload's tokens.  The
    time counts the oracle's own work (reading bf16 / MXFP4 weights into fp64
    and the layer arithmetic); generating the synthetic weights is excluded."""
    import oracle
    from oracle import inputs as oin

    rng = np.random.default_rng(cfg.seed + 1000 + seed_offset)
    sample = np.sort(rng.choice(cfg.T, size=min(n_tokens, cfg.T), replace=False))
    dense = oin.dense_weights(cfg) if dense is None else dense
    x = oin.x_rows(cfg, sample)
    gen_s = [0.0]

    def provider(e):
        t = time.perf_counter()
        raw = [gen.host_expert(cfg, n, e) for n in ("Wg", "Wv", "Wo")]
        gen_s[0] += time.perf_counter() - t
        out = []
        for r in raw:
            out.append(oracle.mxfp4_dequant(*r) if isinstance(r, tuple) else oin.to_f64(r))
        return tuple(out)

    t0 = time.perf_counter()
    oracle.layer_forward_streamed(cfg, dense, x, provider)
    total = time.perf_counter() - t0 - gen_s[0]
    return {"value": round(len(sample) / total, 3), "unit": "tokens/s", "cores": torch.get_num_threads(),
            "kind": "oracle",
            "sample": f"{len(sample)} seeded tokens of the {cfg.name} workload (fp64, torch CPU, "
                      f"{torch.get_num_threads()} threads; weight generation excluded)"}


def run_reference(args, rank, world):
    from oracle import inputs as oin

    cfg = gen.CONFIGS[args.config]
    per_step = max(1, args.cpu_tokens // 4)
    dense = oin.dense_weights(cfg)
    times = []
    for i in range(args.warmup + args.steps):
        cb = cpu_baseline(cfg, per_step, seed_offset=i, dense=dense)
        if i >= args.warmup:
            times.append(per_step / cb["value"])
    total = sum(times)
    value = per_step * args.steps / total
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": round(value, 3),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(1e3 * total / args.steps, 2),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (seeded Philox inputs)",
        "config": {"workload": workload_name(cfg), "tokens_per_step": per_step},
        "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": torch.get_num_threads(),
                         "kind": "oracle",
                         "sample": f"{per_step} seeded tokens per step of the {cfg.name} workload"},
        "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", choices=sorted(gen.CONFIGS), default="prefill")
    ap.add_argument("--y-out", choices=["bf16", "f32"], default="bf16")
    ap.add_argument("--cpu-tokens", type=int, default=8)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        # The CPU oracle runs on rank 0 only; other ranks have nothing to do.
        if rank == 0:
            print(json.dumps(run_reference(args, rank, world)), flush=True)
        return
    if world > 1:
        import datetime

        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        out = run_ours(args, rank, world, local_rank)
        if rank == 0 and out is not None:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
