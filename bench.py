#!/usr/bin/env python
"""Throughput of the Stable LatentMoE layer forward pass on B200.

One step = one moe_layer_forward over one batch of T synthetic tokens (all
stages: router, top-k, latent projection, shared experts, permute, routed
experts, combine + RMSNorm, output projection).

The default run measures five K3-shape workloads, one after the other:
  prefill   T=16384, bf16, Zipf(0.8) expert load  -> the headline line
  decode    T=256, bf16, bias N(0, 0.05)           -> "decode" sub-object
  mxfp4     T=8192, MXFP4 routed weights           -> "mxfp4" sub-object
  mxfp4-a8  T=8192, the same MXFP4 weights, expert inputs quantised to MXFP8,
            block-scaled tensor-core MMA           -> "mxfp4-a8" sub-object
  mxfp4-a4  T=8192, the same MXFP4 weights, expert inputs quantised to MXFP4,
            all-4-bit block-scaled MMA             -> "mxfp4-a4" sub-object
(H=7168, L=3584, 896 experts top-16, I=3072, 2 shared experts, Is=3072).
Each line carries its own device time, stage times, roofline, end-to-end
number, near-tie count, an oracle sample (parity and CPU baseline) and the
balanced expert-parallel plan of its batch on 8 ranks (ep_balance, host
planning only).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--no-extra-lines]
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
NEAR_TIE = 1e-4  # key margin (k-th minus (k+1)-th largest key) counted as a near tie


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
    w = {"mxfp4": "MXFP4 routed weights",
         "mxfp4_a8": "MXFP4 routed weights x MXFP8 expert inputs (block-scaled MMA)",
         "mxfp4_a4": "MXFP4 routed weights x MXFP4 expert inputs (all-4-bit block-scaled MMA)"}.get(
        cfg.routed, f"{cfg.act} weights")
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


def barrier(world: int) -> None:
    if world > 1:
        torch.distributed.barrier()


# ----------------------------------------------------------------------------------- roofline
def routed_weight_bytes_per_element(cfg) -> float:
    if cfg.routed in ("mxfp4", "mxfp4_a8", "mxfp4_a4"):
        return 0.53125  # 4 bits + one E8M0 byte per 32
    return 2.0 if cfg.routed == "bf16" else 4.0


def stage_work(cfg, offsets: np.ndarray, T: int) -> dict:
    """Algorithmic work of the routed-expert gate/up launch: flops of the
    selected (token, expert) pairs only; bytes = weights of the touched
    experts + the permuted latent rows read + h written."""
    R = T * cfg.k
    counts = np.diff(offsets)
    touched = int((counts > 0).sum())
    wbytes = 2 * cfg.I * cfg.L * routed_weight_bytes_per_element(cfg)
    flops = 2.0 * R * cfg.L * 2 * cfg.I
    # MXFP8 rows: E4M3 + E8M0/32; MXFP4 rows: E2M1 + E8M0/32
    act_in = {"mxfp4_a8": 1.03125, "mxfp4_a4": 0.53125}.get(cfg.routed, 2.0)
    bytes_ = touched * wbytes + R * cfg.L * act_in + R * cfg.I * 2
    return {"flops": flops, "bytes": bytes_, "touched_experts": touched}


def layer_bytes(cfg, offsets: np.ndarray, T: int, y_bytes: int) -> float:
    """Algorithmic HBM bytes of one whole layer step: every weight the step
    touches (the three matrices of each expert with at least one row, the
    router, W_down, W_up, the shared experts) plus x read and y written.  This
    is the bound of the weight-streaming decode step."""
    es = 2 if cfg.act == "bf16" else 4
    touched = int((np.diff(offsets) > 0).sum())
    routed = touched * 3 * cfg.I * cfg.L * routed_weight_bytes_per_element(cfg)
    dense = (cfg.E * cfg.H + 2 * cfg.L * cfg.H + 3 * cfg.S * cfg.Is * cfg.H) * es + cfg.E * 4 + cfg.L * 4
    return routed + dense + T * cfg.H * es + T * cfg.H * y_bytes


def gate_up_kernel(cfg) -> str:
    """The routed gate/up kernel the library runs for this workload (the rule
    of moe_api.cu's use_two_tile: bf16 weights whose tiles divide evenly take
    the two-weight-tile kernel unless MOE_EXPERT_KERNEL=one; MXFP4 with bf16
    inputs takes the one-tile kernel)."""
    if cfg.routed in ("mxfp4_a8", "mxfp4_a4"):
        return f"tc_expert_bs_kernel<3, 1, {1 if cfg.routed == 'mxfp4_a4' else 0}>"
    cg = 2 if (cfg.I % 128 == 0 and cfg.L % 256 == 0) else 1
    env = os.environ.get("MOE_EXPERT_KERNEL", "")
    two = cfg.routed == "bf16" and cfg.I % (128 * cg) == 0 and env != "one"
    if two:
        return f"tc_expert2_kernel<3, 1, {cg}>"
    return f"tc_expert_kernel<3, 1, {cg}, {1 if cfg.routed == 'mxfp4' else 0}>"


def gate_up_roofline(cfg, offsets, stage_ms: dict, peaks: dict) -> dict:
    """Roofline of the dominant kernel, the routed gate/up GEMM with the
    SiTU-GLU epilogue, from its CUDA-event time inside the timed region."""
    work = stage_work(cfg, offsets, cfg.T)
    dom_ms = stage_ms["expert_gate_up"]
    if cfg.routed == "mxfp4_a8":
        # kind::mxf8f6f4 runs at the fp8 rate: the measured bf16 peak times the
        # nominal fp8 / bf16 ratio (4.5 / 2.25 PFLOP/s dense)
        tensor_peak = 2.0 * peaks["bf16_tflops_sustained"]
        tsrc = (f"{peaks['source']} sustained bf16 x 2 (nominal fp8/bf16 ratio): the MMA kind is kind::mxf8f6f4 "
                "with E2M1 weights and E4M3 activations")
    elif cfg.routed == "mxfp4_a4":
        # kind::mxf4 runs at the fp4 rate: the measured bf16 peak times the
        # nominal fp4 / bf16 ratio (9 / 2.25 PFLOP/s dense)
        tensor_peak = 4.0 * peaks["bf16_tflops_sustained"]
        tsrc = (f"{peaks['source']} sustained bf16 x 4 (nominal fp4/bf16 ratio): the MMA kind is kind::mxf4 "
                "with E2M1 weights and activations")
    else:
        tensor_peak = peaks["bf16_tflops_sustained"]
        tsrc = f"{peaks['source']} sustained bf16 (the MMA kind is kind::f16 with bf16 operands)"
    bound = "tensor" if (work["flops"] / (tensor_peak * 1e12)) >= (
        work["bytes"] / (peaks["hbm_gbs"] * 1e9)) else "hbm"
    if bound == "tensor":
        achieved = work["flops"] / (dom_ms / 1e3) / 1e12
        peak, unit = tensor_peak, "TFLOP/s"
        src = tsrc
    else:
        achieved = work["bytes"] / (dom_ms / 1e3) / 1e9
        peak, unit = peaks["hbm_gbs"], "GB/s"
        src = f"{peaks['source']} HBM copy (read+write bytes); a read-dominated stream can exceed it"
    kname = gate_up_kernel(cfg)
    traffic = None
    prof = os.path.join(ROOT, "profiles", f"traffic_{cfg.name}_expert_gate_up.json")
    if os.path.exists(prof):
        # dram__bytes_read.sum + dram__bytes_write.sum of one launch, from an ncu
        # capture of this workload; only if it measured the kernel that ran here
        with open(prof) as f:
            rec = json.load(f)
        if rec.get("kernel") == kname:
            traffic = rec.get("dram_bytes_per_launch")
    kern = kname + {"mxfp4": " (2-CTA grouped gate/up, SiTU epilogue, MXFP4 weights decoded to bf16 in shared memory)",
                    "mxfp4_a8": " (2-CTA grouped gate/up, SiTU epilogue, block-scaled MXFP4 x MXFP8 MMA)",
                    "mxfp4_a4": " (2-CTA grouped gate/up, SiTU epilogue, block-scaled MXFP4 x MXFP4 MMA)"}.get(
        cfg.routed, " (2-CTA grouped gate/up, SiTU epilogue)")
    return {"kernel": f"{kern} = stage expert_gate_up", "bound": bound, "achieved": round(achieved, 1),
            "peak": peak, "unit": unit, "frac": round(achieved / peak, 4), "traffic": traffic, "peak_source": src,
            "kernel_ms": round(dom_ms, 4), "algorithmic": {"flops": work["flops"], "bytes": work["bytes"]},
            "touched_experts": work["touched_experts"]}


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
def measure_layer(layer, x, cfg, args, world: int, local_rank: int, sample_clocks: bool) -> dict:
    """Device time of `args.steps` layer steps (after `args.warmup`), the
    per-stage times inside that region, and the end-to-end time through the
    public API with pinned host copies in and out."""
    dev = x.device
    stream = torch.cuda.current_stream(dev)
    y = layer.output(cfg.T)
    offsets = torch.empty(cfg.E + 1, dtype=torch.int32, device=dev)

    def events():
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(2 * moe.MOE_NUM_STAGES)]
        for e in evs:
            e.record(stream)  # creates the event handle
        return evs

    for _ in range(args.warmup):
        layer.forward(x, y)
    torch.cuda.synchronize()
    launches_per_step = moe.moe_last_launch_count()

    step_events = [events() for _ in range(args.steps)]
    auxes = [moe.make_aux(stage_events=ev, expert_offsets=offsets) for ev in step_events]
    torch.cuda.synchronize()
    sampler = ClockSampler(local_rank) if sample_clocks else None
    time.sleep(0.3 if sampler else 0.0)
    barrier(world)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(args.steps):
        moe.check(moe.moe_layer_forward(layer.dims, layer._w, x, y, auxes[i], layer.workspace, None, stream))
    t1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clocks = sampler.stop() if sampler else None
    ms = max_over_ranks(t0.elapsed_time(t1), dev)

    stage_ms = {n: 0.0 for n in moe.STAGE_NAMES}
    for ev in step_events:
        for i, n in enumerate(moe.STAGE_NAMES):
            stage_ms[n] += ev[2 * i].elapsed_time(ev[2 * i + 1]) / args.steps

    e2e_ms = measure_e2e(layer, x, y, cfg, args, world)
    st, code = moe.moe_device_error()
    if st != moe.MOE_OK:
        raise RuntimeError(f"device fault {code} during the bench")
    return {"ms": ms, "stage_ms": stage_ms, "e2e_ms": e2e_ms, "clocks": clocks, "launches": launches_per_step,
            "offsets": offsets.cpu().numpy().astype(np.int64), "y_bytes": y.element_size()}


def measure_e2e(layer, x, y, cfg, args, world: int) -> float:
    """End to end through the public API (MoeLayer.forward): every step copies
    its input from pinned host memory to the device and reads its output back
    to pinned host memory.  Two device buffers each way let the copies of one
    step overlap the compute of the neighbouring steps (a copy-in stream and a
    copy-out stream, ordered by events); the timed region runs from before the
    first copy-in to after the last copy-out."""
    dev = x.device
    compute = torch.cuda.current_stream(dev)
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    x_host = torch.empty(x.shape, dtype=x.dtype, pin_memory=True)
    x_host.copy_(x)
    y_host = [torch.empty(y.shape, dtype=y.dtype, pin_memory=True) for _ in range(2)]
    x_dev = [torch.empty_like(x) for _ in range(2)]
    y_dev = [torch.empty_like(y) for _ in range(2)]
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    for b in range(2):  # every event has been recorded once before it is waited on
        ev_done[b].record(compute)
        ev_out[b].record(compute)

    def run(steps: int):
        for i in range(steps):
            b = i & 1
            with torch.cuda.stream(s_in):
                s_in.wait_event(ev_done[b])  # buffer b's previous step has read its x
                x_dev[b].copy_(x_host, non_blocking=True)
                ev_in[b].record(s_in)
            compute.wait_event(ev_in[b])
            compute.wait_event(ev_out[b])  # buffer b's previous y has been read back
            layer.forward(x_dev[b], y_dev[b], stream=compute)
            ev_done[b].record(compute)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_done[b])
                y_host[b].copy_(y_dev[b], non_blocking=True)
                ev_out[b].record(s_out)

    run(max(2, min(args.warmup, 3)))
    torch.cuda.synchronize()
    barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(compute)
    s_in.wait_event(e0)
    run(args.steps)
    compute.wait_event(ev_out[0])
    compute.wait_event(ev_out[1])
    e1.record(compute)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), dev)
    barrier(world)
    return ms


def routing_of_batch(layer, x, cfg) -> tuple[int, np.ndarray]:
    """(near-tie tokens, the device's expert choice [T, k]) of the whole batch.
    Near ties: tokens whose device-side selection margin (k-th minus (k+1)-th
    largest fp32 key s + b) is below NEAR_TIE, where a device and the fp64
    oracle may legitimately choose different experts.  Outside any timed
    region; scores and choice come from the layer itself (aux outputs)."""
    s = torch.empty(cfg.T, cfg.E, dtype=torch.float32, device=x.device)
    idx = torch.empty(cfg.T, cfg.k, dtype=torch.int32, device=x.device)
    layer.forward(x, aux={"scores": s, "topk_idx": idx})
    idx_np = idx.cpu().numpy().astype(np.int64)
    if cfg.k >= cfg.E:
        return 0, idx_np
    key = s + layer.weights["bias"][None, :]
    top = torch.topk(key, cfg.k + 1, dim=1).values
    return int(((top[:, cfg.k - 1] - top[:, cfg.k]) < NEAR_TIE).sum()), idx_np


def ep_balance(idx: np.ndarray, E: int, G: int = 8) -> dict:
    """The balanced expert-parallel plan (expert_parallel.balanced_plan) on
    this batch's routing, its tokens cut into G contiguous chunks taken as G
    ranks' batches: the largest rank load over the mean with experts split
    over the ranks by the static partition (every row to its expert's owner)
    and with the balanced plan, and the redundant expert copies that plan
    runs.  A host computation outside the timed region; nothing is timed."""
    from sparse_moe_layer_renormalised_b200 import expert_parallel as ep

    chunks = np.array_split(np.arange(idx.shape[0]), G)
    counts = np.stack([np.bincount(idx[c].reshape(-1), minlength=E) for c in chunks]).astype(np.int64)
    bounds = ep.partition(E, G)
    plan = ep.balanced_plan(counts, bounds)
    C = counts.sum(axis=0)
    mean = float(C.sum()) / G
    static = np.array([C[bounds[g]:bounds[g + 1]].sum() for g in range(G)])
    return {"ranks": G, "rows": int(C.sum()),
            "static_max_over_mean": round(float(static.max()) / mean, 4),
            "balanced_max_over_mean": round(float(plan.quota.max()) / mean, 4),
            "copies": int(sum(len(r) for r in plan.replicas)),
            "max_copies_per_rank": int(max(len(r) for r in plan.replicas)),
            "how": "the batch's tokens in G contiguous chunks as the ranks' batches; host planning only"}


def oracle_sample(cfg, layer, x, n_tokens: int, seed_offset: int = 0) -> tuple[dict, dict]:
    """The oracle on a seeded sample of the workload's tokens: the parity of
    the device output there (index sets, near ties, max|dy|/rms(y_ref)) and
    the oracle's own throughput on the host cores (the CPU baseline).  Weight
    generation is excluded from the oracle's time."""
    import oracle
    from oracle import inputs as oin

    tokens = gen.sample_tokens(cfg, n_tokens) if seed_offset == 0 else np.sort(
        np.random.default_rng(cfg.seed + 1000 + seed_offset).choice(cfg.T, size=min(n_tokens, cfg.T),
                                                                    replace=False))
    from dataclasses import replace

    # the same step with an fp32 y (the bf16 y is its rounding), same workspace
    idx = torch.empty(cfg.T, cfg.k, dtype=torch.int32, device=x.device)
    y = torch.empty(cfg.T, cfg.H, dtype=torch.float32, device=x.device)
    d = replace(layer.dims, T=cfg.T, y_out="f32")
    moe.check(moe.moe_layer_forward(d, layer._w, x, y, moe.make_aux(topk_idx=idx), layer.workspace))
    torch.cuda.synchronize()
    sel = torch.as_tensor(tokens)
    y_dev = y.cpu().to(torch.float64)[sel]
    idx_dev = idx.cpu().to(torch.int64)[sel]

    dense = oin.dense_weights(cfg)
    xr = oin.x_rows(cfg, tokens)
    gen_s = [0.0]

    def provider(e):
        t = time.perf_counter()
        w = oin.expert_weights_raw(cfg, e)
        gen_s[0] += time.perf_counter() - t
        return w

    t0 = time.perf_counter()
    ref = oracle.layer_forward_streamed(cfg, dense, xr, provider)
    oracle_s = time.perf_counter() - t0 - gen_s[0]
    differ = (torch.sort(idx_dev, 1).values != torch.sort(ref["idx"], 1).values).any(1)
    near = ref["margin"] < NEAR_TIE
    if bool(differ.any()):
        forced = ref["idx"].clone()
        forced[differ] = idx_dev[differ]
        ref = oracle.layer_forward_streamed(cfg, dense, xr, provider, forced_idx=forced)
    rms = float(ref["y"].pow(2).mean().sqrt())
    parity = {"tokens": len(tokens), "index_set_differences": int(differ.sum()),
              "differences_without_near_tie": int((differ & ~near).sum()), "near_tie_tokens": int(near.sum()),
              "max_abs_dy_over_rms": round(float((y_dev - ref["y"]).abs().max()) / rms, 6),
              "max_rms_dy_over_rms": round(float((y_dev - ref["y"]).pow(2).mean().sqrt()) / rms, 6),
              "tolerance": {"mxfp4": 3e-2, "mxfp4_a8": 1e-1, "mxfp4_a4": 0.5}.get(cfg.routed, 1e-2),
              "oracle": "fp64 C++ oracle (oracle/moe_oracle.cpp), storage-faithful bf16 rounding"}
    cpu = {"value": round(len(tokens) / oracle_s, 4), "unit": "tokens/s", "cores": oracle.num_threads(),
           "kind": "oracle",
           "sample": f"{len(tokens)} seeded tokens of the {cfg.name} workload (fp64 C++ oracle, "
                     f"{oracle.num_threads()} std::thread workers; weight generation excluded)"}
    return parity, cpu


def workload_line(cfg, layer, x, args, world, rank, local_rank, peaks, headline: bool) -> dict:
    m = measure_layer(layer, x, cfg, args, world, local_rank, sample_clocks=(rank == 0))
    off = m["offsets"]
    ms_step = m["ms"] / args.steps
    counts = np.diff(off)
    flops_step = float(cfg.flops_per_token()) * cfg.T
    lb = layer_bytes(cfg, off, cfg.T, m["y_bytes"])
    out = {
        "value": round(job_throughput(cfg.T, args.steps, world, m["ms"]), 1),
        "unit": "tokens/s",
        "ms_per_step": round(ms_step, 4),
        "tflops": round(flops_step / (ms_step / 1e3) / 1e12, 2),
        "stage_ms": {k: round(v, 4) for k, v in m["stage_ms"].items()},
        "roofline": gate_up_roofline(cfg, off, m["stage_ms"], peaks),
        # the whole step against HBM: the bound of the weight-streaming decode step
        "layer_hbm": {"bytes": lb, "achieved": round(lb / (ms_step / 1e3) / 1e9, 1), "peak": peaks["hbm_gbs"],
                      "unit": "GB/s", "frac": round(lb / (ms_step / 1e3) / 1e9 / peaks["hbm_gbs"], 4),
                      "peak_source": f"{peaks['source']} HBM copy (read+write); this stream is read-dominated"},
        "layer_tensor": {"flops": flops_step, "frac_of_sustained_bf16": round(
            flops_step / (ms_step / 1e3) / 1e12 / peaks["bf16_tflops_sustained"], 4)},
        "e2e": {
            "value": round(job_throughput(cfg.T, args.steps, world, m["e2e_ms"]), 1),
            "unit": "tokens/s",
            "h2d_bytes_per_step": x.numel() * x.element_size(),
            "d2h_bytes_per_step": cfg.T * cfg.H * m["y_bytes"],
            "how": "MoeLayer.forward with pinned-host copies in and out every step, double-buffered on copy streams",
        },
        "gpu_launches": m["launches"] * args.steps,
        "clocks": m["clocks"],
        "config": {
            "workload": workload_name(cfg),
            "tokens_per_step_per_gpu": cfg.T,
            "y_dtype": layer.dims.y_out,
            "parallelism": f"replicas x{world} (no data-path collective)",
            "l2": "inputs larger than L2 (routed weights %.1f GB, x %.0f MB per step)" % (
                3 * cfg.E * cfg.I * cfg.L * routed_weight_bytes_per_element(cfg) / 1e9, cfg.T * cfg.H * 2 / 1e6),
            "expert_rows_max": int(counts.max()),
            "expert_rows_min": int(counts.min()),
            "touched_experts": int((counts > 0).sum()),
        },
    }
    if world == 1:
        out["near_tie_tokens"], idx = routing_of_batch(layer, x, cfg)
        if cfg.E >= 8:
            try:  # an informational host statistic: it never costs the measured line
                out["ep_balance"] = ep_balance(idx, cfg.E)
            except Exception as exc:  # noqa: BLE001
                out["ep_balance"] = {"error": f"{type(exc).__name__}: {exc}"}
        if not args.no_oracle:
            parity, cpu = oracle_sample(cfg, layer, x, args.cpu_tokens)
            out["parity"] = parity
            out["cpu_baseline"] = cpu
    return out


# fp32 CUDA-core peak of B200 for the backward pass's contractions: 148 SMs x
# 128 fp32 FMA lanes x 2 flops x the SM clock (1965 MHz maximum).
FP32_ALU_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def backward_flops(cfg) -> float:
    """Algorithmic flops of moe_layer_backward: the forward contractions it
    recomputes (router, W_down, the selected experts' gate/up and down, the
    shared experts' gate/up; not the output projection) plus two contractions
    per forward one for the gradients of its two operands (all of them)."""
    T, H, L, E, k, I, S, Is = cfg.T, cfg.H, cfg.L, cfg.E, cfg.k, cfg.I, cfg.S, cfg.Is
    fwd_all = cfg.flops_per_token() * T
    recompute = fwd_all - T * (2 * L * H + S * 2 * Is * H)  # no output projection
    return recompute + 2 * fwd_all


def measure_backward(cfg, layer, x, reps: int = 3) -> dict:
    """moe_layer_backward (the layer's backward pass with the forward's
    selection held fixed) on this workload, timed with CUDA events after one
    warm-up call; reported against the fp32 CUDA-core peak."""
    dev = x.device
    stream = torch.cuda.current_stream(dev)
    d = dims_for(cfg, "f32")
    idx = torch.empty(cfg.T, cfg.k, dtype=torch.int32, device=dev)
    layer.forward(x, aux={"topk_idx": idx})
    dy = torch.randn(cfg.T, cfg.H, generator=torch.Generator().manual_seed(1)).to(dev)
    shapes = {"dx": (cfg.T, cfg.H), "dWr": (cfg.E, cfg.H), "dWdown": (cfg.L, cfg.H), "dWup": (cfg.H, cfg.L),
              "dgamma": (cfg.L,), "dWg": (cfg.E, cfg.I, cfg.L), "dWv": (cfg.E, cfg.I, cfg.L),
              "dWo": (cfg.E, cfg.L, cfg.I), "dWsg": (cfg.S, cfg.Is, cfg.H), "dWsv": (cfg.S, cfg.Is, cfg.H),
              "dWso": (cfg.S, cfg.H, cfg.Is)}
    grads = {n: torch.empty(s, dtype=torch.float32, device=dev) for n, s in shapes.items()}
    g = moe.make_grads(**grads)
    ws = torch.empty(moe.moe_backward_workspace_size(d), dtype=torch.uint8, device=dev)

    def call():
        moe.check(moe.moe_layer_backward(d, layer._w, x, dy, idx, g, ws, None, stream))

    call()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        call()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    flops = backward_flops(cfg)
    achieved = flops / (ms / 1e3) / 1e12
    del grads, ws
    return {"ms": round(ms, 3), "tokens_per_s": round(cfg.T / (ms / 1e3), 1), "flops": flops, "bound": "alu",
            "achieved": round(achieved, 2), "peak": round(FP32_ALU_PEAK_TFLOPS, 1), "unit": "TFLOP/s",
            "frac": round(achieved / FP32_ALU_PEAK_TFLOPS, 4),
            "peak_source": "derived: 148 SMs x 128 fp32 FMA/clock x 2 x 1965 MHz (contractions on CUDA cores)",
            "workload": workload_name(cfg)}


def build_layer(cfg, dev, y_out: str, weights=None):
    inputs = gen.device_layer(cfg, dev) if weights is None else weights
    x = inputs.pop("x") if "x" in inputs else None
    return moe.MoeLayer(dims_for(cfg, y_out), inputs), x, inputs


def run_ours(args, rank, world, local_rank):
    cfg = gen.CONFIGS[args.config]
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    peaks = load_peaks()
    layer, x, weights = build_layer(cfg, dev, args.y_out)
    line = workload_line(cfg, layer, x, args, world, rank, local_rank, peaks, headline=True)
    stream = torch.cuda.current_stream(dev)
    out = {
        "metric": METRIC,
        "value": line["value"],
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": line["ms_per_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": cfg.act,
        "data": "synthetic (seeded Philox inputs, random-init weights of the K3 layer shape)",
    }
    out.update({k: v for k, v in line.items() if k not in ("value", "unit", "ms_per_step")})
    out["qb_update"] = measure_qb(cfg, dev, stream, peaks)

    extra = [] if args.no_extra_lines or args.config != "prefill" else ["decode", "mxfp4", "mxfp4-a8", "mxfp4-a4"]
    for name in extra:
        sub = gen.CONFIGS[name]
        if name == "decode":
            # same weights as the prefill layer (same seed and shapes), the
            # decode workload's own bias, and the first 256 token rows of x
            w = dict(weights)
            w["bias"] = torch.from_numpy(gen.bias(sub)).to(dev)
            lay = moe.MoeLayer(dims_for(sub, args.y_out), w)
            xs = x[: sub.T].contiguous()
            out["decode"] = workload_line(sub, lay, xs, args, world, rank, local_rank, peaks, headline=False)
            del lay, xs, w
        elif name in ("mxfp4-a8", "mxfp4-a4"):
            # the MXFP4 workload's weights and x (same seed and shapes), routed
            # experts on the block-scaled path
            del layer
            torch.cuda.synchronize()
            layer = moe.MoeLayer(dims_for(sub, args.y_out), weights)
            out[name] = workload_line(sub, layer, x, args, world, rank, local_rank, peaks, headline=False)
        else:
            # the bf16 routed weights are no longer needed
            del layer, weights, x
            torch.cuda.synchronize()
            torch.cuda.empty_cache()
            layer, x, weights = build_layer(sub, dev, args.y_out)
            out[name] = workload_line(sub, layer, x, args, world, rank, local_rank, peaks, headline=False)
    if extra and not args.no_backward:
        # the backward pass on the mid layer (at the K3 shape the fp32 gradients
        # of all 896 experts' weights alone would take 118 GB)
        del layer, weights, x
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
        mid = gen.CONFIGS["mid"]
        layer, x, weights = build_layer(mid, dev, "f32")
        out["backward"] = measure_backward(mid, layer, x)
    return out if rank == 0 else None


# ----------------------------------------------------------------------------------- the oracle
def cpu_baseline(cfg, n_tokens: int, seed_offset: int = 0, dense=None) -> dict:
    """The fp64 C++ oracle on a bounded sample of the workload's tokens.  The
    time counts the oracle's own work (decoding the bf16 / MXFP4 weight bits
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
        w = oin.expert_weights_raw(cfg, e)
        gen_s[0] += time.perf_counter() - t
        return w

    t0 = time.perf_counter()
    oracle.layer_forward_streamed(cfg, dense, x, provider)
    total = time.perf_counter() - t0 - gen_s[0]
    return {"value": round(len(sample) / total, 4), "unit": "tokens/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"{len(sample)} seeded tokens of the {cfg.name} workload (fp64 C++ oracle, "
                      f"{oracle.num_threads()} std::thread workers; weight generation excluded)"}


def run_reference(args, rank, world):
    from oracle import inputs as oin

    cfg = gen.CONFIGS[args.config]
    per_step = max(1, args.cpu_tokens // 8)
    dense = oin.dense_weights(cfg)
    times = []
    cores = None
    for i in range(args.warmup + args.steps):
        cb = cpu_baseline(cfg, per_step, seed_offset=i, dense=dense)
        cores = cb["cores"]
        if i >= args.warmup:
            times.append(per_step / cb["value"])
    total = sum(times)
    value = per_step * args.steps / total
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": round(value, 4),
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
        "cpu_baseline": {"value": round(value, 4), "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"{per_step} seeded tokens per step of the {cfg.name} workload "
                                   f"(fp64 C++ oracle, {cores} std::thread workers)"},
        "e2e": {"value": round(value, 4), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", choices=sorted(gen.CONFIGS), default="prefill")
    ap.add_argument("--y-out", choices=["bf16", "f32"], default="bf16")
    ap.add_argument("--cpu-tokens", type=int, default=16)
    ap.add_argument("--no-oracle", "--no-cpu-baseline", dest="no_oracle", action="store_true",
                    help="skip the oracle sample (parity + CPU baseline)")
    ap.add_argument("--no-extra-lines", action="store_true", help="measure only --config (no decode / mxfp4 lines)")
    ap.add_argument("--no-backward", action="store_true", help="skip the backward-pass measurement")
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
