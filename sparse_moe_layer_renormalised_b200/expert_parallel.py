"""Expert-parallel Stable LatentMoE layer: the routed experts are split over the
ranks of a process group, token rows travel to the rank that holds their
expert and the expert outputs travel back (page "Kimi K3の二軸スケーリング
戦略とは何か", section "MoonEP：疎なMoEを実際に動かす通信層": the expert
parallelism that places the 896 experts across accelerators and exchanges
tokens with all-to-all communication).

Reading (where the page gives only the idea): experts are partitioned into G
contiguous ranges, rank g owning experts [bounds[g], bounds[g+1]); every rank
holds all non-routed weights and runs its own batch of tokens (data parallel
over tokens).  MoonEP's redundant copies of hot experts and its balanced
placement are not built.

One layer step on rank g (every step of the layer runs in libmoe_b200.so;
the exchange is torch.distributed all_to_all, NCCL between GPUs):
  1. moe_router_topk       scores, selection, mixture weights (all E experts)
  2. moe_latent_shared     z = W_down x and the shared experts' h
  3. moe_permute           expert-major order of the local (token, slot)
                           pairs with their z rows; the rows bound for rank r
                           are then one contiguous block
  4. exchange plan         per-expert row counts to and from every rank
  5. dispatch              all_to_all of the z rows
  6. moe_expert_ffn_blocks this rank's experts over the received rows, one
                           expert-major block per sending rank
  7. combine               all_to_all of the fp32 expert outputs back, which
                           arrive in the sender's own expert-major order
  8. moe_combine, moe_output   u, RMSNorm(u), y
Step 4 reads the expert offsets on the host (the all_to_all needs the row
counts), the one host synchronisation of the step.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import numpy as np
import torch
import torch.distributed as dist

from .layer import tile_weight_scales
from ._binding import (BLOCK_SCALED, Dims, check, make_weights, moe_combine, moe_expert_ffn_blocks,
                       moe_expert_ffn_blocks_workspace_size, moe_latent_shared, moe_output, moe_permute,
                       moe_router_topk, moe_workspace_size)

_TORCH_DT = {"f32": torch.float32, "bf16": torch.bfloat16}


def partition(E: int, G: int) -> np.ndarray:
    """Bounds [G + 1] of the contiguous expert ranges: rank g owns experts
    bounds[g] .. bounds[g+1]-1; the first E % G ranks get one more."""
    if not 1 <= G <= E:
        raise ValueError(f"cannot split {E} experts over {G} ranks")
    sizes = np.full(G, E // G, np.int64)
    sizes[: E % G] += 1
    return np.concatenate([[0], np.cumsum(sizes)]).astype(np.int64)


@dataclass
class ExchangePlan:
    """Row counts of one exchange, seen from one rank."""

    send_rows: list  # [G] rows this rank sends to each rank
    recv_rows: list  # [G] rows this rank receives from each rank
    recv_block_offsets: np.ndarray  # [G, E_local + 1] absolute offsets of each source's block
    n_recv: int


def send_counts(offsets: np.ndarray, bounds: np.ndarray) -> np.ndarray:
    """Per-expert row counts this rank sends, grouped by destination:
    [G, Emax] (zero-padded), from its expert-major CSR offsets [E + 1]."""
    offsets = np.asarray(offsets, np.int64)
    G = len(bounds) - 1
    emax = int(np.diff(bounds).max())
    out = np.zeros((G, emax), np.int64)
    counts = np.diff(offsets)
    for r in range(G):
        c = counts[bounds[r]:bounds[r + 1]]
        out[r, : len(c)] = c
    return out


def plan_from_counts(sent: np.ndarray, received: np.ndarray, e_local: int) -> ExchangePlan:
    """sent [G, Emax]: per-expert rows this rank sends to each rank;
    received [G, Emax]: per-expert rows each rank sends to this one (of this
    rank's e_local experts).  The receive buffer holds the sources' blocks in
    rank order; inside a block rows are expert-major, as the sender's order."""
    G = sent.shape[0]
    recv = received[:, :e_local]
    block_offsets = np.zeros((G, e_local + 1), np.int64)
    start = 0
    for b in range(G):
        block_offsets[b, 0] = start
        block_offsets[b, 1:] = start + np.cumsum(recv[b])
        start = int(block_offsets[b, -1])
    return ExchangePlan(send_rows=[int(v) for v in sent.sum(axis=1)],
                        recv_rows=[int(v) for v in recv.sum(axis=1)],
                        recv_block_offsets=block_offsets, n_recv=start)


def exchange_plan(offsets: np.ndarray, bounds: np.ndarray, group=None) -> ExchangePlan:
    """Trades the per-expert row counts with every rank (one small
    all_to_all) and returns this rank's plan."""
    rank = dist.get_rank(group)
    sent = send_counts(offsets, bounds)
    dev = _comm_device(group)
    s = torch.from_numpy(sent.reshape(-1)).to(dev)
    r = torch.empty_like(s)
    dist.all_to_all_single(r, s, group=group)
    received = r.cpu().numpy().reshape(sent.shape)
    return plan_from_counts(sent, received, int(bounds[rank + 1] - bounds[rank]))


def _comm_device(group=None) -> torch.device:
    backend = dist.get_backend(group)
    return torch.device("cuda", torch.cuda.current_device()) if backend == "nccl" else torch.device("cpu")


def dispatch_rows(rows: torch.Tensor, plan: ExchangePlan, group=None) -> torch.Tensor:
    """The sender's expert-major rows [sum send_rows, ...] -> this rank's
    receive buffer [n_recv, ...] (sources in rank order)."""
    out = torch.empty((plan.n_recv,) + tuple(rows.shape[1:]), dtype=rows.dtype, device=rows.device)
    dist.all_to_all_single(out, rows.contiguous(), output_split_sizes=plan.recv_rows,
                           input_split_sizes=plan.send_rows, group=group)
    return out


def combine_rows(rows: torch.Tensor, plan: ExchangePlan, group=None) -> torch.Tensor:
    """The inverse exchange: per-row results in receive order -> the sender's
    rows back in its own expert-major order."""
    out = torch.empty((sum(plan.send_rows),) + tuple(rows.shape[1:]), dtype=rows.dtype, device=rows.device)
    dist.all_to_all_single(out, rows.contiguous(), output_split_sizes=plan.send_rows,
                           input_split_sizes=plan.recv_rows, group=group)
    return out


class ExpertParallelMoeLayer:
    """One rank's share of an expert-parallel layer.

    dims: the full layer (E = all routed experts).  weights: device tensors
    named as moe_weights' fields; Wg / Wv / Wo (and Sg / Sv / So for MXFP4)
    hold only this rank's experts, bounds[rank] .. bounds[rank+1]-1, in order.
    With a block-scaled routed type ("mxfp4_a8", "mxfp4_a4") the dispatched rows stay bf16 and the receiving
    rank quantises them (moe_expert_ffn_blocks).
    max_tokens sizes the local workspaces."""

    def __init__(self, dims: Dims, weights: dict, group=None, max_tokens: int | None = None):
        self.dims = dims
        self.group = group
        self.G = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.bounds = partition(dims.E, self.G)
        self.e_local = int(self.bounds[self.rank + 1] - self.bounds[self.rank])
        if weights["Wg"].shape[0] != self.e_local:
            raise ValueError(f"rank {self.rank} holds {weights['Wg'].shape[0]} experts, expected {self.e_local}")
        self.local_dims = replace(dims, E=self.e_local)
        self.weights = dict(weights)
        if dims.routed in BLOCK_SCALED and "Sgv_tiled" not in weights:
            # the block-scaled experts read their scales in tiled order, made once per rank
            self.weights.update(tile_weight_scales(self.local_dims, weights["Sg"], weights["Sv"], weights["So"]))
        self._w = make_weights(**self.weights)
        self.max_tokens = dims.T if max_tokens is None else max_tokens
        dev = weights["Wr"].device
        self.workspace = torch.empty(moe_workspace_size(replace(dims, T=self.max_tokens)), dtype=torch.uint8,
                                     device=dev)

    def forward(self, x: torch.Tensor, stream=None) -> torch.Tensor:
        d = replace(self.dims, T=x.shape[0])
        T, k, E, L = d.T, d.k, d.E, d.L
        dev = x.device
        act = _TORCH_DT[d.act]
        scores = torch.empty(T, E, dtype=torch.float32, device=dev)
        idx = torch.empty(T, k, dtype=torch.int32, device=dev)
        p = torch.empty(T, k, dtype=torch.float32, device=dev)
        z = torch.empty(T, L, dtype=act, device=dev)
        h_s = torch.empty(T, max(d.S, 1) * max(d.Is, 1), dtype=act, device=dev) if d.S > 0 else None
        offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
        perm_token = torch.empty(T * k, dtype=torch.int32, device=dev)
        inv_perm = torch.empty(T * k, dtype=torch.int32, device=dev)
        z_perm = torch.empty(T * k, L, dtype=act, device=dev)
        w = self.weights
        check(moe_router_topk(d, x, w["Wr"], w["bias"], scores, 0, idx, p, stream))
        check(moe_latent_shared(d, self._w, x, z, h_s, stream))
        check(moe_permute(d, idx, z, offsets, perm_token, inv_perm, z_perm, self.workspace, None, stream))
        plan = exchange_plan(offsets.cpu().numpy(), self.bounds, self.group)
        z_recv = dispatch_rows(z_perm, plan, self.group)
        y_recv = torch.empty(plan.n_recv, L, dtype=torch.float32, device=dev)
        if plan.n_recv > 0:
            blocks = torch.from_numpy(plan.recv_block_offsets.astype(np.int32)).to(dev)
            ws = torch.empty(moe_expert_ffn_blocks_workspace_size(self.local_dims, plan.n_recv, self.G),
                             dtype=torch.uint8, device=dev)
            check(moe_expert_ffn_blocks(self.local_dims, self._w, z_recv, plan.n_recv, blocks, self.G, y_recv, ws,
                                        None, stream))
        y_perm = combine_rows(y_recv, plan, self.group)
        n = torch.empty(T, L, dtype=act, device=dev)
        check(moe_combine(d, y_perm, inv_perm, p, w["gamma"], None, n, stream))
        y = torch.empty(T, d.H, dtype=_TORCH_DT[d.y_out], device=dev)
        check(moe_output(d, self._w, h_s, n, y, stream))
        return y

    __call__ = forward
