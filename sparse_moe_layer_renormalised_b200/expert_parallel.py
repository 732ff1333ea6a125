"""Expert-parallel Stable LatentMoE layer: the routed experts are split over the
ranks of a process group, token rows travel to the rank that holds their
expert and the expert outputs travel back (page "Kimi K3の二軸スケーリング
戦略とは何か", section "MoonEP：疎なMoEを実際に動かす通信層": the expert
parallelism that places the 896 experts across accelerators and exchanges
tokens with all-to-all communication).

Reading (where the page gives only the idea): experts are partitioned into G
contiguous ranges, rank g owning experts [bounds[g], bounds[g+1]); every rank
holds all non-routed weights and runs its own batch of tokens (data parallel
over tokens).

Balanced mode (the default; page "Kimi K3 tech-report summary"
(jiwasawa.github.io), section "Multi-Trillion 規模を支える Infrastructure", the
MoonEP item: redundant experts planned dynamically so that every rank is
assigned the same number of tokens, for static compute shapes).  Reading:
each step the ranks share their per-expert row counts and every rank computes
the same plan (balanced_plan): rank g runs floor(R/G) or ceil(R/G) of the step's
R routed rows; a rank whose own experts draw more rows than that hands rows of
its hottest experts to ranks below their quota, which run those experts as
redundant copies for the step (their weights travel from the owner with the
rows).  The static mode (balance=False) sends every row to its expert's owner.

One layer step on rank g (every step of the layer runs in libmoe_b200.so;
the exchange is torch.distributed all_to_all, NCCL between GPUs):
  1. moe_router_topk       scores, selection, mixture weights (all E experts)
  2. moe_latent_shared     z = W_down x and the shared experts' h
  3. moe_permute           expert-major order of the local (token, slot)
                           pairs with their z rows; the rows bound for rank r
                           are then one contiguous block
  4. exchange plan         per-expert row counts to and from every rank
                           (balanced: all ranks' counts, the plan, and the
                           redundant experts' weights from their owners)
  5. dispatch              all_to_all of the z rows (balanced: first ordered
                           by destination with moe_gather_rows)
  6. moe_expert_ffn_blocks this rank's experts (balanced: and its redundant
                           copies) over the received rows, one expert-major
                           block per sending rank
  7. combine               all_to_all of the fp32 expert outputs back, which
                           arrive in the sender's send order (balanced: put
                           back in expert-major order with moe_gather_rows)
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
                       moe_expert_ffn_blocks_workspace_size, moe_gather_rows, moe_latent_shared, moe_output,
                       moe_permute, moe_router_topk, moe_workspace_size)

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


# ------------------------------------------------------------------------------ balanced mode
@dataclass
class BalancedPlan:
    """One step's assignment of the routed rows to ranks.

    The rows of expert e, in global order (sending ranks in rank order, each
    sender's rows in its own expert-major order), are cut into segments: the
    owner's first, then one per rank that runs a redundant copy of e."""

    bounds: np.ndarray   # [G + 1] home partition (partition(E, G))
    quota: np.ndarray    # [G] rows each rank runs: floor(R / G), the first R % G ranks one more
    segments: list       # [E] lists of (rank, start, count), ordered by start
    replicas: list       # [G] ascending ids of the experts rank g runs without owning them

    def local_experts(self, g: int) -> np.ndarray:
        """The experts rank g runs, in its local order: its own, then its
        redundant copies."""
        home = np.arange(self.bounds[g], self.bounds[g + 1], dtype=np.int64)
        return np.concatenate([home, np.asarray(self.replicas[g], np.int64)])


def balanced_plan(counts: np.ndarray, bounds: np.ndarray) -> BalancedPlan:
    """counts [G, E]: rows each rank sends to each expert this step.

    Every rank's load becomes exactly its quota: ranks whose own experts
    exceed it (donors, in rank order) hand rows of their experts, hottest
    first (ties to the lower id), to the ranks below it (receivers, in rank
    order), a receiver taking from one expert until it is full or the
    donor's excess or the expert's rows are used up.  Each hand-over makes the
    receiver run a redundant copy of that expert.  Deterministic, so every
    rank computes the same plan from the same counts."""
    counts = np.asarray(counts, np.int64)
    G = len(bounds) - 1
    C = counts.sum(axis=0)
    R = int(C.sum())
    quota = np.full(G, R // G, np.int64)
    quota[: R % G] += 1
    home_load = np.array([C[bounds[g]:bounds[g + 1]].sum() for g in range(G)], np.int64)
    excess = home_load - quota
    deficit = np.maximum(-excess, 0)
    receivers = [g for g in range(G) if deficit[g] > 0]
    keep = C.copy()                     # rows the owner keeps
    given: dict = {}                    # expert -> [(rank, rows)] handed over, in order
    ri = 0
    for d in range(G):
        need = int(excess[d])
        if need <= 0:
            continue
        ids = np.arange(bounds[d], bounds[d + 1])
        for e in ids[np.lexsort((ids, -C[ids]))]:  # hottest first, ties to the lower id
            e = int(e)
            while need > 0 and keep[e] > 0:
                r = receivers[ri]
                n = int(min(need, keep[e], deficit[r]))
                given.setdefault(e, []).append((r, n))
                keep[e] -= n
                need -= n
                deficit[r] -= n
                if deficit[r] == 0:
                    ri += 1
            if need == 0:
                break
    owner = np.searchsorted(bounds, np.arange(len(C)), side="right") - 1
    segments = [[(int(o), 0, int(c))] if c > 0 else [] for o, c in zip(owner.tolist(), keep.tolist())]
    replicas = [[] for _ in range(G)]
    for e, lst in given.items():
        start = int(keep[e])
        for r, n in lst:
            segments[e].append((r, start, n))
            replicas[r].append(e)
            start += n
    return BalancedPlan(bounds=np.asarray(bounds, np.int64), quota=quota, segments=segments,
                        replicas=[sorted(set(x)) for x in replicas])


@dataclass
class BalancedExchange:
    """One rank's side of a balanced exchange."""

    send_idx: np.ndarray            # [n_send] rows of the sender's expert-major buffer, in send order
    send_rows: list                 # [G]
    recv_rows: list                 # [G]
    recv_block_offsets: np.ndarray  # [G, n_local + 1] offsets of each source's block, by local expert
    n_recv: int


def _segment_table(plan: BalancedPlan):
    """The plan's segments as arrays (expert, rank, start, rows) and each
    segment's local expert index on its rank (own experts first, then copies
    in ascending id order)."""
    seg = [(e, g, st, n) for e, lst in enumerate(plan.segments) for g, st, n in lst]
    if not seg:
        z = np.zeros(0, np.int64)
        return z, z, z, z, z
    e, g, st, n = (np.array(c, np.int64) for c in zip(*seg))
    n_home = np.diff(plan.bounds)
    local = e - plan.bounds[g]
    own = (local >= 0) & (local < n_home[g])
    for i in np.nonzero(~own)[0]:
        local[i] = n_home[g[i]] + plan.replicas[g[i]].index(int(e[i]))
    return e, g, st, n, local


def balanced_exchange(plan: BalancedPlan, counts: np.ndarray, offsets: np.ndarray, rank: int) -> BalancedExchange:
    """The send order, split sizes and receive blocks of `rank` under the
    plan; offsets [E + 1] are this rank's expert-major CSR offsets.  Rows
    bound for one destination are sent together, in the destination's local
    expert order; a received block (one per source, in rank order) is
    expert-major in this rank's local order."""
    counts = np.asarray(counts, np.int64)
    G = len(plan.quota)
    n_local = len(plan.local_experts(rank))
    e, g, st, n, local = _segment_table(plan)
    # rows of each expert from earlier senders: sender s's rows of expert e
    # are positions [before[s, e], before[s, e] + counts[s, e]) of e's rows
    before = np.cumsum(counts, axis=0) - counts
    lo = before[:, e]
    hi = lo + counts[:, e]
    a = np.maximum(lo, st[None, :])
    overlap = np.maximum(np.minimum(hi, (st + n)[None, :]) - a, 0)  # [senders, segments]
    # this rank's sends: pieces ordered by (destination, its local expert)
    mine = np.nonzero(overlap[rank] > 0)[0]
    order = mine[np.lexsort((local[mine], g[mine]))]
    starts = np.asarray(offsets, np.int64)[e[order]] + (a[rank, order] - lo[rank, order])
    lens = overlap[rank, order]
    total = int(lens.sum())
    first = np.cumsum(lens) - lens
    send_idx = np.repeat(starts - first, lens) + np.arange(total, dtype=np.int64)
    send_rows = np.bincount(g[order], weights=lens, minlength=G).astype(np.int64).tolist()
    # this rank's receives: per source, rows per local expert
    here = np.nonzero(g == rank)[0]
    per = np.zeros((G, n_local), np.int64)
    for s in range(G):
        np.add.at(per[s], local[here], overlap[s, here])
    blocks = np.zeros((G, n_local + 1), np.int64)
    tot = per.sum(axis=1)
    blocks[:, 0] = np.cumsum(tot) - tot
    blocks[:, 1:] = blocks[:, :1] + np.cumsum(per, axis=1)
    return BalancedExchange(send_idx=send_idx, send_rows=[int(v) for v in send_rows],
                            recv_rows=[int(v) for v in tot], recv_block_offsets=blocks, n_recv=int(tot.sum()))


def gather_counts(offsets: np.ndarray, group=None) -> np.ndarray:
    """Every rank's per-expert row counts [G, E] (one all_gather)."""
    c = torch.from_numpy(np.diff(np.asarray(offsets, np.int64)))
    dev = _comm_device(group)
    out = [torch.empty_like(c, device=dev) for _ in range(dist.get_world_size(group))]
    dist.all_gather(out, c.to(dev), group=group)
    return torch.stack(out).cpu().numpy()


def exchange_expert_slices(want: list, bounds: np.ndarray, home: dict, group=None) -> dict:
    """Sends expert weight slices from their owners to the ranks that ask for
    them.  want[g]: ascending ids of the experts rank g needs (none of its
    own), the same list on every rank; home: name -> [n_home, ...] tensor of
    this rank's experts, one slice per expert.  Returns name -> [len(want[rank]),
    ...], the requested slices in ascending id order.  When nobody asks for
    anything every rank returns empty tensors without a collective."""
    rank = dist.get_rank(group)
    G = len(bounds) - 1
    lo = int(bounds[rank])
    if not any(want):
        return {name: t[:0] for name, t in home.items()}
    out = {}
    for name, t in home.items():
        per = t[0].numel() * t.element_size()
        flat = t.reshape(t.shape[0], -1).view(torch.uint8) if t.dtype != torch.uint8 else t.reshape(t.shape[0], -1)
        send, send_sizes = [], []
        for g in range(G):
            mine = [e - lo for e in want[g] if bounds[rank] <= e < bounds[rank + 1]]
            send += [flat[i] for i in mine]
            send_sizes.append(per * len(mine))
        recv_sizes = [per * sum(1 for e in want[rank] if bounds[s] <= e < bounds[s + 1]) for s in range(G)]
        sbuf = torch.cat(send) if send else torch.zeros(0, dtype=torch.uint8, device=t.device)
        rbuf = torch.empty(sum(recv_sizes), dtype=torch.uint8, device=t.device)
        dist.all_to_all_single(rbuf, sbuf.contiguous(), output_split_sizes=recv_sizes, input_split_sizes=send_sizes,
                               group=group)
        out[name] = rbuf.view(t.dtype).reshape((len(want[rank]),) + tuple(t.shape[1:]))
    return out


def exchange_replica_weights(plan: BalancedPlan, home: dict, group=None) -> dict:
    """Every redundant expert's weights from its owner to the ranks that run
    it this step: name -> [len(replicas[rank]), ...] in ascending id order."""
    return exchange_expert_slices(plan.replicas, plan.bounds, home, group)


def missing_copies(plan: BalancedPlan, held: list | None) -> list:
    """Per rank, the redundant experts of the plan whose weights it does not
    hold yet (held[g]: the copies rank g kept from earlier steps)."""
    if held is None:
        return [list(r) for r in plan.replicas]
    return [[e for e in plan.replicas[g] if e not in set(held[g])] for g in range(len(plan.quota))]


def balanced_step(z_perm: torch.Tensor, offsets: np.ndarray, bounds: np.ndarray, home: dict, run_experts, gather,
                  group=None, held: list | None = None):
    """One balanced exchange around this rank's expert computation.

    z_perm [n, L]: this rank's expert-major token rows, offsets [E + 1] their
    CSR offsets; home: name -> [n_home, ...] per-expert weight slices of this
    rank's experts (sent to the ranks that run copies); held (optional, the
    same on every rank): per rank the copies it kept from earlier steps,
    which are not sent again.  gather(src, idx) -> src[idx] on idx int32 rows
    (the layer: moe_gather_rows); run_experts(z_recv, exchange, plan, copies,
    copy_ids) -> fp32 outputs [n_recv, L] for the received rows, copies being
    the weight slices of this rank's redundant experts copy_ids (those it did
    not hold).  Returns (y_perm [n, L] fp32 in expert-major order, plan,
    exchange)."""
    rank = dist.get_rank(group)
    counts = gather_counts(offsets, group)
    plan = balanced_plan(counts, bounds)
    ex = balanced_exchange(plan, counts, offsets, rank)
    want = missing_copies(plan, held)
    copies = exchange_expert_slices(want, plan.bounds, home, group)
    dev, n_send = z_perm.device, len(ex.send_idx)
    z_send = gather(z_perm, torch.from_numpy(ex.send_idx.astype(np.int32)).to(dev))
    z_recv = torch.empty((ex.n_recv,) + tuple(z_perm.shape[1:]), dtype=z_perm.dtype, device=dev)
    dist.all_to_all_single(z_recv, z_send, output_split_sizes=ex.recv_rows, input_split_sizes=ex.send_rows,
                           group=group)
    y_recv = run_experts(z_recv, ex, plan, copies, want[rank])
    y_back = torch.empty((n_send,) + tuple(y_recv.shape[1:]), dtype=y_recv.dtype, device=dev)
    dist.all_to_all_single(y_back, y_recv, output_split_sizes=ex.send_rows, input_split_sizes=ex.recv_rows,
                           group=group)
    inv = np.empty(n_send, np.int64)
    inv[ex.send_idx] = np.arange(n_send)
    return gather(y_back, torch.from_numpy(inv.astype(np.int32)).to(dev)), plan, ex


class ExpertSlots:
    """A rank's routed weights for the balanced mode: per tensor name one
    buffer [n_home + capacity, ...] holding the rank's own expert slices
    first and, behind them, its redundant copies in ascending id order
    (`held`), so that the local expert set (own experts, then copies) is one
    contiguous prefix.  Copies stay from one step to the next; a step whose
    plan repeats a copy does not receive it again."""

    def __init__(self, home: dict, capacity: int):
        self.home = home
        self.n_home = next(iter(home.values())).shape[0]
        self.buf: dict = {}
        self.held: list = []
        self.capacity = 0
        self.grow(capacity)

    def grow(self, capacity: int) -> None:
        """Room for `capacity` copies; the own slices and the held copies move along."""
        keep = self.n_home + len(self.held)
        for n, t in self.home.items():
            b = torch.empty((self.n_home + capacity,) + tuple(t.shape[1:]), dtype=t.dtype, device=t.device)
            if n in self.buf:
                b[:keep].copy_(self.buf[n][:keep])
            else:
                b[: self.n_home].copy_(t)
            self.buf[n] = b
        self.capacity = capacity

    def place(self, copies: dict, ids: list, replicas: list) -> int:
        """Arranges this step's copies, `replicas` (ascending ids), behind the
        own experts: `copies` holds the slices of `ids` (the copies not held
        yet, ascending), the rest come from the held copies.  Returns the local
        expert count."""
        n_rep = len(replicas)
        if n_rep > self.capacity:
            self.grow(max(n_rep, 2 * self.capacity))
        h = len(self.held)
        old = {e: i for i, e in enumerate(self.held)}
        new = {e: h + i for i, e in enumerate(ids)}
        if any(e not in old and e not in new for e in replicas):
            raise ValueError("a redundant copy is neither held nor received")
        src = [new[e] if e in new else old[e] for e in replicas]
        for n, t in copies.items():
            pool = torch.cat([self.buf[n][self.n_home:self.n_home + h], t])  # a fresh tensor: no aliasing
            idx = torch.tensor(src, dtype=torch.long, device=pool.device)
            self.buf[n][self.n_home:self.n_home + n_rep].copy_(pool.index_select(0, idx))
        self.held = list(replicas)
        return self.n_home + n_rep

    def local(self, n_local: int) -> dict:
        """name -> the first n_local expert slices (views, no copy)."""
        return {n: b[:n_local] for n, b in self.buf.items()}

    def forget(self) -> None:
        """Drops the held copies (after the owners' weights changed)."""
        self.held = []


class ExpertParallelMoeLayer:
    """One rank's share of an expert-parallel layer.

    dims: the full layer (E = all routed experts).  weights: device tensors
    named as moe_weights' fields; Wg / Wv / Wo (and Sg / Sv / So for MXFP4)
    hold only this rank's experts, bounds[rank] .. bounds[rank+1]-1, in order.
    With a block-scaled routed type ("mxfp4_a8", "mxfp4_a4") the dispatched
    rows stay bf16 and the receiving rank quantises them
    (moe_expert_ffn_blocks).  balance (default True): every rank runs the
    same number of rows per step, hot experts' rows shared out to redundant
    copies (module docstring); False: every row goes to its expert's owner.
    max_tokens sizes the local workspaces."""

    def __init__(self, dims: Dims, weights: dict, group=None, max_tokens: int | None = None, balance: bool = True):
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
        self.balance = balance
        self.last_plan = None
        if balance:
            # the routed tensors this path reads, one slice per expert, in
            # buffers with room behind this rank's experts for redundant copies
            names = ["Wg", "Wv", "Wo"] + (["Sg", "Sv", "So"] if dims.routed == "mxfp4" else []) + (
                ["Sgv_tiled", "So_tiled"] if dims.routed in BLOCK_SCALED else [])
            self._home = {n: self.weights[n].reshape((self.e_local, -1) if n.endswith("_tiled") else
                                                     tuple(self.weights[n].shape)) for n in names}
            self._slots = ExpertSlots(self._home, self.e_local)
            self._held = None  # per rank, the copies kept from the last step (the same list on every rank)

    def _local_weights(self, n_local: int):
        w = {n: (t.reshape(-1) if n.endswith("_tiled") else t) for n, t in self._slots.local(n_local).items()}
        return make_weights(**w)

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
        if self.balance:
            y_perm = self._balanced_experts(d, offsets.cpu().numpy(), z_perm, stream)
        else:
            y_perm = self._static_experts(d, offsets.cpu().numpy(), z_perm, stream)
        n = torch.empty(T, L, dtype=act, device=dev)
        check(moe_combine(d, y_perm, inv_perm, p, w["gamma"], None, n, stream))
        y = torch.empty(T, d.H, dtype=_TORCH_DT[d.y_out], device=dev)
        check(moe_output(d, self._w, h_s, n, y, stream))
        return y

    def _static_experts(self, d: Dims, offsets: np.ndarray, z_perm: torch.Tensor, stream) -> torch.Tensor:
        """Every row to its expert's owner and back: y_perm [T k, L] fp32."""
        dev, L = z_perm.device, d.L
        plan = exchange_plan(offsets, self.bounds, self.group)
        z_recv = dispatch_rows(z_perm, plan, self.group)
        y_recv = torch.empty(plan.n_recv, L, dtype=torch.float32, device=dev)
        if plan.n_recv > 0:
            blocks = torch.from_numpy(plan.recv_block_offsets.astype(np.int32)).to(dev)
            ws = torch.empty(moe_expert_ffn_blocks_workspace_size(self.local_dims, plan.n_recv, self.G),
                             dtype=torch.uint8, device=dev)
            check(moe_expert_ffn_blocks(self.local_dims, self._w, z_recv, plan.n_recv, blocks, self.G, y_recv, ws,
                                        None, stream))
        return combine_rows(y_recv, plan, self.group)

    def _balanced_experts(self, d: Dims, offsets: np.ndarray, z_perm: torch.Tensor, stream) -> torch.Tensor:
        """The balanced exchange: y_perm [T k, L] fp32 in expert-major order."""
        dev, L = z_perm.device, d.L

        def gather(src: torch.Tensor, idx: torch.Tensor) -> torch.Tensor:
            dst = torch.empty((len(idx),) + tuple(src.shape[1:]), dtype=src.dtype, device=dev)
            check(moe_gather_rows(src, src.shape[0], src[0].numel() * src.element_size(), idx, len(idx), dst,
                                  stream))
            return dst

        def run_experts(z_recv: torch.Tensor, ex: BalancedExchange, plan: BalancedPlan, copies: dict, ids: list):
            n_local = self._slots.place(copies, ids, plan.replicas[self.rank])
            assert n_local == len(plan.local_experts(self.rank))
            y_recv = torch.empty(ex.n_recv, L, dtype=torch.float32, device=dev)
            if ex.n_recv > 0:
                ld = replace(d, E=n_local)
                blocks = torch.from_numpy(ex.recv_block_offsets.astype(np.int32)).to(dev)
                ws = torch.empty(moe_expert_ffn_blocks_workspace_size(ld, ex.n_recv, self.G), dtype=torch.uint8,
                                 device=dev)
                check(moe_expert_ffn_blocks(ld, self._local_weights(n_local), z_recv, ex.n_recv, blocks, self.G,
                                            y_recv, ws, None, stream))
            return y_recv

        y_perm, plan, _ = balanced_step(z_perm, offsets, self.bounds, self._home, run_experts, gather, self.group,
                                        held=self._held)
        self.last_plan = plan
        self._held = [list(r) for r in plan.replicas]
        return y_perm

    def forget_copies(self) -> None:
        """Call on every rank after the routed weights changed: the redundant
        copies kept from earlier steps are dropped and sent again when needed."""
        if self.balance:
            self._held = None
            self._slots.forget()

    __call__ = forward
