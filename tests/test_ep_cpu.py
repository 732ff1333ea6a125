"""The expert-parallel exchange (dispatch and combine of token rows between
the ranks that hold the experts) on CPU: gloo ranks, world sizes 2 to 4, in
the static mode (rows to their expert's owner) and the balanced mode (equal
rows per rank, redundant copies of hot experts; see the last section).

Every rank routes its own tokens, orders its (token, slot) pairs expert-major
(the oracle's stable permutation), and sends each rank the rows of that rank's
experts.  The tests check the exchange tables and the rows against a brute
force over all ranks' data: each rank receives exactly the rows of its experts
(sources in rank order, expert-major within a source), the block offsets label
every received row with its expert, and the results of a stand-in expert
function come back to the sender at the positions of the rows it sent."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from sparse_moe_layer_renormalised_b200 import expert_parallel as ep


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _routing(rank, T, E, k, mode):
    rng = np.random.default_rng(100 + rank)
    if mode == "one_sided" and rank == 1:
        # rank 1 only picks rank 0's experts: it sends nothing to the others
        return np.stack([rng.choice(E // 2, size=k, replace=False) for _ in range(T)])
    w = (np.arange(E) + 1.0) ** -0.8  # Zipf-like expert popularity
    return np.stack([rng.choice(E, size=k, replace=False, p=w / w.sum()) for _ in range(T)])


def _worker(rank, world, port, E, k, mode, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        T, L = 40 + 17 * rank, 6
        idx = _routing(rank, T, E, k, mode)
        z = np.random.default_rng(7 + rank).standard_normal((T, L)).astype(np.float32)
        counts, offsets, perm_token, inv_perm = oracle.permute(idx, E)
        z_perm = torch.from_numpy(z[perm_token])
        bounds = ep.partition(E, world)
        plan = ep.exchange_plan(offsets, bounds)
        z_recv = ep.dispatch_rows(z_perm, plan)

        # brute force over every rank's data
        everyone = [None] * world
        dist.all_gather_object(everyone, (z_perm.numpy(), offsets))
        lo, hi = bounds[rank], bounds[rank + 1]
        want = np.concatenate([zp[off[lo]:off[hi]] for zp, off in everyone])
        assert np.array_equal(z_recv.numpy(), want), "received rows"
        assert plan.n_recv == len(want)
        # the block offsets label each received row with its expert
        label = np.full(plan.n_recv, -1)
        bo = plan.recv_block_offsets
        for b in range(world):
            assert bo[b, 0] == sum(everyone[s][1][hi] - everyone[s][1][lo] for s in range(b))
            for e in range(hi - lo):
                label[bo[b, e]:bo[b, e + 1]] = lo + e
        want_label = np.concatenate([np.repeat(np.arange(lo, hi), np.diff(off[lo:hi + 1])) for _, off in everyone])
        assert np.array_equal(label, want_label), "expert of each received row"

        # stand-in experts: y = z * (expert + 1); the results return to their senders
        y_recv = z_recv * torch.from_numpy((label + 1).astype(np.float32))[:, None]
        y_back = ep.combine_rows(y_recv, plan)
        expert_of_pos = np.repeat(np.arange(E), counts)
        want_back = z_perm.numpy() * (expert_of_pos + 1).astype(np.float32)[:, None]
        assert np.array_equal(y_back.numpy(), want_back), "returned rows"
        # and the slot-ordered gather through inv_perm puts every result at its (token, slot)
        y_slots = y_back.numpy()[inv_perm].reshape(T, k, L)
        assert np.array_equal(y_slots, z[:, None, :] * (idx + 1).astype(np.float32)[:, :, None])
        out[rank] = (plan.n_recv, sum(plan.send_rows))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,E,k,mode", [(2, 13, 3, "zipf"), (2, 12, 4, "one_sided"), (3, 10, 2, "zipf")])
def test_gloo_dispatch_and_combine(world, E, k, mode):
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), E, k, mode, out), nprocs=world, join=True)
    # every row sent is received exactly once
    assert sum(v[0] for v in out.values()) == sum(v[1] for v in out.values())


def test_partition_and_plan_tables():
    assert ep.partition(896, 8).tolist() == [0, 112, 224, 336, 448, 560, 672, 784, 896]
    assert ep.partition(13, 2).tolist() == [0, 7, 13]
    with pytest.raises(ValueError):
        ep.partition(3, 4)
    offsets = np.array([0, 2, 2, 5, 9, 9, 10])  # 6 experts, rows 2, 0, 3, 4, 0, 1
    sent = ep.send_counts(offsets, ep.partition(6, 2))
    assert sent.tolist() == [[2, 0, 3], [4, 0, 1]]
    received = np.array([[5, 1, 0], [2, 2, 2]])  # from ranks 0 and 1, for this rank's 3 experts
    plan = ep.plan_from_counts(sent, received, 3)
    assert plan.send_rows == [5, 5] and plan.recv_rows == [6, 6] and plan.n_recv == 12
    assert plan.recv_block_offsets.tolist() == [[0, 5, 6, 6], [6, 8, 10, 12]]


# ------------------------------------------------------------------------------ balanced mode
def _row_destinations(plan, counts):
    """Brute force: the rank that runs each row, per sender, in the sender's
    expert-major order (global order of expert e's rows: senders in rank
    order)."""
    G, E = counts.shape
    dest = []
    for s in range(G):
        d = []
        for e in range(E):
            before = int(counts[:s, e].sum())
            for j in range(int(counts[s, e])):
                pos = before + j
                owners = [g for g, st, n in plan.segments[e] if st <= pos < st + n]
                assert len(owners) == 1, (s, e, j)
                d.append(owners[0])
        dest.append(np.array(d, np.int64))
    return dest


def _count_cases():
    rng = np.random.default_rng(11)
    cases = []
    for G, E in [(1, 5), (2, 13), (3, 10), (4, 9), (5, 23), (4, 4)]:
        w = (np.arange(E) + 1.0) ** -1.2
        cases.append((G, rng.multinomial(60 * G, w / w.sum(), size=G)))     # Zipf-skewed senders
        cases.append((G, rng.integers(0, 5, size=(G, E))))                    # small, with zeros
    hot = np.zeros((3, 7), np.int64)
    hot[:, 2] = [50, 40, 30]                                                  # one expert holds every row
    cases += [(3, hot), (4, np.zeros((4, 6), np.int64)), (4, np.eye(4, 6, dtype=np.int64))]  # no rows; R < G
    return cases


@pytest.mark.parametrize("case", range(len(_count_cases())))
def test_balanced_plan_invariants(case):
    """Every rank gets floor(R/G) or ceil(R/G) rows (the first R % G one
    more); each expert's rows are cut into consecutive segments, the owner's
    first; ranks other than the owner appear only as listed redundant copies;
    the brute-force destination of every row agrees."""
    G, counts = _count_cases()[case]
    E = counts.shape[1]
    bounds = ep.partition(E, G)
    plan = ep.balanced_plan(counts, bounds)
    C, R = counts.sum(axis=0), int(counts.sum())
    assert plan.quota.tolist() == [R // G + (1 if g < R % G else 0) for g in range(G)]
    load = np.zeros(G, np.int64)
    for e in range(E):
        owner = int(np.searchsorted(bounds, e, side="right") - 1)
        start = 0
        for i, (g, st, n) in enumerate(plan.segments[e]):
            assert st == start and n > 0
            start += n
            load[g] += n
            if g == owner:
                assert i == 0, "the owner's segment comes first"
            else:
                assert e in plan.replicas[g] and not bounds[g] <= e < bounds[g + 1]
        assert start == C[e]
    assert load.tolist() == plan.quota.tolist()
    for g in range(G):
        assert plan.replicas[g] == sorted(set(plan.replicas[g]))
        assert all(any(r == g for r, _, _ in plan.segments[e]) for e in plan.replicas[g])
    dest = _row_destinations(plan, counts)
    assert np.bincount(np.concatenate(dest + [np.zeros(0, np.int64)]), minlength=G).tolist() == plan.quota.tolist()
    # a rank already at its quota keeps all its rows and runs no copies
    home_load = np.array([C[bounds[g]:bounds[g + 1]].sum() for g in range(G)])
    for g in range(G):
        if home_load[g] == plan.quota[g]:
            assert not plan.replicas[g]


@pytest.mark.parametrize("case", range(len(_count_cases())))
def test_balanced_exchange_tables(case):
    """Each sender's send order is a permutation of its rows, grouped by
    destination in rank order and, within a destination, by the
    destination's local expert order; every receiver's blocks match what the
    senders send it."""
    G, counts = _count_cases()[case]
    E = counts.shape[1]
    bounds = ep.partition(E, G)
    plan = ep.balanced_plan(counts, bounds)
    dest = _row_destinations(plan, counts)
    ex = []
    for s in range(G):
        offsets = np.concatenate([[0], np.cumsum(counts[s])])
        x = ep.balanced_exchange(plan, counts, offsets, s)
        assert sorted(x.send_idx.tolist()) == list(range(int(counts[s].sum())))
        expert_of = np.repeat(np.arange(E), counts[s])
        d_of = dest[s][x.send_idx]
        assert np.all(np.diff(d_of) >= 0) and np.bincount(d_of, minlength=G).tolist() == x.send_rows
        for g in range(G):
            local = {int(e): i for i, e in enumerate(plan.local_experts(g))}
            sel = x.send_idx[d_of == g]
            li = np.array([local[int(e)] for e in expert_of[sel]], np.int64)
            assert np.all(np.diff(li) >= 0), "local expert order within a destination"
            assert np.all(np.diff(sel)[np.diff(li) == 0] == 1), "rows of one expert keep their order"
        ex.append(x)
    for g in range(G):
        assert ex[g].n_recv == plan.quota[g]
        for s in range(G):
            assert ex[g].recv_rows[s] == ex[s].send_rows[g]
            blk = ex[g].recv_block_offsets[s]
            assert blk[-1] - blk[0] == ex[s].send_rows[g]


def _balanced_worker(rank, world, port, E, k, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        T, L = 40 + 23 * rank, 6
        idx = _routing(rank, T, E, k, "zipf")
        z = np.random.default_rng(7 + rank).standard_normal((T, L)).astype(np.float32)
        counts_local, offsets, perm_token, inv_perm = oracle.permute(idx, E)
        z_perm = torch.from_numpy(z[perm_token])
        bounds = ep.partition(E, world)
        everyone = [None] * world
        dist.all_gather_object(everyone, (z_perm.numpy(), counts_local))
        counts = np.stack([c for _, c in everyone])
        lo, hi = bounds[rank], bounds[rank + 1]
        # stand-in weight slices: every element of expert e's slice is e
        home = {"Wg": torch.arange(lo, hi, dtype=torch.float32)[:, None, None].repeat(1, 2, 3),
                "So_tiled": (torch.arange(lo, hi, dtype=torch.int64)[:, None].repeat(1, 5) % 251).to(torch.uint8)}
        seen = {}

        def run_experts(z_recv, x, plan, copies, ids):
            # stand-in experts y = z * (e + 1), e the global id of each received row's expert
            local = plan.local_experts(rank)
            label = np.full(x.n_recv, -1)
            for s in range(world):
                b = x.recv_block_offsets[s]
                for i, e in enumerate(local):
                    label[b[i]:b[i + 1]] = e
            assert (label >= 0).all()
            reps = plan.replicas[rank]
            assert ids == reps, "without held copies every copy arrives"
            assert copies["Wg"].shape == (len(reps), 2, 3) and copies["So_tiled"].shape == (len(reps), 5)
            for i, e in enumerate(reps):
                assert torch.all(copies["Wg"][i] == e) and torch.all(copies["So_tiled"][i] == e % 251)
            seen["z_recv"], seen["reps"] = z_recv.clone(), len(reps)
            return z_recv * torch.from_numpy((label + 1).astype(np.float32))[:, None]

        # the layer's own step, with torch indexing for the gather the layer
        # runs as moe_gather_rows on the GPU
        y_perm, plan, x = ep.balanced_step(z_perm, offsets, bounds, home, run_experts,
                                           lambda src, i: src[i.long()])
        assert np.array_equal(plan.quota, ep.balanced_plan(counts, bounds).quota)
        assert x.n_recv == plan.quota[rank], "every rank runs its quota"
        # the received rows are exactly the rows the plan assigns here
        dest = _row_destinations(plan, counts)
        want = np.concatenate([everyone[s][0][np.nonzero(dest[s] == rank)[0]] for s in range(world)])
        assert np.array_equal(np.sort(seen["z_recv"].numpy(), axis=0), np.sort(want, axis=0)), "received rows"
        # the results are back in this rank's expert-major order
        expert_of_pos = np.repeat(np.arange(E), counts_local)
        assert np.array_equal(y_perm.numpy(), z_perm.numpy() * (expert_of_pos + 1).astype(np.float32)[:, None])
        out[rank] = (x.n_recv, seen["reps"])
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,E,k", [(2, 13, 3), (3, 10, 2), (4, 9, 3)])
def test_gloo_balanced_exchange(world, E, k):
    """The balanced exchange end to end on gloo ranks with Zipf-skewed
    routing: per-rank loads equal, rows and results travel correctly, and
    the redundant experts' weight slices arrive from their owners."""
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_balanced_worker, args=(world, _free_port(), E, k, out), nprocs=world, join=True)
    loads = [out[r][0] for r in range(world)]
    assert max(loads) - min(loads) <= 1
    assert sum(out[r][1] for r in range(world)) > 0, "the skew makes some rank run a redundant copy"


def test_expert_slots_place_copies_behind_own_experts():
    """The balanced layer's weight buffers: own slices first, the step's
    copies behind them in ascending id order, growing when a step needs more
    copies than fit; copies held from the previous step are reused (only
    new ones arrive), the own slices never change, and the local views are
    prefixes of the buffers."""
    def sl(ids):
        return {"Wg": torch.tensor(ids, dtype=torch.float32)[:, None, None].repeat(1, 2, 4),
                "So_tiled": (torch.tensor(ids, dtype=torch.int64)[:, None].repeat(1, 7) % 251).to(torch.uint8)}

    home = sl([0, 1, 2])
    slots = ep.ExpertSlots(home, capacity=1)
    assert slots.place(sl([]), [], []) == 3
    assert torch.equal(slots.local(3)["Wg"], home["Wg"])

    def check(replicas):
        loc = slots.local(3 + len(replicas))
        assert torch.equal(loc["Wg"][:3], home["Wg"]) and torch.equal(loc["So_tiled"][:3], home["So_tiled"])
        for i, e in enumerate(replicas):
            assert torch.all(loc["Wg"][3 + i] == e) and torch.all(loc["So_tiled"][3 + i] == e % 251)
        assert slots.held == replicas

    assert slots.place(sl([9, 40]), [9, 40], [9, 40]) == 5 and slots.capacity >= 2  # grown
    check([9, 40])
    assert slots.local(5)["Wg"].data_ptr() == slots.buf["Wg"].data_ptr()           # a view of the buffer
    # next step: 9 and 40 are held; only 17 and 300 arrive; the order is by id
    assert slots.place(sl([17, 300]), [17, 300], [9, 17, 40, 300]) == 7
    check([9, 17, 40, 300])
    # a step that drops copies and reuses one
    assert slots.place(sl([]), [], [40]) == 4
    check([40])
    with pytest.raises(ValueError):
        slots.place(sl([]), [], [40, 41])      # 41 neither held nor received
    slots.forget()
    assert slots.held == [] and slots.place(sl([5]), [5], [5]) == 4
    check([5])


def _no_copy_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        counts = np.array([[3, 1, 2, 2], [1, 3, 2, 2]])  # every rank already at its quota (8 rows)
        plan = ep.balanced_plan(counts, ep.partition(4, world))
        assert not any(plan.replicas)
        home = {"Wg": torch.zeros(2, 3)}
        copies = ep.exchange_replica_weights(plan, home)
        out[rank] = tuple(copies["Wg"].shape)
    finally:
        dist.destroy_process_group()


def test_no_copies_no_weight_exchange():
    """A plan without copies returns empty copy sets on every rank (the ranks
    skip the weight collectives together)."""
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_no_copy_worker, args=(2, _free_port(), out), nprocs=2, join=True)
    assert out[0] == out[1] == (0, 3)


# ------------------------------------------------------------------------------ the layer's own step on gloo
def _fake_library(layer, cfg, wd):
    """fp64 oracle stand-ins for the library entries the expert-parallel layer
    calls, with the library's argument lists, so that the layer's own step runs
    on CPU ranks.  The routed experts read the layer's own local weight set
    (its experts, then its redundant copies), which is what the test checks."""
    F64 = torch.float64
    rnd = oracle.storage_round(cfg.act)
    state = {}

    def router_topk(d, x, Wr, bias, scores, from_scores, idx, p, stream=None):
        s = oracle.router_scores(x.to(F64), wd["Wr"])
        i, pp, _ = oracle.select_experts(s, wd["bias"], d.k)
        scores.copy_(s)
        idx.copy_(i)
        p.copy_(pp)
        return 0

    def latent_shared(d, w, x, z, h_s, stream=None):
        xf = x.to(F64)
        z.copy_(rnd(xf @ wd["Wdown"].T))
        state["y_shared"] = oracle.shared_experts(xf, wd["Wsg"], wd["Wsv"], wd["Wso"], cfg.situ_c, rnd)
        return 0

    def permute(d, idx, z, offsets, perm_token, inv_perm, z_perm, ws, ws_bytes=None, stream=None):
        _, off, pt, ip = oracle.permute(idx.numpy().astype(np.int64), d.E)
        offsets.copy_(torch.from_numpy(off))
        perm_token.copy_(torch.from_numpy(pt))
        inv_perm.copy_(torch.from_numpy(ip))
        z_perm.copy_(z[torch.from_numpy(pt).long()])
        return 0

    def gather_rows(src, src_rows, row_bytes, idx, n, dst, stream=None):
        dst.copy_(src[idx.long()])
        return 0

    def expert_ffn_blocks(d, w, x_rows, n_rows, blocks, n_blocks, y_rows, ws, ws_bytes=None, stream=None):
        loc = layer._slots.local(d.E) if layer.balance else {n: layer.weights[n] for n in ("Wg", "Wv", "Wo")}
        b = blocks.numpy().reshape(n_blocks, d.E + 1)
        for s in range(n_blocks):
            for i in range(d.E):
                lo, hi = int(b[s, i]), int(b[s, i + 1])
                if lo < hi:
                    y_rows[lo:hi] = oracle.expert_forward(x_rows[lo:hi].to(F64), loc["Wg"][i].to(F64),
                                                          loc["Wv"][i].to(F64), loc["Wo"][i].to(F64), cfg.situ_c,
                                                          rnd).to(y_rows.dtype)
        return 0

    def combine(d, y_perm, inv_perm, p, gamma, u_out, n_out, stream=None):
        T, k = p.shape
        u = oracle.combine(y_perm.to(F64)[inv_perm.long()].reshape(T, k, -1), p.to(F64))
        n_out.copy_(rnd(oracle.rms_norm(u, wd["gamma"], cfg.rms_eps)))
        return 0

    def output(d, w, h_s, n, y, stream=None):
        y.copy_(state["y_shared"] + n.to(F64) @ wd["Wup"].T)
        return 0

    return {"moe_router_topk": router_topk, "moe_latent_shared": latent_shared, "moe_permute": permute,
            "moe_gather_rows": gather_rows, "moe_expert_ffn_blocks": expert_ffn_blocks, "moe_combine": combine,
            "moe_output": output}


def _layer_worker(rank, world, port, balance, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import gen
        from oracle import inputs as oin
        from sparse_moe_layer_renormalised_b200 import Dims

        T_r = 24
        cfg = gen.CONFIGS["tiny"].with_(T=2 * T_r * world)
        wd = oin.all_weights(cfg)                       # fp64, the generator's fp32 values
        bounds = ep.partition(cfg.E, world)
        lo, hi = int(bounds[rank]), int(bounds[rank + 1])
        w = {n: wd[n].to(torch.float32) for n in ("Wr", "bias", "Wdown", "Wup", "gamma", "Wsg", "Wsv", "Wso")}
        w.update({n: wd[n][lo:hi].to(torch.float32).contiguous() for n in ("Wg", "Wv", "Wo")})
        dims = Dims(T=T_r, H=cfg.H, L=cfg.L, E=cfg.E, k=cfg.k, I=cfg.I, S=cfg.S, Is=cfg.Is, act="f32", routed="f32",
                    y_out="f32", situ_c=cfg.situ_c, rms_eps=cfg.rms_eps)
        layer = ep.ExpertParallelMoeLayer(dims, w, balance=balance)
        for name, f in _fake_library(layer, cfg, wd).items():
            setattr(ep, name, f)
        sent = []  # the copies requested from their owners, per step
        orig = ep.exchange_expert_slices

        def recorded(want, *a, **kw):
            sent.append([list(v) for v in want])
            return orig(want, *a, **kw)

        ep.exchange_expert_slices = recorded
        # three steps: a batch, the same batch again (its copies are all held),
        # then another batch (only the copies not held travel)
        errs, copies = [], []
        for b in (0, 0, 1):
            x = oin.x_rows(cfg, np.arange((b * world + rank) * T_r, (b * world + rank + 1) * T_r))
            y = layer(x.to(torch.float32))
            ref = oracle.layer_forward(cfg, wd, x)["y"]
            errs.append(float((y.to(torch.float64) - ref).abs().max() / ref.pow(2).mean().sqrt()))
            copies.append(len(layer.last_plan.replicas[rank]) if balance else 0)
        if balance:
            assert not any(sent[1]), "a repeated plan sends no weights"
            assert all(set(sent[2][g]) <= set(layer.last_plan.replicas[g]) for g in range(world))
        out[rank] = (max(errs), sum(copies))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,balance", [(1, True), (2, True), (3, True), (3, False)])
def test_gloo_layer_step_matches_the_oracle(world, balance):
    """The expert-parallel layer's own forward step on gloo ranks, each with
    its own tokens and only its own experts' weights, the library entries
    replaced by fp64 oracle stand-ins: every rank's y equals the oracle layer
    on its tokens (fp32 storage between the steps), in the balanced mode with
    redundant copies whose weights came from other ranks."""
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_layer_worker, args=(world, _free_port(), balance, out), nprocs=world, join=True)
    for r in range(world):
        assert out[r][0] <= 1e-5, (r, out[r])
    if balance and world > 1:
        assert sum(out[r][1] for r in range(world)) > 0, "some rank ran a redundant copy"


def test_balanced_plan_at_k3_scale():
    """8 ranks, 896 experts, 2^19 rows with a Zipf-skewed load (the prefill
    mix): exact quotas, each expert's rows tiled by its segments, few copies,
    and a plan computed in well under a second."""
    import time

    rng = np.random.default_rng(17)
    G, E = 8, 896
    w = (np.arange(E) + 1.0) ** -0.8
    rng.shuffle(w)
    counts = rng.multinomial(2 ** 16, w / w.sum(), size=G).astype(np.int64)
    bounds = ep.partition(E, G)
    t0 = time.perf_counter()
    plan = ep.balanced_plan(counts, bounds)
    dt = time.perf_counter() - t0
    R = int(counts.sum())
    assert plan.quota.tolist() == [R // G] * G
    load = np.zeros(G, np.int64)
    C = counts.sum(axis=0)
    for e in range(E):
        assert sum(n for _, _, n in plan.segments[e]) == C[e]
        for g, _, n in plan.segments[e]:
            load[g] += n
    assert load.tolist() == plan.quota.tolist()
    assert sum(len(r) for r in plan.replicas) <= 2 * G
    assert dt < 1.0, dt
