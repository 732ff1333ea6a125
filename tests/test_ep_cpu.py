"""The expert-parallel exchange (dispatch and combine of token rows between
the ranks that hold the experts) on CPU: gloo ranks, world size 2 and 3.

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
