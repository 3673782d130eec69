"""Expert-parallel exchange plan (host logic) on CPU.

The plan must place every kept dispatch exactly where the single-GPU layer on
the ranks' batches laid end to end would group it ("Mixture of Experts MoE:
how sparse activation saves compute" §3.5, §3.6, §3.8), which the oracle's
permutation of the concatenated batch fixes.  A gloo run then moves real
token rows with all-to-all by the plan, evaluates the experts on their owners
with the oracle, sends the results back, combines them, and must reproduce
the oracle's single-GPU layer output bit for bit.
"""
import os
import socket

import numpy as np
import pytest

import oracle as O
from sparse_mixture_experts_15_b200 import ep


def test_hand_worked_plan():
    """Two ranks, four experts (0, 1 on rank 0; 2, 3 on rank 1), capacity 3.
    Expert 0: rank 0 fills all 3 slots, rank 1's one dispatch drops; expert 1:
    rank 1 keeps 3 of 4; expert 3: rank 0 keeps 1, rank 1 keeps the last 2."""
    counts = [[3, 0, 2, 1], [1, 4, 0, 2]]
    p0, p1 = ep.plan(counts, 3, 0), ep.plan(counts, 3, 1)
    assert p0.kept.tolist() == [3, 0, 2, 1] and p1.kept.tolist() == [0, 3, 0, 2]
    assert p0.local_offsets.tolist() == [0, 3, 3, 5, 6]
    assert p0.send_base.tolist() == [0, 3, 0, 2]
    assert p1.send_base.tolist() == [3, 3, 2, 3]
    assert p0.send_counts.tolist() == [3, 3] and p1.send_counts.tolist() == [3, 2]
    assert p0.recv_offsets.tolist() == [0, 3, 6] and p1.recv_offsets.tolist() == [0, 2, 5]
    assert p0.recv_src_base.tolist() == [[0, 3], [3, 3]]
    assert p1.recv_src_base.tolist() == [[0, 2], [2, 3]]
    assert p0.recv_counts.tolist() == [3, 3] and p1.recv_counts.tolist() == [3, 2]
    assert p0.overflow.tolist() == [1, 1, 0, 0]


def test_plan_rejects_bad_input():
    with pytest.raises(ValueError):
        ep.plan([[1, 2, 3], [1, 1, 1]], 0, 0)  # 3 experts over 2 ranks
    with pytest.raises(ValueError):
        ep.plan([[1, 2], [1, 1]], -1, 0)
    with pytest.raises(ValueError):
        ep.plan([[1, 2], [1, 1]], 0, 2)


def _routing(seed, T, N, k):
    rng = np.random.default_rng(seed)
    z = rng.standard_normal((T, N)) + np.linspace(1.0, 0.0, N)[None, :]
    return np.argsort(-z, axis=1, kind="stable")[:, :k].astype(np.int32)


def _local_rank_in_expert(idx, N):
    """j of each dispatch: its index among this rank's dispatches to the same
    expert, in token order (the grouping of a capacity-0 permutation)."""
    p = O.permute(idx, N, 0)
    return p["row_of"] - p["offsets"][idx], p


@pytest.mark.parametrize("R,N,k,C", [(1, 8, 2, 5), (2, 8, 2, 0), (2, 8, 2, 9), (4, 16, 3, 7),
                                     (4, 8, 1, 2), (3, 6, 2, 4)])
def test_plan_matches_global_permutation(R, N, k, C):
    Ts = [37, 50, 1, 64][:R]
    idxs = [_routing(100 * R + r, Ts[r], N, k) for r in range(R)]
    counts = np.stack([np.bincount(i.ravel(), minlength=N) for i in idxs])
    glob = O.permute(np.concatenate(idxs), N, C)
    E = N // R
    t0 = 0
    seen = {o: [] for o in range(R)}
    for r in range(R):
        p = ep.plan(counts, C, r)
        j, _ = _local_rank_in_expert(idxs[r], N)
        for t in range(Ts[r]):
            for s in range(k):
                e = int(idxs[r][t, s])
                o = p.owner(e)
                assert o == ep.owner_of(e, N, R)
                g = int(glob["row_of"][t0 + t, s])
                if j[t, s] < p.kept[e]:
                    pos = int(p.send_base[e] + j[t, s])
                    assert g - int(glob["offsets"][o * E]) == pos
                    seen[o].append(pos)
                else:
                    assert g == -1
        t0 += Ts[r]
    for o in range(R):
        po = ep.plan(counts, C, o)
        assert sorted(seen[o]) == list(range(po.recv_rows))  # the buffer is tiled exactly
        assert po.recv_rows == int(glob["offsets"][(o + 1) * E] - glob["offsets"][o * E])
    assert np.array_equal(ep.plan(counts, C, 0).overflow, glob["overflow"])
    # send and receive sizes agree pairwise
    plans = [ep.plan(counts, C, r) for r in range(R)]
    for a in range(R):
        for b in range(R):
            assert plans[a].send_counts[b] == plans[b].recv_counts[a]


# ------------------------------------------------------------- gloo data flow
def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


D, H, NE, K, CAP = 16, 24, 6, 2, 9


def _experts():
    rng = np.random.default_rng(7)
    mk = lambda rows, cols: O.Mat(O.F64, rows, cols, data=rng.normal(0, 0.3, (rows, cols)))  # noqa
    return [(mk(H, D), mk(H, D), mk(D, H)) for _ in range(NE)]


def _batch(r):
    rng = np.random.default_rng(50 + r)
    T = [21, 30, 17][r]
    u = rng.normal(0, 1.0, (T, D))
    idx = _routing(300 + r, T, NE, K)
    w = rng.random((T, K))
    return u, idx, w / w.sum(1, keepdims=True)


def _ep_worker(rank, world, port, q):
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mats = _experts()
        u, idx, w = _batch(rank)
        T = u.shape[0]
        j, _ = _local_rank_in_expert(idx, NE)
        counts_all = ep.exchange_counts(np.bincount(idx.ravel(), minlength=NE))
        p = ep.plan(counts_all, CAP, rank)
        kept_all = np.stack([ep.plan(counts_all, CAP, r).kept for r in range(world)])
        E = p.experts_per_rank
        # dispatch: my kept rows in my grouped layout (experts in order, so the
        # rows for one owner form one chunk)
        send = np.zeros((int(p.kept.sum()), D))
        slot_of = {}
        for t in range(T):
            for s in range(K):
                e = int(idx[t, s])
                if j[t, s] < p.kept[e]:
                    row = int(p.local_offsets[e] + j[t, s])
                    send[row] = u[t]
                    slot_of[(t, s)] = row
        recv = torch.empty((p.recv_rows, D), dtype=torch.float64)
        dist.all_to_all_single(recv, torch.from_numpy(send), p.recv_counts.tolist(),
                               p.send_counts.tolist())
        recv = recv.numpy()
        # source r's chunk holds its kept rows for my experts in expert order;
        # each lands at recv_src_base in my expert-major buffer
        out = np.zeros((p.recv_rows, D))
        chunk = 0
        for r in range(world):
            for el in range(E):
                e = rank * E + el
                base = int(p.recv_src_base[el, r])
                for i in range(int(kept_all[r, e])):
                    out[base + i] = O.expert(*mats[e], recv[chunk + i])
                chunk += int(kept_all[r, e])
        # combine route: the results go back source-major
        back_send = np.zeros((p.recv_rows, D))
        chunk = 0
        for r in range(world):
            for el in range(E):
                n, base = int(kept_all[r, rank * E + el]), int(p.recv_src_base[el, r])
                back_send[chunk:chunk + n] = out[base:base + n]
                chunk += n
        back = torch.empty((int(p.kept.sum()), D), dtype=torch.float64)
        dist.all_to_all_single(back, torch.from_numpy(back_send), p.send_counts.tolist(),
                               p.recv_counts.tolist())
        rows = back.numpy()
        y = np.zeros((T, D))
        for t in range(T):
            for s in range(K):
                if (t, s) in slot_of:
                    y[t] += w[t, s] * rows[slot_of[(t, s)]]
        q.put((rank, y))
    finally:
        dist.barrier()
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_gloo_ranks_reproduce_the_single_gpu_layer(world):
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ep_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # the single-GPU layer on the batches laid end to end
    mats = _experts()
    batches = [_batch(r) for r in range(world)]
    u = np.concatenate([b[0] for b in batches])
    idx = np.concatenate([b[1] for b in batches])
    w = np.concatenate([b[2] for b in batches])
    perm = O.permute(idx, NE, CAP)
    assert perm["totals"][1] > 0, "the case should drop some dispatches"
    ref = O.moe_tokens([m[0] for m in mats], [m[1] for m in mats], [m[2] for m in mats], u, idx,
                       w, row_of=perm["row_of"])
    t0 = 0
    for r in range(world):
        T = batches[r][0].shape[0]
        assert np.array_equal(got[r], ref[t0:t0 + T]), f"rank {r}"
        t0 += T


def test_plan_invariants_on_random_counts():
    """For random per-rank counts and capacities: every owner's receive
    buffer is tiled exactly by the sources' kept rows, send and receive sizes
    agree pairwise, each expert keeps min(C, all dispatches) rows (all of them
    for C = 0), and a rank keeps rows for an expert only while the ranks
    before it left room."""
    from hypothesis import given, settings, strategies as st

    @settings(max_examples=200, deadline=None)
    @given(st.integers(1, 4), st.integers(1, 4), st.integers(0, 12), st.data())
    def check(R, E, C, data):
        N = R * E
        counts = np.array(data.draw(st.lists(st.lists(st.integers(0, 9), min_size=N, max_size=N),
                                             min_size=R, max_size=R)))
        plans = [ep.plan(counts, C, r) for r in range(R)]
        kept = np.stack([p.kept for p in plans])
        tot = counts.sum(0)
        assert np.array_equal(kept.sum(0), np.minimum(tot, C) if C else tot)
        assert np.array_equal(plans[0].overflow, tot - kept.sum(0))
        for r in range(1, R):  # a later rank keeps rows only if the earlier ranks kept all theirs
            later = kept[r] > 0
            assert np.array_equal(kept[:r, later], counts[:r, later])
        for a in range(R):
            for b in range(R):
                assert plans[a].send_counts[b] == plans[b].recv_counts[a]
        for o in range(R):
            cover = []
            for r in range(R):
                for e in range(o * E, (o + 1) * E):
                    cover += list(range(plans[r].send_base[e], plans[r].send_base[e] + kept[r, e]))
                    el = e - o * E
                    assert plans[o].recv_src_base[el, r] == plans[r].send_base[e]
            assert sorted(cover) == list(range(plans[o].recv_rows))
            assert plans[o].recv_rows == int(plans[o].recv_counts.sum())

    check()
