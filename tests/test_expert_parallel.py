"""Expert parallelism on CPU ranks (gloo): the dispatch and combine index
arithmetic against brute force, and whole expert-parallel forwards -- each
rank holding only its share of the routed experts, the oracle as each rank's
expert compute -- against the single-process oracle."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from sparse_moe_transformer_router_b200 import expert_parallel as ep


def test_dispatch_plan_is_a_stable_bijection_grouped_by_destination():
    rng = np.random.default_rng(0)
    for _ in range(200):
        G = int(rng.choice([1, 2, 4, 8]))
        E = G * int(rng.integers(1, 9))
        T, k = int(rng.integers(0, 60)), int(rng.integers(1, min(4, E) + 1))
        idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]) if T else np.zeros((0, k), np.int64)
        plan = ep.plan_dispatch(idx, E, G)
        flat = idx.reshape(-1)
        assert sorted(plan.order.tolist()) == list(range(T * k))          # bijection
        assert plan.send_counts.sum() == T * k
        # brute force: entries sorted by (destination, expert, entry number)
        ref = sorted(range(T * k), key=lambda n: (flat[n] // (E // G), flat[n], n))
        assert plan.order.tolist() == ref
        # the entries of destination q are the q-th consecutive run of the order
        starts = np.concatenate([[0], np.cumsum(plan.send_counts)])
        for q in range(G):
            run = plan.order[starts[q]:starts[q + 1]]
            assert np.all(flat[run] // (E // G) == q)


def test_local_groups_order_received_entries_by_expert_then_source():
    rng = np.random.default_rng(1)
    for _ in range(200):
        G, n_local = int(rng.integers(1, 5)), int(rng.integers(1, 6))
        first = int(rng.integers(0, 3)) * n_local
        recv_counts = rng.integers(0, 7, size=G)
        recv_e = np.concatenate([np.sort(rng.integers(first, first + n_local, size=c)) for c in recv_counts]) \
            if recv_counts.sum() else np.zeros(0, np.int64)
        src = np.repeat(np.arange(G), recv_counts)
        lg = ep.local_groups(recv_e, recv_counts, first, n_local)
        ref = sorted(range(recv_e.size), key=lambda i: (recv_e[i], src[i], i))
        assert lg.order.tolist() == ref
        assert lg.counts.sum() == recv_e.size
        assert lg.counts.tolist() == np.bincount(recv_e - first, minlength=n_local).tolist()


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, k, result):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), OMP_NUM_THREADS="1")
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        from sparse_moe_transformer_router_b200.workloads import LayerConfig, generate, to_storage_numpy
        E = 8
        cfg = LayerConfig("ep", 24 + 7 * rank, 64, E, 64, 128, "bf16", wr_std=0.2)
        layer = generate(cfg, seed=0, device="cpu")                  # the same weights on every rank
        x_mine = to_storage_numpy(generate(cfg, seed=100 + rank, device="cpu").x)  # this rank's tokens
        Wr = to_storage_numpy(layer.W_router)
        Ws_gu, Ws_dn = to_storage_numpy(layer.Ws_gate_up), to_storage_numpy(layer.Ws_down)
        mine = set(ep.experts_of_rank(E, world, rank))
        W_gu = {e: to_storage_numpy(layer.W_gate_up[e]) for e in mine}  # only this rank's experts
        W_dn = {e: to_storage_numpy(layer.W_down[e]) for e in mine}

        def route(x):
            xs = x.numpy().view(np.uint16)
            if k == 1:
                idx, lmax, _ = oracle.route(xs, Wr)
                return idx, 1.0 / (1.0 + np.exp(-lmax.astype(np.float64)))
            idx, lsel, _ = oracle.route_topk(xs, Wr, k)
            return idx, 1.0 / (1.0 + np.exp(-lsel.astype(np.float64)))

        def expert(e, rows, gates):
            assert e in mine
            return oracle.expert_rows(rows.numpy().view(np.uint16), gates, W_gu[e], W_dn[e])

        def shared(x):
            return oracle.forward(x.numpy().view(np.uint16), np.zeros((cfg.d_model, 0), np.uint16), [], [],
                                  Ws_gu, Ws_dn)[0]

        x_t = torch.from_numpy(x_mine.view(np.int16).copy())
        out = ep.ep_forward(x_t, route, expert, shared, E, k=k).numpy()
        full = [to_storage_numpy(w) for w in layer.W_gate_up], [to_storage_numpy(w) for w in layer.W_down]
        ref = oracle.forward(x_mine, Wr, full[0], full[1], Ws_gu, Ws_dn, k=k)[0]
        err = float(np.max(np.abs(out - ref)) / np.sqrt(np.mean(ref ** 2)))
        # every routed entry was computed exactly once, somewhere
        idx, _ = route(x_t)
        n = torch.tensor([np.asarray(idx).size], dtype=torch.int64)
        dist.all_reduce(n)
        result[rank] = (err, int(n.item()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,k", [(2, 1), (4, 1), (2, 2)])
def test_expert_parallel_forward_equals_the_single_process_oracle(world, k):
    with mp.Manager() as m:
        result = m.dict()
        mp.spawn(_rank, args=(world, _free_port(), k, result), nprocs=world, join=True)
        res = dict(result)
    assert len(res) == world
    for rank, (err, n) in res.items():
        assert err < 1e-12, (rank, err)       # fp64 on both sides: only the order of the final sum differs
        assert n == sum(24 + 7 * r for r in range(world)) * k
