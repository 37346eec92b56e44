"""Expert parallelism on the CPU: the send-plan construction the GPU tests compare the dispatch
kernel with, and the all-to-all orchestration of ExpertParallelRank.forward over real gloo process
groups (world sizes 2 and 4), with the experts' arithmetic replaced by a checkable stand-in."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from tests import helpers as H


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _routing(T, E, k_max, seed, elastic=False):
    rng = np.random.default_rng(seed)
    k_t = rng.integers(1, k_max + 1, size=T) if elastic else np.full(T, k_max)
    ids = np.full((T, k_max), -1, dtype=np.int32)
    w = np.zeros((T, k_max), dtype=np.float32)
    for t in range(T):
        ids[t, :k_t[t]] = rng.choice(E, size=k_t[t], replace=False)
        p = rng.random(k_t[t]).astype(np.float32) + 0.1
        w[t, :k_t[t]] = p / p.sum()
    return ids, w, k_t


@pytest.mark.parametrize("T,E,k_max,n,elastic", [(30, 16, 4, 4, False), (25, 8, 2, 8, False),
                                                 (40, 64, 8, 2, True), (12, 4, 4, 1, False)])
def test_send_plan_reconstructs_the_routing(T, E, k_max, n, elastic):
    ids, w, k_t = _routing(T, E, k_max, seed=T + E, elastic=elastic)
    ref = H.ep_dispatch_reference(ids, w, k_t, E, n)
    El = E // n
    assert ref["counts"].sum() == len(ref["tokens"])
    # segments are rank-major, tokens ascending inside each
    start = np.concatenate([[0], np.cumsum(ref["counts"])])
    for r in range(n):
        seg = ref["tokens"][start[r]:start[r + 1]]
        assert np.all(np.diff(seg) > 0)
    # every (token, expert, weight) appears exactly once, on the rank that holds the expert
    for t in range(T):
        got = {}
        for r in range(n):
            row = ref["slot_of"][t, r]
            if row < 0:
                assert not any(r * El <= e < (r + 1) * El for e in ids[t, :k_t[t]])
                continue
            assert start[r] <= row < start[r + 1] and ref["tokens"][row] == t
            for q in range(ref["kl"]):
                e = ref["send_ids"][row, q]
                if e >= 0:
                    got[r * El + int(e)] = float(ref["send_w"][row, q])
        want = {int(e): float(x) for e, x in zip(ids[t, :k_t[t]], w[t, :k_t[t]])}
        assert got == want
        # slot order is kept inside a rank
        for r in range(n):
            row = ref["slot_of"][t, r]
            if row >= 0:
                loc = [int(e) for e in ref["send_ids"][row] if e >= 0]
                glob = [int(e) - r * El for e in ids[t, :k_t[t]] if r * El <= e < (r + 1) * El]
                assert loc == glob


# ------------------------------------------------------------------ orchestration over gloo
def _stand_in_rank(EP, rank, n, E, k_max, d):
    """An ExpertParallelRank whose three compute steps are CPU stand-ins: dispatch builds the send
    rows from the reference plan, expert e multiplies a row by (e + 1), the shared expert by 0.5."""

    class StandIn(EP.ExpertParallelRank):
        def dispatch(self, hidden, k_per_token=None):
            ids, w, k_t = self.routing
            ref = H.ep_dispatch_reference(ids, w, k_t, self.E, self.n_ranks)
            return EP.Dispatched(hidden.shape[0], hidden[ref["tokens"]].contiguous(),
                                 torch.from_numpy(ref["send_ids"]),
                                 torch.from_numpy(ref["send_w"]),
                                 [int(c) for c in ref["counts"]],
                                 torch.from_numpy(ref["slot_of"]),
                                 torch.from_numpy(ref["slot_w"]), 0.5 * hidden)

        def experts(self, recv_hidden, recv_ids, recv_w):
            out = torch.zeros_like(recv_hidden)
            for q in range(recv_ids.shape[1]):
                e = recv_ids[:, q].to(torch.float64)
                mult = torch.where(e >= 0, self.rank * self.E_local + e + 1.0, 0.0)
                out += (recv_w[:, q].to(torch.float64) * mult)[:, None] * recv_hidden
            return out

        def combine(self, disp, returned):
            y = disp.shared_out.clone()
            for r in range(self.n_ranks):
                rows = disp.slot_of[:, r].long()
                m = rows >= 0
                y[m] += disp.slot_w[m, r].to(torch.float64)[:, None] * returned[rows[m]]
            return y

    El = E // n
    z = torch.zeros
    return StandIn(rank, n, z(E, d), None, k_max, k_max, z(El, 32, d, dtype=torch.uint8),
                   z(El, 32), z(El, d, 16, dtype=torch.uint8), z(El, d))


def _worker(rank, n, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=n, timeout=datetime.timedelta(seconds=60))
    from fp8_moe_layer_b200 import expert_parallel as EP
    ex = EP.TorchDistExchange()
    assert ex.n_ranks == n and ex.device.type == "cpu"

    # raw exchange: rank r sends (r + i) % 3 rows to rank i (some segments empty), three dtypes
    send = [(rank + i) % 3 for i in range(n)]
    recv = ex.counts(send)
    assert recv == [(s + rank) % 3 for s in range(n)]
    for dt in (torch.bfloat16, torch.int32, torch.float32):
        x = torch.cat([torch.full((send[i], 5), 100 * rank + i).to(dt) for i in range(n)])
        y = ex.rows(x, send, recv)
        want = torch.cat([torch.full((recv[s], 5), 100 * s + rank).to(dt) for s in range(n)])
        assert y.dtype == dt and torch.equal(y, want)
        back = ex.rows(y, recv, send)
        assert torch.equal(back, x)

    # the layer's forward with stand-in arithmetic: y = (0.5 + sum_j w_j (e_j + 1)) x
    E, k_max, d = 8 * n, 4, 24
    T = 0 if (n == 4 and rank == 2) else 10 + 7 * rank        # one rank with an empty batch
    layer = _stand_in_rank(EP, rank, n, E, k_max, d)
    ids, w, k_t = _routing(T, E, k_max, seed=1000 + rank, elastic=True)
    layer.routing = (ids, w, k_t)
    x = torch.from_numpy(np.random.default_rng(rank).standard_normal((T, d)))
    y = layer.forward(x, ex)
    coef = 0.5 + np.array([sum(float(w[t, j]) * (int(ids[t, j]) + 1) for j in range(k_t[t]))
                           for t in range(T)])
    np.testing.assert_allclose(y.numpy(), coef[:, None] * x.numpy(), rtol=1e-6, atol=1e-12)
    dist.barrier()
    dist.destroy_process_group()
    open(os.path.join(out_dir, f"ok{rank}"), "w").close()


@pytest.fixture(scope="module")
def built():
    from fp8_moe_layer_b200 import build
    build.build()


@pytest.mark.parametrize("n", [2, 4])
def test_forward_orchestration_over_gloo(built, tmp_path, n):
    mp.start_processes(_worker, args=(n, _free_port(), str(tmp_path)), nprocs=n,
                       start_method="spawn")
    assert sorted(os.listdir(tmp_path)) == [f"ok{r}" for r in range(n)]


@pytest.mark.parametrize("n,Ts", [(3, (9, 0, 14)), (1, (6,)), (5, (1, 2, 3, 4, 5))])
def test_loopback_exchange_with_stand_in_ranks(built, n, Ts):
    """loopback_forward's segment bookkeeping (who receives which rows, where the partial sums go
    back) on the CPU, with the same stand-in arithmetic as the gloo test."""
    from fp8_moe_layer_b200 import expert_parallel as EP
    E, k_max, d = 4 * n, 3, 8
    ranks, xs, want = [], [], []
    for r, T in enumerate(Ts):
        layer = _stand_in_rank(EP, r, n, E, k_max, d)
        ids, w, k_t = _routing(T, E, k_max, seed=50 + r, elastic=True)
        layer.routing = (ids, w, k_t)
        x = torch.from_numpy(np.random.default_rng(7 + r).standard_normal((T, d)))
        coef = 0.5 + np.array([sum(float(w[t, j]) * (int(ids[t, j]) + 1) for j in range(k_t[t]))
                               for t in range(T)])
        ranks.append(layer)
        xs.append(x)
        want.append(coef[:, None] * x.numpy())
    ys = EP.loopback_forward(ranks, xs)
    for y, wnt in zip(ys, want):
        np.testing.assert_allclose(y.numpy(), wnt, rtol=1e-6, atol=1e-12)
