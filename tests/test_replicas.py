"""The multi-GPU path is independent replicas: checked with world_size-2 gloo process groups on
the CPU (each rank runs the oracle on its own batch; timings reduce to the max over ranks)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from fp8_moe_layer_b200 import replicas


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    from fp8_moe_layer_b200 import inputs as I
    from oracle import moe_oracle as O
    r, w, lr = replicas.rank_env()
    assert (r, w, lr) == (rank, world, rank)
    shape = I.MoEShape("replica", 12, 64, 4, 32, 2, 2)
    inp = I.make_inputs(shape, seed=replicas.replica_seed(100, rank))
    out = O.moe_forward(inp.hidden.view(torch.int16).numpy().view(np.uint16),
                        inp.router_w.numpy(), None, shape.k, None, inp.w13.numpy(),
                        inp.w13_scale.numpy(), inp.w2.numpy(), inp.w2_scale.numpy())
    np.save(os.path.join(out_dir, f"y{rank}.npy"), out["y64"])
    # pretend timings: rank r took (r + 1) ms; the reduction must return the slowest
    got = replicas.max_over_ranks([rank + 1.0, 10.0 - rank])
    assert got == [float(world), 10.0]
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_replicas(tmp_path):
    world = 2
    mp.spawn(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    y0, y1 = np.load(tmp_path / "y0.npy"), np.load(tmp_path / "y1.npy")
    assert y0.shape == y1.shape and not np.array_equal(y0, y1)   # independent batches


def test_single_process_and_throughput():
    assert replicas.max_over_ranks([1.5, 2.5]) == [1.5, 2.5]
    assert replicas.aggregate_tokens_per_s(512, 4, 2.0) == pytest.approx(512 * 4 / 2e-3)
    assert replicas.replica_seed(7, 3) == 10
