"""The data-parallel path (N > 1) on CPU: two gloo ranks, gradient averaging, identical
updates on every rank, max-over-ranks timing, and a rank failure seen by the other rank."""
import os
import socket
import tempfile

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import model as om


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, outdir):
    import numpy as np
    from layer_streamed_nf4_lut_b200 import dp
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    torch.manual_seed(0)
    params = torch.randn(1000, dtype=torch.float64)
    m = torch.zeros_like(params)
    v = torch.zeros_like(params)
    grads = torch.zeros_like(params)
    rng = np.random.default_rng(100 + rank)
    local_g = torch.from_numpy(rng.standard_normal(1000))

    def fwd_bwd():
        grads.copy_(local_g)
        return float(rank + 1)

    def update():
        p, mm, vv = om.adamw(params.numpy(), grads.numpy(), m.numpy(), v.numpy(), 1, 1e-3)
        params.copy_(torch.from_numpy(p))

    loss, mean_loss = dp.dp_step(fwd_bwd, grads, update)
    slow = dp.max_over_ranks(0.5 + rank)
    torch.save(dict(params=params, grads=grads, mean_loss=mean_loss, slow=slow), os.path.join(outdir, f"r{rank}.pt"))
    dist.barrier()
    dist.destroy_process_group()


def test_dp_two_ranks_gloo():
    import numpy as np
    with tempfile.TemporaryDirectory() as d:
        mp.spawn(_worker, args=(2, _free_port(), d), nprocs=2, join=True)
        r0, r1 = torch.load(os.path.join(d, "r0.pt")), torch.load(os.path.join(d, "r1.pt"))
    g_mean = (np.random.default_rng(100).standard_normal(1000) + np.random.default_rng(101).standard_normal(1000)) / 2
    assert torch.allclose(r0["grads"], torch.from_numpy(g_mean), atol=1e-14)
    assert torch.equal(r0["params"], r1["params"])  # replicas stay identical
    assert r0["mean_loss"] == 1.5 and r1["slow"] == 1.5


def _failing_worker(rank, world, port, outdir):
    import datetime
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=3))
    if rank == 1:
        raise SystemExit(0)  # leaves between steps, before the collective
    t = torch.ones(4)
    try:
        dist.all_reduce(t)
        status = "no error"
    except Exception as ex:  # the short process-group timeout / closed peer ends the collective
        status = "error: " + type(ex).__name__
    open(os.path.join(outdir, "r0.txt"), "w").write(status)


def test_dp_rank_leaving_is_reported():
    with tempfile.TemporaryDirectory() as d:
        ctx = mp.start_processes(_failing_worker, args=(2, _free_port(), d), nprocs=2, join=False,
                                 start_method="spawn")
        for p in ctx.processes:
            p.join(60)
        status = open(os.path.join(d, "r0.txt")).read()
    assert status.startswith("error"), status
