"""The multi-rank logic on CPU with gloo, world size 2.

bench.py runs one independent batch per rank (weak scaling) and takes the
max of the per-rank step time over the process group.  These tests run that
reduction and the per-rank seeding as two gloo processes, and check the
data-parallel identity a training step would rely on: summing per-rank loss
numerators, counts and dW over ranks reproduces the unsharded oracle.
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import oracle
        from ckl_synth import make_inputs

        # max over ranks of a per-rank time
        t = bench.max_over_ranks(10.0 + rank, world)
        # per-rank seeds differ, so each rank draws its own batch
        seed = bench.rank_seed(0, rank)
        # data-parallel shard of one global batch: rows split between ranks
        c = make_inputs(40, 16, 60, 5, seed=5, w_std=0.4, mask=("bernoulli", 0.2))
        lo, hi = rank * 20, (rank + 1) * 20
        part = oracle.dense(c["H"][lo:hi], c["W"], c["idx"][lo:hi], c["logp"][lo:hi],
                            c["mask"][lo:hi], g=1.0)
        n_local = torch.tensor([float(part["N"])], dtype=torch.float64)
        num = torch.tensor([part["loss"] * part["N"]], dtype=torch.float64)
        dist.all_reduce(n_local)
        dist.all_reduce(num)
        # the local backward scale is g/N_local; re-weight to the global N
        dw = torch.from_numpy(part["dW"] * part["N"])
        dist.all_reduce(dw)
        np.savez(os.path.join(out_dir, f"r{rank}.npz"), t=t, seed=seed,
                 loss=(num / n_local).item(), dw=(dw / n_local).numpy())
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    world = 2
    mp.spawn(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    r = [np.load(tmp_path / f"r{i}.npz") for i in range(world)]
    assert float(r[0]["t"]) == float(r[1]["t"]) == 11.0
    assert int(r[0]["seed"]) != int(r[1]["seed"])

    import oracle
    from ckl_synth import make_inputs
    c = make_inputs(40, 16, 60, 5, seed=5, w_std=0.4, mask=("bernoulli", 0.2))
    full = oracle.dense(c["H"], c["W"], c["idx"], c["logp"], c["mask"], g=1.0)
    for x in r:
        assert abs(float(x["loss"]) - full["loss"]) < 1e-12 * full["loss"]
        np.testing.assert_allclose(x["dw"], full["dW"], rtol=1e-10, atol=1e-14)
