"""GPU side of the data-parallel exchange, on the one GPU this suite has.

* ckl_backward_ex reports dW row ranges that partition [0, V), one per
  vocabulary slab on the last row chunk of a sliced backward, and its results
  are bitwise those of ckl_backward;
* dp_forward_backward under a one-rank NCCL process group (the all-reduces
  then sum one term) is bitwise the plain forward + backward, and matches the
  fp64 oracle at the contract tolerances, also when no position counts;
* two ranks as two processes sharing the one GPU, exchanging over gloo (the
  collectives run on the host, so no kernel of one rank waits for the
  other's): uneven shards of one batch through the real kernels, checked
  against the unsharded oracle -- the loss, every dH row and dW -- and a
  shard with no counted position (N_r = 0).
"""

import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from ckl_synth import make_inputs
from gpu_util import assert_parity, to_device

pytestmark = pytest.mark.gpu


def _ranges_and_grads(ckl, c, chunk):
    H, W, idx, logp, m = to_device(c)
    T, d, V, K = c["T"], c["d"], c["V"], c["K"]
    ws = ckl.new_workspace(T, d, V, K, chunk)
    loss, lse = ckl.forward(H, W, idx, logp, m, chunk, workspace=ws)
    seen = []
    dH1, dW1 = ckl.backward(H, W, idx, logp, m, lse, chunk=chunk, workspace=ws,
                            on_dw_ready=lambda a, b: seen.append((a, b)))
    dH1, dW1 = dH1.clone(), dW1.clone()
    dH2, dW2 = ckl.backward(H, W, idx, logp, m, lse, chunk=chunk, workspace=ws)
    torch.cuda.synchronize()
    return seen, (dH1, dW1), (dH2, dW2)


@pytest.mark.parametrize("shape,chunk", [((3072, 1024, 8192, 16), 512),
                                         ((1000, 328, 3000, 32), 256)])
def test_dw_ready_ranges_partition_V(gpu_lib, shape, chunk):
    T, d, V, K = shape
    c = make_inputs(T, d, V, K, seed=21, w_std=0.05, mask=("bernoulli", 0.1))
    seen, a, b = _ranges_and_grads(gpu_lib, c, chunk)
    Cr, Sv, n = gpu_lib.backward_plan(T, d, V, K, chunk)
    want = [(s * Sv, min(V, (s + 1) * Sv)) for s in range(n)] if n > 1 else [(0, V)]
    assert seen == want
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_dp_step_one_rank_nccl_is_the_plain_step(gpu_lib, tmp_path):
    from chunked_kl_loss_ckl_b200.dp import dp_forward_backward
    c = make_inputs(3072, 1024, 8192, 16, seed=22, w_std=0.05, mask=("bernoulli", 0.1))
    H, W, idx, logp, m = to_device(c)
    dist.init_process_group("nccl", init_method=f"file://{tmp_path}/store", rank=0,
                            world_size=1, timeout=datetime.timedelta(seconds=60))
    try:
        g = torch.tensor([0.5], dtype=torch.float32, device="cuda")
        loss, lse, dH, dW = dp_forward_backward(H, W, idx, logp, m, chunk=512, grad_loss=g)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    l2, lse2 = gpu_lib.forward(H, W, idx, logp, m, 512)
    dH2, dW2 = gpu_lib.backward(H, W, idx, logp, m, lse2, grad_loss=g, chunk=512)
    torch.cuda.synchronize()
    assert loss.item() == l2.item()
    assert torch.equal(lse, lse2) and torch.equal(dH, dH2) and torch.equal(dW, dW2)
    assert np.isfinite(loss.item()) and dW.abs().max().item() > 0
    ref = oracle.dense(c["H"], c["W"], c["idx"], c["logp"], c["mask"], g=0.5)
    out = dict(loss=float(loss.item()), lse=lse.cpu().numpy().astype(np.float64),
               dH=dH.float().cpu().numpy().astype(np.float64),
               dW=dW.cpu().numpy().astype(np.float64), status_f=(0, 0), status_b=(0, 0))
    assert_parity(out, ref, "dp one rank vs oracle")


def test_dp_step_one_rank_no_position_counts(gpu_lib, tmp_path):
    from chunked_kl_loss_ckl_b200.dp import dp_forward_backward
    c = make_inputs(600, 256, 3000, 16, seed=23, w_std=0.1, mask=("none",))
    H, W, idx, logp, m = to_device(c)
    dist.init_process_group("nccl", init_method=f"file://{tmp_path}/store", rank=0,
                            world_size=1, timeout=datetime.timedelta(seconds=60))
    try:
        loss, lse, dH, dW = dp_forward_backward(H, W, idx, logp, m, chunk=256)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    ref = oracle.dense(c["H"], c["W"], c["idx"], c["logp"], c["mask"])
    assert loss.item() == 0.0 and ref["loss"] == 0.0
    assert dH.abs().max().item() == 0.0 and dW.abs().max().item() == 0.0
    assert np.abs(lse.cpu().numpy() - ref["lse"]).max() <= 2e-3


# ------------------------------------------------------ two ranks, one GPU
def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


_TWO_RANK = dict(T=3072, d=1024, V=8192, K=16, split=1100, chunk=512)


def _two_rank_inputs(kind):
    p = _TWO_RANK
    c = make_inputs(p["T"], p["d"], p["V"], p["K"], seed=24, w_std=0.05,
                    mask=("bernoulli", 0.1))
    if kind == "empty_shard":          # rank 1's rows never count: N_1 = 0
        c["mask"] = c["mask"].copy()
        c["mask"][p["split"]:] = 0
    return c


def _two_rank_worker(rank, world, port, out_dir, kind):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        from chunked_kl_loss_ckl_b200.dp import dp_forward_backward
        p = _TWO_RANK
        c = _two_rank_inputs(kind)
        lo, hi = (0, p["split"]) if rank == 0 else (p["split"], p["T"])   # 1100 / 1972 rows
        part = dict(c, H=c["H"][lo:hi], idx=c["idx"][lo:hi], logp=c["logp"][lo:hi],
                    mask=c["mask"][lo:hi], T=hi - lo)
        H, W, idx, logp, m = to_device(part)
        g = torch.tensor([0.8], dtype=torch.float32, device="cuda")
        loss, lse, dH, dW = dp_forward_backward(H, W, idx, logp, m, chunk=p["chunk"],
                                                grad_loss=g)
        torch.cuda.synchronize()
        np.savez(os.path.join(out_dir, f"{kind}{rank}.npz"), loss=loss.cpu().numpy(),
                 lse=lse.cpu().numpy(), dH=dH.float().cpu().numpy(), dW=dW.cpu().numpy(),
                 lo=lo, hi=hi)
    finally:
        dist.barrier()
        dist.destroy_process_group()


@pytest.mark.parametrize("kind", ["uneven", "empty_shard"])
def test_dp_two_processes_one_gpu_against_the_oracle(gpu_lib, tmp_path, kind):
    world = 2
    mp.spawn(_two_rank_worker, args=(world, _free_port(), str(tmp_path), kind), nprocs=world,
             join=True)
    r = [np.load(tmp_path / f"{kind}{i}.npz") for i in range(world)]
    c = _two_rank_inputs(kind)
    ref = oracle.dense(c["H"], c["W"], c["idx"], c["logp"], c["mask"], g=0.8)
    dH = np.concatenate([x["dH"] for x in r]).astype(np.float64)
    lse = np.concatenate([x["lse"] for x in r]).astype(np.float64)
    for x in r:   # every rank holds the global loss and the summed dW
        out = dict(loss=float(x["loss"][0]), lse=lse, dH=dH, dW=x["dW"].astype(np.float64),
                   status_f=(0, 0), status_b=(0, 0))
        assert_parity(out, ref, f"dp two processes ({kind})")
    assert np.array_equal(r[0]["dW"], r[1]["dW"])
    if kind == "empty_shard":
        assert np.abs(r[1]["dH"]).max() == 0.0
