"""GPU parity of the vocabulary-parallel loss against the fp64 oracle.

The head is split by rows into shards; each shard's forward reduces its
logits to per-row (max, sum of exp, sum of p z) partials, the partials of all
shards are merged into lse and the loss, and each shard's backward yields its
dW rows and its fp32 share of dH.  The merged results must match the
unsharded oracle at the contract tolerances:

* all shards in one process (the exchange done by hand), with shard
  boundaries that are not multiples of the 256-column tile, teacher ids on
  both sides of each boundary, a mask, and both backward schedules;
* two ranks as two processes sharing the one GPU over gloo (host-side
  collectives; no kernel waits for another process) through
  ``vp_forward_backward``.
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


def _by_hand(ckl, c, bounds, chunk, g=None):
    H, W, idx, logp, m = to_device(c)
    V, K = c["V"], c["K"]
    parts, wss = [], []
    for vb, ve in bounds:
        part, ws = ckl.forward_vocab_shard(H, W[vb:ve], idx, logp, m, V, vb, ve, chunk)
        parts.append(part)
        wss.append(ws)
    gathered = torch.stack(parts).contiguous()
    loss, lse = ckl.combine_vocab_shards(gathered, m, K, wss[0])
    gl = None if g is None else torch.tensor([g], dtype=torch.float32, device="cuda")
    dHp = torch.zeros(c["T"], c["d"], dtype=torch.float32, device="cuda")
    dWs = []
    for (vb, ve), ws in zip(bounds, wss):
        dh, dw = ckl.backward_vocab_shard(H, W[vb:ve], idx, logp, m, V, vb, ve, lse, grad_loss=gl,
                                          chunk=chunk, workspace=ws)
        dHp += dh
        dWs.append(dw)
    dH = ckl.dh_to_bf16(dHp)
    st = [ckl.read_device_status(ws) for ws in wss]
    torch.cuda.synchronize()
    return dict(loss=float(loss.item()), lse=lse.cpu().numpy().astype(np.float64),
                dH=dH.float().cpu().numpy().astype(np.float64),
                dW=torch.cat(dWs).cpu().numpy().astype(np.float64),
                status_f=st[0], status_b=max(st, key=lambda x: x[0]))


@pytest.mark.parametrize("shape,bounds,chunk", [
    ((300, 200, 3000, 16), [(0, 1111), (1111, 2222), (2222, 3000)], 128),
    ((3072, 512, 8192, 16), [(0, 4000), (4000, 8192)], 512),
])
def test_vocab_shards_in_one_process_match_the_oracle(gpu_lib, shape, bounds, chunk):
    T, d, V, K = shape
    c = make_inputs(T, d, V, K, seed=31, w_std=0.1, mask=("bernoulli", 0.1))
    # teacher ids right at every shard boundary in the first rows
    for i, (vb, _) in enumerate(bounds[1:]):
        c["idx"][i, :2] = [vb - 1, vb]
        assert len(set(c["idx"][i].tolist())) == K
    ref = oracle.dense(c["H"], c["W"], c["idx"], c["logp"], c["mask"], g=0.6)
    assert_parity(_by_hand(gpu_lib, c, bounds, chunk, g=0.6), ref, f"vocab shards {shape}")


def test_one_shard_is_the_plain_loss(gpu_lib):
    c = make_inputs(500, 128, 2000, 16, seed=32, w_std=0.2)
    out = _by_hand(gpu_lib, c, [(0, 2000)], 256)
    ref = oracle.dense(c["H"], c["W"], c["idx"], c["logp"], None)
    assert_parity(out, ref, "one vocabulary shard")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


_SHAPE = dict(T=1000, d=256, V=5000, K=32, chunk=256)


def _inputs():
    p = _SHAPE
    return make_inputs(p["T"], p["d"], p["V"], p["K"], seed=33, w_std=0.1, mask=("tail", 50))


def _vp_worker(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        from chunked_kl_loss_ckl_b200.vp import shard_bounds, vp_forward_backward
        c = _inputs()
        H, W, idx, logp, m = to_device(c)
        vb, ve = shard_bounds(c["V"], world, rank)
        g = torch.tensor([1.3], dtype=torch.float32, device="cuda")
        loss, lse, dH, dW = vp_forward_backward(H, W[vb:ve].contiguous(), c["V"], vb, ve, idx,
                                                logp, m, chunk=_SHAPE["chunk"], grad_loss=g)
        torch.cuda.synchronize()
        np.savez(os.path.join(out_dir, f"vp{rank}.npz"), loss=loss.cpu().numpy(),
                 lse=lse.cpu().numpy(), dH=dH.float().cpu().numpy(), dW=dW.cpu().numpy(),
                 vb=vb, ve=ve)
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_vp_two_processes_one_gpu_against_the_oracle(gpu_lib, tmp_path):
    world = 2
    mp.spawn(_vp_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    r = [np.load(tmp_path / f"vp{i}.npz") for i in range(world)]
    c = _inputs()
    ref = oracle.dense(c["H"], c["W"], c["idx"], c["logp"], c["mask"], g=1.3)
    assert int(r[0]["ve"]) == int(r[1]["vb"]) and int(r[1]["ve"]) == c["V"]
    dW = np.concatenate([x["dW"] for x in r]).astype(np.float64)
    for x in r:
        out = dict(loss=float(x["loss"][0]), lse=x["lse"].astype(np.float64),
                   dH=x["dH"].astype(np.float64), dW=dW, status_f=(0, 0), status_b=(0, 0))
        assert_parity(out, ref, "vocabulary parallel, two processes")
    assert np.array_equal(r[0]["dH"], r[1]["dH"]) and np.array_equal(r[0]["lse"], r[1]["lse"])
