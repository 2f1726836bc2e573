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


# ---------------------------------------------------------------- data parallel
class _OracleOps:
    """Stands in for the CUDA library on CPU: the oracle's dense forward and
    backward of the rank's own rows, with the library's interface (fp32/bf16
    outputs, the fp64 (sum of KL, N_r) stats, dW written range by range with
    on_dw_ready after each range)."""

    def __init__(self, c):
        self.c = c
        self.fwd = None

    def new_workspace(self, T, d, V, K, chunk, device=None):
        return torch.zeros(1, dtype=torch.uint8)

    def forward(self, H, W, idx, logp, mask, chunk, workspace=None):
        import oracle
        c = self.c
        r = oracle.dense(c["H"], c["W"], c["idx"], c["logp"], c["mask"], g=1.0)
        self.fwd = r
        return (torch.tensor([r["loss"]], dtype=torch.float32),
                torch.from_numpy(r["lse"].astype(np.float32)))

    def dp_local_stats(self, workspace):
        r = self.fwd
        num = r["loss"] * r["N"]
        return torch.tensor([num, r["N"], num, r["N"]], dtype=torch.float64)

    def dp_finish(self, stats, grad_loss=None):
        num, n, n_r = float(stats[0]), float(stats[1]), float(stats[3])
        g = 1.0 if grad_loss is None else float(grad_loss.item())
        loss = num / n if n > 0 else 0.0
        return (torch.tensor([loss], dtype=torch.float32),
                torch.tensor([g * n_r / n if n > 0 else 0.0], dtype=torch.float32))

    def backward(self, H, W, idx, logp, mask, lse, grad_loss=None, chunk=1024, dW=None,
                 workspace=None, on_dw_ready=None):
        import oracle
        c = self.c
        g = 1.0 if grad_loss is None else float(grad_loss.item())
        r = oracle.dense(c["H"], c["W"], c["idx"], c["logp"], c["mask"], g=g)
        # ranges that depend on the rank's row count, as the library's
        # blocking does: ranks report different ranges
        V = dW.shape[0]
        n = 1 + H.shape[0] % 4
        cuts = [V * i // n for i in range(n + 1)]
        for v0, v1 in zip(cuts[:-1], cuts[1:]):
            dW[v0:v1] = torch.from_numpy(r["dW"][v0:v1].astype(np.float32))
            on_dw_ready(v0, v1)
        return torch.from_numpy(r["dH"].astype(np.float32)), dW


def _dp_worker(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        from chunked_kl_loss_ckl_b200.dp import dp_forward_backward
        from ckl_synth import make_inputs
        c = make_inputs(40, 16, 60, 5, seed=5, w_std=0.4, mask=("bernoulli", 0.2))
        lo, hi = (0, 13) if rank == 0 else (13, 40)   # uneven shards
        part = dict(c, H=c["H"][lo:hi], idx=c["idx"][lo:hi], logp=c["logp"][lo:hi],
                    mask=c["mask"][lo:hi], T=hi - lo)
        ops = _OracleOps(part)
        Ht = torch.zeros(hi - lo, 16)
        Wt = torch.zeros(60, 16)
        g = torch.tensor([0.7], dtype=torch.float32)
        mt = torch.from_numpy(np.ascontiguousarray(part["mask"], dtype=np.uint8))
        it = torch.from_numpy(part["idx"])
        lt = torch.from_numpy(part["logp"])
        loss, lse, dH, dW = dp_forward_backward(Ht, Wt, it, lt, mask=mt, chunk=8,
                                                grad_loss=g, ops=ops)
        np.savez(os.path.join(out_dir, f"dp{rank}.npz"), loss=loss.numpy(), dH=dH.numpy(),
                 dW=dW.numpy(), lo=lo, hi=hi)
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_data_parallel_step_two_gloo_ranks(tmp_path):
    """dp_forward_backward on two ranks with uneven shards equals the
    unsharded loss and gradients: the global mean, dH rows scaled by the
    global N, dW summed over ranks piece by piece (the same pieces on both
    ranks although their backwards report different ranges)."""
    world = 2
    mp.spawn(_dp_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    r = [np.load(tmp_path / f"dp{i}.npz") for i in range(world)]
    import oracle
    from ckl_synth import make_inputs
    c = make_inputs(40, 16, 60, 5, seed=5, w_std=0.4, mask=("bernoulli", 0.2))
    full = oracle.dense(c["H"], c["W"], c["idx"], c["logp"], c["mask"], g=0.7)
    for x in r:
        assert abs(float(x["loss"][0]) - full["loss"]) <= 1e-6 * full["loss"]
        np.testing.assert_allclose(x["dW"], full["dW"], rtol=1e-5, atol=1e-7)
        lo, hi = int(x["lo"]), int(x["hi"])
        np.testing.assert_allclose(x["dH"], full["dH"][lo:hi], rtol=1e-5, atol=1e-7)


# ---------------------------------------------------------------- vocabulary parallel
class _OracleVPOps:
    """Stands in for the CUDA library's vocabulary-shard entry points on CPU:
    per-row (max z log2 e, sum of 2^(z log2 e - max), sum of p z over the
    shard's teacher ids) from the oracle's logits of the shard, their merge,
    and the shard's share of the closed-form gradient."""

    LOG2E = 1.0 / np.log(2.0)

    def __init__(self, c):
        import oracle
        self.c = c
        self.H = oracle.widen_bf16(c["H"])
        self.W = oracle.widen_bf16(c["W"])
        self.p, self.logp_n = oracle.renormalise_topk(c["logp"])
        m = np.ones(c["T"]) if c["mask"] is None else (c["mask"] != 0).astype(float)
        self.m, self.N = m, m.sum()

    def _shard_logits(self, vb, ve):
        import oracle
        return oracle.logits(self.H, self.W[vb:ve])

    def forward_vocab_shard(self, H, W_shard, idx, logp, mask, V, vb, ve, chunk):
        Z = self._shard_logits(vb, ve)
        y = Z * self.LOG2E
        mx = y.max(axis=1)
        s = np.exp2(y - mx[:, None]).sum(axis=1)
        ids = self.c["idx"].astype(np.int64)
        inside = (ids >= vb) & (ids < ve)
        zg = np.take_along_axis(Z, np.clip(ids - vb, 0, ve - vb - 1), axis=1)
        pz = np.where(inside, self.p * zg, 0.0).sum(axis=1)
        part = np.stack([mx, s, pz, np.zeros_like(mx)], axis=1)
        return torch.from_numpy(part.astype(np.float32)), torch.zeros(1)

    def combine_vocab_shards(self, gathered, mask, K, ws):
        g = gathered.double().numpy()
        M = g[:, :, 0].max(axis=0)
        S = (g[:, :, 1] * np.exp2(g[:, :, 0] - M[None, :])).sum(axis=0)
        pz = g[:, :, 2].sum(axis=0)
        lse = (M + np.log2(S)) * np.log(2.0)
        hp = np.where(self.p > 0, self.p * np.where(self.p > 0, self.logp_n, 0.0), 0.0).sum(1)
        kl = hp - pz + lse
        loss = (self.m * kl).sum() / self.N if self.N > 0 else 0.0
        self.lse = lse
        return torch.tensor([loss], dtype=torch.float32), torch.from_numpy(lse.astype(np.float32))

    def backward_vocab_shard(self, H, W_shard, idx, logp, mask, V, vb, ve, lse, grad_loss=None,
                             chunk=1024, workspace=None):
        g = 1.0 if grad_loss is None else float(grad_loss.item())
        Z = self._shard_logits(vb, ve)
        G = np.exp(Z - self.lse[:, None])
        ids = self.c["idx"].astype(np.int64)
        for t in range(Z.shape[0]):
            for k in range(ids.shape[1]):
                if vb <= ids[t, k] < ve:
                    G[t, ids[t, k] - vb] -= self.p[t, k]
        G *= (g * self.m / self.N)[:, None] if self.N > 0 else 0.0
        return torch.from_numpy(G @ self.W[vb:ve]), torch.from_numpy(G.T @ self.H)

    def dh_to_bf16(self, x):
        return x.to(torch.bfloat16)


def _vp_worker(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        from chunked_kl_loss_ckl_b200.vp import vp_forward_backward
        from ckl_synth import make_inputs
        c = make_inputs(40, 16, 60, 5, seed=5, w_std=0.4, mask=("bernoulli", 0.2))
        vb, ve = (0, 23) if rank == 0 else (23, 60)          # uneven, unaligned
        ops = _OracleVPOps(c)
        g = torch.tensor([0.7], dtype=torch.float32)
        loss, lse, dH, dW = vp_forward_backward(
            torch.zeros(40, 16), torch.zeros(ve - vb, 16), 60, vb, ve,
            torch.from_numpy(c["idx"]), torch.from_numpy(c["logp"]),
            torch.from_numpy(c["mask"]), chunk=8, grad_loss=g, ops=ops)
        np.savez(os.path.join(out_dir, f"vp{rank}.npz"), loss=loss.numpy(), lse=lse.numpy(),
                 dH=dH.float().numpy(), dW=dW.numpy(), vb=vb, ve=ve)
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_vocab_parallel_step_two_gloo_ranks(tmp_path):
    """vp_forward_backward on two ranks holding uneven vocabulary shards of
    the head equals the unsharded loss, lse, dH and (concatenated) dW: the
    per-row (max, sum of exp, sum of p z) partials merge exactly."""
    world = 2
    mp.spawn(_vp_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    r = [np.load(tmp_path / f"vp{i}.npz") for i in range(world)]
    import oracle
    from ckl_synth import make_inputs
    c = make_inputs(40, 16, 60, 5, seed=5, w_std=0.4, mask=("bernoulli", 0.2))
    full = oracle.dense(c["H"], c["W"], c["idx"], c["logp"], c["mask"], g=0.7)
    for x in r:
        assert abs(float(x["loss"][0]) - full["loss"]) <= 1e-6 * full["loss"]
        np.testing.assert_allclose(x["lse"], full["lse"], rtol=1e-6, atol=1e-6)
        # dH is rounded to bf16 once, after the sum over the shards
        np.testing.assert_allclose(x["dH"], full["dH"], rtol=1e-2, atol=1e-4)
        np.testing.assert_allclose(x["dW"], full["dW"][int(x["vb"]):int(x["ve"])], rtol=1e-5,
                                   atol=1e-7)
    assert np.array_equal(r[0]["dH"], r[1]["dH"])
