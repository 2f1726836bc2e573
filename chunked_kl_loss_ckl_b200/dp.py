"""Data-parallel forward + backward over torch.distributed.

Each rank holds its own rows of the batch (H, the teacher cache, the mask)
and the whole output head W.  The loss is the mean over the positions that
count on ALL ranks, so:

* the forward's per-rank loss (a mean over the rank's own N_r positions) and
  N_r are summed over ranks (one all-reduce of two fp64 numbers):
  loss = sum_r loss_r N_r / sum_r N_r;
* the backward runs with the upstream gradient scaled by N_r / N (the library
  divides by its own N_r), so the rank's dH rows are final and its dW is its
  share of the global gradient;
* dW is summed over ranks with all-reduces issued while the backward is still
  running: the library reports each range of dW rows as soon as the launches
  that last write them are enqueued (``on_dw_ready``, one range per
  vocabulary slab when the backward is sliced), and the all-reduce of that
  range is queued right then, behind them, on the collective's stream.

The pages run on one GPU (their multi-node setup is the one the loss lets
them leave); this is the exchange a data-parallel training step adds around
the same loss.  With NCCL the collectives run over NVLink; the tests run the
same host logic with gloo on CPU.
"""

from __future__ import annotations

import torch
import torch.distributed as dist

__all__ = ["dp_forward_backward"]


def _count(mask, T: int, device) -> torch.Tensor:
    if mask is None:
        return torch.tensor(float(T), dtype=torch.float64, device=device)
    return (mask != 0).sum(dtype=torch.float64)


def dp_forward_backward(H, W, idx, logp, mask=None, chunk: int = 1024, grad_loss=None,
                        group=None, workspace=None, dW=None, ops=None):
    """Loss over all ranks' rows, this rank's lse and dH, and dW summed over ranks.

    ``grad_loss`` is the upstream gradient g of the global loss (a float32
    [1] tensor on H's device, or None for 1).  ``ops`` supplies
    ``forward(H, W, idx, logp, mask, chunk, workspace=...)`` and
    ``backward(H, W, idx, logp, mask, lse, grad_loss=..., chunk=..., dW=...,
    workspace=..., on_dw_ready=...)``; by default the CUDA library.
    Returns (loss, lse, dH, dW); every rank gets the same loss and dW.
    """
    if ops is None:
        import chunked_kl_loss_ckl_b200 as ops
    T = H.shape[0]
    loss_r, lse = ops.forward(H, W, idx, logp, mask, chunk, workspace=workspace)
    n_r = _count(mask, T, loss_r.device)
    stats = torch.stack([loss_r.reshape(()).double() * n_r, n_r])
    dist.all_reduce(stats, group=group)
    n = stats[1]
    has = n > 0
    loss = torch.where(has, stats[0] / torch.where(has, n, torch.ones_like(n)),
                       torch.zeros_like(n)).float().reshape(1)
    g = torch.ones((), dtype=torch.float64, device=n.device) if grad_loss is None \
        else grad_loss.reshape(()).double()
    g_r = torch.where(has, g * n_r / torch.where(has, n, torch.ones_like(n)),
                      torch.zeros_like(n)).float().reshape(1)

    works = []
    out = {}

    def ready(v0: int, v1: int):
        works.append(dist.all_reduce(out["dW"][v0:v1], group=group, async_op=True))

    if dW is None:
        dW = torch.empty(W.shape[0], W.shape[1], dtype=torch.float32, device=H.device)
    out["dW"] = dW
    dH, dW = ops.backward(H, W, idx, logp, mask, lse, grad_loss=g_r, chunk=chunk, dW=dW,
                          workspace=workspace, on_dw_ready=ready)
    for w in works:
        w.wait()
    return loss, lse, dH, dW
