"""Data-parallel forward + backward over torch.distributed.

Each rank holds its own rows of the batch (H, the teacher cache, the mask)
and the whole output head W.  The loss is the mean over the positions that
count on ALL ranks, so:

* after the forward, the library writes this rank's (sum of KL over its
  counted positions, N_r) in fp64 (``ckl_dp_local_stats``); those two numbers
  are summed over the ranks (one all-reduce) and the library turns them into
  the global loss and this rank's upstream gradient g N_r / N
  (``ckl_dp_finish``), so that the backward, which divides by its own N_r,
  scales by g / N: the rank's dH rows are final and its dW is its share of
  the global gradient;
* dW is summed over ranks with all-reduces issued while the backward is still
  running: the library reports each range of dW rows as soon as the launches
  that last write them are enqueued (``on_dw_ready``, one range per
  vocabulary slab when the backward is sliced).  The ranges depend on the
  rank's own row count (the blocking of its backward), but collectives must
  be issued in the same order with the same sizes on every rank, so dW is
  exchanged in fixed pieces that are the same on every rank: a piece's
  all-reduce is queued, behind the launches that finish it, as soon as the
  reported ranges cover it.

The pages run on one GPU (their multi-node setup is the one the loss lets
them leave); this is the exchange a data-parallel training step adds around
the same loss.  With NCCL the collectives run over NVLink; the tests run the
same host logic with gloo, on CPU and between two processes on one GPU.
"""

from __future__ import annotations

import torch
import torch.distributed as dist

__all__ = ["dp_forward_backward", "dw_pieces"]


def dp_forward_backward(H, W, idx, logp, mask=None, chunk: int = 1024, grad_loss=None,
                        group=None, workspace=None, dW=None, ops=None):
    """Loss over all ranks' rows, this rank's lse and dH, and dW summed over ranks.

    ``grad_loss`` is the upstream gradient g of the global loss (a float32
    [1] tensor on H's device, or None for 1).  ``ops`` supplies the library's
    ``new_workspace``, ``forward``, ``dp_local_stats``, ``dp_finish`` and
    ``backward`` (with ``on_dw_ready``); by default the CUDA library.
    Returns (loss, lse, dH, dW); every rank gets the same loss and dW.
    """
    if ops is None:
        import chunked_kl_loss_ckl_b200 as ops
    T, d = H.shape
    V = W.shape[0]
    K = idx.shape[1]
    if workspace is None:
        workspace = ops.new_workspace(T, d, V, K, chunk, H.device)
    _, lse = ops.forward(H, W, idx, logp, mask, chunk, workspace=workspace)
    stats = ops.dp_local_stats(workspace)
    dist.all_reduce(stats[0:2], group=group)
    loss, g_local = ops.dp_finish(stats, grad_loss)

    works = []
    if dW is None:
        dW = torch.empty(V, d, dtype=torch.float32, device=H.device)
    bounds = dw_pieces(V)
    state = {"next": 0}

    def ready(v0: int, v1: int):
        # ranges arrive in increasing order and partition [0, V): rows below
        # v1 are final; exchange every piece that lies below it
        while state["next"] < len(bounds) and bounds[state["next"]][1] <= v1:
            b, e = bounds[state["next"]]
            works.append(dist.all_reduce(dW[b:e], group=group, async_op=True))
            state["next"] += 1

    dH, dW = ops.backward(H, W, idx, logp, mask, lse, grad_loss=g_local, chunk=chunk, dW=dW,
                          workspace=workspace, on_dw_ready=ready)
    if state["next"] != len(bounds):
        raise RuntimeError("the backward did not report every dW row as final")
    for w in works:
        w.wait()
    return loss, lse, dH, dW


def dw_pieces(V: int, pieces: int = 8, align: int = 256):
    """The fixed pieces [begin, end) of dW's rows exchanged one all-reduce
    each: the same on every rank, since they depend on V alone."""
    step = -(-V // pieces)
    if V >= pieces * align:
        step = -(-step // align) * align
    return [(b, min(V, b + step)) for b in range(0, V, step)]
