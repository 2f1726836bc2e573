"""Vocabulary-parallel forward + backward over torch.distributed.

The output head is split by rows: rank r holds W[v_begin_r, v_end_r) (and
computes only that slice of dW), while every rank holds all T rows of H and
of the teacher cache.  One step:

* each rank runs the logit GEMM over its shard and reduces it, per row, to
  (max, sum of exp, sum of p z over the teacher ids in the shard)
  (``ckl_forward_vocab_shard``);
* those T x 16 bytes per rank are gathered from every rank (an all-reduce of
  a zero-filled [g, T, 4] tensor into which each rank wrote its own row, so
  that the same call works under NCCL and gloo) and merged into lse and the
  loss, the same on every rank (``ckl_combine_vocab_shards``);
* the backward recomputes the shard's logits with the global lse; the shard's
  dW rows are final where they are, and the shard's fp32 share of dH is
  summed over the ranks (an all-reduce of T x d fp32) and rounded to bf16
  once (``ckl_dh_to_bf16``).

The pages run one GPU; this is the split a head takes when it (V x d) and
its fp32 gradient do not fit on one device.
"""

from __future__ import annotations

import torch
import torch.distributed as dist

__all__ = ["shard_bounds", "vp_forward_backward"]


def shard_bounds(V: int, world: int, rank: int, align: int = 256):
    """[v_begin, v_end) of rank's shard: near-equal, boundaries on multiples
    of ``align`` (the last shard takes the rest)."""
    per = -(-V // world)
    per = -(-per // align) * align
    b = min(V, rank * per)
    e = min(V, (rank + 1) * per)
    return b, e


def vp_forward_backward(H, W_shard, V: int, v_begin: int, v_end: int, idx, logp, mask=None,
                        chunk: int = 1024, grad_loss=None, group=None, ops=None):
    """(loss, lse, dH, dW_shard) of the loss over all of V, each rank holding
    the shard [v_begin, v_end) of the head.  ``ops`` is the CUDA library by
    default; every rank gets the same loss, lse and dH."""
    if ops is None:
        import chunked_kl_loss_ckl_b200 as ops
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    T = H.shape[0]
    K = idx.shape[1]
    part, ws = ops.forward_vocab_shard(H, W_shard, idx, logp, mask, V, v_begin, v_end, chunk)
    gathered = torch.zeros(world, T, 4, dtype=torch.float32, device=part.device)
    gathered[rank].copy_(part)
    dist.all_reduce(gathered, group=group)
    loss, lse = ops.combine_vocab_shards(gathered, mask, K, ws)
    dHp, dW = ops.backward_vocab_shard(H, W_shard, idx, logp, mask, V, v_begin, v_end, lse,
                                       grad_loss=grad_loss, chunk=chunk, workspace=ws)
    dist.all_reduce(dHp, group=group)
    dH = ops.dh_to_bf16(dHp)
    return loss, lse, dH, dW
