"""GPU side of the data-parallel exchange, on the one GPU this suite has.

* ckl_backward_ex reports dW row ranges that partition [0, V), one per
  vocabulary slab on the last row chunk of a sliced backward, and its results
  are bitwise those of ckl_backward;
* dp_forward_backward under a one-rank NCCL process group (the all-reduces
  then sum one term) is bitwise the plain forward + backward: the callback
  path, the stream ordering of the collectives and the loss/N bookkeeping
  run for real; the two-rank arithmetic is covered with gloo on CPU
  (test_multirank.py).
"""

import datetime

import numpy as np
import pytest
import torch
import torch.distributed as dist

from ckl_synth import make_inputs
from gpu_util import to_device

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
