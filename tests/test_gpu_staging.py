"""The double-buffered host -> device stager: batches staged on a side stream
give exactly the results of the same batches copied in place, in order (the
copy of batch i + 1 overlaps the loss of batch i without overwriting what
that loss still reads)."""

import numpy as np
import pytest
import torch

from ckl_synth import make_inputs

pytestmark = pytest.mark.gpu


def test_staged_batches_match_direct_calls(gpu_lib):
    from chunked_kl_loss_ckl_b200.staging import Stager
    T, d, V, K, chunk = 600, 256, 3000, 16, 256
    batches = [make_inputs(T, d, V, K, seed=30 + i, w_std=0.1, mask=("bernoulli", 0.1))
               for i in range(5)]
    W = torch.from_numpy(batches[0]["W"].view(np.int16)).cuda().view(torch.bfloat16)
    pin = lambda a: torch.from_numpy(np.ascontiguousarray(a)).pin_memory()
    hosts = [[pin(b["H"].view(np.int16)), pin(b["idx"]), pin(b["logp"]), pin(b["mask"])]
             for b in batches]
    stream = torch.cuda.current_stream()
    stager = Stager(hosts[0], "cuda", stream)
    got = []
    stager.put(hosts[0])
    for i in range(len(hosts)):
        bufs = stager.get()
        if i + 1 < len(hosts):
            stager.put(hosts[i + 1])
        H, idx, logp, m = bufs[0].view(torch.bfloat16), bufs[1], bufs[2], bufs[3]
        loss, lse = gpu_lib.forward(H, W, idx, logp, m, chunk)
        dH, dW = gpu_lib.backward(H, W, idx, logp, m, lse, chunk=chunk)
        stager.release()
        got.append((loss.clone(), dH.clone(), dW.clone()))
    torch.cuda.synchronize()
    for (loss, dH, dW), h in zip(got, hosts):
        H = h[0].cuda().view(torch.bfloat16)
        idx, logp, m = h[1].cuda(), h[2].cuda(), h[3].cuda()
        l2, lse2 = gpu_lib.forward(H, W, idx, logp, m, chunk)
        dH2, dW2 = gpu_lib.backward(H, W, idx, logp, m, lse2, chunk=chunk)
        torch.cuda.synchronize()
        assert loss.item() == l2.item()
        assert torch.equal(dH, dH2) and torch.equal(dW, dW2)
