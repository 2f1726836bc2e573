"""Double-buffered host -> device staging of per-step inputs.

A training loop feeds the loss a new batch every step: the student's hidden
states and the cached teacher top-K (ids, log-probs, mask) come from pinned
host memory, while the output head stays resident.  ``Stager`` keeps two
device copies of the step's inputs and copies batch i + 1 on a side stream
while the loss of batch i runs, so the copy engine and the tensor cores
overlap; each batch still crosses PCIe exactly once.

    stager = Stager([hH, hidx, hlogp, hmask], device)
    stager.put(next_host_batch)          # starts the copy (side stream)
    dev_batch = stager.get()             # the compute stream waits for it
    ... loss on dev_batch ...
    stager.release()                     # the buffer may be refilled
"""

from __future__ import annotations

import torch

__all__ = ["Stager"]


class Stager:
    """Two device buffers per input; ``put`` fills the next one on a copy
    stream, ``get`` hands it to the current stream once its copy is done,
    ``release`` marks the buffer ``get`` returned as no longer read."""

    def __init__(self, like, device, stream=None):
        self.device = torch.device(device)
        self.copy_stream = torch.cuda.Stream(self.device)
        self.compute = stream or torch.cuda.current_stream(self.device)
        self.bufs = [[torch.empty(t.shape, dtype=t.dtype, device=self.device) for t in like]
                     for _ in range(2)]
        self.ready = [torch.cuda.Event(), torch.cuda.Event()]
        self.free = [torch.cuda.Event(), torch.cuda.Event()]
        self.freed = [False, False]
        self.next = 0      # buffer the next put fills
        self.cur = None    # buffer the last get returned
        self.filled = []   # buffers filled and not yet taken, in order

    def put(self, host_tensors) -> None:
        b = self.next
        if len(self.filled) == 2:
            raise RuntimeError("both buffers hold batches not yet taken")
        with torch.cuda.stream(self.copy_stream):
            if self.freed[b]:
                self.copy_stream.wait_event(self.free[b])
            for dst, src in zip(self.bufs[b], host_tensors):
                dst.copy_(src, non_blocking=True)
            self.ready[b].record(self.copy_stream)
        self.filled.append(b)
        self.next = 1 - b

    def get(self):
        if not self.filled:
            raise RuntimeError("no batch was put")
        b = self.filled.pop(0)
        self.compute.wait_event(self.ready[b])
        self.cur = b
        return self.bufs[b]

    def release(self) -> None:
        if self.cur is None:
            return
        self.free[self.cur].record(self.compute)
        self.freed[self.cur] = True
        self.cur = None
