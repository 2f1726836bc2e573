"""Failure detection on the GPU without a fault: a bounded wait that nothing
satisfies runs out, the kernel records the timeout in the status word and
returns, and the context stays usable for the next call."""

import time

import numpy as np
import pytest
import torch

from ckl_synth import make_config
from gpu_util import assert_parity, run_library

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_and_is_reported(gpu_lib):
    ws = torch.empty(4096, dtype=torch.uint8, device="cuda")
    t0 = time.perf_counter()
    gpu_lib.selftest_wait_timeout(0.05, ws)
    rc, word = gpu_lib.read_device_status(ws)    # synchronises the stream
    dt = time.perf_counter() - t0
    assert rc == 7 and word & 4                  # CKL_ERR_TIMEOUT, CKL_DEV_TIMEOUT
    assert 0.05 <= dt < 2.0
    # the context is still good: a normal call on the same workspace memory
    import oracle
    c = make_config("tiny")
    assert_parity(run_library(gpu_lib, c), oracle.dense(c["H"], c["W"], c["idx"], c["logp"], None),
                  "after a timed-out wait")
