"""The allocation-free forward, ckl_forward_static_scratch.

Some callers cannot allocate device memory: a plugin whose host runtime owns
every device allocation and passes it only input and output pointers, or code
on a latency-critical path where an allocation (which may synchronise the
device) is not allowed.  They cannot hand ckl_forward a workspace, so this
entry point keeps its scratch in one static device buffer inside the library.

The tests call it through the C ABI, twice in a row on two different problems
(so contents left in the shared buffer by the first call would show up in the
second), then on a problem whose H is too large for L2 (the forward's
split-fastest schedule), then right at its documented size limit and one
token past it.  Each result is compared with ckl_forward's on the same inputs
and with the fp64 oracle, within the tolerances the other GPU tests use.
This file is collected last.
"""

import ctypes

import numpy as np
import pytest
import torch

import oracle
from ckl_synth import make_inputs

pytestmark = pytest.mark.gpu

LOSS_RTOL = 1e-3
LSE_ATOL = 2e-3
CKL_ERR_WORKSPACE = 3
SCRATCH_BYTES = 32 << 20


def _r256(x):
    return (x + 255) // 256 * 256


def scratch_needed(T, K):
    """Bytes of static scratch a forward of T rows needs, as ckl.h states it."""
    return 256 + _r256(8 * K * T) + _r256(4 * T) + _r256(1024 * T) + _r256(8 * -(-T // 256))


def _bind():
    import chunked_kl_loss_ckl_b200 as ckl

    raw = ctypes.CDLL(ckl.LIB_PATH)
    vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32
    f = raw.ckl_forward_static_scratch
    f.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i32, vp, vp, vp, vp]
    f.restype = ctypes.c_int
    return ckl, f


def _device(c):
    H = torch.from_numpy(c["H"].view(np.int16)).cuda().view(torch.bfloat16)
    W = torch.from_numpy(c["W"].view(np.int16)).cuda().view(torch.bfloat16)
    idx = torch.from_numpy(c["idx"]).cuda()
    logp = torch.from_numpy(c["logp"]).cuda()
    m = None if c["mask"] is None else torch.from_numpy(c["mask"]).cuda()
    return H, W, idx, logp, m


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _static_forward(fwd_static, c):
    H, W, idx, logp, m = _device(c)
    T, d, V, K = c["T"], c["d"], c["V"], c["K"]
    loss = torch.empty(1, dtype=torch.float32, device="cuda")
    lse = torch.empty(T, dtype=torch.float32, device="cuda")
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    rc = fwd_static(_p(H), _p(W), _p(idx), _p(logp), _p(m), T, d, V, K, _p(loss), _p(lse),
                    _p(status), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    return rc, int(status.item()), loss, lse


def _check_against_both(ckl, fwd_static, c):
    rc, status, loss, lse = _static_forward(fwd_static, c)
    assert rc == 0 and status == 0, (rc, status)
    # the existing entry point, with a caller-owned workspace
    H, W, idx, logp, m = _device(c)
    ref_loss, ref_lse = ckl.forward(H, W, idx, logp, m, chunk=128)
    torch.cuda.synchronize()
    rl, l = ref_loss.item(), loss.item()
    assert abs(l - rl) <= LOSS_RTOL * abs(rl), (l, rl)
    assert (lse - ref_lse).abs().max().item() <= LSE_ATOL
    # and the fp64 oracle
    ref = oracle.dense(c["H"], c["W"], c["idx"], c["logp"], c["mask"], want_grad=False)
    assert abs(l - ref["loss"]) <= LOSS_RTOL * abs(ref["loss"]), (l, ref["loss"])
    assert np.abs(lse.cpu().numpy().astype(np.float64) - ref["lse"]).max() <= LSE_ATOL


def test_static_scratch_forward_matches_workspace_forward_on_two_calls():
    ckl, fwd_static = _bind()
    problems = [
        make_inputs(300, 200, 1000, 16, seed=21, w_std=0.3, mask=("bernoulli", 0.2)),
        make_inputs(1000, 328, 3000, 32, seed=22, w_std=0.1, mask=("tail", 37)),
    ]
    for c in problems:
        _check_against_both(ckl, fwd_static, c)


def test_static_scratch_forward_with_h_larger_than_l2():
    # 36 row blocks of 256 x 3072 bf16 (57 MB) exceed the forward's 48 MiB L2
    # budget for H, so its units run split-fastest, as in ckl_forward
    ckl, fwd_static = _bind()
    _check_against_both(ckl, fwd_static,
                        make_inputs(9000, 3072, 2000, 16, seed=25, w_std=0.02,
                                    mask=("bernoulli", 0.05)))


def test_static_scratch_size_limit_is_exact():
    ckl, fwd_static = _bind()
    K = 100
    T_max = max(T for T in range(18000, 19000) if scratch_needed(T, K) <= SCRATCH_BYTES)
    assert T_max == 18355 and scratch_needed(T_max + 1, K) > SCRATCH_BYTES
    c = make_inputs(T_max + 1, 64, 1000, K, seed=26, w_std=0.2)
    # one token past the limit: rejected before anything runs (real buffers)
    rc, status, _, _ = _static_forward(fwd_static, c)
    assert rc == CKL_ERR_WORKSPACE and status == -1
    # at the limit: runs, and matches
    c_max = dict(c, T=T_max, H=c["H"][:T_max], idx=c["idx"][:T_max], logp=c["logp"][:T_max])
    _check_against_both(ckl, fwd_static, c_max)
