"""GPU parity of the single-pass entry point (ckl_forward_backward) against the
fp64 oracle, and its agreement with the two-pass path (ckl_forward +
ckl_backward) on the same inputs.

The single pass computes each chunk's logits once, keeps them in fp32 and
derives dZ from them after the chunk's lse is known, so its results are the
same quantities as the two-pass path's.  Tolerances against the oracle: loss
relative 1e-3, lse absolute 2e-3, dH and dW relative Frobenius 1e-2.  Against
the two-pass path the only difference is the grouping of the fp32 sums that
make lse (the vocabulary is split per chunk here, over all T there), so the
bounds are much tighter.
"""

import numpy as np
import pytest
import torch

import oracle
from ckl_synth import make_config, make_inputs
from gpu_util import assert_parity, rel_fro, run_library, to_device

pytestmark = pytest.mark.gpu


def _ref(c, g=1.0, mask="config"):
    m = c["mask"] if isinstance(mask, str) else mask
    return oracle.dense(c["H"], c["W"], c["idx"], c["logp"], m, g=g)


def run_single_pass(ckl, c, chunk=None, g=None, mask="config", dW0=None):
    H, W, idx, logp, m = to_device(c, mask)
    chunk = chunk or c["chunk"]
    T, d, V, K = c["T"], c["d"], c["V"], c["K"]
    ws = torch.empty(ckl.single_pass_workspace_bytes(T, d, V, K, chunk), dtype=torch.uint8,
                     device="cuda")
    gl = None if g is None else torch.tensor([g], dtype=torch.float32, device="cuda")
    dW = None
    if dW0 is not None:
        dW = torch.from_numpy(np.ascontiguousarray(dW0, dtype=np.float32)).cuda()
    loss, lse, dH, dW = ckl.forward_backward(H, W, idx, logp, m, grad_loss=gl, chunk=chunk, dW=dW,
                                             accumulate_dW=dW0 is not None, workspace=ws)
    st = ckl.read_device_status(ws)
    torch.cuda.synchronize()
    return dict(loss=float(loss.item()), lse=lse.cpu().numpy().astype(np.float64),
                dH=dH.float().cpu().numpy().astype(np.float64),
                dW=dW.cpu().numpy().astype(np.float64), status_f=st, status_b=st)


def test_tiny_config(gpu_lib):
    c = make_config("tiny")
    assert_parity(run_single_pass(gpu_lib, c), _ref(c), "single pass tiny")


@pytest.mark.parametrize("chunk", [64, 100, 128, 300])
def test_ragged_shapes_all_chunk_sizes(gpu_lib, chunk):
    c = make_inputs(300, 200, 1000, 16, seed=3, w_std=0.3, mask=("bernoulli", 0.2))
    assert_parity(run_single_pass(gpu_lib, c, chunk=chunk), _ref(c), f"single pass chunk={chunk}")


def test_vocab_not_multiple_of_8_and_small_d(gpu_lib):
    # V = 1003: the fp32 logit rows are padded to 1004, dZ panels to 1024
    c = make_inputs(130, 8, 1003, 5, seed=4, w_std=0.5)
    assert_parity(run_single_pass(gpu_lib, c, chunk=64), _ref(c), "single pass V=1003 d=8")


def test_many_row_blocks_and_vocab_tiles(gpu_lib):
    c = make_inputs(1000, 328, 3000, 32, seed=5, w_std=0.1, mask=("tail", 37))
    assert_parity(run_single_pass(gpu_lib, c, chunk=512), _ref(c), "single pass 1000x3000x328")


def test_agrees_with_the_two_pass_path(gpu_lib):
    c = make_inputs(1000, 328, 3000, 32, seed=16, w_std=0.1, mask=("bernoulli", 0.1))
    a = run_single_pass(gpu_lib, c, chunk=256)
    b = run_library(gpu_lib, c, chunk=256)
    e_loss = abs(a["loss"] - b["loss"]) / abs(b["loss"])
    e_lse = float(np.abs(a["lse"] - b["lse"]).max())
    e_dH, e_dW = rel_fro(a["dH"], b["dH"]), rel_fro(a["dW"], b["dW"])
    print(f"[single vs two-pass] loss {e_loss:.2e} lse {e_lse:.2e} dH {e_dH:.2e} dW {e_dW:.2e}")
    assert e_loss <= 1e-5 and e_lse <= 1e-4
    assert e_dH <= 1e-3 and e_dW <= 1e-3


def test_runs_are_deterministic(gpu_lib):
    c = make_inputs(300, 200, 1000, 16, seed=7, w_std=0.3, mask=("bernoulli", 0.1))
    a = run_single_pass(gpu_lib, c, chunk=128)
    b = run_single_pass(gpu_lib, c, chunk=128)
    for k in ("lse", "dH", "dW"):
        assert np.array_equal(a[k], b[k]), k
    assert a["loss"] == b["loss"]


def test_upstream_gradient_and_dw_accumulation(gpu_lib):
    c = make_inputs(260, 64, 700, 8, seed=8, w_std=0.4)
    ref = dict(_ref(c, g=0.37))
    dW0 = np.random.default_rng(0).normal(0, 1e-3, (700, 64))
    out = run_single_pass(gpu_lib, c, chunk=100, g=0.37, dW0=dW0)
    ref["dW"] = ref["dW"] + dW0.astype(np.float32)
    assert_parity(out, ref, "single pass g=0.37 accumulate")


def test_all_positions_masked(gpu_lib):
    c = make_inputs(200, 64, 600, 8, seed=9, w_std=0.4)
    mask = np.zeros(200, np.uint8)
    out = run_single_pass(gpu_lib, c, chunk=128, mask=mask)
    ref = _ref(c, mask=mask)
    assert out["loss"] == 0.0
    assert np.abs(out["dH"]).max() == 0.0 and np.abs(out["dW"]).max() == 0.0
    assert np.abs(out["lse"] - ref["lse"]).max() <= 2e-3


def test_empty_batch(gpu_lib):
    c = make_inputs(0, 64, 600, 8, seed=1, w_std=0.4)
    H, W, idx, logp, m = to_device(c)
    dW = torch.full((600, 64), 7.0, device="cuda")
    loss, lse, dH, dW = gpu_lib.forward_backward(H, W, idx, logp, None, chunk=64, dW=dW)
    torch.cuda.synchronize()
    assert loss.item() == 0.0 and lse.numel() == 0 and dH.numel() == 0
    assert dW.abs().max().item() == 0.0


def test_repeated_teacher_ids(gpu_lib):
    c = make_inputs(150, 64, 500, 6, seed=10, w_std=0.4)
    idx = c["idx"].copy()
    idx[:, 3] = idx[:, 0]
    idx[::3, 5] = idx[::3, 1]
    c = dict(c, idx=idx)
    assert_parity(run_single_pass(gpu_lib, c, chunk=64), _ref(c), "single pass repeated ids")


@pytest.mark.parametrize("K", [1, 256])
def test_smallest_and_largest_K(gpu_lib, K):
    c = make_inputs(140, 64, 1500, K, seed=11, w_std=0.4)
    assert_parity(run_single_pass(gpu_lib, c, chunk=128), _ref(c), f"single pass K={K}")


def test_minus_inf_teacher_entries(gpu_lib):
    c = make_inputs(140, 64, 800, 10, seed=12, w_std=0.4)
    logp = c["logp"].copy()
    logp[:, -3:] = -np.inf
    c = dict(c, logp=logp)
    assert_parity(run_single_pass(gpu_lib, c, chunk=128), _ref(c), "single pass -inf entries")


def test_bad_teacher_id_is_reported_not_faulted(gpu_lib):
    c = make_inputs(64, 64, 300, 4, seed=13, w_std=0.4)
    idx = c["idx"].copy()
    idx[5, 2] = 300
    idx[9, 0] = -1
    out = run_single_pass(gpu_lib, dict(c, idx=idx), chunk=64)
    rc, word = out["status_f"]
    assert rc == 5 and word & 1
