"""GPU parity of the fp32 entry points (tf32 tensor-core products) against the
fp64 oracle on the fp32 inputs themselves (no bf16 rounding).

Tolerances derived from the arithmetic.  The tensor core reads each fp32
factor to 10 mantissa bits (relative error below 2^-10), so a product h w is
off by at most 2^-9 |h w|, and with fp32 accumulation over d terms each logit
by at most  tau_tv = (2^-9 + d 2^-23) sum_j |H_tj| |W_vj|.  lse moves by at
most max_v tau_tv (it is 1-Lipschitz in the max norm) and each row's KL by at
most twice that; so lse is checked per row against max_v tau_tv and the loss
against the mean of 2 max_v tau_tv over the rows that count (plus 1e-5 for
the fp32 softmax).  dH and dW keep the relative Frobenius bound 1e-2.  On
bf16-valued inputs tf32 is exact and the bf16 path's tolerances apply.
"""

import numpy as np
import pytest
import torch

import oracle
from ckl_synth import bf16_bits_to_f32, make_config, make_inputs
from gpu_util import rel_fro

pytestmark = pytest.mark.gpu


def _dev(c, mask="config"):
    H = torch.from_numpy(np.ascontiguousarray(c["H"], dtype=np.float32)).cuda()
    W = torch.from_numpy(np.ascontiguousarray(c["W"], dtype=np.float32)).cuda()
    idx = torch.from_numpy(c["idx"]).cuda()
    logp = torch.from_numpy(c["logp"]).cuda()
    m = c["mask"] if isinstance(mask, str) else mask
    mt = None if m is None else torch.from_numpy(np.ascontiguousarray(m, dtype=np.uint8)).cuda()
    return H, W, idx, logp, mt


def run_f32(ckl, c, chunk=None, g=None, dW0=None):
    H, W, idx, logp, m = _dev(c)
    chunk = chunk or c["chunk"]
    T, d, V, K = c["T"], c["d"], c["V"], c["K"]
    ws = torch.empty(ckl.lib.ckl_workspace_bytes_f32(T, d, V, K, chunk), dtype=torch.uint8,
                     device="cuda")
    loss, lse = ckl.forward_f32(H, W, idx, logp, m, chunk, workspace=ws)
    st_f = ckl.read_device_status(ws)
    gl = None if g is None else torch.tensor([g], dtype=torch.float32, device="cuda")
    dW = None
    if dW0 is not None:
        dW = torch.from_numpy(np.ascontiguousarray(dW0, dtype=np.float32)).cuda()
    dH, dW = ckl.backward_f32(H, W, idx, logp, m, lse, grad_loss=gl, chunk=chunk, dW=dW,
                              accumulate_dW=dW0 is not None, workspace=ws)
    st_b = ckl.read_device_status(ws)
    torch.cuda.synchronize()
    assert st_f[0] == 0 and st_b[0] == 0, (st_f, st_b)
    return dict(loss=float(loss.item()), lse=lse.cpu().numpy().astype(np.float64),
                dH=dH.cpu().numpy().astype(np.float64), dW=dW.cpu().numpy().astype(np.float64),
                status_f=st_f, status_b=st_b)


def _ref(c, g=1.0):
    return oracle.dense_values(np.asarray(c["H"], np.float64), np.asarray(c["W"], np.float64),
                               c["idx"], c["logp"], c["mask"], g=g)


def assert_parity_tf32(out, ref, c, tag=""):
    H = np.abs(np.asarray(c["H"], np.float64))
    W = np.abs(np.asarray(c["W"], np.float64))
    d = H.shape[1]
    tau = (2.0 ** -9 + d * 2.0 ** -23) * (H @ W.T).max(axis=1) + 1e-5   # per row
    m = np.ones(len(tau)) if c["mask"] is None else (np.asarray(c["mask"]) != 0).astype(float)
    lse_err = np.abs(out["lse"] - ref["lse"])
    loss_tol = 2 * (tau * m).sum() / max(m.sum(), 1) + 1e-5
    e_dH, e_dW = rel_fro(out["dH"], ref["dH"]), rel_fro(out["dW"], ref["dW"])
    print(f"[parity {tag}] loss_err={abs(out['loss'] - ref['loss']):.3e} (tol {loss_tol:.3e}) "
          f"lse_err/tol max={float((lse_err / tau).max()):.3f} dH_rfro={e_dH:.3e} "
          f"dW_rfro={e_dW:.3e}")
    assert abs(out["loss"] - ref["loss"]) <= loss_tol
    assert (lse_err <= tau).all()
    assert e_dH <= 1e-2 and e_dW <= 1e-2


def test_tiny_fp32_config(gpu_lib):
    # the tiny workload is an fp32 case: besides the tf32-derived bounds, its
    # results meet the contract tolerances themselves (loss 1e-3 relative,
    # lse 2e-3 absolute, dH and dW 1e-2 relative Frobenius)
    from gpu_util import assert_parity
    c = make_config("tiny", fp32=True)
    assert c["H"].dtype == np.float32
    out, ref = run_f32(gpu_lib, c), _ref(c)
    assert_parity_tf32(out, ref, c, "fp32 tiny")
    assert_parity(out, ref, "fp32 tiny, contract tolerances")


@pytest.mark.parametrize("chunk", [100, 300])
def test_ragged_fp32_both_schedules(gpu_lib, chunk):
    # chunk 100: sliced (dH summed in fp32 over vocabulary slabs in the output
    # itself); chunk 300: one chunk of all rows
    c = make_inputs(300, 200, 1000, 16, seed=3, w_std=0.3, mask=("bernoulli", 0.2), fp32=True)
    assert_parity_tf32(run_f32(gpu_lib, c, chunk=chunk), _ref(c), c, f"fp32 ragged chunk={chunk}")


def test_fp32_vocab_not_multiple_of_32_and_small_d(gpu_lib):
    c = make_inputs(130, 8, 1003, 5, seed=4, w_std=0.5, fp32=True)
    assert_parity_tf32(run_f32(gpu_lib, c, chunk=64), _ref(c), c, "fp32 V=1003 d=8")


def test_fp32_many_tiles_upstream_gradient_and_accumulation(gpu_lib):
    c = make_inputs(1000, 328, 3000, 32, seed=5, w_std=0.1, mask=("tail", 37), fp32=True)
    dW0 = np.random.default_rng(0).normal(0, 1e-3, (3000, 328))
    ref = dict(_ref(c, g=0.37))
    ref["dW"] = ref["dW"] + dW0.astype(np.float32)
    assert_parity_tf32(run_f32(gpu_lib, c, chunk=512, g=0.37, dW0=dW0), ref, c,
                       "fp32 1000x3000x328")


def test_fp32_path_on_bf16_values_matches_the_bf16_path(gpu_lib):
    # bf16 values are exact in tf32, so both paths multiply the same numbers;
    # they differ in accumulation order and in dZ (fp32 here, bf16 there).
    from gpu_util import run_library
    c = make_inputs(1000, 328, 3000, 32, seed=6, w_std=0.1, mask=("bernoulli", 0.1))
    c32 = dict(c, H=bf16_bits_to_f32(c["H"]), W=bf16_bits_to_f32(c["W"]))
    a = run_f32(gpu_lib, c32, chunk=256)
    b = run_library(gpu_lib, c, chunk=256)
    e = (abs(a["loss"] - b["loss"]) / abs(b["loss"]), float(np.abs(a["lse"] - b["lse"]).max()),
         rel_fro(a["dH"], b["dH"]), rel_fro(a["dW"], b["dW"]))
    print(f"[fp32 vs bf16 path] loss {e[0]:.2e} lse {e[1]:.2e} dH {e[2]:.2e} dW {e[3]:.2e}")
    assert e[0] <= 1e-5 and e[1] <= 1e-4 and e[2] <= 5e-3 and e[3] <= 5e-3
