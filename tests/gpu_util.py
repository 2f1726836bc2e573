"""Helpers shared by the GPU tests: move a workload to the device, run the
library's forward + backward, and compare with the oracle."""

from __future__ import annotations

import numpy as np
import torch

# Tolerances for floating point, as the contract fixes them.
LOSS_RTOL = 1e-3     # |loss - ref| <= 1e-3 |ref|
LSE_ATOL = 2e-3      # max_t |lse_t - ref_t|
GRAD_RFRO = 1e-2     # ||g - ref||_F / ||ref||_F for dH and dW


def to_device(c: dict, mask="config"):
    H = torch.from_numpy(c["H"].view(np.int16)).cuda().view(torch.bfloat16)
    W = torch.from_numpy(c["W"].view(np.int16)).cuda().view(torch.bfloat16)
    idx = torch.from_numpy(c["idx"]).cuda()
    logp = torch.from_numpy(c["logp"]).cuda()
    m = c["mask"] if isinstance(mask, str) else mask
    mt = None if m is None else torch.from_numpy(np.ascontiguousarray(m, dtype=np.uint8)).cuda()
    return H, W, idx, logp, mt


def run_library(ckl, c, chunk=None, g=None, mask="config", dW0=None, workspace=None):
    """forward + backward on the GPU; returns numpy results and the status."""
    H, W, idx, logp, m = to_device(c, mask)
    chunk = chunk or c["chunk"]
    T, d, V, K = c["T"], c["d"], c["V"], c["K"]
    ws = workspace if workspace is not None else ckl.new_workspace(T, d, V, K, chunk)
    loss, lse = ckl.forward(H, W, idx, logp, m, chunk, workspace=ws)
    st_f = ckl.read_device_status(ws)
    gl = None if g is None else torch.tensor([g], dtype=torch.float32, device="cuda")
    dW = None
    if dW0 is not None:
        dW = torch.from_numpy(np.ascontiguousarray(dW0, dtype=np.float32)).cuda()
    dH, dW = ckl.backward(H, W, idx, logp, m, lse, grad_loss=gl, chunk=chunk, dW=dW,
                          accumulate_dW=dW0 is not None, workspace=ws)
    st_b = ckl.read_device_status(ws)
    torch.cuda.synchronize()
    return dict(loss=float(loss.item()), lse=lse.cpu().numpy().astype(np.float64),
                dH=dH.float().cpu().numpy().astype(np.float64),
                dW=dW.cpu().numpy().astype(np.float64), status_f=st_f, status_b=st_b)


def rel_fro(a, b) -> float:
    nb = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / nb) if nb > 0 else float(np.linalg.norm(a))


def errors(out, ref) -> dict:
    e = dict(loss_rel=abs(out["loss"] - ref["loss"]) / max(abs(ref["loss"]), 1e-30),
             lse_abs=float(np.abs(out["lse"] - ref["lse"]).max()) if ref["lse"].size else 0.0)
    if "dH" in ref:
        e["dH_rfro"] = rel_fro(out["dH"], ref["dH"])
    if "dW" in ref:
        e["dW_rfro"] = rel_fro(out["dW"], ref["dW"])
    return e


def assert_parity(out, ref, tag=""):
    e = errors(out, ref)
    print(f"[parity {tag}] " + " ".join(f"{k}={v:.3e}" for k, v in e.items()))
    assert out["status_f"][0] == 0 and out["status_b"][0] == 0, (out["status_f"], out["status_b"])
    if ref["loss"] == 0.0:
        assert abs(out["loss"]) <= 1e-6
    else:
        assert e["loss_rel"] <= LOSS_RTOL, e
    assert e["lse_abs"] <= LSE_ATOL, e
    if "dH_rfro" in e:
        assert e["dH_rfro"] <= GRAD_RFRO, e
    if "dW_rfro" in e:
        assert e["dW_rfro"] <= GRAD_RFRO, e
    return e


from ckl_synth import student_topk_torch  # noqa: E402,F401  (re-exported for the tests)
