"""GPU parity at the five workloads' full sizes, in the launch configuration
bench.py times (the workload's own chunk and mask).

The oracle cannot build a [T, V] grid of this size on the host, so each
check uses outputs it can compute one row at a time, or a property that
holds at any size:

* run A (the workload as given): lse and dH on sampled rows against the
  oracle (dH needs only its own row and N), and the column sum of dW, which
  is zero in exact arithmetic (every row of the logit gradient sums to 0);
* run B (the same launch with the mask restricted to a few rows): the loss is
  then the mean KL of those rows, and dW = sum over them of G_t^T h_t, so
  both are compared with the oracle directly; dH must be exactly 0 on every
  other row.

Tolerances: loss relative 1e-3, lse absolute 2e-3, dH and dW relative
Frobenius 1e-2 (over the sampled rows).
"""

import numpy as np
import pytest
import torch

import oracle
from ckl_synth import make_config
from gpu_util import GRAD_RFRO, LOSS_RTOL, LSE_ATOL, rel_fro, student_topk_torch, to_device

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

def _config(name):
    topk = student_topk_torch if name == "oss" else None
    return make_config(name, seed=0, student_topk=topk)


def _sample_rows(c, n=10, seed=123):
    T = c["T"]
    rows = {0, 1, T // 2, T - 1}
    if c["mask"] is not None and (c["mask"] == 0).any():
        rows.add(int(np.nonzero(c["mask"] == 0)[0][0]))
    rng = np.random.default_rng(seed)
    rows.update(int(r) for r in rng.choice(T, n, replace=False))
    return np.array(sorted(rows))


def _run(ckl, c, mask, rows, vrows=None, single_pass=False):
    """One forward + backward at full size (two calls, or the single-pass
    call); returns only what the checks use (the full outputs are gigabytes)."""
    H, W, idx, logp, m = to_device(c, mask)
    T, d, V, K, chunk = c["T"], c["d"], c["V"], c["K"], c["chunk"]
    if single_pass:
        ws = torch.empty(ckl.single_pass_workspace_bytes(T, d, V, K, chunk), dtype=torch.uint8,
                         device="cuda")
        loss, lse, dH, dW = ckl.forward_backward(H, W, idx, logp, m, chunk=chunk, workspace=ws)
        st_f = st_b = ckl.read_device_status(ws)
    else:
        ws = ckl.new_workspace(T, d, V, K, chunk)
        loss, lse = ckl.forward(H, W, idx, logp, m, chunk, workspace=ws)
        st_f = ckl.read_device_status(ws)
        dH, dW = ckl.backward(H, W, idx, logp, m, lse, chunk=chunk, workspace=ws)
        st_b = ckl.read_device_status(ws)
    r = torch.from_numpy(rows).cuda()
    out = dict(loss=float(loss.item()), lse=lse[r].double().cpu().numpy(),
               dH=dH[r].double().cpu().numpy(), status=(st_f[0], st_b[0]),
               colsum_rel=float(dW.double().sum(0).norm() / dW.double().norm()))
    if vrows is not None:
        out["dW"] = dW[torch.from_numpy(vrows).cuda()].double().cpu().numpy()
        keep = torch.ones(T, dtype=torch.bool, device="cuda")
        keep[r] = False
        out["dH_others_max"] = float(dH[keep].float().abs().max()) if keep.any() else 0.0
    del H, W, idx, logp, m, ws, dH, dW
    torch.cuda.empty_cache()
    return out


@pytest.mark.parametrize("name,single_pass", [("8k", False), ("32k", False), ("oss", False),
                                              ("256k", False), ("8k", True), ("oss", True)])
def test_full_size_workload(gpu_lib, name, single_pass):
    c = _config(name)
    T, V = c["T"], c["V"]
    if single_pass:
        name += " single pass"
    # --- run A: the workload as given
    rows = _sample_rows(c)
    a = _run(gpu_lib, c, "config", rows, single_pass=single_pass)
    assert a["status"] == (0, 0)
    assert np.isfinite(a["loss"]) and a["loss"] > 0
    N = T if c["mask"] is None else int((c["mask"] != 0).sum())
    ref = oracle.rows_subset(c["H"], c["W"], c["idx"], c["logp"], rows, N=N, mask=c["mask"])
    lse_err = float(np.abs(a["lse"] - ref["lse"]).max())
    dh_err = rel_fro(a["dH"], ref["dH"])
    print(f"[{name} run A] lse_abs={lse_err:.3e} dH_rfro(rows)={dh_err:.3e} "
          f"|colsum dW|/|dW|={a['colsum_rel']:.3e} loss={a['loss']:.6f}")
    assert lse_err <= LSE_ATOL
    assert dh_err <= GRAD_RFRO
    assert a["colsum_rel"] <= GRAD_RFRO
    # --- run B: same launch, mask restricted to a few rows
    rows_b = _sample_rows(c, n=12, seed=7)
    mask = np.zeros(T, np.uint8)
    mask[rows_b] = 1
    vset = set(range(64)) | set(int(v) for v in c["idx"][rows_b].ravel()) | {V - 1}
    vset |= set(int(v) for v in np.random.default_rng(11).choice(V, 1024, replace=False))
    vrows = np.array(sorted(vset))
    b = _run(gpu_lib, c, mask, rows_b, vrows, single_pass=single_pass)
    assert b["status"] == (0, 0)
    ref_b = oracle.rows_subset(c["H"], c["W"], c["idx"], c["logp"], rows_b, N=len(rows_b),
                               mask=mask)
    want_loss = float(ref_b["kl"].mean())
    loss_err = abs(b["loss"] - want_loss) / want_loss
    ref_dw = oracle.dw_rows_from_subset(c["H"], ref_b["G"], rows_b, vrows)
    dw_err = rel_fro(b["dW"], ref_dw)
    dh_err_b = rel_fro(b["dH"], ref_b["dH"])
    print(f"[{name} run B] loss_rel={loss_err:.3e} dW_rfro(vrows)={dw_err:.3e} "
          f"dH_rfro(rows)={dh_err_b:.3e} lse_abs={np.abs(b['lse'] - ref_b['lse']).max():.3e}")
    assert loss_err <= LOSS_RTOL
    assert dw_err <= GRAD_RFRO
    assert dh_err_b <= GRAD_RFRO
    assert b["dH_others_max"] == 0.0
