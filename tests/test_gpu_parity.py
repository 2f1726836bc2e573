"""GPU parity: the CUDA library against the fp64 oracle, element by element.

Sizes here span several tiles in every dimension with ragged tails (T not a
multiple of 128, V not a multiple of 256 or 8, d not a multiple of 64), so the
oracle's dense form finishes in seconds.  Tolerances: loss relative 1e-3, lse
absolute 2e-3, dH and dW relative Frobenius 1e-2.
"""

import numpy as np
import pytest
import torch

import oracle
from ckl_synth import f32_to_bf16_bits, make_config, make_inputs
from gpu_util import assert_parity, run_library, to_device

pytestmark = pytest.mark.gpu


def _ref(c, g=1.0, mask="config"):
    m = c["mask"] if isinstance(mask, str) else mask
    return oracle.dense(c["H"], c["W"], c["idx"], c["logp"], m, g=g)


def test_tiny_config(gpu_lib):
    c = make_config("tiny")
    assert_parity(run_library(gpu_lib, c), _ref(c), "tiny")


@pytest.mark.parametrize("chunk", [64, 100, 128, 300])
def test_ragged_shapes_all_chunk_sizes(gpu_lib, chunk):
    c = make_inputs(300, 200, 1000, 16, seed=3, w_std=0.3, mask=("bernoulli", 0.2))
    assert_parity(run_library(gpu_lib, c, chunk=chunk), _ref(c), f"ragged chunk={chunk}")


def test_vocab_not_multiple_of_8_and_small_d(gpu_lib):
    c = make_inputs(130, 8, 1003, 5, seed=4, w_std=0.5)
    assert_parity(run_library(gpu_lib, c, chunk=64), _ref(c), "V=1003 d=8")


def test_many_row_blocks_and_vocab_tiles(gpu_lib):
    # 8 row blocks x 12 vocabulary tiles, d spanning 5 k-blocks + a tail
    c = make_inputs(1000, 328, 3000, 32, seed=5, w_std=0.1, mask=("tail", 37))
    assert_parity(run_library(gpu_lib, c, chunk=512), _ref(c), "1000x3000x328")


def test_sliced_backward_both_dw_schedules(gpu_lib):
    # Taller row chunks swept in vocabulary slabs: the first row chunk (2048
    # rows) deals its dW tiles in rounds, the second (1024 rows) gives each
    # slot a contiguous range; dH is summed in fp32 over the slabs.
    c = make_inputs(3072, 1024, 8192, 16, seed=17, w_std=0.05, mask=("bernoulli", 0.1))
    Cr, Sv, n = gpu_lib.backward_plan(3072, 1024, 8192, 16, 512)
    assert (Cr, n) == (2048, 4) and Cr * Sv <= 512 * 8192
    assert_parity(run_library(gpu_lib, c, chunk=512), _ref(c), "sliced 3072x8192x1024")


def test_forward_units_split_fastest_when_H_exceeds_L2(gpu_lib):
    # 25 row blocks of 256 x 4096 bf16 (52 MB) do not fit the forward's 48 MiB
    # L2 budget together: its units are numbered split-fastest
    c = make_inputs(6400, 4096, 1536, 8, seed=18, w_std=0.02, mask=("bernoulli", 0.1))
    assert_parity(run_library(gpu_lib, c, chunk=1024), _ref(c), "split-fastest forward")


def test_lse_is_bitwise_identical_across_chunk_sizes(gpu_lib):
    c = make_inputs(300, 200, 1000, 16, seed=6, w_std=0.3)
    outs = [run_library(gpu_lib, c, chunk=ch) for ch in (64, 128, 300)]
    for o in outs[1:]:
        assert np.array_equal(o["lse"], outs[0]["lse"])
        assert o["loss"] == outs[0]["loss"]


def test_runs_are_deterministic(gpu_lib):
    c = make_inputs(300, 200, 1000, 16, seed=7, w_std=0.3, mask=("bernoulli", 0.1))
    a = run_library(gpu_lib, c, chunk=128)
    b = run_library(gpu_lib, c, chunk=128)
    for k in ("lse", "dH", "dW"):
        assert np.array_equal(a[k], b[k]), k
    assert a["loss"] == b["loss"]


def test_upstream_gradient_and_dw_accumulation(gpu_lib):
    c = make_inputs(260, 64, 700, 8, seed=8, w_std=0.4)
    ref = _ref(c, g=0.37)
    dW0 = np.random.default_rng(0).normal(0, 1e-3, (700, 64))
    out = run_library(gpu_lib, c, chunk=100, g=0.37, dW0=dW0)
    ref = dict(ref)
    ref["dW"] = ref["dW"] + dW0.astype(np.float32)
    assert_parity(out, ref, "g=0.37 accumulate")


def test_all_positions_masked(gpu_lib):
    c = make_inputs(200, 64, 600, 8, seed=9, w_std=0.4)
    mask = np.zeros(200, np.uint8)
    out = run_library(gpu_lib, c, chunk=128, mask=mask)
    ref = _ref(c, mask=mask)
    assert out["loss"] == 0.0
    assert np.abs(out["dH"]).max() == 0.0 and np.abs(out["dW"]).max() == 0.0
    assert np.abs(out["lse"] - ref["lse"]).max() <= 2e-3


def test_empty_batch(gpu_lib):
    c = make_inputs(0, 64, 600, 8, seed=1, w_std=0.4)
    H, W, idx, logp, m = to_device(c)
    ws = gpu_lib.new_workspace(0, 64, 600, 8, 64)
    loss, lse = gpu_lib.forward(H, W, idx, logp, None, 64, workspace=ws)
    dW = torch.full((600, 64), 7.0, device="cuda")
    dH, dW = gpu_lib.backward(H, W, idx, logp, None, lse, chunk=64, dW=dW, workspace=ws)
    torch.cuda.synchronize()
    assert loss.item() == 0.0 and lse.numel() == 0 and dH.numel() == 0
    assert dW.abs().max().item() == 0.0


def test_repeated_teacher_ids(gpu_lib):
    c = make_inputs(150, 64, 500, 6, seed=10, w_std=0.4)
    idx = c["idx"].copy()
    idx[:, 3] = idx[:, 0]
    idx[::3, 5] = idx[::3, 1]
    c = dict(c, idx=idx)
    assert_parity(run_library(gpu_lib, c, chunk=64), _ref(c), "repeated ids")


@pytest.mark.parametrize("K", [1, 256])
def test_smallest_and_largest_K(gpu_lib, K):
    c = make_inputs(140, 64, 1500, K, seed=11, w_std=0.4)
    assert_parity(run_library(gpu_lib, c, chunk=128), _ref(c), f"K={K}")


@pytest.mark.parametrize("K", [257, 1000, 2048])
def test_large_K_takes_the_block_prep(gpu_lib, K):
    # K above 256: the prep runs one CTA per row; ids uniform and distinct per
    # row (a Zipf draw of 2048 distinct ids out of a few thousand is slow to
    # make), with repeats in some rows, -inf entries and a few masked rows
    rng = np.random.default_rng(K)
    c = make_inputs(150, 64, 3000, 4, seed=13, w_std=0.4, mask=("bernoulli", 0.1))
    idx = np.stack([rng.permutation(3000)[:K] for _ in range(150)]).astype(np.int32)
    idx[:10, 1] = idx[:10, 0]                      # repeated ids
    logp = np.log(rng.dirichlet(np.ones(K), 150)).astype(np.float32)
    logp[10:20, -5:] = -np.inf
    c = dict(c, idx=idx, logp=logp, K=K)
    assert_parity(run_library(gpu_lib, c, chunk=64), _ref(c), f"K={K}")
    out = run_library(gpu_lib, c, chunk=64)
    assert out["status_f"][0] == 0


def test_minus_inf_teacher_entries(gpu_lib):
    c = make_inputs(140, 64, 800, 10, seed=12, w_std=0.4)
    logp = c["logp"].copy()
    logp[:, -3:] = -np.inf
    c = dict(c, logp=logp)
    assert_parity(run_library(gpu_lib, c, chunk=128), _ref(c), "-inf entries")


def test_student_matching_teacher_gives_zero_loss(gpu_lib):
    # d = V, W = I, h = bf16(teacher log-probs) on the ids and -60 elsewhere.
    rng = np.random.default_rng(4)
    T, V, K = 130, 128, 6
    idx = np.stack([rng.permutation(V)[:K] for _ in range(T)]).astype(np.int32)
    h = np.full((T, V), -60.0, np.float32)
    np.put_along_axis(h, idx.astype(np.int64), rng.normal(0, 2, (T, K)).astype(np.float32), axis=1)
    H = f32_to_bf16_bits(h)
    logp = np.take_along_axis(oracle.widen_bf16(H), idx.astype(np.int64), axis=1).astype(np.float32)
    c = dict(T=T, d=V, V=V, K=K, chunk=64, H=H, W=f32_to_bf16_bits(np.eye(V, dtype=np.float32)),
             idx=idx, logp=logp, mask=None)
    out = run_library(gpu_lib, c)
    assert abs(out["loss"]) < 1e-4


def test_bad_teacher_id_is_reported_not_faulted(gpu_lib):
    c = make_inputs(64, 64, 300, 4, seed=13, w_std=0.4)
    idx = c["idx"].copy()
    idx[5, 2] = 300
    idx[9, 0] = -1
    H, W, idxd, logp, m = to_device(dict(c, idx=idx))
    ws = gpu_lib.new_workspace(64, 64, 300, 4, 64)
    gpu_lib.forward(H, W, idxd, logp, None, 64, workspace=ws)
    rc, word = gpu_lib.read_device_status(ws)
    assert rc == 5 and word & 1


def test_row_without_finite_logprob_is_reported(gpu_lib):
    c = make_inputs(64, 64, 300, 4, seed=14, w_std=0.4)
    logp = c["logp"].copy()
    logp[7, :] = -np.inf
    H, W, idx, lp, m = to_device(dict(c, logp=logp))
    ws = gpu_lib.new_workspace(64, 64, 300, 4, 64)
    gpu_lib.forward(H, W, idx, lp, None, 64, workspace=ws)
    rc, word = gpu_lib.read_device_status(ws)
    assert rc == 6 and word & 2


def test_autograd_function(gpu_lib):
    c = make_inputs(200, 64, 900, 8, seed=15, w_std=0.4, mask=("bernoulli", 0.2))
    H, W, idx, logp, m = to_device(c)
    H.requires_grad_(True)
    W32 = W.float().requires_grad_(True)
    Wb = W32.to(torch.bfloat16)
    loss = gpu_lib.chunked_kl_loss(H, Wb, idx, logp, m, 64) * 2.0
    loss.backward()
    ref = _ref(c, g=2.0)
    assert abs(loss.item() / 2.0 - ref["loss"]) <= 1e-3 * ref["loss"]
    gH = H.grad.float().cpu().numpy()
    assert np.linalg.norm(gH - ref["dH"]) / np.linalg.norm(ref["dH"]) < 1e-2
    gW = W32.grad.cpu().numpy()
    assert np.linalg.norm(gW - ref["dW"]) / np.linalg.norm(ref["dW"]) < 1e-2


def test_comparator_losses_agree_with_the_library(gpu_lib):
    # The dense and forward-chunked PyTorch losses that bench.py --compare
    # measures compute the same loss and gradients as the fused library.
    import bench

    c = make_inputs(400, 256, 3000, 16, seed=16, w_std=0.1, mask=("bernoulli", 0.1))
    H, W, idx, logp, m = to_device(c)
    out = run_library(gpu_lib, c, chunk=128)
    for fn in (lambda h, w: bench.dense_kl_torch(h, w, idx, logp, m),
               lambda h, w: bench.forward_chunked_kl_torch(h, w, idx, logp, m, 128)):
        h = H.detach().clone().requires_grad_(True)
        w = W.detach().clone().requires_grad_(True)
        loss = fn(h, w)
        loss.backward()
        assert abs(loss.item() - out["loss"]) <= 1e-3 * out["loss"]
        gh = h.grad.float().cpu().numpy()
        gw = w.grad.float().cpu().numpy()
        assert np.linalg.norm(gh - out["dH"]) / np.linalg.norm(out["dH"]) < 2e-2
        assert np.linalg.norm(gw - out["dW"]) / np.linalg.norm(out["dW"]) < 2e-2


def _first_dup_row(idx):
    return next((r for r in range(idx.shape[0]) if len(np.unique(idx[r])) < idx.shape[1]), -1)


@pytest.mark.parametrize("T,K", [(700, 100), (40, 2048), (5, 1), (0, 16)])
def test_duplicate_id_check_finds_the_first_repeat(gpu_lib, T, K):
    # distinct ids everywhere (-1), then repeats planted in three rows: the
    # smallest of them is reported; 700 rows > the CTAs' rows per pass
    rng = np.random.default_rng(T + K)
    idx = np.zeros((T, K), dtype=np.int32)
    for r in range(T):
        idx[r] = rng.permutation(200000)[:K]
    got = gpu_lib.find_duplicate_ids(torch.from_numpy(idx).cuda()).item()
    assert got == -1 == _first_dup_row(idx)
    if K > 1 and T > 0:
        for r in rng.choice(T, min(3, T), replace=False):
            a, b = rng.choice(K, 2, replace=False)
            idx[r, b] = idx[r, a]
        got = gpu_lib.find_duplicate_ids(torch.from_numpy(idx).cuda()).item()
        assert got == _first_dup_row(idx) >= 0
