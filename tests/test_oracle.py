"""Pins for the fp64 oracle: what the pages and the mathematics fix.

None of these compares the oracle with itself.  Each checks a property any
correct implementation must have: Gibbs' inequality, the zero case, the
pages' statement that dense and chunked compute the same loss ("Tối ưu hóa
chi phí chưng cất tri thức ...", section "Hai thay đổi hệ thống"), central
finite differences for the closed-form gradient, reductions to library
routines (K = 1 is cross-entropy, K = V with all ids is the full KL), a
closed form (W = 0), and invariants of the definition.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from ckl_synth import f32_to_bf16_bits, make_inputs


def _rand_case(T=37, d=24, V=50, K=6, seed=1, mask_frac=0.2, w_std=0.4):
    c = make_inputs(T, d, V, K, seed=seed, w_std=w_std, mask=("bernoulli", mask_frac))
    return c


def _values(c):
    return oracle.widen_bf16(c["H"]), oracle.widen_bf16(c["W"])


# --- the input widening -------------------------------------------------------

def test_widen_bf16_every_bit_pattern_matches_torch():
    # All 65 536 bf16 patterns, against torch's own bf16 -> fp64 conversion:
    # finite values equal (signed zeros and subnormals included), infinities
    # with their sign, NaN patterns NaN.
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    got = oracle.widen_bf16(bits)
    ref = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).double().numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))
    assert got.dtype == np.float64 and got.shape == bits.shape
    # a few by hand: 1.0, -2.0, the smallest subnormal, the largest finite
    assert oracle.widen_bf16(np.array([0x3F80, 0xC000, 0x0001, 0x7F7F], np.uint16)).tolist() == [
        1.0, -2.0, 2.0 ** -133, (2 - 2 ** -7) * 2.0 ** 127]


# --- Gibbs' inequality and the zero case -----------------------------------

def test_kl_nonnegative_per_row():
    for seed in range(5):
        c = _rand_case(seed=seed)
        out = oracle.dense(c["H"], c["W"], c["idx"], c["logp"], c["mask"])
        assert (out["kl"] >= -1e-12).all()
        assert out["loss"] >= 0.0


def test_kl_zero_when_student_matches_teacher_exactly():
    # Logit-level: z = log p on the K ids and -inf elsewhere gives q = p on
    # the support and no mass outside it, so every KL term vanishes.
    rng = np.random.default_rng(3)
    T, V, K = 5, 40, 7
    idx = np.stack([rng.permutation(V)[:K] for _ in range(T)]).astype(np.int32)
    logp = rng.normal(0, 2, (T, K)).astype(np.float32)
    p, logp_n = oracle.renormalise_topk(logp)
    Z = np.full((T, V), -np.inf)
    np.put_along_axis(Z, idx.astype(np.int64), logp_n + 3.0, axis=1)  # any shift
    lse = oracle.logsumexp_rows(Z)
    kl = oracle.kl_rows(Z, lse, idx, p, logp_n)
    assert np.abs(kl).max() < 1e-14


def test_kl_zero_via_identity_head():
    # Through H and W: d = V, W = I (exact in bf16), h_t = bf16(log p) on the
    # ids and -60 elsewhere; the teacher log-probs are the same bf16 values,
    # so the only residual is the e^-60 mass outside the support (~1e-25),
    # below fp64 rounding of the O(1) terms.
    rng = np.random.default_rng(4)
    T, V, K = 6, 32, 5
    idx = np.stack([rng.permutation(V)[:K] for _ in range(T)]).astype(np.int32)
    raw = rng.normal(0, 2, (T, K)).astype(np.float32)
    h = np.full((T, V), -60.0, dtype=np.float32)
    np.put_along_axis(h, idx.astype(np.int64), raw, axis=1)
    H = f32_to_bf16_bits(h)
    hv = oracle.widen_bf16(H)
    logp = np.take_along_axis(hv, idx.astype(np.int64), axis=1).astype(np.float32)
    W = f32_to_bf16_bits(np.eye(V, dtype=np.float32))
    out = oracle.dense(H, W, idx, logp)
    assert abs(out["loss"]) < 1e-14
    assert np.abs(out["kl"]).max() < 1e-14


# --- the pages: dense and chunked compute the same loss ---------------------

@pytest.mark.parametrize("chunk", [1, 7, 64, 37])
def test_chunked_equals_dense(chunk):
    c = _rand_case(T=37)
    a = oracle.dense(c["H"], c["W"], c["idx"], c["logp"], c["mask"], g=0.7)
    b = oracle.chunked(c["H"], c["W"], c["idx"], c["logp"], c["mask"], g=0.7, chunk=chunk)
    assert abs(a["loss"] - b["loss"]) <= 1e-12 * abs(a["loss"])
    np.testing.assert_allclose(b["lse"], a["lse"], rtol=1e-13, atol=0)
    np.testing.assert_allclose(b["dH"], a["dH"], rtol=1e-11, atol=1e-15)
    np.testing.assert_allclose(b["dW"], a["dW"], rtol=1e-11, atol=1e-15)


# --- the closed-form gradient against central differences -------------------

def test_gradient_matches_central_differences():
    rng = np.random.default_rng(11)
    T, d, V, K = 6, 5, 11, 3
    H = rng.normal(0, 1, (T, d))
    W = rng.normal(0, 0.5, (V, d))
    idx = np.stack([rng.permutation(V)[:K] for _ in range(T)]).astype(np.int32)
    logp = rng.normal(0, 2, (T, K)).astype(np.float32)
    mask = np.ones(T, np.uint8)
    mask[2] = 0
    g = 1.3
    out = oracle.dense_values(H, W, idx, logp, mask, g=g)
    h = 1e-6

    def L(Hx, Wx):
        return g * oracle.dense_values(Hx, Wx, idx, logp, mask, want_grad=False)["loss"]

    num_dH = np.zeros_like(H)
    for i in range(T):
        for j in range(d):
            Hp, Hm = H.copy(), H.copy()
            Hp[i, j] += h
            Hm[i, j] -= h
            num_dH[i, j] = (L(Hp, W) - L(Hm, W)) / (2 * h)
    num_dW = np.zeros_like(W)
    for i in range(V):
        for j in range(d):
            Wp, Wm = W.copy(), W.copy()
            Wp[i, j] += h
            Wm[i, j] -= h
            num_dW[i, j] = (L(H, Wp) - L(H, Wm)) / (2 * h)
    rel = lambda a, b: np.linalg.norm(a - b) / np.linalg.norm(b)
    assert rel(out["dH"], num_dH) < 1e-6
    assert rel(out["dW"], num_dW) < 1e-6
    assert np.abs(out["dH"][2]).max() == 0.0   # the masked row


# --- reductions to library routines ------------------------------------------

def test_k1_is_cross_entropy():
    # K = 1: p = 1, log p = 0, so KL_t = -log q_{t, idx_t}: cross-entropy.
    c = make_inputs(29, 16, 70, 1, seed=5, w_std=0.5, mask=("bernoulli", 0.25))
    Hv, Wv = _values(c)
    out = oracle.dense(c["H"], c["W"], c["idx"], c["logp"], c["mask"], g=1.0)
    Ht = torch.tensor(Hv, requires_grad=True)
    Wt = torch.tensor(Wv, requires_grad=True)
    m = torch.tensor(c["mask"] != 0)
    tgt = torch.tensor(c["idx"][:, 0], dtype=torch.long)
    ce = torch.nn.functional.cross_entropy(Ht @ Wt.T, tgt, reduction="none")
    loss = ce[m].mean()
    loss.backward()
    assert abs(out["loss"] - loss.item()) < 1e-12
    np.testing.assert_allclose(out["dH"], Ht.grad.numpy(), rtol=1e-10, atol=1e-14)
    np.testing.assert_allclose(out["dW"], Wt.grad.numpy(), rtol=1e-10, atol=1e-14)


def test_k_equals_v_is_full_kl():
    # Every vocabulary id cached once (a permutation): the loss is the full
    # KL(p || q) over the vocabulary, torch's kl_div with log targets.
    rng = np.random.default_rng(8)
    T, d, V = 13, 12, 17
    c = make_inputs(T, d, V, V, seed=9, w_std=0.5)
    idx = np.stack([rng.permutation(V) for _ in range(T)]).astype(np.int32)
    logp = c["logp"]
    Hv, Wv = _values(c)
    out = oracle.dense(c["H"], c["W"], idx, logp, None, g=1.0)
    Ht = torch.tensor(Hv, requires_grad=True)
    Wt = torch.tensor(Wv, requires_grad=True)
    logp_t = torch.log_softmax(torch.tensor(logp, dtype=torch.float64), dim=1)
    # teacher log-probs placed at their vocabulary ids
    target = torch.empty(T, V, dtype=torch.float64)
    target.scatter_(1, torch.tensor(idx, dtype=torch.long), logp_t)
    logq = torch.log_softmax(Ht @ Wt.T, dim=1)
    loss = torch.nn.functional.kl_div(logq, target, reduction="sum", log_target=True) / T
    loss.backward()
    assert abs(out["loss"] - loss.item()) < 1e-12
    np.testing.assert_allclose(out["dH"], Ht.grad.numpy(), rtol=1e-10, atol=1e-14)
    np.testing.assert_allclose(out["dW"], Wt.grad.numpy(), rtol=1e-10, atol=1e-14)


def test_repeated_id_reduces_to_entropy_plus_cross_entropy():
    # Both entries of a row name the same id v: sum_k p_k = 1, so
    # KL_t = sum_k p_k log p_k - log q_v = -entropy(p) + CE(v).
    from scipy.stats import entropy

    c = make_inputs(9, 8, 30, 2, seed=12, w_std=0.5)
    idx = np.repeat(c["idx"][:, :1], 2, axis=1)
    out = oracle.dense(c["H"], c["W"], idx, c["logp"], None)
    Hv, Wv = _values(c)
    ce = torch.nn.functional.cross_entropy(torch.tensor(Hv @ Wv.T),
                                           torch.tensor(idx[:, 0], dtype=torch.long),
                                           reduction="none").numpy()
    p = np.exp(c["logp"].astype(np.float64))
    p /= p.sum(axis=1, keepdims=True)
    want = -entropy(p, axis=1) + ce
    np.testing.assert_allclose(out["kl"], want, rtol=1e-12, atol=1e-13)


# --- a closed form ------------------------------------------------------------

def test_zero_head_closed_form():
    # W = 0: every z_tv = 0, q = 1/V, lse = log V.  With a uniform teacher
    # (equal log-probs) p = 1/K and KL_t = log(V / K).  The gradient is
    # G_tv = (1/N)(1/V - [v in row t]/K): dH = G W = 0, dW = G^T H.
    T, d, V, K = 11, 6, 40, 4
    c = make_inputs(T, d, V, K, seed=2)
    W = np.zeros((V, d), np.uint16)
    logp = np.full((T, K), -1.25, np.float32)
    out = oracle.dense(c["H"], W, c["idx"], logp, None)
    assert abs(out["loss"] - math.log(V / K)) < 1e-13
    np.testing.assert_allclose(out["lse"], np.full(T, math.log(V)), rtol=1e-15)
    assert np.abs(out["dH"]).max() == 0.0
    Hv = oracle.widen_bf16(c["H"])
    G = np.full((T, V), 1.0 / V)
    for t in range(T):
        G[t, c["idx"][t]] -= 1.0 / K
    np.testing.assert_allclose(out["dW"], (G / T).T @ Hv, rtol=1e-12, atol=1e-15)


# --- invariants of the definition ----------------------------------------------

def test_dw_column_sum_is_zero_and_masked_rows_have_no_gradient():
    c = _rand_case(T=40, mask_frac=0.3)
    out = oracle.dense(c["H"], c["W"], c["idx"], c["logp"], c["mask"])
    # sum_v G_tv = 0 for every row, hence 1^T dW = 0
    assert np.abs(out["dW"].sum(axis=0)).max() < 1e-13 * np.abs(out["dW"]).max() * out["dW"].shape[0]
    masked = c["mask"] == 0
    assert masked.any()
    assert np.abs(out["dH"][masked]).max() == 0.0
    assert np.isfinite(out["lse"]).all()


def test_teacher_logprob_shift_invariance():
    c = _rand_case()
    a = oracle.dense(c["H"], c["W"], c["idx"], c["logp"], c["mask"])
    b = oracle.dense(c["H"], c["W"], c["idx"], c["logp"] + np.float32(3.5), c["mask"])
    assert abs(a["loss"] - b["loss"]) < 1e-6 * a["loss"]
    np.testing.assert_allclose(b["dW"], a["dW"], rtol=1e-5, atol=1e-12)


def test_row_permutation_equivariance():
    c = _rand_case(T=33)
    perm = np.random.default_rng(7).permutation(33)
    a = oracle.dense(c["H"], c["W"], c["idx"], c["logp"], c["mask"])
    b = oracle.dense(c["H"][perm], c["W"], c["idx"][perm], c["logp"][perm], c["mask"][perm])
    assert abs(a["loss"] - b["loss"]) < 1e-12 * a["loss"]
    np.testing.assert_allclose(b["lse"], a["lse"][perm], rtol=1e-14)
    np.testing.assert_allclose(b["dH"], a["dH"][perm], rtol=1e-12, atol=1e-16)
    np.testing.assert_allclose(b["dW"], a["dW"], rtol=1e-11, atol=1e-15)


def test_all_masked_gives_zero_loss_and_gradients():
    c = _rand_case(T=12)
    mask = np.zeros(12, np.uint8)
    out = oracle.dense(c["H"], c["W"], c["idx"], c["logp"], mask)
    assert out["loss"] == 0.0 and out["N"] == 0
    assert np.abs(out["dH"]).max() == 0.0 and np.abs(out["dW"]).max() == 0.0
    assert np.isfinite(out["lse"]).all()


def test_minus_inf_teacher_entries_contribute_nothing():
    # A -inf cached log-prob means p = 0: dropping that entry changes nothing.
    c = _rand_case(T=10, K=5)
    logp = c["logp"].copy()
    logp[:, -1] = -np.inf
    a = oracle.dense(c["H"], c["W"], c["idx"], logp, c["mask"])
    b = oracle.dense(c["H"], c["W"], c["idx"][:, :-1], c["logp"][:, :-1], c["mask"])
    assert abs(a["loss"] - b["loss"]) < 1e-12 * b["loss"]
    np.testing.assert_allclose(a["dW"], b["dW"], rtol=1e-12, atol=1e-15)


def test_bad_inputs_are_rejected():
    c = _rand_case(T=4, K=3)
    bad = c["idx"].copy()
    bad[1, 2] = c["V"]
    with pytest.raises(ValueError):
        oracle.dense(c["H"], c["W"], bad, c["logp"])
    lp = c["logp"].copy()
    lp[2, :] = -np.inf
    with pytest.raises(ValueError):
        oracle.dense(c["H"], c["W"], c["idx"], lp)
    lp = c["logp"].copy()
    lp[0, 0] = np.nan
    with pytest.raises(ValueError):
        oracle.dense(c["H"], c["W"], c["idx"], lp)


# --- the sampled-row helpers used at full size agree with the dense form ------

def test_rows_subset_and_dw_from_subset_match_dense():
    c = _rand_case(T=30, V=70, mask_frac=0.0)
    rows = np.array([0, 5, 17, 29])
    mask = np.zeros(30, np.uint8)
    mask[rows] = 1
    out = oracle.dense(c["H"], c["W"], c["idx"], c["logp"], mask, g=0.5)
    sub = oracle.rows_subset(c["H"], c["W"], c["idx"], c["logp"], rows, N=4, g=0.5,
                             mask=mask, block_v=16)
    np.testing.assert_allclose(sub["lse"], out["lse"][rows], rtol=1e-14)
    np.testing.assert_allclose(sub["kl"], out["kl"][rows], rtol=1e-13)
    np.testing.assert_allclose(sub["dH"], out["dH"][rows], rtol=1e-12, atol=1e-16)
    vrows = np.array([0, 3, 69, 40])
    dw = oracle.dw_rows_from_subset(c["H"], sub["G"], rows, vrows)
    np.testing.assert_allclose(dw, out["dW"][vrows], rtol=1e-12, atol=1e-16)


# --- the offline top-K cache producer ------------------------------------------

def test_topk_cache_matches_torch_topk_and_log_softmax():
    # Distinct logits: the selection is torch.topk's, the log-probs are
    # torch.log_softmax's at those ids.
    rng = np.random.default_rng(21)
    T, V, K = 7, 300, 10
    # distinct bf16 values: every pattern with exponent field 121..130, both signs
    pos = np.arange(121 * 128, 131 * 128, dtype=np.uint16)
    pool = np.concatenate([pos, pos | np.uint16(0x8000)])
    bits = rng.choice(pool, T * V, replace=False).astype(np.uint16).reshape(T, V)
    zb = oracle.widen_bf16(bits)
    assert len(np.unique(zb)) == T * V  # exactly representable, no ties
    ids, logp = oracle.topk_cache(bits, K)
    zt = torch.tensor(zb)
    want_ids = torch.topk(zt, K, dim=1).indices.numpy()
    assert np.array_equal(ids, want_ids)
    want = torch.log_softmax(zt, dim=1).gather(1, torch.tensor(want_ids)).numpy()
    np.testing.assert_allclose(logp, want, rtol=0, atol=1e-12)


def test_topk_cache_breaks_ties_by_smaller_id():
    bits = f32_to_bf16_bits(np.array([[1.0, 3.0, 3.0, 2.0, 3.0, 0.5]], np.float32))
    ids, logp = oracle.topk_cache(bits, 4)
    assert ids.tolist() == [[1, 2, 4, 3]]
    assert logp[0, 0] == logp[0, 1] == logp[0, 2]
