"""GPU parity of the teacher top-K cache producer against the oracle.

The ids must match exactly (the selection compares bf16 values, exact in any
precision; equal logits go to the smaller id); the log-probabilities within
1e-4 absolute (fp32 log-sum-exp over the row).
"""

import numpy as np
import pytest
import torch

import oracle
from ckl_synth import f32_to_bf16_bits

pytestmark = pytest.mark.gpu

LOGP_ATOL = 1e-4
LOGP_RTOL = 1e-6   # log-probs of logits far from 1 carry fp32 relative error


def _run(ckl, bits, K):
    x = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda()
    idx, logp, st = ckl.topk_cache(x, K)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), logp.cpu().numpy().astype(np.float64), int(st.item())


def _check(ckl, bits, K, rows=None):
    idx, logp, st = _run(ckl, bits, K)
    assert st == 0
    sel = slice(None) if rows is None else rows
    ref_idx, ref_logp = oracle.topk_cache(bits[sel], K)
    assert np.array_equal(idx[sel], ref_idx)
    assert (np.abs(logp[sel] - ref_logp) <= LOGP_ATOL + LOGP_RTOL * np.abs(ref_logp)).all()
    return idx, logp


def test_teacher_sized_rows(gpu_lib):
    rng = np.random.default_rng(1)
    bits = f32_to_bf16_bits(rng.normal(0, 2, (48, 128256)).astype(np.float32))
    _check(gpu_lib, bits, 100)


def test_unaligned_rows_and_heavy_ties(gpu_lib):
    # V not a multiple of 8 (scalar loads); logits on a 0.25 grid tie often
    rng = np.random.default_rng(2)
    z = np.round(rng.normal(0, 2, (33, 1001)) * 4) / 4
    _check(gpu_lib, f32_to_bf16_bits(z.astype(np.float32)), 16)


@pytest.mark.parametrize("K", [1, 300])
def test_k_one_and_k_equals_v(gpu_lib, K):
    rng = np.random.default_rng(3)
    _check(gpu_lib, f32_to_bf16_bits(rng.normal(0, 1, (17, 300)).astype(np.float32)), K)


def test_signed_zeros_and_wide_value_range(gpu_lib):
    # -0 and +0 are equal logits (ties by id); values spread over many binades
    # so the histogram window has to slide below the largest key
    rng = np.random.default_rng(4)
    z = rng.normal(0, 1, (9, 5000)).astype(np.float32)
    z[0, :50] = -0.0
    z[0, 50:100] = 0.0
    z[0, 100:] = -rng.uniform(1, 2, 4900)
    z[1] = np.exp(rng.uniform(-80, 80, 5000)).astype(np.float32) * rng.choice([-1, 1], 5000)
    _check(gpu_lib, f32_to_bf16_bits(z), 80)


def test_too_many_ties_is_reported_and_other_rows_are_right(gpu_lib):
    rng = np.random.default_rng(5)
    z = rng.normal(0, 1, (4, 10000)).astype(np.float32)
    z[2] = 1.5                                    # 10 000 equal logits
    bits = f32_to_bf16_bits(z)
    idx, logp, st = _run(gpu_lib, bits, 10)
    assert st & 8
    rows = np.array([0, 1, 3])
    ref_idx, ref_logp = oracle.topk_cache(bits[rows], 10)
    assert np.array_equal(idx[rows], ref_idx)
    assert np.abs(logp[rows] - ref_logp).max() <= LOGP_ATOL


@pytest.mark.parametrize("V", [1001, 1024])
def test_many_rows_per_cta_heavy_ties_every_row(gpu_lib, V):
    # far more rows than the launch has CTAs, so every CTA handles many rows
    # in turn (state left from a previous row would show); logits on a 0.25
    # grid tie often, also at the K-th value; V = 1001 takes the scalar loads
    rng = np.random.default_rng(7)
    z = np.round(rng.normal(0, 2, (1500, V)) * 4) / 4
    z[1400] = 0.5                                   # a row of equal logits, late
    z[1401, ::3] = 3.0                              # many ties above the K-th value
    _check(gpu_lib, f32_to_bf16_bits(z.astype(np.float32)), 16)


def test_teacher_sized_many_rows_sampled(gpu_lib):
    # 1500 teacher-sized rows (several per CTA); ids checked exactly on a
    # seeded sample of 160 rows, most of them past the first row of each CTA,
    # plus a late row whose top values tie heavily
    rng = np.random.default_rng(8)
    T, V, K = 1500, 128256, 100
    z = rng.normal(0, 2, (T, V)).astype(np.float32)
    z[1333, rng.choice(V, 400, replace=False)] = 7.5      # 400 equal top logits
    bits = f32_to_bf16_bits(z)
    del z
    sample = np.unique(np.concatenate([rng.choice(296, 32, replace=False),
                                       296 + rng.choice(T - 296, 128, replace=False),
                                       [1333, T - 1]]))
    _check(gpu_lib, bits, K, rows=sample)


def test_rows_whose_large_values_crowd_into_few_threads(gpu_lib):
    # The streaming pass thresholds at the K-th largest of its 256 threads'
    # maxima; thread t reads the 8-element vectors t, t + 256, ...  Giving
    # every element of threads 0-11 a large value (about 6000 elements) puts
    # far more than 2048 of them above that threshold, so the row is handed
    # to the histogram kernel, which must still return the exact top K.
    rng = np.random.default_rng(9)
    T, V, K = 6, 128256, 100
    z = rng.normal(0, 2, (T, V)).astype(np.float32)
    vec = np.arange(V // 8)
    crowd = np.concatenate([8 * vec[vec % 256 == t][:, None] + np.arange(8)[None, :]
                            for t in range(12)]).ravel()
    assert crowd.size > 2048 + K
    for r in (1, 4):
        z[r, crowd] = 100.0 + rng.normal(0, 1, crowd.size).astype(np.float32)
    _check(gpu_lib, f32_to_bf16_bits(z), K)


@pytest.mark.parametrize("V,K", [(1024, 200), (2048, 256), (4096, 256), (8, 8)])
def test_rows_with_fewer_vectors_than_threads(gpu_lib, V, K):
    # 8-element vectors: 1024 logits give 128 thread maxima, fewer than K =
    # 200, so every element is a candidate (and they are sorted, not ranked);
    # 2048 and 4096 give exactly and twice 256 maxima at the largest K the
    # streaming form takes; V = K = 8 is one vector
    rng = np.random.default_rng(V + K)
    z = np.round(rng.normal(0, 2, (37, V)) * 8) / 8   # ties on a 1/8 grid
    _check(gpu_lib, f32_to_bf16_bits(z.astype(np.float32)), K)


@pytest.mark.parametrize("n_top", [300, 700])
def test_many_marked_vectors_rank_or_fallback(gpu_lib, n_top):
    # n_top equal top logits, each in its own 8-element vector: 300 are
    # ranked in the streaming kernel (more candidates than threads), 700 mark
    # more vectors than its list holds and the row goes to the histogram
    # kernel; both must return the first K of the ties by id
    rng = np.random.default_rng(11 + n_top)
    T, V, K = 4, 128256, 100
    z = rng.normal(0, 2, (T, V)).astype(np.float32)
    for r in (0, 2):
        vecs = rng.choice(V // 8, n_top, replace=False)
        z[r, 8 * vecs + rng.integers(0, 8, n_top)] = 11.0
    _check(gpu_lib, f32_to_bf16_bits(z), K)


@pytest.mark.parametrize("V", [262144, 262152])
def test_widest_rows_with_and_without_vector_marks(gpu_lib, V):
    # 262 144 is the widest row whose 8-element vector maxima the streaming
    # kernel keeps in shared memory (64 KB per CTA, fewer CTAs per SM); one
    # vector wider and it reads the row a second time to gather instead.
    # Row 3 has 150 equal logits across the K-th value.
    rng = np.random.default_rng(10)
    z = rng.normal(0, 2, (5, V)).astype(np.float32)
    z[3, rng.choice(V, 150, replace=False)] = 9.0
    _check(gpu_lib, f32_to_bf16_bits(z), 100)


def test_cache_feeds_the_loss(gpu_lib):
    # The producer's output is a valid teacher cache for the fused loss.
    from ckl_synth import make_inputs
    from gpu_util import assert_parity, run_library

    rng = np.random.default_rng(6)
    c = make_inputs(200, 64, 2000, 20, seed=17, w_std=0.3)
    teacher = f32_to_bf16_bits(rng.normal(0, 2, (200, 2000)).astype(np.float32))
    idx, logp, st = _run(gpu_lib, teacher, 20)
    assert st == 0
    c = dict(c, idx=idx.astype(np.int32), logp=logp.astype(np.float32))
    ref = oracle.dense(c["H"], c["W"], c["idx"], c["logp"], None)
    assert_parity(run_library(gpu_lib, c, chunk=64), ref, "top-K cache -> loss")
