"""The seeded input generator: determinism, layout and the stated recipes."""

import numpy as np
import torch

from ckl_synth import (CONFIGS, bf16_bits_to_f32, f32_to_bf16_bits, make_config,
                       make_inputs)


def test_bf16_rounding_matches_torch_round_to_nearest_even():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.normal(0, 1, 100000).astype(np.float32),
                        np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875, 3.0e38, -1e-40],
                                 np.float32)])
    ours = f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    back = bf16_bits_to_f32(ours)
    assert np.array_equal(back, torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_same_seed_same_arrays_and_different_seed_differs():
    a = make_config("tiny", seed=0)
    b = make_config("tiny", seed=0)
    c = make_config("tiny", seed=1)
    for k in ("H", "W", "idx", "logp"):
        assert np.array_equal(a[k], b[k])
        assert not np.array_equal(a[k], c[k])


def test_tiny_shapes_and_teacher_cache_layout():
    c = make_config("tiny")
    T, d, V, K = (CONFIGS["tiny"][k] for k in ("T", "d", "V", "K"))
    assert c["H"].shape == (T, d) and c["H"].dtype == np.uint16
    assert c["W"].shape == (V, d) and c["W"].dtype == np.uint16
    assert c["idx"].shape == (T, K) and c["idx"].dtype == np.int32
    assert c["logp"].shape == (T, K) and c["logp"].dtype == np.float32
    assert c["mask"] is None
    assert all(len(set(r)) == K for r in c["idx"])
    assert (c["idx"] >= 0).all() and (c["idx"] < V).all()
    # log-softmax over K: each row sums to one in probability, descending
    np.testing.assert_allclose(np.exp(c["logp"].astype(np.float64)).sum(1), 1.0, rtol=1e-5)
    assert (np.diff(c["logp"], axis=1) <= 0).all()
    # tiny W has variance 1/d
    w = bf16_bits_to_f32(c["W"])
    assert abs(w.std() - d ** -0.5) < 0.01


def test_zipf_first_draw_follows_the_law():
    # The first id of each row is one plain Zipf(1.1) draw.
    V = 1000
    c = make_inputs(20000, 8, V, 3, seed=4)
    first = c["idx"][:, 0]
    w = np.arange(1, V + 1, dtype=np.float64) ** -1.1
    w /= w.sum()
    for v in (0, 1, 2, 10):
        assert abs((first == v).mean() - w[v]) < 4 * np.sqrt(w[v] / 20000) + 1e-3


def test_masks():
    m = make_inputs(100, 8, 50, 3, mask=("tail", 5))["mask"]
    assert m.sum() == 95 and (m[-5:] == 0).all()
    m = make_inputs(64, 8, 50, 3, mask=("packed", 4, 16, 2))["mask"]
    assert m.sum() == 56
    for s in range(4):
        assert (m[s * 16 + 14:(s + 1) * 16] == 0).all() and (m[s * 16:s * 16 + 14] == 1).all()
    m = make_inputs(10, 8, 50, 3, mask=("rows", [1, 7]))["mask"]
    assert list(np.nonzero(m)[0]) == [1, 7]


def test_neighbourhood_case_takes_half_from_student_top():
    c = make_inputs(30, 16, 400, 10, neighbourhood=(20, 5), w_std=0.3, seed=3)
    hf = bf16_bits_to_f32(c["H"])
    wf = bf16_bits_to_f32(c["W"])
    z = hf @ wf.T
    top = np.argsort(-z, axis=1)[:, :20]
    for t in range(30):
        assert set(c["idx"][t, :5]) <= set(top[t])
        assert len(set(c["idx"][t])) == 10


def test_fp32_option_keeps_the_same_draws_unrounded():
    from ckl_synth import f32_to_bf16_bits, make_inputs
    a = make_inputs(50, 24, 300, 7, seed=3, w_std=0.3, mask=("bernoulli", 0.2))
    b = make_inputs(50, 24, 300, 7, seed=3, w_std=0.3, mask=("bernoulli", 0.2), fp32=True)
    assert b["H"].dtype == np.float32 and b["W"].dtype == np.float32
    assert np.array_equal(f32_to_bf16_bits(b["H"]), a["H"])
    assert np.array_equal(f32_to_bf16_bits(b["W"]), a["W"])
    for k in ("idx", "logp", "mask"):
        assert np.array_equal(a[k], b[k])
