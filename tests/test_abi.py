"""The C ABI without a GPU: the library loads, exports what ckl.h declares,
and rejects bad arguments on the host before touching the device."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "ckl.h")).read()
    return sorted(set(re.findall(r"CKL_API\s+[\w\s\*]+?\b(ckl_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def ckl():
    import chunked_kl_loss_ckl_b200 as m
    return m


def test_header_declares_the_entry_points():
    assert _declared() == ["ckl_backward", "ckl_backward_ex", "ckl_backward_f32",
                           "ckl_backward_plan", "ckl_backward_vocab_shard",
                           "ckl_combine_vocab_shards", "ckl_dh_to_bf16", "ckl_dp_finish",
                           "ckl_dp_local_stats", "ckl_find_duplicate_ids", "ckl_forward",
                           "ckl_forward_backward",
                           "ckl_forward_f32", "ckl_forward_static_scratch",
                           "ckl_forward_vocab_shard",
                           "ckl_read_device_status", "ckl_selftest_wait_timeout",
                           "ckl_single_pass_workspace_bytes",
                           "ckl_status_string", "ckl_topk_cache", "ckl_version",
                           "ckl_workspace_bytes", "ckl_workspace_bytes_f32"]


def test_library_exports_every_declared_symbol(ckl):
    raw = ctypes.CDLL(ckl.LIB_PATH)
    for name in _declared():
        assert hasattr(raw, name), name


def test_status_strings_and_version(ckl):
    for code in range(10):
        assert ckl.status_string(code) and ckl.status_string(code) != "unknown status"
    assert ckl.status_string(99) == "unknown status"
    assert ckl.lib.ckl_version() >= 100


def test_workspace_is_linear_in_T(ckl):
    d, V, K, chunk = 3072, 128256, 100, 1024
    ws = [ckl.lib.ckl_workspace_bytes(T, d, V, K, chunk) for T in (8192, 16384, 32768, 65536)]
    # constant second difference (up to 256-byte alignment) = a + b T
    slope1, slope2, slope3 = ws[1] - ws[0], (ws[2] - ws[1]) / 2, (ws[3] - ws[2]) / 4
    assert abs(slope1 - slope2) <= 2048 and abs(slope2 - slope3) <= 2048
    # the per-token part: sorted pairs, p log p, split partials, block sums
    assert abs(slope1 / 8192 - (K * 8 + 4 + 64 * 16 + 8 / 256)) < 1.0
    # the dZ buffer is chunk x round_up(V, 8) bf16
    assert ws[0] - 8192 * (K * 8 + 4 + 64 * 16) >= chunk * V * 2


def test_single_pass_workspace_adds_the_chunk_logits(ckl):
    # fp32 logits of one chunk, the rows' loss terms, and dZ for up to four
    # chunks (one dH / dW launch per four chunks) instead of one
    d, V, K, chunk = 3072, 128256, 100, 1024
    for T in (100, 2500, 8192, 32768):
        base = ckl.lib.ckl_workspace_bytes(T, d, V, K, chunk)
        sp = ckl.lib.ckl_single_pass_workspace_bytes(T, d, V, K, chunk)
        rows = min(chunk, T)
        group = min(4, -(-T // rows))
        extra = rows * ((V + 3) // 4 * 4) * 4 + T * 4 + (group - 1) * rows * (-(-V // 64) * 64) * 2
        assert extra <= sp - base <= extra + 1024 + d * group * rows * 2, T
    assert ckl.lib.ckl_single_pass_workspace_bytes(10, 60, 100, 4, 8) == 0


def test_backward_plan_fits_the_dz_buffer_and_covers_V(ckl):
    """The blocking of the backward: either the row-chunked schedule, or taller
    row chunks x vocabulary slabs whose dZ block fits the same chunk x V
    buffer, covering every column exactly once."""
    import numpy as np
    rng = np.random.default_rng(0)
    shapes = [(256, 64, 1024, 16, 64), (8192, 3072, 128256, 100, 1024),
              (32768, 4096, 128256, 100, 2048), (32768, 2880, 201088, 100, 2048),
              (262144, 4096, 128256, 100, 4096), (300, 200, 1000, 16, 100), (64, 64, 300, 4, 64),
              (1, 8, 1, 1, 1), (5000, 8, 70, 3, 7)]
    for _ in range(300):
        shapes.append((int(rng.integers(1, 70000)), 8 * int(rng.integers(1, 600)),
                       int(rng.integers(1, 300000)), int(rng.integers(1, 257)),
                       int(rng.integers(1, 9000))))
    n_sliced = 0
    for T, d, V, K, chunk in shapes:
        Cr, Sv, n = ckl.backward_plan(T, d, V, K, chunk)
        cap, Vp = min(chunk, T), -(-V // 64) * 64
        if n == 1:
            assert (Cr, Sv) == (cap, Vp), (T, d, V, K, chunk)
            continue
        n_sliced += 1
        assert T > cap and cap < Cr <= T
        assert Sv % 256 == 0 and Sv >= 256
        assert -(-Vp // Sv) == n and (n - 1) * Sv < V
        assert Cr * Sv <= cap * Vp, (T, d, V, K, chunk)
        # the sliced schedule's extra buffers are in the workspace
        ws = ckl.lib.ckl_workspace_bytes(T, d, V, K, chunk)
        assert ws >= cap * Vp * 2 + Cr * d * 6
    assert n_sliced > 50
    # the pages' configs: the 8K head is swept in slabs over all of its rows
    assert ckl.backward_plan(8192, 3072, 128256, 100, 1024) == (8192, 14336, 9)
    assert ckl.backward_plan(1000, 64, 5000, 8, 1000) == (1000, 5056, 1)  # one chunk


def test_f32_workspace_holds_fp32_dz(ckl):
    for T, d, V, K, chunk in ((256, 64, 1024, 16, 64), (8192, 3072, 128256, 100, 1024),
                              (100, 8, 1003, 5, 64)):
        f32 = ckl.lib.ckl_workspace_bytes_f32(T, d, V, K, chunk)
        dz = min(chunk, T) * (-(-V // 64) * 64)          # dZ entries
        assert f32 >= dz * 4 + T * K * 8                  # fp32 dZ + sorted pairs
        assert f32 > ckl.lib.ckl_workspace_bytes(T, d, V, K, chunk) - T * d * 4
    assert ckl.lib.ckl_workspace_bytes_f32(10, 60, 100, 4, 8) == 0


def test_workspace_rejects_bad_sizes(ckl):
    f = ckl.lib.ckl_workspace_bytes
    assert f(-1, 64, 100, 4, 8) == 0
    assert f(10, 60, 100, 4, 8) == 0      # d % 8 != 0
    assert f(10, 64, 0, 4, 8) == 0
    assert f(10, 64, 100, 0, 8) == 0
    assert f(10, 64, 100, 4, 0) == 0
    assert f(0, 64, 100, 4, 8) > 0         # an empty batch is allowed


def test_host_checks_return_before_any_device_work(ckl):
    L = ckl.lib
    nul = None
    # null inputs
    assert L.ckl_forward(nul, nul, nul, nul, nul, 4, 64, 100, 4, 8, nul, nul, nul, 0, nul,
                         nul) == 1
    fake = ctypes.c_void_p(4096)
    # bad sizes with non-null pointers
    assert L.ckl_forward(fake, fake, fake, fake, nul, 4, 60, 100, 4, 8, fake, fake, fake, 1 << 20,
                         nul, nul) == 1
    # misaligned H
    assert L.ckl_forward(ctypes.c_void_p(4098), fake, fake, fake, nul, 4, 64, 100, 4, 8, fake,
                         fake, fake, 1 << 20, nul, nul) == 1
    # workspace too small
    assert L.ckl_forward(fake, fake, fake, fake, nul, 4, 64, 100, 4, 8, fake, fake, fake, 16, nul,
                         nul) == 3
    # K above the supported maximum (2048)
    assert L.ckl_forward(fake, fake, fake, fake, nul, 4, 64, 100, 3000, 8, fake, fake, fake,
                         1 << 30, nul, nul) == 2
    # backward: null dW
    assert L.ckl_backward(fake, fake, fake, fake, nul, 4, 64, 100, 4, 8, fake, nul, fake, nul, 0,
                          fake, 1 << 20, nul, nul) == 1
    # single pass: null dW, null loss, and the larger workspace it needs
    assert L.ckl_forward_backward(fake, fake, fake, fake, nul, 4, 64, 100, 4, 8, nul, fake, fake,
                                  fake, nul, 0, fake, 1 << 20, nul, nul) == 1
    assert L.ckl_forward_backward(fake, fake, fake, fake, nul, 4, 64, 100, 4, 8, nul, nul, fake,
                                  fake, fake, 0, fake, 1 << 20, nul, nul) == 1
    small = L.ckl_workspace_bytes(4, 64, 100, 4, 8)
    assert small < L.ckl_single_pass_workspace_bytes(4, 64, 100, 4, 8)
    assert L.ckl_forward_backward(fake, fake, fake, fake, nul, 4, 64, 100, 4, 8, nul, fake, fake,
                                  fake, fake, 0, fake, small, nul, nul) == 3
    assert L.ckl_read_device_status(nul, nul, nul) == 1
    # the wait self-test: limit outside [1 ms, 4 s], or no workspace
    assert L.ckl_selftest_wait_timeout(10, fake, 1 << 20, nul) == 1
    assert L.ckl_selftest_wait_timeout(5_000_000_000, fake, 1 << 20, nul) == 1
    assert L.ckl_selftest_wait_timeout(50_000_000, nul, 1 << 20, nul) == 1
    assert L.ckl_selftest_wait_timeout(50_000_000, fake, 16, nul) == 1
    # top-K cache: K must be in [1, min(V, 2048)]
    assert L.ckl_topk_cache(fake, 4, 100, 0, fake, fake, nul, nul) == 1
    assert L.ckl_topk_cache(fake, 4, 100, 101, fake, fake, nul, nul) == 1
    assert L.ckl_topk_cache(fake, 4, 5000, 3000, fake, fake, nul, nul) == 2
    # data-parallel stats: null or misaligned buffers
    L.ckl_dp_local_stats.argtypes = [ctypes.c_void_p] * 3
    L.ckl_dp_finish.argtypes = [ctypes.c_void_p] * 5
    assert L.ckl_dp_local_stats(nul, fake, nul) == 1
    assert L.ckl_dp_local_stats(fake, ctypes.c_void_p(4100), nul) == 1
    assert L.ckl_dp_finish(nul, nul, fake, fake, nul) == 1
    assert L.ckl_dp_finish(fake, nul, fake, ctypes.c_void_p(4097), nul) == 1
    # vocabulary shards: the shard must lie inside [0, V) and be non-empty
    for vb, ve in ((-1, 10), (10, 10), (50, 101)):
        assert L.ckl_forward_vocab_shard(fake, fake, fake, fake, nul, 4, 64, 100, vb, ve, 4, 8,
                                         fake, fake, 1 << 20, nul, nul) == 1
        assert L.ckl_backward_vocab_shard(fake, fake, fake, fake, nul, 4, 64, 100, vb, ve, 4, 8,
                                          fake, nul, fake, fake, 0, fake, 1 << 20, nul, nul) == 1
    assert L.ckl_combine_vocab_shards(fake, 0, nul, 4, 4, fake, fake, fake, 1 << 20, nul,
                                      nul) == 1
    assert L.ckl_combine_vocab_shards(fake, 2, nul, 4, 4, fake, fake, fake, 16, nul, nul) == 3
    assert L.ckl_dh_to_bf16(fake, fake, 6, nul) == 1
    assert L.ckl_dh_to_bf16(ctypes.c_void_p(4100), fake, 8, nul) == 1
    # duplicate-id check: K in [1, 2048], aligned non-null buffers
    assert L.ckl_find_duplicate_ids(fake, 4, 0, fake, nul) == 1
    assert L.ckl_find_duplicate_ids(fake, -1, 4, fake, nul) == 1
    assert L.ckl_find_duplicate_ids(fake, 4, 4, nul, nul) == 1
    assert L.ckl_find_duplicate_ids(nul, 4, 4, fake, nul) == 1
    assert L.ckl_find_duplicate_ids(fake, 4, 4, ctypes.c_void_p(4098), nul) == 1
    assert L.ckl_find_duplicate_ids(fake, 4, 3000, fake, nul) == 2


def test_static_scratch_limit_is_checked_on_the_host(ckl):
    """ckl_forward_static_scratch rejects a problem one token past the limit
    ckl.h states (T = 18 355 at K = 100) before any CUDA call.  Without a
    device, a problem at the limit gets as far as the device query."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is visible: the GPU test checks the limit with real buffers")
    vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32
    f = ctypes.CDLL(ckl.LIB_PATH).ckl_forward_static_scratch
    f.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i32, vp, vp, vp, vp]
    fake = ctypes.c_void_p(1 << 20)
    assert f(fake, fake, fake, fake, None, 18356, 64, 1000, 100, fake, fake, None, None) == 3
    assert f(fake, fake, fake, fake, None, 18355, 64, 1000, 100, fake, fake, None, None) == 4
