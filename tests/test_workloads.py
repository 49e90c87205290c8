"""The seeded input recipe (bit_weight_quantized_nvq_b200/workloads.py), on
the CPU: determinism, independence of tensors, the thread split of weight
generation, and each distribution feature the workloads ask for (weight
std 0.02, 1 % of weight columns x20, 0.1 % of activation channels x50 in
every token, Student-t(4) small-batch activations)."""
import math
import os
import sys

import numpy as np
import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
from bit_weight_quantized_nvq_b200 import workloads as wl  # noqa: E402


def test_generators_are_deterministic_and_tensors_independent():
    a = wl.weights("t", "W", 300, 256)
    b = wl.weights("t", "W", 300, 256)
    assert a.dtype == np.float32 and a.shape == (300, 256)
    assert np.array_equal(a, b)
    assert not np.array_equal(a, wl.weights("t", "W2", 300, 256))
    assert not np.array_equal(a, wl.weights("t2", "W", 300, 256))
    x1 = wl.activations("t", "x", 3, 512)
    assert np.array_equal(x1, wl.activations("t", "x", 3, 512))
    assert not np.array_equal(x1, wl.activations("t", "y", 3, 512))


def test_weight_blocks_do_not_depend_on_the_thread_count():
    N = 3 * wl.ROW_BLOCK + 17   # four row blocks, a ragged last one
    one = wl.weights("t", "W", N, 64, threads=1)
    many = wl.weights("t", "W", N, 64, threads=4)
    assert np.array_equal(one, many)
    # distinct blocks draw distinct streams
    assert not np.array_equal(one[:wl.ROW_BLOCK], one[wl.ROW_BLOCK:2 * wl.ROW_BLOCK])


def test_weight_std_and_boosted_columns():
    N, K = 2048, 1024
    plain = wl.weights("t", "W", N, K)
    boosted = wl.weights("t", "W", N, K, boost_columns=True)
    cols = wl.boosted_columns("t", "W", K)
    assert len(cols) == math.ceil(0.01 * K) and len(set(cols.tolist())) == len(cols)
    assert np.all(np.diff(cols) > 0) and cols[0] >= 0 and cols[-1] < K
    # the boost multiplies exactly those columns by 20, nothing else changes
    others = np.setdiff1d(np.arange(K), cols)
    assert np.array_equal(boosted[:, others], plain[:, others])
    assert np.array_equal(boosted[:, cols], plain[:, cols] * np.float32(20.0))
    # N(0, 0.02^2): sample std within a few standard errors
    std = float(plain.std(dtype=np.float64))
    assert abs(std - 0.02) < 0.02 * 5 / math.sqrt(N * K / 2)
    assert abs(float(plain.mean(dtype=np.float64))) < 0.02 * 5 / math.sqrt(N * K)


def test_outlier_channels_are_the_same_in_every_token():
    M, K = 64, 4096
    plain = wl.activations("t", "x", M, K, "normal")
    out = wl.activations("t", "x", M, K, "normal", outliers=True)
    ch = wl.outlier_channels("t", "x", K)
    assert len(ch) == math.ceil(0.001 * K)
    others = np.setdiff1d(np.arange(K), ch)
    assert np.array_equal(out[:, others], plain[:, others])
    assert np.array_equal(out[:, ch], plain[:, ch] * np.float32(50.0))
    # N(0, 1)
    assert abs(float(plain.std(dtype=np.float64)) - 1.0) < 5 / math.sqrt(M * K / 2)


def test_student_t_activations_have_heavy_tails():
    x = wl.activations("t", "x", 16, 1 << 14, "student_t4").astype(np.float64)
    # Student-t with nu = 4: variance nu / (nu - 2) = 2, infinite kurtosis in
    # theory; a normal sample of this size has excess kurtosis ~0
    assert abs(x.var() - 2.0) < 0.15
    kurt = ((x - x.mean()) ** 4).mean() / x.var() ** 2 - 3.0
    assert kurt > 2.0
    with pytest.raises(ValueError):
        wl.activations("t", "x", 1, 64, "uniform")


def test_workload_cases_follow_the_recipe():
    W, x = wl.small_batch_case(2, 256, 64)
    assert W.shape == (64, 256) and x.shape == (2, 256)
    cols = wl.boosted_columns("small_batch", "W", 256)
    assert np.array_equal(W[:, cols], wl.weights("small_batch", "W", 64, 256)[:, cols] * 20)
    W, x = wl.prefill_case(8, 1024, 32)
    ch = wl.outlier_channels("prefill", "x", 1024)
    plain = wl.activations("prefill", "x", 8, 1024, "normal")
    assert np.array_equal(x[:, ch], plain[:, ch] * 50)
    assert [name for name, _, _ in wl.STACK_LINEARS] == ["q", "k", "v", "o", "up", "gate", "down"]
    assert sum(K * N for _, K, N in wl.STACK_LINEARS) * wl.STACK_LAYERS * 0.5625 / 1e9 == pytest.approx(17.93, abs=0.01)


def test_weight_rows_equal_the_leading_rows_of_the_full_matrix():
    full = wl.weights("wl_test", "W", 2500, 128, boost_columns=True)
    for rows in (1, 1024, 1500, 2500, 9999):
        part = wl.weight_rows("wl_test", "W", 2500, 128, rows, boost_columns=True)
        assert np.array_equal(part, full[:rows])
