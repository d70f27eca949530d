"""Pins for the oracle's storage rounding, generator and Haar rotation (CPU only)."""
import json
import math
import os

import numpy as np
import pytest
import torch
from scipy import stats

from conftest import GOLDEN
from oracle import numerics as nm


def test_bf16_rounding_matches_torch_conversion():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(200000) * 10.0 ** rng.integers(-30, 30, 200000),
                        rng.standard_normal(1000) * 1e-39])          # bf16 subnormals
    x32 = x.astype(np.float32)
    ref = torch.from_numpy(x32).to(torch.bfloat16).to(torch.float32).numpy().astype(np.float64)
    got = nm.round_bf16(x32.astype(np.float64))
    assert np.array_equal(got, ref)


def test_bf16_round_half_even_ties():
    # 1 + 2^-8 lies halfway between 1 and 1 + 2^-7: ties go to the even significand (1.0).
    assert nm.round_bf16(np.array([1.0 + 2.0 ** -8]))[0] == 1.0
    assert nm.round_bf16(np.array([1.0 + 3 * 2.0 ** -8]))[0] == 1.0 + 2.0 ** -6


def test_fp16_rounding_matches_numpy_and_saturates():
    rng = np.random.default_rng(1)
    x = rng.standard_normal(200000) * 10.0 ** rng.uniform(-9, 4.5, 200000)
    x = x[np.abs(x) < 65504]
    ref = x.astype(np.float16).astype(np.float64)
    assert np.array_equal(nm.round_fp16_sat(x), ref)
    assert nm.round_fp16_sat(np.array([1e6, -1e6]))[0] == 65504.0
    assert nm.round_fp16_sat(np.array([1e6, -1e6]))[1] == -65504.0


def test_bit_patterns_roundtrip():
    v = nm.round_bf16(np.random.default_rng(2).standard_normal(1000))
    assert np.array_equal(nm.bf16_from_bits(nm.bf16_bits(v)), v)
    h = nm.round_fp16_sat(np.random.default_rng(3).standard_normal(1000))
    assert np.array_equal(nm.fp16_from_bits(nm.fp16_bits(h)), h)


def test_splitmix64_published_outputs():
    g = json.load(open(os.path.join(GOLDEN, "splitmix64_state0.json")))
    out = nm.splitmix64_outputs(g["state"], len(g["outputs_hex"]))
    assert [format(int(v), "016x") for v in out] == g["outputs_hex"]


def test_stream_words_are_splitmix_sequences_from_the_key():
    key = nm.stream_key(42, 7)
    assert np.array_equal(nm.stream_words(42, 7, 0, 16), nm.splitmix64_outputs(key, 16))
    assert np.array_equal(nm.stream_words(42, 7, 5, 3), nm.splitmix64_outputs(key, 8)[5:])
    assert nm.stream_key(42, 7) != nm.stream_key(42, 8) != nm.stream_key(43, 7)


def test_uniforms_and_gaussians_have_the_right_law():
    w = nm.stream_words(5, 3, 0, 400000)
    u = nm.uniform53(w)
    assert u.min() >= 0.0 and u.max() < 1.0
    assert stats.kstest(u, "uniform").pvalue > 1e-3
    z = nm.gaussians(5, 3, 400001)
    assert abs(z.mean()) < 5e-3 and abs(z.var() - 1.0) < 1e-2
    assert abs(stats.kurtosis(z, fisher=False) - 3.0) < 3e-2
    assert stats.kstest(z, "norm").pvalue > 1e-3
    # an odd count is the prefix of the even count
    assert np.array_equal(nm.gaussians(5, 3, 7), nm.gaussians(5, 3, 8)[:7])


@pytest.mark.parametrize("D", [8, 64, 128])
def test_haar_rotation_orthogonal_and_unique_qr(D):
    Pi = nm.haar_rotation(42, D)
    assert np.abs(Pi.T @ Pi - np.eye(D)).max() <= 1e-12
    assert abs(abs(np.linalg.det(Pi)) - 1.0) < 1e-10
    # G = Pi R with R upper triangular and a positive diagonal (the unique QR of G)
    G = nm.gaussians(42, nm.STREAM_ROTATION, D * D).reshape(D, D)
    R = Pi.T @ G
    assert np.abs(np.tril(R, -1)).max() < 1e-10
    assert (np.diag(R) > 0).all()
    assert np.array_equal(nm.haar_rotation(42, D), Pi)          # regenerated bit-identically
    assert not np.allclose(nm.haar_rotation(43, D), Pi)


def test_haar_rotation_law_first_column_uniform_on_sphere():
    # Pi e_1 is uniform on the sphere: each coordinate squared has mean 1/D.
    D = 16
    cols = np.stack([nm.haar_rotation(s, D)[:, 0] for s in range(400)])
    m = (cols ** 2).mean(0)
    assert np.abs(m - 1.0 / D).max() < 0.03


def test_sketch_matrix_on_bf16_grid_and_seeded():
    Om = nm.sketch_matrix(42, 3, 64, 24)
    assert Om.shape == (64, 24)
    assert np.array_equal(nm.round_bf16(Om), Om)
    assert np.array_equal(nm.sketch_matrix(42, 3, 64, 24), Om)
    assert not np.array_equal(nm.sketch_matrix(42, 4, 64, 24), Om)
    z = nm.gaussians(42, nm.STREAM_SKETCH0 + 3, 64 * 24).reshape(64, 24)
    assert np.abs(Om - z).max() <= 2.0 ** -8 * np.abs(z).max()
