"""Pins for the randomized Hadamard rotation of the oracle (CPU only).

The structured Johnson-Lindenstrauss rotation Pi = diag(s) H / sqrt(D) (Ailon & Chazelle 2006)
replaces the dense Haar matrix as an option: H is the Sylvester Hadamard matrix and s a vector of
random signs drawn from the seed's rotation stream. Applying it costs one fast Walsh-Hadamard
transform (log2 D butterfly stages) instead of a D x D product.
"""
import numpy as np
import pytest
import scipy.linalg

import synth
from oracle import jolt, numerics as nm
from oracle import stream as ostream


@pytest.mark.parametrize("D", [2, 4, 16, 128])
def test_hadamard_matrix_is_sylvesters(D):
    assert np.array_equal(nm.hadamard_matrix(D), scipy.linalg.hadamard(D).astype(np.float64))


def test_rotation_is_orthogonal_with_equal_magnitudes():
    Pi = nm.hadamard_rotation(42, 128)
    assert np.abs(Pi.T @ Pi - np.eye(128)).max() <= 1e-15
    assert np.allclose(np.abs(Pi), 1.0 / np.sqrt(128), rtol=0, atol=0)


def test_signs_reproducible_and_balanced():
    s = nm.hadamard_signs(42, 128)
    assert np.array_equal(s, nm.hadamard_signs(42, 128))
    assert not np.array_equal(s, nm.hadamard_signs(43, 128))
    neg = np.stack([nm.hadamard_signs(k, 128) for k in range(200)]) < 0
    assert abs(neg.mean() - 0.5) < 0.01            # 25,600 draws: 4 sigma is 0.0125


def test_fast_transform_equals_the_dense_product():
    """x Pi = FWHT(x * s) / sqrt(D): in-place butterflies (a + b, a - b) with strides 1, 2, ..."""
    rng = np.random.default_rng(0)
    X = rng.standard_normal((64, 128))
    s = nm.hadamard_signs(7, 128)
    Y = X * s
    h = 1
    while h < 128:
        Y = Y.reshape(64, -1, 2, h)
        a, b = Y[:, :, 0, :].copy(), Y[:, :, 1, :].copy()
        Y = np.stack([a + b, a - b], axis=2).reshape(64, 128)
        h *= 2
    Y = Y / np.sqrt(128)
    assert np.abs(Y - X @ nm.hadamard_rotation(7, 128)).max() <= 1e-13


def test_codec_with_hadamard_rotation():
    """The quantiser's error keeps the uniform model after the structured rotation, the stream
    records the rotation kind and decoding the parsed stream uses it."""
    cfg = synth.config(0)
    K, _ = synth.gen_cache_numpy(cfg)
    X = K.astype(np.float64)
    _, H, T, D = X.shape
    p = jolt.Plan(L=1, H=H, T=T, D=D, has_v=False, budget=10 ** 9, num_groups=1, encoder="exact",
                  rt_cap=0, bits=(4,), rotation="hadamard")
    st, dbg = jolt.encode(p, X, None, seed=3, spec=False)
    assert np.array_equal(dbg["Pi"], nm.hadamard_rotation(3, D))
    Xh, _ = jolt.decode(st, rounded=False)
    Y = np.einsum("htd,de->hte", X[0], dbg["Pi"])
    s = np.abs(Y).max(-1, keepdims=True).astype(np.float16).astype(np.float64)
    ratio = float(np.mean((X[0] - Xh[0]) ** 2)) / float(np.mean((2 * s / 16) ** 2 / 12.0))
    assert 0.85 < ratio < 1.15
    st, _ = jolt.encode(p, X, None, seed=3, spec=True)          # storage rounding, as serialized
    st2 = ostream.parse(ostream.serialize(st))
    assert st2.rotation == "hadamard"
    assert np.array_equal(jolt.decode(st, rounded=False)[0], jolt.decode(st2, rounded=False)[0])
