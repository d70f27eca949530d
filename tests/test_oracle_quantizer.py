"""Pins for the oracle's residual quantiser, bit packing and error model (CPU only)."""
import json
import math
import os

import numpy as np
import pytest

from conftest import GOLDEN
from oracle import jolt, numerics as nm


def test_worked_example():
    g = json.load(open(os.path.join(GOLDEN, "quantizer_example.json")))
    y = np.array([g["y"]])
    s, c, _ = jolt.quantize_rows(y, g["b"])
    assert s[0] == g["scale"]
    assert c[0].tolist() == g["codes"]
    assert jolt.pack_codes(c, g["b"])[0].tobytes().hex() == g["packed_hex"]
    assert np.allclose(jolt.dequantize_rows(s, c, g["b"])[0], g["dequant"])


@pytest.mark.parametrize("b", range(1, 9))
def test_pack_unpack_roundtrip(b):
    rng = np.random.default_rng(b)
    c = rng.integers(0, 2 ** b, (5, 7, 128))
    p = jolt.pack_codes(c, b)
    assert p.shape == (5, 7, 128 * b // 8) and p.dtype == np.uint8
    assert np.array_equal(jolt.unpack_codes(p, b, 128), c)


def test_packing_bit_order_little_endian():
    # code i sits at bits [i b, i b + b): with b = 3, codes (1, 2, 4, 7, 0, 5, 3, 6)
    c = np.array([[1, 2, 4, 7, 0, 5, 3, 6]])
    bits = "".join(format(v, "03b")[::-1] for v in c[0])           # LSB first per code
    expect = bytes(int(bits[8 * k:8 * k + 8][::-1], 2) for k in range(3))
    assert jolt.pack_codes(c, 3)[0].tobytes() == expect


@pytest.mark.parametrize("b", [1, 2, 3, 4, 8])
def test_boundaries_go_up_and_cells_are_exhaustive(b):
    s = 1.0
    half = 2 ** (b - 1)
    k = np.arange(0, 2 ** b + 1)
    y = (k - half) / half * s                                  # every cell boundary in [-s, s]
    y = np.concatenate([y, [0.0]])
    _, c, _ = jolt.quantize_rows(y[None, :], b, spec=False)
    expect = np.clip(np.concatenate([k, [half]]), 0, 2 ** b - 1)
    assert c[0].tolist() == expect.tolist()


@pytest.mark.parametrize("b", range(1, 9))
def test_error_at_most_half_a_cell(b):
    rng = np.random.default_rng(10 + b)
    Y = rng.standard_normal((2000, 128)) * rng.uniform(0.01, 3.0, (2000, 1))
    s, c, _ = jolt.quantize_rows(Y, b, spec=False)
    err = np.abs(jolt.dequantize_rows(s, c, b) - Y)
    delta = 2.0 * s / 2 ** b
    assert (err <= delta[:, None] / 2 * (1 + 1e-12)).all()


def test_spec_scale_is_fp16_absmax_and_clamps():
    rng = np.random.default_rng(4)
    Y = rng.standard_normal((500, 128))
    s, c, _ = jolt.quantize_rows(Y, 4, spec=True)
    assert np.array_equal(s, nm.round_fp16_sat(np.abs(Y).max(1)))
    assert c.min() >= 0 and c.max() <= 15


def test_zero_rows():
    s, c, d = jolt.quantize_rows(np.zeros((3, 16)), 3)
    assert (s == 0).all() and (c == 0).all() and np.isinf(d).all()
    assert (jolt.dequantize_rows(s, c, 3) == 0).all()


def test_uniform_error_model_on_rotated_rows():
    """Rotated Gaussian rows: mean squared error is close to Delta^2 / 12 (uniform model)."""
    rng = np.random.default_rng(7)
    Pi = nm.haar_rotation(1, 128)
    Y = (rng.standard_normal((20000, 128)) * np.linspace(0.1, 3, 128)) @ Pi
    for b in (2, 4, 6):
        s, c, _ = jolt.quantize_rows(Y, b, spec=False)
        mse = ((jolt.dequantize_rows(s, c, b) - Y) ** 2).mean(1)
        model = (2.0 * s / 2 ** b) ** 2 / 12.0
        assert abs(mse.mean() / model.mean() - 1.0) < 0.03


def test_kappa_closed_forms_and_monte_carlo():
    g = json.load(open(os.path.join(GOLDEN, "kappa_closed_forms.json")))
    for D, v in g["cases"]:
        assert abs(jolt.kappa(D) - v) < 1e-10
    rng = np.random.default_rng(0)
    z = rng.standard_normal((200000, 128))
    mc = (z ** 2).max(1).mean()
    assert abs(jolt.kappa(128) / mc - 1.0) < 0.01


def test_phi_matches_measured_whitened_error():
    """phi(b) * ||y||^2 predicts the b-bit error of Gaussian (whitened) rows."""
    rng = np.random.default_rng(3)
    Y = rng.standard_normal((40000, 128))
    kap = jolt.kappa(128)
    # The uniform-cell model is coarse at 1 bit (two cells over a Gaussian row): 15% there.
    for b, tol in ((1, 0.16), (2, 0.08), (3, 0.05), (5, 0.05)):
        s, c, _ = jolt.quantize_rows(Y, b, spec=False)
        err = ((jolt.dequantize_rows(s, c, b) - Y) ** 2).sum()
        assert abs(err / (Y ** 2).sum() / jolt.phi(b, kap) - 1.0) < tol
    assert jolt.phi(0, kap) == 1.0
