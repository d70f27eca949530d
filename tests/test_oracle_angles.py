"""Pins for the oracle's principal angles, the checker behind the factor-subspace tolerance.

The GPU's factors are compared with the oracle's as subspaces (they are defined only up to the
signs and rotations of their columns), by the principal angles between the column spaces. These
tests fix that function against answers known in closed form, on bases that are neither
orthonormal nor aligned with the axes, so that a checker that skipped the orthonormalisation,
returned cosines instead of angles, or returned zeros would fail.
"""
import math

import numpy as np
import scipy.linalg

from oracle import jolt


def _rotate_and_mix(U, rng):
    """The same subspace in a rotated frame, spanned by a non-orthonormal basis."""
    n, k = U.shape
    Q = np.linalg.qr(rng.standard_normal((n, n)))[0]
    M = rng.standard_normal((k, k)) + 3.0 * np.eye(k)      # invertible column mixing
    return Q, Q @ U @ M


def test_two_planes_at_known_angles():
    """span(e1, e2) against span(cos a e1 + sin a e3, cos b e2 + sin b e4) in R^4: angles (a, b)."""
    rng = np.random.default_rng(3)
    a, b = 0.3, 0.7
    U1 = np.eye(4)[:, :2]
    U2 = np.zeros((4, 2))
    U2[0, 0], U2[2, 0] = math.cos(a), math.sin(a)
    U2[1, 1], U2[3, 1] = math.cos(b), math.sin(b)
    Q, V1 = _rotate_and_mix(U1, rng)
    V2 = Q @ U2 @ (rng.standard_normal((2, 2)) + 3.0 * np.eye(2))
    ang = np.sort(jolt.principal_angles(V1, V2))
    assert np.abs(ang - [a, b]).max() < 1e-12, ang


def test_subspace_against_itself_is_zero():
    rng = np.random.default_rng(4)
    U = rng.standard_normal((40, 6))
    _, V = _rotate_and_mix(np.linalg.qr(U)[0], rng)
    W = np.linalg.qr(V)[0] @ (rng.standard_normal((6, 6)) + 4.0 * np.eye(6))
    assert jolt.principal_angles(V, W).max() < 1e-7


def test_orthogonal_complement_is_a_right_angle():
    rng = np.random.default_rng(5)
    Q = np.linalg.qr(rng.standard_normal((10, 10)))[0]
    ang = jolt.principal_angles(Q[:, :4] @ (np.eye(4) + 0.5), Q[:, 4:8])
    assert np.abs(ang - math.pi / 2).max() < 1e-12


def test_small_angle_is_resolved():
    """An angle at the scale of the parity tolerance (1e-4 rad) comes out to 1e-10 absolute."""
    rng = np.random.default_rng(6)
    t = 1e-4
    U1 = np.eye(6)[:, :3]
    U2 = U1.copy()
    U2[:, 1] = math.cos(t) * np.eye(6)[:, 1] + math.sin(t) * np.eye(6)[:, 5]
    Q, V1 = _rotate_and_mix(U1, rng)
    V2 = Q @ U2
    ang = np.sort(jolt.principal_angles(V1, V2))
    assert abs(ang[-1] - t) < 1e-10 and ang[:2].max() < 1e-7, ang


def test_agrees_with_scipy_on_random_subspaces():
    """Against SciPy's independent routine (complement-based sines for small angles)."""
    rng = np.random.default_rng(7)
    for k in (1, 3, 8):
        A = rng.standard_normal((30, k))
        B = A + 0.05 * rng.standard_normal((30, k))
        got = np.sort(jolt.principal_angles(A, B))
        ref = np.sort(scipy.linalg.subspace_angles(A, B))
        assert np.abs(got - ref).max() < 1e-9
