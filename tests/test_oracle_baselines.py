"""Pins for the oracle's in-codec baselines (CPU only).

Two restrictions of the same codec serve as baselines for the JoLT allocation: residual only
(r_t = r_d = 0 for every layer-tensor, one fixed bit-width: per-row b-bit quantisation of the
rotated cache) and Tucker only (b = 0: the dual picks ranks and no residual is stored). The
"A JoLT for the KV Cache" abstract compares the joint allocation against quantisation-only and
decomposition-only methods; these are the plainest members of each family inside the codec.
"""
import numpy as np
import pytest

import synth
from oracle import jolt


def quant_plan(H, T, D, b, L=1, **kw):
    d = dict(L=L, H=H, T=T, D=D, has_v=False, budget=10 ** 9, num_groups=1, encoder="exact",
             rt_cap=0, bits=(b,))
    d.update(kw)
    return jolt.Plan(**d)


@pytest.fixture(scope="module")
def x0():
    K, _ = synth.gen_cache_numpy(synth.config(0))
    return K.astype(np.float64)          # [1][H][T][D]


def test_residual_only_allocation_and_bytes(x0):
    """rt_cap = 0 leaves the single grid point (0, 0): every unit takes (0, 0, b) and spends
    H T (D b / 8 + 2) bytes per layer-tensor, whatever the budget."""
    _, H, T, D = x0.shape
    for b in (2, 4, 8):
        p = quant_plan(H, T, D, b)
        assert p.R() == 0 and p.grid() == [(0, 0)]
        st, _ = jolt.encode(p, x0, None, seed=3, spec=True)
        assert st.alloc[0, 0].tolist() == [0, 0, b]
        assert jolt.layer_bytes(H, T, D, 0, 0, b) == H * T * (D * b // 8 + 2)


def test_residual_only_error_is_the_rotated_quantisation_error(x0):
    """Pi is orthogonal, so ||X - X_hat|| equals the norm of the quantisation error of the
    rotated rows; each entry's error is at most half a cell of the row's fp16 scale (plus the
    clamp where the fp16 scale rounded below the absmax)."""
    _, H, T, D = x0.shape
    b = 4
    p = quant_plan(H, T, D, b)
    st, dbg = jolt.encode(p, x0, None, seed=3, spec=True)
    Xh, _ = jolt.decode(st, rounded=False)
    Pi = dbg["Pi"]
    Y = np.einsum("htd,de->hte", x0[0], Pi)
    Yh = np.einsum("htd,de->hte", Xh[0], Pi)
    err = Y - Yh
    assert abs(np.linalg.norm(err) - np.linalg.norm(x0[0] - Xh[0])) <= 1e-9 * np.linalg.norm(x0[0])
    m = np.abs(Y).max(-1, keepdims=True)
    s = m.astype(np.float16).astype(np.float64)
    bound = s / 2 ** b + np.maximum(m - s, 0.0) + 1e-12 * m
    assert (np.abs(err) <= bound).all()


def test_residual_only_error_follows_the_uniform_model(x0):
    """The error of a b-bit mid-rise quantiser is ~uniform over a cell of width 2 s / 2^b
    (the pages' "approximately independent uniform" claim): mean squared error ~ cell^2 / 12,
    and one more bit divides it by ~4."""
    _, H, T, D = x0.shape
    mse = {}
    for b in (3, 4, 5, 6):
        p = quant_plan(H, T, D, b)
        st, dbg = jolt.encode(p, x0, None, seed=3, spec=False)
        Xh, _ = jolt.decode(st, rounded=False)
        Pi = dbg["Pi"]
        Y = np.einsum("htd,de->hte", x0[0], Pi)
        s = np.abs(Y).max(-1, keepdims=True).astype(np.float16).astype(np.float64)
        model = float(np.mean((2 * s / 2 ** b) ** 2 / 12.0))
        mse[b] = float(np.mean((x0[0] - Xh[0]) ** 2))
        assert 0.85 < mse[b] / model < 1.15, (b, mse[b] / model)
    for b in (3, 4, 5):
        assert 3.4 < mse[b] / mse[b + 1] < 4.6, (b, mse[b] / mse[b + 1])


def test_tucker_only_error_is_the_truncation_energy():
    """b = 0 everywhere: the reconstruction is the orthogonal projection onto the chosen
    factors, so ||X - X_hat||^2 = ||X||^2 - ||G||^2 (ideal mode, float64), and the allocation
    spends no residual bytes and stays within the budget."""
    cfg = synth.config(0)
    K, _ = synth.gen_cache_numpy(cfg)
    X = K.astype(np.float64)
    _, H, T, D = X.shape
    budget = X[0].size * 2 // 4
    p = jolt.Plan(L=1, H=H, T=T, D=D, has_v=False, budget=budget, num_groups=1, encoder="exact", bits=(0,))
    st, _ = jolt.encode(p, X, None, seed=5, spec=False)
    rt, rd, b = (int(v) for v in st.alloc[0, 0])
    assert b == 0 and rt > 0 and rd > 0
    assert jolt.layer_bytes(H, T, D, rt, rd, 0) <= budget
    Xh, _ = jolt.decode(st, rounded=False)
    G = np.asarray(st.lts[0].G, dtype=np.float64)
    lhs = np.sum((X[0] - Xh[0]) ** 2)
    rhs = np.sum(X[0] ** 2) - np.sum(G ** 2)
    assert abs(lhs - rhs) <= 1e-9 * np.sum(X[0] ** 2)
