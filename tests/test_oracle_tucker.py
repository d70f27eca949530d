"""Pins for the oracle's partial Tucker factors, core, sketch and error table (CPU only)."""
import numpy as np
import pytest

import synth
from oracle import jolt, numerics as nm


def tiny_plan(H, T, D, **kw):
    d = dict(L=1, H=H, T=T, D=D, has_v=False, budget=10 ** 9, num_groups=1, encoder="exact",
             rank_step=1, rt_cap=10 ** 6, bits=(0, 1, 2, 3, 4))
    d.update(kw)
    return jolt.Plan(**d)


def forced(plan, X, alloc, spec=False, seed=7):
    a = np.zeros((plan.num_groups, 2, 3), dtype=np.int64)
    a[0, 0] = alloc
    st, dbg = jolt.encode(plan, X[None], None, seed, spec=spec, alloc=a)
    Xh, _ = jolt.decode(st, rounded=False)
    return st, dbg, Xh[0]


@pytest.fixture(scope="module")
def x0():
    K, _ = synth.gen_cache_numpy(synth.config(0))
    return K[0].astype(np.float64)


def test_full_rank_b0_reproduces_x():
    rng = np.random.default_rng(0)
    X = rng.standard_normal((2, 8, 8))
    for enc in ("exact", "sketch"):
        p = tiny_plan(2, 8, 8, encoder=enc, oversample=16)
        _, _, Xh = forced(p, X, (8, 8, 0))
        assert jolt.rel_frob(X, Xh) <= 1e-12


@pytest.mark.parametrize("enc", ["exact", "sketch"])
def test_exact_multilinear_rank_recovered(enc):
    rng = np.random.default_rng(1)
    H, T, D, rt, rd = 4, 12, 16, 3, 5
    U = np.linalg.qr(rng.standard_normal((T, rt)))[0]
    V = np.linalg.qr(rng.standard_normal((D, rd)))[0]
    C = rng.standard_normal((H, rt, rd))
    X = np.einsum("tr,hre,de->htd", U, C, V)
    p = tiny_plan(H, T, D, encoder=enc, rt_cap=4, oversample=2)
    _, _, Xh = forced(p, X, (rt, rd, 0))
    assert jolt.rel_frob(X, Xh) <= 1e-10


def test_factors_match_svd_of_the_unfoldings(x0):
    """eigh of the Grams and SVD of the mode-2 / mode-3 unfoldings give the same columns."""
    H, T, D = x0.shape
    UD, wD = jolt.feature_factor(x0)
    Usvd = np.linalg.svd(x0.reshape(H * T, D).T, full_matrices=False)[0]
    UT, wT = jolt.exact_token_factor(x0, 32)
    Tsvd = np.linalg.svd(x0.transpose(1, 0, 2).reshape(T, H * D), full_matrices=False)[0]
    for U, S, w in ((UD, Usvd, wD), (UT, Tsvd, wT)):
        gaps = -np.diff(w) / w[0]
        k = int(np.argmax(gaps[:24] < 1e-4)) if (gaps[:24] < 1e-4).any() else 24
        cos = np.abs(np.sum(U[:, :k] * S[:, :k], axis=0))
        assert (cos > 1 - 1e-8).all()
    assert np.allclose(wD[:10], np.linalg.svd(x0.reshape(H * T, D), compute_uv=False)[:10] ** 2)


def test_sign_rule():
    U = np.array([[0.1, -0.9, 0.5], [-0.8, 0.1, -0.5], [0.2, 0.3, 0.1]])
    s = jolt.column_signs(U)
    assert s.tolist() == [-1.0, -1.0, 1.0]          # tie in column 2 -> first index decides


def test_table_is_the_true_b0_error_for_orthonormal_factors(x0):
    """Ideal mode: E(r_t, r_d) equals ||X - U_T G U_D^T||^2 at every grid point (Pythagoras)."""
    p = jolt.Plan(L=1, H=8, T=256, D=128, has_v=False, budget=262144, num_groups=1,
                  encoder="exact")
    a = jolt.analyse_layer_tensor(p, x0, 42, 0, spec=False)
    for i, (rt, rd) in enumerate(p.grid()):
        if rt % 32 or rd % 32:
            continue
        rec = jolt.tucker_part(a["U_T"][:, :rt], a["Gmax"][:, :rt, :rd], a["U_D"][:, :rd], 8, 256, 128)
        true = ((x0 - rec) ** 2).sum()
        assert abs(a["E"][i] - true) <= 1e-9 * a["xx"]
    E = a["E"][1:].reshape(p.R() // 16, 8)
    assert (np.diff(E, axis=0) <= 1e-12).all() and (np.diff(E, axis=1) <= 1e-12).all()


def test_sketch_core_identity(x0):
    H, T, D = x0.shape
    UT, WR, B, Q, _ = jolt.sketch_token_factor(x0, 48, 16, 1, 42, 0)
    UD, _ = jolt.feature_factor(x0)
    assert np.abs(Q.T @ Q - np.eye(Q.shape[1])).max() < 1e-12
    G1 = jolt.core_sketch(B, WR, UD, H, D)
    G2 = jolt.core_exact(x0, UT, UD)
    assert np.abs(G1 - G2).max() <= 1e-10 * np.abs(G2).max()


def test_full_width_sketch_equals_exact_factor(x0):
    """With l = T the sketch spans R^T and the Rayleigh-Ritz factor is the exact one."""
    H, T, D = x0.shape
    UT_s = jolt.sketch_token_factor(x0, 40, T - 40, 0, 42, 0)[0]
    UT_e, w = jolt.exact_token_factor(x0, 40)
    assert (w[39] - w[40]) / w[0] > 1e-4
    assert jolt.principal_angles(UT_s, UT_e).max() < 1e-6


def test_power_iteration_improves_the_sketch(x0):
    """Randomized subspace iteration: more power iterations never hurt the captured energy."""
    H, T, D = x0.shape
    A = jolt.token_unfolding(x0)
    caught = []
    for q in (0, 1, 2):
        UT = jolt.sketch_token_factor(x0, 32, 16, q, 42, 0)[0]
        caught.append(np.linalg.norm(UT.T @ A) ** 2)
    best = np.sum(np.linalg.svd(A, compute_uv=False)[:32] ** 2)
    assert caught[0] <= caught[1] * (1 + 1e-9) <= caught[2] * (1 + 1e-9) <= best * (1 + 1e-9)
    assert caught[1] >= 0.99 * best


def test_monotone_in_bits_and_ranks():
    """Config-0 layer, seeds 0..9: rel. error falls with b at fixed ranks, and with ranks at fixed b."""
    cfg = synth.config(0)
    p = jolt.Plan(L=1, H=8, T=256, D=128, has_v=False, budget=262144, num_groups=1,
                  encoder="exact")
    worst = 0.0
    for s in range(10):
        X = synth.gen_layer_tensor(synth.config(0, seed=2000 + s), 0, 0).astype(np.float64)
        a = jolt.analyse_layer_tensor(p, X, s, 0)
        Pi = nm.haar_rotation(s, 128)
        errs = {}
        for rt, rd in ((16, 16), (32, 32), (64, 64)):
            G = nm.round_bf16(a["Gmax"][:, :rt, :rd])
            Y = jolt.residual_rotated(X, a["U_T"][:, :rt], G, a["U_D"][:, :rd], Pi)
            for b in range(1, 9):
                sc, c, _ = jolt.quantize_rows(Y, b)
                rec = jolt.tucker_part(a["U_T"][:, :rt], G, a["U_D"][:, :rd], 8, 256, 128) + \
                    np.einsum("hte,de->htd", jolt.dequantize_rows(sc, c, b), Pi)
                errs[(rt, b)] = jolt.rel_frob(X, rec)
        for rt in (16, 32, 64):
            e = [errs[(rt, b)] for b in range(1, 9)]
            assert all(e1 > e2 for e1, e2 in zip(e, e[1:]))
        for b in range(1, 9):
            e = [errs[(rt, b)] for rt in (16, 32, 64)]
            worst = max(worst, max(e2 / e1 - 1.0 for e1, e2 in zip(e, e[1:])))
    assert worst < 0.02, worst
