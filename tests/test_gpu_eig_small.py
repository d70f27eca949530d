"""The eigensolver of the feature and sketch eigenproblems (n <= 128) through its C-ABI self-test,
against properties that fix the answer whatever the solver: eigenvalues of symmetric float64
matrices against LAPACK's (numpy.linalg.eigvalsh), orthonormal float32 eigenvectors, and small
residuals ||A v - lambda v||. Clustered, repeated and zero spectra have no unique vectors, but
these properties still hold. The tridiagonal solver is also checked against the one-sided Jacobi
solver on the Gram matrices of the workloads' caches.

Tolerances: the outputs are float32, so an eigenvalue carries a relative rounding of 6e-8 and a
vector entry 6e-8 of its size; the float64 computation adds a few eps ||A|| to the eigenvalues and
~eps ||A|| / gap to the vectors. Bounds: |lambda - lambda_ref| <= 2e-7 |lambda_ref| + 1e-12 ||A||,
|V^T V - I| <= 2e-6, ||A v - lambda v||_max <= 2e-6 ||A||.
"""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def J():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from tensor_decomposition_b200 import build
    build.build()
    from tensor_decomposition_b200 import jolt
    return jolt


def _matrix(kind, n, rng):
    M = rng.standard_normal((n, n))
    if kind == "symmetric":
        return 0.5 * (M + M.T)
    if kind == "psd":
        return M @ M.T / n
    if kind == "decaying":       # eigenvalues 1 .. e^-25: tiny ones far below eps^(1/2) ||A||
        Q = np.linalg.qr(M)[0]
        return (Q * np.exp(-np.arange(n) / (n / 25.0))) @ Q.T
    if kind == "repeated":
        Q = np.linalg.qr(M)[0]
        lam = np.repeat([9.0, 4.0, 4.0, 1.0], n // 4 + 1)[:n]
        return (Q * lam) @ Q.T
    if kind == "rank3":
        X = rng.standard_normal((n, 3))
        return X @ X.T
    if kind == "diagonal":
        return np.diag(np.floor(rng.uniform(0, 5, n)))
    if kind == "tridiagonal":
        T = np.diag(rng.uniform(1, 5, n)) + np.diag(rng.uniform(0.1, 1, n - 1), 1) if n > 1 else np.eye(1)
        return np.triu(T) + np.triu(T, 1).T
    if kind == "zero":
        return np.zeros((n, n))
    if kind == "scaled_identity":
        return 3.0 * np.eye(n)
    raise ValueError(kind)


def _solve(J, A, solver):
    import torch
    b, n = A.shape[0], A.shape[1]
    V = torch.full((b, n, n), float("nan"), dtype=torch.float32, device="cuda")
    L = torch.full((b, n), float("nan"), dtype=torch.float32, device="cuda")
    J.jolt_selftest_eig_small(torch.from_numpy(A).cuda(), V, L, solver)
    return V.cpu().numpy().astype(np.float64), L.cpu().numpy().astype(np.float64)


def _check(A, V, L):
    for b in range(A.shape[0]):
        a = 0.5 * (A[b] + A[b].T)
        ref = np.sort(np.linalg.eigvalsh(a))[::-1]
        nrm = max(np.abs(ref).max(), 1e-300) if ref.size else 1.0
        assert np.all(np.diff(L[b]) <= 0), "eigenvalues must come out descending"
        assert np.abs(L[b] - ref).max() <= (2e-7 * np.abs(ref) + 1e-12 * nrm).max() + 1e-30, \
            np.abs(L[b] - ref).max()
        n = a.shape[0]
        assert np.abs(V[b].T @ V[b] - np.eye(n)).max() <= 2e-6
        assert np.abs(a @ V[b] - V[b] * L[b]).max() <= 2e-6 * nrm + 1e-30


@pytest.mark.parametrize("n,kind", [
    (128, "symmetric"), (128, "psd"), (128, "decaying"), (128, "repeated"), (128, "rank3"),
    (128, "diagonal"), (128, "tridiagonal"), (128, "zero"), (128, "scaled_identity"),
    (100, "psd"), (97, "symmetric"), (64, "psd"), (33, "decaying"), (32, "symmetric"), (31, "psd"),
    (3, "symmetric"), (2, "symmetric"), (1, "symmetric")])
def test_tridiagonal_solver_properties(J, n, kind):
    rng = np.random.default_rng(1000 + n)
    A = np.stack([_matrix(kind, n, rng) for _ in range(3)])
    # the solver reads the lower triangle only: the upper one is garbage here
    A_in = np.tril(A) + np.triu(np.full_like(A, 7.5), 1)
    V, L = _solve(J, A_in, J.JOLT_EIG_TRIDIAG)
    _check(A, V, L)


def test_nonfinite_input_is_reported(J):
    import torch
    A = np.eye(16)[None].repeat(2, 0)
    A[1, 3, 2] = np.nan
    V = torch.empty((2, 16, 16), dtype=torch.float32, device="cuda")
    L = torch.empty((2, 16), dtype=torch.float32, device="cuda")
    with pytest.raises(J.JoltError) as e:
        J.jolt_selftest_eig_small(torch.from_numpy(A).cuda(), V, L, J.JOLT_EIG_TRIDIAG)
    assert e.value.status == 6
    assert np.allclose(L[0].cpu().numpy(), 1.0) and np.isnan(L[1].cpu().numpy()).all()


@pytest.mark.parametrize("cfg_idx", [1, 2])
def test_agrees_with_jacobi_on_workload_grams(J, cfg_idx):
    """Feature Grams C_D = sum_h X_h^T X_h of the first layers of the synthetic caches (K and V):
    both solvers satisfy the properties, their eigenvalues agree and the leading vectors span the
    same lines wherever the eigengap is clear."""
    import synth
    from oracle import jolt as oj
    cfg = synth.config(cfg_idx, layers=2)
    A = np.stack([oj.feature_gram(synth.kv.gen_layer_tensor(cfg, layer, kind).astype(np.float64))
                  for layer in range(2) for kind in (0, 1)])
    Vt, Lt = _solve(J, A, J.JOLT_EIG_TRIDIAG)
    Vj, Lj = _solve(J, A, J.JOLT_EIG_JACOBI)
    _check(A, Vt, Lt)
    _check(A, Vj, Lj)
    for b in range(A.shape[0]):
        assert np.abs(Lt[b] - Lj[b]).max() <= 4e-7 * np.abs(Lj[b]).max()
        lam = np.sort(np.linalg.eigvalsh(A[b]))[::-1]
        gap = np.minimum(np.r_[np.inf, lam[:-1] - lam[1:]], np.r_[lam[:-1] - lam[1:], np.inf])
        clear = gap > 1e-4 * lam[0]
        cos = np.abs(np.sum(Vt[b] * Vj[b], axis=0))
        assert np.all(cos[clear] >= 1 - 1e-6), cos[clear].min()
