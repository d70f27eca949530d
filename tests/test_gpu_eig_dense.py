"""The dense eigensolver of the exact token factor (token Grams above 128 tokens) through its C-ABI
self-test, against properties that fix the answer: float64 eigenpairs of symmetric matrices with a
known spectrum (eigenvalues to ~1e-12 of the norm, residual ||A v - lambda v|| and orthonormality of
the R vectors to rounding), including clustered, repeated and zero spectra where individual vectors
are not unique but these properties still are."""
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


def _spectrum(kind, n, rng):
    if kind == "separated":
        return np.sort(rng.uniform(0.1, 10.0, n))[::-1] * np.linspace(1.0, 2.0, n)[::-1]
    if kind == "gram_like":
        # 64 signal values over a noise bulk of width ~1 (the shape of a token Gram)
        sig = 50.0 * np.exp(-np.arange(64) / 12.0) + 2.0
        bulk = np.sort(rng.uniform(0.0, 1.6, n - 64))[::-1]
        return np.concatenate([sig, bulk])
    if kind == "repeated":
        return np.repeat([9.0, 4.0, 4.0, 1.0], n // 4 + 1)[:n]
    if kind == "zero":
        return np.zeros(n)
    raise ValueError(kind)


@pytest.mark.parametrize("n,R,kind", [(130, 16, "separated"), (257, 112, "gram_like"), (256, 112, "repeated"),
                                      (200, 40, "zero"), (1024, 112, "gram_like")])
def test_dense_eigenpairs(J, n, R, kind):
    import torch
    rng = np.random.default_rng(n + R)
    batch = 2
    A = np.empty((batch, n, n))
    lams = []
    for b in range(batch):
        Q = np.linalg.qr(rng.standard_normal((n, n)))[0]
        lam = _spectrum(kind, n, rng)
        A[b] = (Q * lam) @ Q.T
        A[b] = 0.5 * (A[b] + A[b].T)
        lams.append(np.sort(np.linalg.eigvalsh(A[b]))[::-1])
    Ad = torch.from_numpy(A).cuda()
    V = torch.full((batch, n, R), float("nan"), dtype=torch.float64, device="cuda")
    L = torch.full((batch, R), float("nan"), dtype=torch.float64, device="cuda")
    J.jolt_selftest_eig_dense(Ad, R, V, L)
    V, L = V.cpu().numpy(), L.cpu().numpy()
    for b in range(batch):
        nrm = max(np.abs(lams[b]).max(), 1.0)
        assert np.abs(L[b] - lams[b][:R]).max() <= 1e-12 * nrm, np.abs(L[b] - lams[b][:R]).max()
        assert np.abs(V[b].T @ V[b] - np.eye(R)).max() <= 1e-12
        res = A[b] @ V[b] - V[b] * L[b]
        assert np.abs(res).max() <= 1e-11 * nrm, np.abs(res).max()


def test_already_tridiagonal_and_diagonal(J):
    """No reflection to make (tau = 0) and a split tridiagonal (zero off-diagonals)."""
    import torch
    n, R = 300, 24
    rng = np.random.default_rng(9)
    T1 = np.diag(rng.uniform(1, 5, n)) + np.diag(rng.uniform(0.1, 1, n - 1), 1)
    T1 = T1 + np.triu(T1, 1).T
    T2 = np.diag(np.arange(n, dtype=np.float64))
    A = np.stack([T1, T2])
    V = torch.empty((2, n, R), dtype=torch.float64, device="cuda")
    L = torch.empty((2, R), dtype=torch.float64, device="cuda")
    J.jolt_selftest_eig_dense(torch.from_numpy(A).cuda(), R, V, L)
    V, L = V.cpu().numpy(), L.cpu().numpy()
    for b in range(2):
        w = np.sort(np.linalg.eigvalsh(A[b]))[::-1][:R]
        assert np.abs(L[b] - w).max() <= 1e-12 * np.abs(w).max()
        assert np.abs(A[b] @ V[b] - V[b] * L[b]).max() <= 1e-11 * np.abs(w).max()
        assert np.abs(V[b].T @ V[b] - np.eye(R)).max() <= 1e-12
