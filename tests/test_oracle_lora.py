"""Pins for the oracle's LoRA linear (CPU only): B = 0 reduction and central
finite differences of every analytic gradient on tiny shapes."""
import numpy as np

from oracle import lora_linear as LL


def _case(M=3, K=64, N=5, r=2, seed=0):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((M, K))
    Wd = rng.standard_normal((N, K)) * 0.1
    A = rng.standard_normal((r, K)) / np.sqrt(K)
    B = rng.standard_normal((N, r)) * 0.5
    dY = rng.standard_normal((M, N))
    return X, Wd, A, B, dY


def test_b_zero_is_base_linear():
    X, Wd, A, B, _ = _case()
    Y, U = LL.lora_forward(X, Wd, A, np.zeros_like(B), 2.0)
    base = np.array([[sum(X[m, k] * Wd[n, k] for k in range(X.shape[1])) for n in range(Wd.shape[0])]
                     for m in range(X.shape[0])])
    np.testing.assert_allclose(Y, base, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(U, X @ A.T, rtol=1e-13)


def test_forward_brute_force():
    X, Wd, A, B, _ = _case(M=2, K=64, N=3, r=2, seed=3)
    s = 1.5
    Y, _ = LL.lora_forward(X, Wd, A, B, s)
    for m in range(2):
        for n in range(3):
            u = [sum(X[m, k] * A[j, k] for k in range(64)) for j in range(2)]
            want = sum(X[m, k] * Wd[n, k] for k in range(64)) + s * sum(u[j] * B[n, j] for j in range(2))
            assert abs(Y[m, n] - want) < 1e-12


def _fd(f, P, h=1e-6):
    g = np.zeros_like(P)
    it = np.nditer(P, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        old = P[i]
        P[i] = old + h
        fp = f()
        P[i] = old - h
        fm = f()
        P[i] = old
        g[i] = (fp - fm) / (2 * h)
    return g


def test_gradients_match_central_differences():
    X, Wd, A, B, dY = _case(M=3, K=64, N=5, r=2, seed=1)
    s = 2.0
    dX, dA, dB, G = LL.lora_backward(X, Wd, A, B, s, dY)
    f = lambda: LL.lora_loss(X, Wd, A, B, s, dY)
    for analytic, P in ((dX, X), (dA, A), (dB, B)):
        num = _fd(f, P)
        rel = np.linalg.norm(num - analytic) / np.linalg.norm(analytic)
        assert rel < 1e-6, rel
    np.testing.assert_allclose(G, dY @ B)
