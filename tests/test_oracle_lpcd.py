"""Pins of the oracle's LPCD reading (two-layer linear submodule).

The pages give no LPCD formula, so the pins check what the reading's
mathematics fixes: the relaxed steps are exact least-squares minimisers (a
brute-force solve of the vectorised problem, an augmented lstsq, and
perturbations must agree), the identity special case returns the weights, and
one round improves on the layer-wise start, as the pages say LPCD does over
layer-wise quantisation.
"""
import numpy as np
import pytest

import oracle


def _case(n, d, m, N, seed, noise=0.1):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((N, n))
    x[:, :3] *= 5.0
    xh = x + noise * rng.standard_normal((N, n))
    W1 = 0.1 * rng.standard_normal((d, n))
    W2 = 0.1 * rng.standard_normal((m, d))
    return x, xh, W1, W2


def test_left_project_is_the_ridge_minimiser():
    rng = np.random.default_rng(1)
    m, d, n = 30, 12, 9
    B = rng.standard_normal((m, d))
    W2 = rng.standard_normal((m, d))
    V = rng.standard_normal((d, n))
    damp = 0.05
    W = oracle.lpcd_left_project(B, W2, V, damp)
    mu = damp * np.mean(np.diag(B.T @ B))
    # augmented least squares [B; sqrt(mu) I] W = [W2 V; 0], solved by SVD
    A = np.vstack([B, np.sqrt(mu) * np.eye(d)])
    rhs = np.vstack([W2 @ V, np.zeros((d, n))])
    ref = np.linalg.lstsq(A, rhs, rcond=None)[0]
    assert np.allclose(W, ref, rtol=1e-10, atol=1e-12)

    def f(X):
        return np.sum((B @ X - W2 @ V) ** 2) + mu * np.sum(X ** 2)

    f0 = f(W)
    for _ in range(5):
        P = rng.standard_normal(W.shape)
        assert f(W + 1e-3 * P) > f0
        assert f(W - 1e-3 * P) > f0


def test_layer1_step_is_the_exact_least_squares_solution():
    # with damp = 0 both ridge terms vanish and the relaxed layer-1 step must be
    # the minimiser of ||x W1^T W2^T - xh W^T Q2^T||_F^2 over W
    x, xh, W1, W2 = _case(n=5, d=6, m=7, N=40, seed=2)
    rng = np.random.default_rng(3)
    Q2 = W2 + 0.02 * rng.standard_normal(W2.shape)
    V1 = oracle.qep_correct(W1, x, xh, 1.0, 0.0)
    Ws = oracle.lpcd_left_project(Q2, W2, V1, 0.0)
    # brute force: vec(xh W^T Q2^T) = (Q2 kron xh) vec(W^T), column-major vec
    Y = x @ W1.T @ W2.T
    K = np.kron(Q2, xh)
    vecWt = np.linalg.lstsq(K, Y.reshape(-1, order="F"), rcond=None)[0]
    ref = vecWt.reshape((xh.shape[1], Q2.shape[1]), order="F").T
    assert np.allclose(Ws, ref, rtol=1e-8, atol=1e-10)

    def g(W):
        return np.sum((Y - xh @ W.T @ Q2.T) ** 2)

    g0 = g(Ws)
    for _ in range(5):
        P = rng.standard_normal(Ws.shape)
        assert g(Ws + 1e-4 * P) >= g0


def test_layer2_step_is_qep_alpha_one_least_squares():
    # the layer-2 relaxed step is QEP with alpha = 1: with damp = 0 it is the
    # minimiser of ||z W2^T - zh W^T||_F^2 over W
    rng = np.random.default_rng(4)
    z = rng.standard_normal((60, 8))
    zh = z + 0.1 * rng.standard_normal(z.shape)
    W2 = rng.standard_normal((5, 8))
    Wp = oracle.qep_correct(W2, z, zh, 1.0, 0.0)
    ref = np.linalg.lstsq(zh, z @ W2.T, rcond=None)[0].T
    assert np.allclose(Wp, ref, rtol=1e-9, atol=1e-11)


def test_identity_case_returns_the_first_layer():
    # unchanged second layer (square, invertible), no input error, no damping
    x, _, W1, _ = _case(n=8, d=6, m=6, N=50, seed=5)
    rng = np.random.default_rng(6)
    W2 = rng.standard_normal((6, 6)) + 3.0 * np.eye(6)
    V1 = oracle.qep_correct(W1, x, x, 1.0, 0.0)
    assert np.allclose(V1, W1, rtol=1e-10, atol=1e-12)
    assert np.allclose(oracle.lpcd_left_project(W2, W2, V1, 0.0), W1, rtol=1e-9, atol=1e-11)


def test_lpcd_pair_round_solves_its_least_squares_problem():
    # the loop's own composition: with damp = 0 each round's relaxed W1 is the
    # brute-force minimiser against the quantised second layer it was given
    x, xh, W1, W2 = _case(n=5, d=6, m=7, N=40, seed=7)
    r = oracle.lpcd_pair(W1, W2, x, xh, 0.5, 0.0, 4, -1, False, rounds=2)
    xb, xhb = oracle._bf16(x), oracle._bf16(xh)
    Y = xb @ W1.T @ W2.T
    for Ws, Q2 in zip(r["W1_star"], r["Q2_used"]):
        vecWt = np.linalg.lstsq(np.kron(Q2, xhb), Y.reshape(-1, order="F"), rcond=None)[0]
        ref = vecWt.reshape((xb.shape[1], Q2.shape[1]), order="F").T
        assert np.allclose(Ws, ref, rtol=1e-7, atol=1e-9)


@pytest.mark.parametrize("wbits", [3, 4])
def test_one_round_improves_on_the_layer_wise_start(wbits):
    x, xh, W1, W2 = _case(n=64, d=48, m=40, N=1200, seed=5)
    r = oracle.lpcd_pair(W1, W2, x, xh, 0.5, 0.01, wbits, 16, False, rounds=1)
    assert len(r["errors"]) == 2 and len(r["W1_star"]) == 1
    assert r["errors"][1] < 0.9 * r["errors"][0]
    assert r["errors"][0] < 0.05 * r["ref"]
