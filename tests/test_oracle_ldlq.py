"""Pins of the oracle's LDLQ (oracle/ldlq.py), CPU only.

  - the block factorisation reproduces H (U D U^T = H), with U unit
    block-upper-triangular and D block-diagonal and positive definite;
  - with H = I, or any block-diagonal H, there is no feedback and LDLQ is the
    plain trellis encoding of W, bit for bit;
  - for a general H the proxy loss tr(E^T H E) equals sum_b tr(F_b^T D_b F_b)
    with F_b = W_hat_b - T_b computed from the returned W_hat: an identity of
    the LDL feedback that a wrong sign, index or transpose breaks;
  - with a strongly correlated H, LDLQ's proxy loss is well below that of
    encoding W without feedback.
"""
import numpy as np
import pytest

import oracle
from oracle import ldlq as L


def correlated_hessian(k, rng, rho=0.9, ridge=1e-3):
    # inputs x = z C with an AR(1)-like mixing: neighbouring channels correlated
    idx = np.arange(k)
    c = rho ** np.abs(idx[:, None] - idx[None, :])
    z = rng.standard_normal((4 * k, k))
    x = z @ np.linalg.cholesky(c).T
    h = x.T @ x / x.shape[0]
    return h + ridge * np.trace(h) / k * np.eye(k)


@pytest.mark.parametrize("k", [16, 48, 96])
def test_udu_reproduces_h(k):
    rng = np.random.default_rng(k)
    h = correlated_hessian(k, rng)
    U, D = L.udu(h)
    assert np.allclose(U @ D @ U.T, h, rtol=1e-10, atol=1e-10 * np.abs(h).max())
    B = 16
    for a in range(k // B):
        for b in range(k // B):
            ub = U[a * B:(a + 1) * B, b * B:(b + 1) * B]
            db = D[a * B:(a + 1) * B, b * B:(b + 1) * B]
            if a == b:
                assert np.array_equal(ub, np.eye(B))
                assert np.allclose(db, db.T) and np.linalg.eigvalsh(db).min() > 0
            else:
                assert not db.any()
                if a > b:
                    assert not ub.any()


@pytest.mark.parametrize("K", [2, 4])
def test_identity_and_block_diagonal_h_give_plain_encoding(K):
    rng = np.random.default_rng(10 + K)
    k, n = 48, 32
    w = rng.standard_normal((k, n)).astype(np.float32)
    plain, _ = oracle.encode(w, K)
    tr, _, targets, _, _ = L.ldlq(w, np.eye(k), K)
    assert np.array_equal(tr, plain)
    assert np.array_equal(targets, w)
    # block-diagonal SPD H: U = I, still no feedback
    h = np.zeros((k, k))
    for b in range(k // 16):
        a = rng.standard_normal((16, 16))
        h[16 * b:16 * b + 16, 16 * b:16 * b + 16] = a @ a.T + 16 * np.eye(16)
    tr2, _, _, U, _ = L.ldlq(w, h, K)
    assert np.array_equal(U, np.eye(k))
    assert np.array_equal(tr2, plain)


@pytest.mark.parametrize("K", [2, 3])
def test_proxy_loss_is_the_sum_of_block_residuals(K):
    rng = np.random.default_rng(20 + K)
    k, n = 64, 32
    w = rng.standard_normal((k, n)).astype(np.float32)
    h = correlated_hessian(k, rng)
    tr, what, targets, U, D = L.ldlq(w, h, K)
    # the code decodes to W_hat
    assert np.array_equal(oracle.half_to_double(oracle.decode_tiles(tr, k, n, K)), what)
    e = what - w.astype(np.float64)
    total = 0.0
    for b in range(k // 16):
        r0, r1 = 16 * b, 16 * b + 16
        t = w[r0:r1].astype(np.float64) - U[:r0, r0:r1].T @ e[:r0]
        assert np.allclose(t.astype(np.float32), targets[r0:r1], rtol=0, atol=1e-6 * np.abs(t).max())
        f = what[r0:r1] - t
        total += np.trace(f.T @ D[r0:r1, r0:r1] @ f)
    loss = L.proxy_loss(what, w, h)
    assert abs(loss - total) <= 1e-9 * loss


def test_ldlq_beats_encoding_without_feedback_on_a_correlated_hessian():
    ratios = []
    for seed in range(3):
        rng = np.random.default_rng(30 + seed)
        k, n, K = 96, 32, 2
        w = rng.standard_normal((k, n)).astype(np.float32)
        h = correlated_hessian(k, rng, rho=0.95)
        _, what, _, _, _ = L.ldlq(w, h, K)
        plain, _ = oracle.encode(w, K)
        pdec = oracle.half_to_double(oracle.decode_tiles(plain, k, n, K))
        ratios.append(L.proxy_loss(what, w, h) / L.proxy_loss(pdec, w, h))
    assert max(ratios) < 0.8, ratios
