"""GPU parity of the block factorisation (exl3_udu) and of LDLQ (exl3_ldlq),
through the C ABI, against the oracle (oracle/ldlq.py).

The factor is fp64 on both sides (different summation orders, so compared to
a tight relative tolerance).  LDLQ's targets are fp64 sums rounded to fp32 on
both sides and the encoder decides in fp32, so the trellis words must match
bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import ldlq as OL
from test_oracle_ldlq import correlated_hessian
from trellis_coded_bit_b200 import exl3

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    exl3.load()
    yield


@pytest.mark.parametrize("k", [16, 64, 208])
def test_udu_matches_oracle(k):
    rng = np.random.default_rng(5000 + k)
    h = correlated_hessian(k, rng)
    ud = exl3.exl3_udu(torch.from_numpy(h).cuda()).cpu().numpy()
    U, D = OL.udu(h)
    B = 16
    scale = np.abs(h).max()
    for a in range(k // B):
        for b in range(k // B):
            blk = ud[a * B:(a + 1) * B, b * B:(b + 1) * B]
            if a == b:
                ref = D[a * B:(a + 1) * B, b * B:(b + 1) * B]
                assert np.allclose(blk, ref, rtol=1e-9, atol=1e-12 * scale)
            elif a < b:
                ref = U[a * B:(a + 1) * B, b * B:(b + 1) * B]
                assert np.allclose(blk, ref, rtol=1e-9, atol=1e-10)
            else:
                assert not blk.any()


def _run_ldlq(w, h, K):
    k, n = w.shape
    ws = exl3.new_workspace(exl3.exl3_ldlq_workspace_size(k, n, K))
    t, wh = exl3.exl3_ldlq(torch.from_numpy(w).cuda(), torch.from_numpy(h).cuda(), K, workspace=ws)
    torch.cuda.synchronize()
    return t.cpu().numpy(), wh.cpu().numpy()


@pytest.mark.parametrize("K", [2, 4])
def test_ldlq_with_identity_hessian_is_plain_encoding(K):
    rng = np.random.default_rng(5100 + K)
    k, n = 48, 80
    w = rng.standard_normal((k, n)).astype(np.float32)
    t, wh = _run_ldlq(w, np.eye(k), K)
    ws = exl3.new_workspace(exl3.exl3_encode_workspace_size(k, n, K))
    plain, _ = exl3.exl3_encode(torch.from_numpy(w).cuda(), K, workspace=ws)
    assert np.array_equal(t, plain.cpu().numpy())
    assert np.array_equal(wh, oracle.half_to_double(oracle.decode_tiles(t, k, n, K)).astype(np.float32))


@pytest.mark.parametrize("k,n,K", [(64, 48, 2), (64, 48, 4), (112, 160, 3)])
def test_ldlq_matches_oracle_bit_exact(k, n, K):
    rng = np.random.default_rng(5200 + k + n + K)
    w = rng.standard_normal((k, n)).astype(np.float32)
    h = correlated_hessian(k, rng, rho=0.95)
    t, wh = _run_ldlq(w, h, K)
    rt, rwhat, _, _, _ = OL.ldlq(w, h, K, threads=oracle.threads_available())
    assert np.array_equal(t, rt)
    assert np.array_equal(wh.astype(np.float64), rwhat)
    # and the Hessian-weighted error is the oracle's
    assert OL.proxy_loss(wh, w, h) == pytest.approx(OL.proxy_loss(rwhat, w, h), rel=1e-12)


@pytest.mark.parametrize("K", [1, 8])
def test_ldlq_single_tile_row_is_plain_encoding(K):
    # k = 16: one block, nothing to feed back, whatever H is (K = 1 also takes
    # the encoder's global-memory cost vectors)
    rng = np.random.default_rng(5300 + K)
    k, n = 16, 48
    w = rng.standard_normal((k, n)).astype(np.float32)
    a = rng.standard_normal((k, k))
    h = a @ a.T + k * np.eye(k)
    t, _ = _run_ldlq(w, h, K)
    rt, _ = oracle.encode(w, K)
    assert np.array_equal(t, rt)
