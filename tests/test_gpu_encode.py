"""GPU parity of the tail-biting trellis encoder (exl3_encode, through the C ABI)
against the oracle's encoder.

Both take the same decisions in the same precision (fp32 costs, one fused
multiply-add per weight, ties to the smallest index), so the trellis words
must be bit-exact and the per-tile costs equal.  Decoding the GPU's code with
the GPU decoder must give back the targets when they are decodable.
"""
import numpy as np
import pytest
import torch

import oracle
from trellis_coded_bit_b200 import exl3

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    exl3.load()
    yield


def gpu_encode(w, K):
    k, n = w.shape
    ws = exl3.new_workspace(exl3.exl3_encode_workspace_size(k, n, K))
    t, c = exl3.exl3_encode(torch.from_numpy(np.ascontiguousarray(w, dtype=np.float32)).cuda(), K, workspace=ws)
    torch.cuda.synchronize()
    return t.cpu().numpy(), c.cpu().numpy()


@pytest.mark.parametrize("K", range(1, 9))
def test_encode_bit_exact_against_oracle(K):
    rng = np.random.default_rng(4000 + K)
    w = (1.2 * rng.standard_normal((32, 48))).astype(np.float32)
    t, c = gpu_encode(w, K)
    rt, rc = oracle.encode(w, K, threads=oracle.threads_available())
    assert np.array_equal(t, rt), K
    assert np.array_equal(c, rc), K


@pytest.mark.parametrize("K", [2, 5, 8])
def test_encode_decodable_targets_round_trip(K):
    rng = np.random.default_rng(4100 + K)
    k, n = 32, 32
    tr = torch.from_numpy(rng.integers(0, 65536, size=(k // 16, n // 16, 16 * K), dtype=np.uint16)).cuda()
    target = exl3.exl3_decode_tiles(tr, k, n, K).float()
    ws = exl3.new_workspace(exl3.exl3_encode_workspace_size(k, n, K))
    t, c = exl3.exl3_encode(target, K, workspace=ws)
    back = exl3.exl3_decode_tiles(t, k, n, K).float()
    torch.cuda.synchronize()
    assert float(c.abs().max()) == 0.0
    assert torch.equal(back, target)


def test_encode_more_tiles_than_ctas():
    # K = 2 keeps one CTA per SM, so 160 tiles on fewer CTAs take the grid-stride loop
    K = 2
    rng = np.random.default_rng(4200)
    w = rng.standard_normal((16, 2560)).astype(np.float32)
    t, c = gpu_encode(w, K)
    rt, rc = oracle.encode(w, K, threads=oracle.threads_available())
    assert np.array_equal(t, rt)
    assert np.array_equal(c, rc)


def test_encode_sampled_tiles_of_a_large_layer():
    K = 4
    rng = np.random.default_rng(4300)
    k = n = 1024
    w = rng.standard_normal((k, n)).astype(np.float32)
    t, c = gpu_encode(w, K)
    # the reported costs are the decoded code's squared errors
    dec = exl3.exl3_decode_tiles(torch.from_numpy(t).cuda(), k, n, K).double().cpu().numpy()
    sse = ((dec - w) ** 2).reshape(k // 16, 16, n // 16, 16).sum(axis=(1, 3))
    assert np.allclose(sse, c, rtol=1e-4, atol=1e-5)
    for tk, tn in zip(rng.integers(0, k // 16, 12), rng.integers(0, n // 16, 12)):
        rt, rc = oracle.encode(w[16 * tk:16 * tk + 16, 16 * tn:16 * tn + 16], K)
        assert np.array_equal(t[tk, tn], rt[0, 0]), (tk, tn)
        assert c[tk, tn] == rc[0, 0]
