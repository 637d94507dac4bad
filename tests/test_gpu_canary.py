"""Out-of-bounds write checks through the C ABI.

Every output array and every workspace is placed between two 4 KiB guard
regions filled with a byte pattern; after each call the guards must be
unchanged, so a kernel that writes past either end of what it was given is
caught without a fault.  Each result is also compared with the same call on
plain (unguarded) buffers: the calls are deterministic, so the two must agree
bit for bit, which shows that the guarded views were the buffers used.
Shapes are the tiny and ragged ones (one tile, one 128-channel block, m not a
multiple of 8) where index arithmetic is most likely to step outside.
"""
import numpy as np
import pytest
import torch

from test_oracle_ldlq import correlated_hessian
from trellis_coded_bit_b200 import exl3, inputs

pytestmark = pytest.mark.gpu

GUARD = 4096
PATTERN = 0xA5


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    exl3.load()
    yield


class Guarded:
    """A device buffer of `nbytes` between two guard regions; `.view` is the
    usable part as `dtype` with `shape` (zero-filled if `zero`)."""

    def __init__(self, nbytes, dtype, shape=None, zero=False):
        self.nbytes = int(nbytes)
        self.buf = torch.full((2 * GUARD + self.nbytes,), PATTERN, dtype=torch.uint8, device="cuda")
        body = self.buf[GUARD:GUARD + self.nbytes]
        if zero:
            body.zero_()
        self.view = body.view(dtype)
        if shape is not None:
            self.view = self.view.view(shape)

    def intact(self):
        torch.cuda.synchronize()
        head = self.buf[:GUARD]
        tail = self.buf[GUARD + self.nbytes:]
        return bool((head == PATTERN).all()) and bool((tail == PATTERN).all())


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def test_hadamard_guards():
    x = torch.randn(3, 256, dtype=torch.float16, device="cuda")
    y = Guarded(3 * 256 * 2, torch.float16, (3, 256))
    exl3.exl3_hadamard(x, y=y.view)
    assert y.intact()
    assert torch.equal(y.view, exl3.exl3_hadamard(x))


@pytest.mark.parametrize("k,n,K", [(16, 16, 1), (128, 384, 3), (256, 128, 8)])
def test_decode_guards(k, n, K):
    rng = np.random.default_rng(8000 + k + K)
    t = dev(inputs.make_trellis(rng, k, n, K))
    w = Guarded(k * n * 2, torch.float16, (k, n))
    exl3.exl3_decode_tiles(t, k, n, K, w=w.view)
    assert w.intact()
    assert torch.equal(w.view, exl3.exl3_decode_tiles(t, k, n, K))


def _linear_guarded(fn, size_fn, layer):
    m, k, n, K = layer.m, layer.k, layer.n, layer.K
    args = (dev(layer.x), dev(layer.trellis), dev(layer.suh), dev(layer.svh), K)
    wsb = size_fn(m, k, n, K)
    y = Guarded(m * n * 2, torch.float16, (m, n))
    ws = Guarded(wsb, torch.uint8, zero=True)
    fn(*args, y=y.view, workspace=ws.view)
    assert y.intact(), "y guard overwritten"
    assert ws.intact(), "workspace guard overwritten"
    assert exl3.exl3_workspace_status(ws.view) == exl3.EXL3_OK
    # a second call on the same guarded workspace (counters re-armed) and a
    # call on plain buffers give the same bits
    y2 = Guarded(m * n * 2, torch.float16, (m, n))
    fn(*args, y=y2.view, workspace=ws.view)
    assert y2.intact() and ws.intact()
    plain = fn(*args, workspace=exl3.new_workspace(wsb))
    torch.cuda.synchronize()
    assert torch.equal(y.view, y2.view) and torch.equal(y.view, plain)


@pytest.mark.parametrize("m,k,n,K", [(1, 128, 128, 4), (3, 256, 384, 2), (9, 512, 256, 7), (16, 1024, 640, 5)])
def test_gemv_guards(m, k, n, K):
    layer = inputs.make_layer(m, k, n, K, seed=8100 + m + K)
    _linear_guarded(exl3.exl3_gemv, exl3.exl3_gemv_workspace_size, layer)


@pytest.mark.parametrize("m,k,n,K", [(1, 128, 256, 3), (33, 512, 256, 5), (64, 256, 512, 1), (65, 128, 256, 2),
                                     (200, 384, 768, 8), (32, 512, 384, 3), (130, 256, 128, 4)])
def test_gemm_guards(m, k, n, K):
    layer = inputs.make_layer(m, k, n, K, seed=8200 + m + K)
    _linear_guarded(exl3.exl3_gemm, exl3.exl3_gemm_workspace_size, layer)


@pytest.mark.parametrize("m", [3, 40])
def test_matmul_guards(m):
    layer = inputs.make_layer(m, 256, 384, 4, seed=8250 + m)
    _linear_guarded(exl3.exl3_matmul, exl3.exl3_matmul_workspace_size, layer)


def test_gemv_multi_guards():
    m = 3
    layers = [inputs.make_layer(m, k, n, K, seed=8300 + i) for i, (k, n, K) in
              enumerate([(128, 256, 2), (384, 128, 6), (256, 640, 3)])]
    ys = [Guarded(m * L.n * 2, torch.float16, (m, L.n)) for L in layers]
    descs = [(dev(L.x), dev(L.trellis), dev(L.suh), dev(L.svh), L.K, y.view) for L, y in zip(layers, ys)]
    wsb = exl3.exl3_gemv_multi_workspace_size(descs, m)
    ws = Guarded(wsb, torch.uint8, zero=True)
    exl3.exl3_gemv_multi(descs, workspace=ws.view)
    assert all(y.intact() for y in ys) and ws.intact()
    plain = exl3.exl3_gemv_multi([d[:5] + (None,) for d in descs], workspace=exl3.new_workspace(wsb))
    torch.cuda.synchronize()
    for d, p in zip(descs, plain):
        assert torch.equal(d[5], p)


@pytest.mark.parametrize("k,n,K", [(16, 16, 1), (32, 48, 3), (48, 32, 8)])
def test_encode_guards(k, n, K):
    rng = np.random.default_rng(8500 + k + K)
    w = dev((1.2 * rng.standard_normal((k, n))).astype(np.float32))
    t = Guarded(k * n * K // 8, torch.uint16, (k // 16, n // 16, 16 * K))
    c = Guarded((k // 16) * (n // 16) * 4, torch.float32, (k // 16, n // 16))
    ws = Guarded(exl3.exl3_encode_workspace_size(k, n, K), torch.uint8, zero=True)
    exl3.exl3_encode(w, K, trellis=t.view, cost=c.view, workspace=ws.view)
    assert t.intact() and c.intact() and ws.intact()
    t2, c2 = exl3.exl3_encode(w, K, workspace=exl3.new_workspace(exl3.exl3_encode_workspace_size(k, n, K)))
    torch.cuda.synchronize()
    assert torch.equal(t.view, t2) and torch.equal(c.view, c2)


def test_udu_and_ldlq_guards():
    k, n, K = 48, 32, 2
    rng = np.random.default_rng(8600)
    h = dev(correlated_hessian(k, rng))
    ud = Guarded(k * k * 8, torch.float64, (k, k))
    exl3.exl3_udu(h, ud=ud.view)
    assert ud.intact()
    assert torch.equal(ud.view, exl3.exl3_udu(h))
    w = dev((1.2 * rng.standard_normal((k, n))).astype(np.float32))
    t = Guarded(k * n * K // 8, torch.uint16, (k // 16, n // 16, 16 * K))
    wh = Guarded(k * n * 4, torch.float32, (k, n))
    ws = Guarded(exl3.exl3_ldlq_workspace_size(k, n, K), torch.uint8, zero=True)
    exl3.exl3_ldlq(w, h, K, trellis=t.view, w_hat=wh.view, workspace=ws.view)
    assert t.intact() and wh.intact() and ws.intact()
    t2, wh2 = exl3.exl3_ldlq(w, h, K, workspace=exl3.new_workspace(exl3.exl3_ldlq_workspace_size(k, n, K)))
    torch.cuda.synchronize()
    assert torch.equal(t.view, t2) and torch.equal(wh.view, wh2)
