"""The allocation-free GEMV entry point, exl3_gemv_noalloc.

It exists for callers that cannot allocate device memory (a host framework
that owns all device memory, a fixed memory budget, or a path where an
allocation and its implied synchronisation are not allowed): instead of a
caller-provided workspace it uses a fixed scratch array compiled into the
library.  These tests call it through the C ABI and check that it gives the
same outputs as exl3_gemv, within the stated output tolerance, on two calls in
a row (the array keeps the previous call's contents, so the second call
checks that nothing stale leaks through).  The file is named to be collected
last; it passes alone in a fresh process as well.  The outputs are also
checked against the fp64 oracle, so that a fault shared by both entry points
(the scratch layout, say) cannot pass unseen.
"""
import numpy as np
import pytest
import torch

import oracle
from conftest import within_tolerance
from trellis_coded_bit_b200 import exl3, inputs

pytestmark = pytest.mark.gpu


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    exl3.load()
    yield


@pytest.mark.parametrize("m,k,n,K", [(1, 4096, 4096, 4), (5, 2048, 1024, 3), (16, 1024, 2048, 2)])
def test_noalloc_matches_gemv_on_two_calls_in_a_row(m, k, n, K):
    assert exl3.exl3_gemv_workspace_size(m, k, n, K) <= exl3.exl3_gemv_noalloc_max_scratch()
    layers = [inputs.make_layer(m, k, n, K, seed=900 + i) for i in range(2)]
    for L in layers:  # two different inputs, one call each, back to back
        args = (dev(L.x), dev(L.trellis), dev(L.suh), dev(L.svh), K)
        ws = exl3.new_workspace(exl3.exl3_gemv_workspace_size(m, k, n, K))
        ref = exl3.exl3_gemv(*args, workspace=ws).cpu().numpy().astype(np.float64)
        y1 = torch.empty((m, n), dtype=torch.float16, device="cuda")
        y2 = torch.empty((m, n), dtype=torch.float16, device="cuda")
        exl3.exl3_gemv_noalloc(*args, y=y1)
        exl3.exl3_gemv_noalloc(*args, y=y2)
        torch.cuda.synchronize()
        for y in (y1, y2):
            got = y.cpu().numpy().astype(np.float64)
            ok, err, bound = within_tolerance(got, ref)
            assert ok, "max err %.4g > bound %.4g" % (err, bound)
        # against the oracle, on the first, a middle and the last column block
        nb = n // 128
        for cb in sorted({0, nb // 2, nb - 1}):
            want = oracle.linear(L.x, L.trellis, L.suh, L.svh, K, col_blocks=(cb, cb + 1))
            got = y2.cpu().numpy().astype(np.float64)[:, cb * 128:(cb + 1) * 128]
            ok, err, bound = within_tolerance(got, want)
            assert ok, "block %d: max err %.4g > bound %.4g" % (cb, err, bound)


def test_noalloc_split_k_shape_matches_the_oracle():
    # k = 8192 with 256 column blocks: more CTAs than column blocks, so every
    # block is split over several CTAs whose partials meet in the scratch array
    m, k, n, K = 2, 8192, 2048, 3
    assert exl3.exl3_gemv_workspace_size(m, k, n, K) <= exl3.exl3_gemv_noalloc_max_scratch()
    L = inputs.make_layer(m, k, n, K, seed=930)
    y = torch.empty((m, n), dtype=torch.float16, device="cuda")
    exl3.exl3_gemv_noalloc(dev(L.x), dev(L.trellis), dev(L.suh), dev(L.svh), K, y=y)
    got = y.cpu().numpy().astype(np.float64)
    for cb in (0, 7, 15):
        want = oracle.linear(L.x, L.trellis, L.suh, L.svh, K, col_blocks=(cb, cb + 1))
        ok, err, bound = within_tolerance(got[:, cb * 128:(cb + 1) * 128], want)
        assert ok, "block %d: max err %.4g > bound %.4g" % (cb, err, bound)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    # split partials alone for 448 column blocks x 16 batches need far more than the array
    m, k, n, K = 16, 8192, 57344, 4
    assert exl3.exl3_gemv_workspace_size(m, k, n, K) > 1.5 * exl3.exl3_gemv_noalloc_max_scratch()
    x = torch.zeros((m, k), dtype=torch.float16, device="cuda")
    t = torch.zeros((k // 16, n // 16, 16 * K), dtype=torch.uint16, device="cuda")
    suh = torch.ones(k, dtype=torch.float16, device="cuda")
    svh = torch.ones(n, dtype=torch.float16, device="cuda")
    y = torch.empty((m, n), dtype=torch.float16, device="cuda")
    with pytest.raises(exl3.Exl3Error) as e:
        exl3.exl3_gemv_noalloc(x, t, suh, svh, K, y=y)
    assert e.value.status == exl3.EXL3_ERR_WORKSPACE
