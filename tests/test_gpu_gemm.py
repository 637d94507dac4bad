"""GPU parity of the tensor-core GEMM path (exl3_gemm, through the C ABI)
against the fp64 oracle: max|y - y_ref| <= 1e-2 * rms(y_ref) + 1e-3."""
import numpy as np
import pytest
import torch

import oracle
from conftest import within_tolerance
from trellis_coded_bit_b200 import exl3, inputs, workloads

pytestmark = pytest.mark.gpu


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    exl3.load()
    yield


def run_gemm(layer, ws=None):
    m, k, n, K = layer.m, layer.k, layer.n, layer.K
    if ws is None:
        ws = exl3.new_workspace(exl3.exl3_gemm_workspace_size(m, k, n, K))
    y = exl3.exl3_gemm(dev(layer.x), dev(layer.trellis), dev(layer.suh), dev(layer.svh), K, workspace=ws)
    torch.cuda.synchronize()
    assert exl3.exl3_workspace_status(ws) == exl3.EXL3_OK
    return y.cpu().numpy().astype(np.float64), ws


def check(layer, y, rows=None, col_blocks=None):
    x = layer.x if rows is None else layer.x[rows]
    ref = oracle.linear(x, layer.trellis, layer.suh, layer.svh, layer.K, col_blocks=col_blocks)
    yy = y if rows is None else y[rows]
    if col_blocks is not None:
        yy = yy[:, col_blocks[0] * 128:col_blocks[1] * 128]
    ok, err, bound = within_tolerance(yy, ref)
    assert ok, "max err %.4g > bound %.4g" % (err, bound)


@pytest.mark.parametrize("m,k,n,K", [(1, 128, 256, 3), (64, 256, 256, 4), (128, 512, 512, 2),
                                     (200, 384, 256, 8), (256, 256, 512, 1), (300, 512, 256, 5),
                                     (513, 256, 256, 6), (256, 1024, 768, 7)])
def test_gemm_small(m, k, n, K):
    layer = inputs.make_layer(m, k, n, K, seed=6000 + m + K)
    y, _ = run_gemm(layer)
    check(layer, y)


def test_gemm_closed_form_constant_weights():
    layer = inputs.make_layer(130, 256, 256, 3, seed=3)
    layer.trellis[:] = 0
    y, _ = run_gemm(layer)
    check(layer, y)
    mask = np.ones(256, dtype=bool)
    mask[::128] = False
    assert np.abs(y[:, mask]).max() <= 1e-3 * np.abs(y[:, ~mask]).max()


def test_gemm_agrees_with_gemv_at_m16():
    layer = inputs.make_layer(16, 1024, 512, 4, seed=4)
    yg, ws = run_gemm(layer)
    yv = exl3.exl3_gemv(dev(layer.x), dev(layer.trellis), dev(layer.suh), dev(layer.svh), 4,
                        workspace=exl3.new_workspace(exl3.exl3_gemv_workspace_size(16, 1024, 512, 4)))
    yv = yv.cpu().numpy().astype(np.float64)
    ok, err, bound = within_tolerance(yg, yv)
    assert ok, (err, bound)
    # deterministic across calls with the same workspace
    yg2, _ = run_gemm(layer, ws)
    assert np.array_equal(yg, yg2)


@pytest.mark.parametrize("case", range(len(workloads.PREFILL)))
def test_gemm_prefill_sampled(case):
    name, m, k, n, K, outl = workloads.PREFILL[case]
    layer = inputs.make_layer(m, k, n, K, inputs.seed_for(3, case), outl)
    y, _ = run_gemm(layer)
    assert np.isfinite(y).all()
    rng = np.random.default_rng(case)
    rows = np.sort(rng.choice(m, 64, replace=False))
    nb = n // 128
    check(layer, y, rows=rows, col_blocks=(0, 1))
    check(layer, y, rows=rows, col_blocks=(nb - 2, nb))


# m <= 64: the decoded weights are the MMA's A operand (128 output channels per
# MMA) and x' its B operand (N = m rounded up to 32).  Shapes with many k
# blocks per tile split tiles over several CTAs (partial sums and tickets);
# m = 65 is the first size on the other form.
@pytest.mark.parametrize("m,k,n,K", [(17, 4096, 2048, 2), (32, 1024, 768, 3), (33, 512, 512, 4),
                                     (48, 2048, 256, 6), (63, 256, 1024, 8), (64, 4096, 512, 1),
                                     (2, 8192, 512, 5), (65, 512, 256, 7)])
def test_gemm_small_m(m, k, n, K):
    layer = inputs.make_layer(m, k, n, K, seed=6100 + m + K)
    y, ws = run_gemm(layer)
    check(layer, y)
    y2, _ = run_gemm(layer, ws)  # deterministic with the workspace reused
    assert np.array_equal(y, y2)


def test_gemm_small_m_agrees_with_gemv_halves():
    # m = 32 against two m = 16 GEMV calls on the rows' halves
    layer = inputs.make_layer(32, 2048, 1024, 3, seed=5)
    yg, _ = run_gemm(layer)
    ws = exl3.new_workspace(exl3.exl3_gemv_workspace_size(16, 2048, 1024, 3))
    for h in range(2):
        rows = slice(16 * h, 16 * h + 16)
        yv = exl3.exl3_gemv(dev(layer.x[rows]), dev(layer.trellis), dev(layer.suh), dev(layer.svh), 3,
                            workspace=ws)
        yv = yv.cpu().numpy().astype(np.float64)
        ok, err, bound = within_tolerance(yg[rows], yv)
        assert ok, (h, err, bound)


@pytest.mark.parametrize("m,k,n,K", [(32, 1024, 384, 3), (32, 2048, 1152, 4), (17, 512, 128, 2),
                                     (200, 512, 384, 5), (64, 1024, 640, 8)])
def test_gemm_half_width_last_tile(m, k, n, K):
    # n = 256j + 128: the last output tile carries 128 columns; every column
    # must match the oracle (guard regions around y: tests/test_gpu_canary.py)
    layer = inputs.make_layer(m, k, n, K, seed=6500 + m + n + K)
    y, _ = run_gemm(layer)
    check(layer, y)


@pytest.mark.parametrize("m", [1, 16, 17, 32, 65])
def test_matmul_dispatch_matches_the_oracle(m):
    # exl3_matmul runs the GEMV for m <= 16 and the GEMM above; both must give
    # the layer to the stated tolerance, n = 384 included
    k, n, K = 1024, 384, 3
    layer = inputs.make_layer(m, k, n, K, seed=6600 + m)
    ws = exl3.new_workspace(exl3.exl3_matmul_workspace_size(m, k, n, K))
    y = exl3.exl3_matmul(dev(layer.x), dev(layer.trellis), dev(layer.suh), dev(layer.svh), K, workspace=ws)
    torch.cuda.synchronize()
    assert exl3.exl3_workspace_status(ws) == exl3.EXL3_OK
    check(layer, y.cpu().numpy().astype(np.float64))


def _multi_layers(m, specs, seed):
    """Layers of one multi call: each spec (k, n, K) gets its own x, trellis,
    suh and svh."""
    return [inputs.make_layer(m, k, n, K, seed=seed + i) for i, (k, n, K) in enumerate(specs)]


def _multi_args(layers):
    return [(dev(L.x), dev(L.trellis), dev(L.suh), dev(L.svh), L.K, None) for L in layers]


@pytest.mark.parametrize("m,specs", [
    (32, [(512, 1024, 3), (512, 256, 3), (512, 256, 3)]),              # q/k/v-like: one wide, two narrow
    (40, [(256, 384, 2), (256, 128, 2)]),                              # half-width tiles in both layers
    (200, [(384, 512, 4), (384, 640, 4), (384, 128, 4)]),              # weights-as-B form, ragged m
    (17, [(1024, 256, 8)] * 3 + [(1024, 384, 8)] * 7),                 # 10 layers: two launches
])
def test_gemm_multi_matches_the_oracle(m, specs):
    """exl3_gemm_multi: every layer's y equals the oracle's (each layer with its
    own x, suh, svh; tiles of all layers share one launch's stream-K split)."""
    layers = _multi_layers(m, specs, seed=7100 + m)
    args = _multi_args(layers)
    ws = exl3.new_workspace(exl3.exl3_gemm_multi_workspace_size(args, m))
    ys = exl3.exl3_gemm_multi(args, workspace=ws)
    torch.cuda.synchronize()
    assert exl3.exl3_workspace_status(ws) == exl3.EXL3_OK
    for L, y in zip(layers, ys):
        check(L, y.cpu().numpy().astype(np.float64))
    # a second call on the same workspace (counters back at zero) gives the same bits
    ys2 = exl3.exl3_gemm_multi(args, workspace=ws)
    torch.cuda.synchronize()
    for y, y2 in zip(ys, ys2):
        assert torch.equal(y, y2)


def test_gemm_multi_rejects_mixed_k_or_K():
    for specs in ([(256, 256, 3), (512, 256, 3)], [(256, 256, 3), (256, 256, 4)]):
        args = _multi_args(_multi_layers(32, specs, seed=7300))
        assert exl3.exl3_gemm_multi_workspace_size(args, 32) == 0
        with pytest.raises(exl3.Exl3Error) as e:
            exl3.exl3_gemm_multi(args, workspace=exl3.new_workspace(1 << 20))
        assert e.value.status == exl3.EXL3_ERR_UNSUPPORTED


@pytest.mark.parametrize("m", [8, 40])
def test_matmul_multi_matches_the_oracle(m):
    """exl3_matmul_multi: the GEMV multi call below m = 17 (any mix of k and K
    is allowed there), the GEMM multi call above."""
    specs = [(512, 384, 2), (512, 256, 2)] if m > 16 else [(512, 384, 2), (256, 256, 5)]
    layers = _multi_layers(m, specs, seed=7400 + m)
    args = _multi_args(layers)
    ws = exl3.new_workspace(exl3.exl3_matmul_multi_workspace_size(args, m))
    ys = exl3.exl3_matmul_multi(args, workspace=ws)
    torch.cuda.synchronize()
    for L, y in zip(layers, ys):
        check(L, y.cpu().numpy().astype(np.float64))
