"""exl3_gemv_multi: several independent layers in one call, through the C ABI.

Each layer's output must satisfy the stated tolerance against the fp64
oracle, agree with exl3_gemv on the same layer to that tolerance, and be
bitwise reproducible from call to call.
"""
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


def run_multi(layers):
    args = [(dev(L.x), dev(L.trellis), dev(L.suh), dev(L.svh), L.K, None) for L in layers]
    ws = exl3.new_workspace(exl3.exl3_gemv_multi_workspace_size(args, layers[0].m))
    ys = exl3.exl3_gemv_multi(args, workspace=ws)
    torch.cuda.synchronize()
    return [y.cpu().numpy().astype(np.float64) for y in ys], args, ws


def check(L, y, col_blocks=None):
    ref = oracle.linear(L.x, L.trellis, L.suh, L.svh, L.K, col_blocks=col_blocks)
    yy = y if col_blocks is None else y[:, col_blocks[0] * 128:col_blocks[1] * 128]
    ok, err, bound = within_tolerance(yy, ref)
    assert ok, "max err %.4g > bound %.4g" % (err, bound)


@pytest.mark.parametrize("m", [1, 3, 9, 16])
def test_multi_mixed_shapes_and_bits(m):
    shapes = [(384, 256, 4), (256, 640, 2), (1024, 128, 4), (128, 384, 7), (512, 256, 2), (256, 256, 4)]
    layers = [inputs.make_layer(m, k, n, K, seed=8000 + 10 * i + m) for i, (k, n, K) in enumerate(shapes)]
    ys, _, _ = run_multi(layers)
    for L, y in zip(layers, ys):
        check(L, y)


def test_multi_decode_set_matches_oracle_and_single_calls():
    layers = [inputs.make_layer(m, k, n, K, inputs.seed_for(1, c), o)
              for c, (nm, m, k, n, K, o) in enumerate(workloads.LLAMA8B_DECODE)]
    ys, args, _ = run_multi(layers)
    for L, y, a in zip(layers, ys, args):
        nb = L.n // 128
        check(L, y, col_blocks=(0, 1))
        check(L, y, col_blocks=(nb - 1, nb))
        ws = exl3.new_workspace(exl3.exl3_gemv_workspace_size(L.m, L.k, L.n, L.K))
        y1 = exl3.exl3_gemv(*a[:5], workspace=ws).cpu().numpy().astype(np.float64)
        ok, err, bound = within_tolerance(y, y1)
        assert ok, "multi vs single: max diff %.4g > %.4g" % (err, bound)


def test_multi_more_layers_than_one_launch_takes():
    # one launch takes up to 32 layers; 34 of mixed K run as two launches
    layers = [inputs.make_layer(2, 256, 256, 2 + i % 3, seed=8500 + i) for i in range(34)]
    ys, _, _ = run_multi(layers)
    for L, y in zip(layers, ys):
        check(L, y)


def test_multi_is_deterministic():
    layers = [inputs.make_layer(1, 1024, 512, K, seed=8600 + K) for K in (3, 3, 5)]
    ys, args, ws = run_multi(layers)
    for _ in range(2):
        again = exl3.exl3_gemv_multi([a[:5] + (None,) for a in args], workspace=ws)
        torch.cuda.synchronize()
        for y, z in zip(ys, again):
            assert np.array_equal(y, z.cpu().numpy().astype(np.float64))


def test_multi_with_views_into_contiguous_buffers():
    # x and y of every layer are views into one device buffer each (as an
    # application batching a decode step's activations would hold them)
    shapes = [(256, 384, 3), (1024, 128, 2), (128, 256, 8), (384, 640, 4)]
    layers = [inputs.make_layer(2, k, n, K, seed=8700 + i) for i, (k, n, K) in enumerate(shapes)]
    ref, _, _ = run_multi(layers)
    xs = torch.cat([dev(L.x).reshape(-1) for L in layers])
    ys = torch.empty(sum(2 * L.n for L in layers), dtype=torch.float16, device="cuda")
    args, ox, oy = [], 0, 0
    for L in layers:
        xv = xs[ox:ox + 2 * L.k].view(2, L.k)
        yv = ys[oy:oy + 2 * L.n].view(2, L.n)
        args.append((xv, dev(L.trellis), dev(L.suh), dev(L.svh), L.K, yv))
        ox += 2 * L.k
        oy += 2 * L.n
    ws = exl3.new_workspace(exl3.exl3_gemv_multi_workspace_size(args, 2))
    exl3.exl3_gemv_multi(args, workspace=ws)
    torch.cuda.synchronize()
    for a, r in zip(args, ref):
        assert np.array_equal(a[5].cpu().numpy().astype(np.float64), r)


@pytest.mark.parametrize("m", [1, 12])
def test_multi_tiny_and_large_k_groups(m):
    # a one-block K = 1 layer (8 units: its CTA group is a single CTA) beside a
    # large K = 8 layer that takes the rest of the grid
    layers = [inputs.make_layer(m, 128, 128, 1, seed=8800 + m), inputs.make_layer(m, 2048, 2048, 8, seed=8900 + m)]
    ys, _, _ = run_multi(layers)
    check(layers[0], ys[0])
    check(layers[1], ys[1], col_blocks=(0, 2))
    check(layers[1], ys[1], col_blocks=(14, 16))
