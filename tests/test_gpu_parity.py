"""GPU parity of the CUDA path (through the C ABI) against the fp64 oracle.

Decoded weights must be bit-exact; layer outputs must satisfy
max|y - y_ref| <= 1e-2 * rms(y_ref) + 1e-3.  Inputs come from the seeded
generator shared by both sides; expected values come only from ``oracle``.
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


def host(t):
    return t.cpu().numpy()


def fp16_ulp(x):
    a = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -14)))
    return 2.0 ** (e - 10)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    exl3.load()
    yield


# -------------------------------------------------------------- hadamard ---

@pytest.mark.parametrize("rows,cols,pre,post", [(1, 128, False, False), (3, 4096, True, True),
                                                (17, 384, True, False), (64, 1024, False, True)])
def test_hadamard(rows, cols, pre, post):
    rng = np.random.default_rng(rows * 1000 + cols)
    x = rng.standard_normal((rows, cols)).astype(np.float16)
    p = rng.choice([-1.0, 1.0], cols).astype(np.float16) if pre else None
    q = rng.uniform(0.01, 0.05, cols).astype(np.float16) if post else None
    y = host(exl3.exl3_hadamard(dev(x), pre=None if p is None else dev(p),
                                post=None if q is None else dev(q)))
    ref = oracle.hadamard(x.astype(np.float64), None if p is None else p.astype(np.float64),
                          None if q is None else q.astype(np.float64))
    err = np.abs(y.astype(np.float64) - ref)
    assert (err <= fp16_ulp(ref) + 1e-7).all()


def test_hadamard_in_place_and_empty():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((5, 256)).astype(np.float16)
    t = dev(x)
    exl3.exl3_hadamard(t, y=t)
    ref = oracle.hadamard(x.astype(np.float64))
    assert (np.abs(host(t).astype(np.float64) - ref) <= fp16_ulp(ref) + 1e-7).all()
    e = torch.empty((0, 128), dtype=torch.float16, device="cuda")
    exl3.exl3_hadamard(e, y=e)


# ---------------------------------------------------------------- decode ---

def _patterns(k, n, K, rng):
    shape = (k // 16, n // 16, 16 * K)
    wrap = np.zeros(shape, dtype=np.uint16)
    wrap[:, :, -1] = 1  # only the last bit of every tile: exercises the tail-biting wrap
    first = np.zeros(shape, dtype=np.uint16)
    first[:, :, 0] = 0x8000
    return {"random": rng.integers(0, 65536, size=shape, dtype=np.uint16),
            "zeros": np.zeros(shape, dtype=np.uint16),
            "ones": np.full(shape, 0xFFFF, dtype=np.uint16),
            "wrap": wrap, "first": first}


@pytest.mark.parametrize("K", range(1, 9))
def test_decode_tiles_bit_exact(K):
    rng = np.random.default_rng(K)
    k, n = 64, 96
    for name, tr in _patterns(k, n, K, rng).items():
        w = host(exl3.exl3_decode_tiles(dev(tr), k, n, K))
        ref = oracle.decode_tiles(tr, k, n, K)
        assert np.array_equal(w.view(np.uint16), ref), (name, K)


def test_decode_tiles_large_grid():
    # more tiles than one wave of warps: the grid-stride loop
    rng = np.random.default_rng(11)
    k, n, K = 2048, 2048, 3
    tr = rng.integers(0, 65536, size=(k // 16, n // 16, 16 * K), dtype=np.uint16)
    w = host(exl3.exl3_decode_tiles(dev(tr), k, n, K)).view(np.uint16)
    ref = oracle.decode_tiles(tr, k, n, K)
    assert np.array_equal(w, ref)


# ------------------------------------------------------------------ gemv ---

def run_gemv(layer, ws=None):
    m, k, n, K = layer.m, layer.k, layer.n, layer.K
    if ws is None:
        ws = exl3.new_workspace(exl3.exl3_gemv_workspace_size(m, k, n, K))
    y = exl3.exl3_gemv(dev(layer.x), dev(layer.trellis), dev(layer.suh), dev(layer.svh), K,
                       workspace=ws)
    return host(y).astype(np.float64), ws


def check_layer(layer, y, col_blocks=None):
    ref = oracle.linear(layer.x, layer.trellis, layer.suh, layer.svh, layer.K, col_blocks=col_blocks)
    if col_blocks is not None:
        y = y[:, col_blocks[0] * 128:col_blocks[1] * 128]
    ok, err, bound = within_tolerance(y, ref)
    assert ok, "max err %.4g > bound %.4g" % (err, bound)
    assert np.isfinite(y).all()


@pytest.mark.parametrize("K", range(1, 9))
@pytest.mark.parametrize("m", [1, 3, 8, 9, 16])
def test_gemv_small(K, m):
    layer = inputs.make_layer(m, 384, 256, K, seed=7000 + 10 * K + m)
    y, _ = run_gemv(layer)
    check_layer(layer, y)


@pytest.mark.parametrize("m,k,n,K", [(1, 896, 128, 4),       # 7 splits of one block each
                                     (16, 2560, 5120, 2),    # ragged last split
                                     (2, 128, 128, 8),       # single block, no split
                                     (5, 1152, 384, 5)])
def test_gemv_splits_and_tails(m, k, n, K):
    layer = inputs.make_layer(m, k, n, K, seed=8000 + m + K)
    y, ws = run_gemv(layer)
    check_layer(layer, y)
    # counters re-armed: a second call with the same workspace gives identical output
    y2, _ = run_gemv(layer, ws)
    assert np.array_equal(y, y2)
    assert exl3.exl3_workspace_status(ws) == exl3.EXL3_OK


def test_gemv_closed_form_constant_weights():
    # all-zero trellis: every weight is c = 0.76806640625 and only the first column of each
    # 128-block is nonzero: y[r,128j] = 128 c svh[128j] sum_b x'... (oracle pins the formula)
    layer = inputs.make_layer(2, 512, 384, 3, seed=9)
    layer.trellis[:] = 0
    y, _ = run_gemv(layer)
    check_layer(layer, y)
    mask = np.ones(384, dtype=bool)
    mask[::128] = False
    assert (y[:, mask] == 0).all()


def test_gemv_pr1_layer():
    (name, m, k, n, K, outl), = workloads.PR1
    layer = inputs.make_layer(m, k, n, K, inputs.seed_for(0, 0), outl)
    y, _ = run_gemv(layer)
    check_layer(layer, y)


@pytest.mark.parametrize("case", range(len(workloads.LLAMA8B_DECODE)))
def test_gemv_llama8b_decode_set(case):
    name, m, k, n, K, outl = workloads.LLAMA8B_DECODE[case]
    layer = inputs.make_layer(m, k, n, K, inputs.seed_for(1, case), outl)
    y, _ = run_gemv(layer)
    check_layer(layer, y, col_blocks=(0, min(n // 128, 8)))
    check_layer(layer, y, col_blocks=(n // 128 - 1, n // 128))


@pytest.mark.parametrize("case", list(range(0, len(workloads.SMALL_BATCH), 7)))
def test_gemv_llama70b_small_batch_sampled(case):
    name, m, k, n, K, outl = workloads.SMALL_BATCH[case]
    layer = inputs.make_layer(m, k, n, K, inputs.seed_for(2, case), outl)
    y, _ = run_gemv(layer)
    nb = n // 128
    check_layer(layer, y, col_blocks=(0, 1))
    check_layer(layer, y, col_blocks=(nb // 2, nb // 2 + 1))
    check_layer(layer, y, col_blocks=(nb - 1, nb))


# Where the GEMV's input rotation runs follows from the plan: inside the main
# kernel (each CTA rotates the blocks its own units read) when every CTA's
# unit range is at most the smallest tile-row count k/16 of its K group and
# (range/8 + 2) * m <= 16; otherwise in a rotation kernel launched just
# before.  The shapes below fall on both sides (ranges from the plan's grid:
# min(296, units/16) CTAs, aligned to whole column blocks for one layer).
@pytest.mark.parametrize("m,k,n,K,where", [
    (1, 4096, 4096, 4, "in kernel"),          # 8192 units / 288 CTAs: 29 rows of 256
    (4, 1024, 1024, 3, "in kernel"),          # 512 units / 32 CTAs: 16 rows of 64, 16 jobs per CTA
    (16, 1024, 1024, 3, "separate"),          # the same ranges, 64 jobs per CTA
    (1, 256, 38016, 2, "separate"),           # 297 column blocks: ranges of 17 > 16 tile rows
])
def test_gemv_rotation_in_kernel_or_separate(m, k, n, K, where):
    layer = inputs.make_layer(m, k, n, K, seed=7600 + m + K)
    y, _ = run_gemv(layer)
    nb = n // 128
    check_layer(layer, y, col_blocks=(0, min(nb, 4)))
    check_layer(layer, y, col_blocks=(nb - 2, nb))


def test_gemv_multi_in_kernel_rotation_across_layers():
    # two layers of one K group, 360 units on 22 CTAs: ranges of 16-17 units
    # (<= 24 tile rows), so each CTA rotates its own blocks, and CTA 14's range
    # [229, 245) ends layer 0 (rows 13..23 of its last column block) and starts
    # layer 1 (rows 0..4 of its first)
    layers = [inputs.make_layer(1, 384, 1280, 3, seed=7700), inputs.make_layer(1, 384, 640, 3, seed=7701)]
    args = [(dev(L.x), dev(L.trellis), dev(L.suh), dev(L.svh), L.K, None) for L in layers]
    ws = exl3.new_workspace(exl3.exl3_gemv_multi_workspace_size(args, 1))
    ys = exl3.exl3_gemv_multi(args, workspace=ws)
    for L, y in zip(layers, ys):
        check_layer(L, host(y).astype(np.float64))


def test_gemm_timeout_reports_status_without_hang():
    # the GEMM's stage hand-offs are bounded waits: with a 1 ns bound they run
    # out, the kernel records EXL3_ERR_TIMEOUT and returns -- no fault, no hang
    layer = inputs.make_layer(256, 1024, 512, 4, seed=5)
    ws = exl3.new_workspace(exl3.exl3_gemm_workspace_size(256, 1024, 512, 4))
    args = (dev(layer.x), dev(layer.trellis), dev(layer.suh), dev(layer.svh), 4)
    try:
        exl3.exl3_debug_set_wait_limit_ns(1)
        exl3.exl3_gemm(*args, workspace=ws)
        torch.cuda.synchronize()
        st = exl3.exl3_workspace_status(ws, clear=True)
    finally:
        exl3.exl3_debug_set_wait_limit_ns(0)
    assert st == exl3.EXL3_ERR_TIMEOUT
    # the context is still usable; the status read with clear also returned the
    # split-tile counters (which a timed-out call may leave part-way) to zero,
    # so the next call on the same workspace is correct
    y = exl3.exl3_gemm(*args, workspace=ws).cpu().numpy().astype(np.float64)
    assert exl3.exl3_workspace_status(ws) == exl3.EXL3_OK
    check_layer(layer, y)


def test_pdl_launches_give_identical_results():
    # a chain of dependent calls (each layer's input is the previous layer's output) run with
    # and without programmatic dependent launch must agree bit for bit
    layers = [inputs.make_layer(1, 1024, 1024, K, seed=40 + K) for K in (2, 3, 4)]
    big = inputs.make_layer(256, 1024, 1024, 4, seed=44)
    dl = [(dev(L.trellis), dev(L.suh), dev(L.svh), L.K) for L in layers]
    db = (dev(big.trellis), dev(big.suh), dev(big.svh), big.K)
    x0 = dev(layers[0].x)
    xb = dev(big.x)
    ws = exl3.new_workspace(max(exl3.exl3_gemv_workspace_size(1, 1024, 1024, 4),
                                exl3.exl3_gemm_workspace_size(256, 1024, 1024, 4)))

    def chain():
        y = x0
        for t, suh, svh, K in dl * 3:
            y = exl3.exl3_gemv(y, t, suh, svh, K, workspace=ws)
        z = xb
        for _ in range(3):
            z = exl3.exl3_gemm(z, db[0], db[1], db[2], db[3], workspace=ws)
        torch.cuda.synchronize()
        return y.cpu().numpy(), z.cpu().numpy()

    ref = chain()
    try:
        exl3.exl3_set_launch_flags(exl3.EXL3_LAUNCH_PDL)
        got = chain()
    finally:
        exl3.exl3_set_launch_flags(0)
    assert np.array_equal(ref[0], got[0]) and np.array_equal(ref[1], got[1])
    assert np.isfinite(ref[0]).all() and np.isfinite(ref[1]).all()


def test_native_library_is_the_in_tree_build():
    import os

    maps = open("/proc/self/maps").read()
    assert exl3.library_path() in maps
    assert os.path.dirname(exl3.library_path()).endswith("trellis_coded_bit_b200")
