"""Pins of the fp64 oracle against what the pages and the mathematics fix.

None of these calls the CUDA library.  Each pin is chosen so that a plausible
mistake in the oracle (a dropped term, a flipped sign or bit, a transposed
operand, a missing wrap) fails at least one of them.
"""
import hashlib

import numpy as np
import pytest
import scipy.linalg

import oracle
from oracle import recurrence
from conftest import read_golden

H128 = scipy.linalg.hadamard(128).astype(np.float64)  # Sylvester construction


# ------------------------------------------------------------------ fp16 ---

def test_half_to_double_all_patterns():
    bits = np.arange(65536, dtype=np.uint16)
    got = oracle.half_to_double(bits)
    ref = bits.view(np.float16).astype(np.float64)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    # signed zero kept
    assert np.signbit(got[0x8000]) and not np.signbit(got[0])


def test_double_to_half_rne_matches_numpy():
    rng = np.random.default_rng(7)
    vals = np.concatenate([
        rng.standard_normal(4000) * 4.0,
        rng.standard_normal(1000) * 1e-5,          # subnormal range
        rng.uniform(-70000, 70000, 500),           # includes overflow
        # exact ties between neighbouring fp16 values (round half to even)
        (np.arange(1, 2048, dtype=np.float64) + 0.5) * 2.0 ** -10,
        (np.arange(1, 1024, dtype=np.float64) + 0.5) * 2.0 ** -24,
        [0.0, -0.0, 65504.0, 65519.99, 65520.0, -65520.0, 2.0 ** -24, 2.0 ** -25, 3 * 2.0 ** -26],
    ])
    got = oracle.double_to_half(vals)
    with np.errstate(over="ignore"):
        ref = vals.astype(np.float16).view(np.uint16)
    assert np.array_equal(got, ref)


# ------------------------------------------------------------- codebook ---

@pytest.fixture(scope="module")
def table():
    return oracle.codebook_table()


def test_codebook_spot_values(table):
    for st, v, hi, lo, wbits, wval in read_golden("codebook_spot.txt"):
        s = int(st, 16)
        assert table[s] == int(wbits, 16), st
        assert np.float64(np.uint16(table[s]).view(np.float16)) == float(wval)
        assert float(hi) + float(lo) == pytest.approx(float(wval), abs=2.0 ** -10)


def test_codebook_whole_table_invariants(table):
    g = {row[0]: row[1] for row in read_golden("codebook_stats.txt")}
    w = table.view(np.float16)
    wd = w.astype(np.float64)
    assert hashlib.sha256(table.astype("<u2").tobytes()).hexdigest() == g["sha256_le_fp16"]
    assert np.isfinite(wd).all()
    assert int((wd == 0).sum()) == int(g["zeros"])
    assert len(np.unique(wd)) == int(g["distinct"])
    assert int((wd < 0).sum()) == int(g["negative"])
    assert int(table[np.argmin(wd)]) == int(g["min_bits"], 16)
    assert int(table[np.argmax(wd)]) == int(g["max_bits"], 16)
    assert np.abs(wd[wd != 0]).min() == float(g["min_abs_nonzero"])
    assert wd.sum() == float(g["sum"])
    assert (wd ** 2).sum() == pytest.approx(float(g["sum_sq"]), rel=1e-15)


def test_codebook_split_sum_bound(table):
    # The word's two halves, from the definition with numpy (not the oracle's
    # code): their exact sum rounds (nearest even) to the oracle's value, the
    # count of states where that rounding changes anything is the golden one,
    # and the change is at most half an fp16 ulp, i.e. at most 2^-11 relative
    # -- the bound behind computing x * (hi + lo) exactly instead of with the
    # rounded weight.
    g = {row[0]: row[1] for row in read_golden("codebook_stats.txt")}
    s = np.arange(65536, dtype=np.uint64)
    v = (s * 89226354 + 64248484) & 0xffffffff
    v = (v & 0x8fff8fff) ^ 0x3b603b60
    hi = (v >> 16).astype(np.uint16).view(np.float16).astype(np.float64)
    lo = (v & 0xffff).astype(np.uint16).view(np.float16).astype(np.float64)
    exact = hi + lo  # exact in fp64: both halves are fp16 with exponents -3..0
    w = table.view(np.float16).astype(np.float64)
    assert np.array_equal(exact.astype(np.float16).view(np.uint16), table)
    d = np.abs(exact - w)
    assert int((d > 0).sum()) == int(g["rounded_sums"])
    nz = w != 0
    ulp = 2.0 ** (np.floor(np.log2(np.abs(w[nz]))) - 10)
    assert (d[nz] <= 0.5 * ulp).all()
    assert (d[nz] / np.abs(w[nz])).max() == 2.0 ** -11
    assert (d[~nz] == 0).all()


def test_codebook_halves_range(table):
    # |w| < 4 since each half is in +-[0.125, 2); and w never subnormal
    wd = table.view(np.float16).astype(np.float64)
    assert np.abs(wd).max() < 4.0
    nz = wd[wd != 0]
    assert (np.abs(nz) >= 2.0 ** -14).all()


# --------------------------------------------------------------- trellis ---

@pytest.mark.parametrize("K", range(1, 9))
def test_states_two_formulations_agree(K):
    rng = np.random.default_rng(100 + K)
    k, n = 32, 48
    trellis = rng.integers(0, 65536, size=(k // 16, n // 16, 16 * K), dtype=np.uint16)
    st = oracle.states(trellis, k, n, K)
    for tk in range(k // 16):
        for tn in range(n // 16):
            assert list(st[tk, tn]) == recurrence.tile_states(trellis[tk, tn], K)


@pytest.mark.parametrize("K", range(1, 9))
def test_states_constant_streams(K):
    zeros = np.zeros((1, 1, 16 * K), dtype=np.uint16)
    ones = np.full((1, 1, 16 * K), 0xFFFF, dtype=np.uint16)
    assert (oracle.states(zeros, 16, 16, K) == 0).all()
    assert (oracle.states(ones, 16, 16, K) == 0xFFFF).all()


def test_states_wrap_case_K4():
    words = np.zeros(64, dtype=np.uint16)
    words[63] = 0x0001
    expect = {int(i): int(s, 16) for i, s in read_golden("trellis_wrap_K4.txt")}
    for i in range(256):
        assert oracle.state(words, 4, i) == expect.get(i, 0), i


@pytest.mark.parametrize("K", [1, 2, 4, 8])
def test_states_popcount_invariant(K):
    # when K divides 16 every stream bit appears in exactly 16/K windows
    rng = np.random.default_rng(K)
    words = rng.integers(0, 65536, size=16 * K, dtype=np.uint16)
    total = sum(bin(oracle.state(words, K, i)).count("1") for i in range(256))
    assert total == (16 // K) * sum(bin(int(w)).count("1") for w in words)


@pytest.mark.parametrize("K", [1, 3, 4, 7])
def test_single_bit_walks_through_windows(K):
    # one set bit at stream position p appears in the states of exactly the weights whose
    # windows cover p, at bit index (window end - 1 - p); brute force over all p of a tile
    rng = np.random.default_rng(K)
    for p in rng.choice(256 * K, 12, replace=False):
        words = np.zeros(16 * K, dtype=np.uint16)
        words[p // 16] = 1 << (15 - p % 16)
        for i in range(256):
            end = (i + 1) * K  # exclusive end of the window, cyclic
            off = (end - 1 - p) % (256 * K)
            want = (1 << off) if off < 16 else 0
            assert oracle.state(words, K, i) == want


@pytest.mark.parametrize("K", [2, 5])
def test_decode_layout_row_major_tiles(K):
    rng = np.random.default_rng(K)
    k, n = 48, 32
    trellis = rng.integers(0, 65536, size=(k // 16, n // 16, 16 * K), dtype=np.uint16)
    table = oracle.codebook_table()
    w = oracle.decode_tiles(trellis, k, n, K)
    for tk in range(k // 16):
        for tn in range(n // 16):
            st = recurrence.tile_states(trellis[tk, tn], K)
            blk = np.array([table[s] for s in st], dtype=np.uint16).reshape(16, 16)
            assert np.array_equal(w[16 * tk:16 * tk + 16, 16 * tn:16 * tn + 16], blk)


# -------------------------------------------------------------- hadamard ---

def test_hadamard_matches_sylvester_matrix():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((3, 256))
    pre = rng.choice([-1.0, 1.0], 256)
    post = rng.uniform(0.5, 2.0, 256)
    y = oracle.hadamard(x, pre, post)
    xs = (x * pre).reshape(3, 2, 128)
    ref = (xs @ H128.T / np.sqrt(128)).reshape(3, 256) * post
    np.testing.assert_allclose(y, ref, rtol=0, atol=1e-12)


def test_hadamard_orthogonality_and_involution():
    eye = np.eye(128)
    h = oracle.hadamard(eye)              # rows: H e_j / sqrt(128)
    np.testing.assert_allclose(h @ h.T, eye, atol=1e-13)        # H H^T = 128 I
    np.testing.assert_allclose(oracle.hadamard(h), eye, atol=1e-13)  # involution
    np.testing.assert_allclose(h[0], np.full(128, 1 / np.sqrt(128)), atol=1e-15)  # H e0 = 1
    ones = oracle.hadamard(np.ones((1, 128)))
    np.testing.assert_allclose(ones[0], np.eye(128)[0] * np.sqrt(128), atol=1e-12)


def test_hadamard_parseval():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((5, 384))
    pre = rng.choice([-1.0, 1.0], 384)
    y = oracle.hadamard(x, pre)
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x * pre, axis=1), rtol=1e-13)


# ---------------------------------------------------------------- linear ---

def _f16(a):
    return np.asarray(a, dtype=np.float16)


def test_linear_closed_form_constant_weights():
    # all-zero words: every state 0, every weight c = codebook(0); then
    # y[r,128j] = 128 c svh[128j] sum_b x[r,128b] suh[128b] (shown below), other columns 0
    rng = np.random.default_rng(5)
    m, k, n, K = 2, 256, 384, 3
    x = _f16(rng.standard_normal((m, k)))
    suh = _f16(rng.choice([-1.0, 1.0], k))
    svh = _f16(rng.uniform(-0.05, 0.05, n))
    trellis = np.zeros((k // 16, n // 16, 16 * K), dtype=np.uint16)
    y = oracle.linear(x, trellis, suh, svh, K)
    c = 0.76806640625
    xs = x.astype(np.float64) * suh.astype(np.float64)
    # x' = H(xs)/sqrt(128) per block; sum over all k of x' = sum_b sqrt(128) * xs[128b]
    # (only H's first row sums to 128); y' = c * sum_k x' for every column; then the
    # output rotation concentrates the constant on each block's first column.
    s = np.sqrt(128) * xs[:, ::128].sum(axis=1)
    ref = np.zeros((m, n))
    ref[:, ::128] = (c * s)[:, None] * np.sqrt(128) * svh.astype(np.float64)[::128]
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)


def test_linear_hand_case_wrap_tile():
    # k = n = 128, m = 1, x = e0, suh = svh = 1; tile (0,0) at K = 4 holds the wrap
    # pattern (word 63 = 1), every other tile is zero.  Weights: (0,0)=w(0x10),
    # (0,1)=w(0x100), (0,2)=w(0x1000), (15,15)=w(0x1), all others c = w(0).
    spot = {int(r[0], 16): float(r[5]) for r in read_golden("codebook_spot.txt")}
    c = spot[0]
    d = {0: spot[0x10] - c, 1: spot[0x100] - c, 2: spot[0x1000] - c, 15: spot[0x1] - c}
    K = 4
    trellis = np.zeros((8, 8, 64), dtype=np.uint16)
    trellis[0, 0, 63] = 1
    x = np.zeros((1, 128), dtype=np.float16)
    x[0, 0] = 1
    ones = np.ones(128, dtype=np.float16)
    y = oracle.linear(x, trellis, ones, ones, K)[0]
    # x' = 1/sqrt(128) everywhere, y'[col] = colsum/sqrt(128), y = H y'/sqrt(128):
    # y[i] = (1/128) sum_col H[i][col] colsum[col]
    ref = np.zeros(128)
    for i in range(128):
        acc = 128 * c * 128 if i == 0 else 0.0
        for col, dv in d.items():
            acc += (-1) ** bin(i & col).count("1") * dv
        ref[i] = acc / 128
    np.testing.assert_allclose(y, ref, rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("K", range(1, 9))
def test_linear_dense_formulation(K):
    # y = x diag(suh) Hk W Hn diag(svh) / 128 with scipy's Hadamard and numpy matmuls;
    # W from the shift-register states and the (pinned) codebook table
    rng = np.random.default_rng(50 + K)
    m, k, n = 3, 256, 128
    x = _f16(rng.standard_normal((m, k)))
    suh = _f16(rng.choice([-1.0, 1.0], k))
    svh = _f16(rng.choice([-1.0, 1.0], n) * rng.uniform(0.01, 0.05, n))
    trellis = rng.integers(0, 65536, size=(k // 16, n // 16, 16 * K), dtype=np.uint16)
    table = oracle.codebook_table().view(np.float16).astype(np.float64)
    W = np.zeros((k, n))
    for tk in range(k // 16):
        for tn in range(n // 16):
            st = recurrence.tile_states(trellis[tk, tn], K)
            W[16 * tk:16 * tk + 16, 16 * tn:16 * tn + 16] = table[st].reshape(16, 16)
    Hk = scipy.linalg.block_diag(*([H128] * (k // 128)))
    Hn = scipy.linalg.block_diag(*([H128] * (n // 128)))
    ref = x.astype(np.float64) @ np.diag(suh.astype(np.float64)) @ Hk @ W @ Hn \
        @ np.diag(svh.astype(np.float64)) / 128.0
    y = oracle.linear(x, trellis, suh, svh, K)
    np.testing.assert_allclose(y, ref, rtol=1e-10, atol=1e-10)


def test_linear_column_blocks_and_threads():
    rng = np.random.default_rng(9)
    m, k, n, K = 2, 128, 512, 2
    x = _f16(rng.standard_normal((m, k)))
    suh = _f16(rng.choice([-1.0, 1.0], k))
    svh = _f16(rng.uniform(-0.05, 0.05, n))
    trellis = rng.integers(0, 65536, size=(k // 16, n // 16, 16 * K), dtype=np.uint16)
    full = oracle.linear(x, trellis, suh, svh, K)
    part = oracle.linear(x, trellis, suh, svh, K, col_blocks=(1, 3), threads=4)
    np.testing.assert_array_equal(part, full[:, 128:384])
