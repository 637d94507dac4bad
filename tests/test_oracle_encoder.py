"""Pins of the oracle's tail-biting trellis encoder (CPU only).

The encoder (oracle_encode_seq / oracle_encode) follows the page "ExLlamaV3推理快的
秘密: EXL3 GEMM内核与融合Viterbi编码CUDA实现剖析", section Viterbi编码内核剖析: a
Viterbi search over the trellis for the cheapest path, closed into a
tail-biting code.  These tests check it against things that do not use its
recursion:
  - exhaustive search over every bit string of a small trellis (8-bit states),
    with states taken as cyclic windows of the string: the encoder's code must
    cost exactly the cheapest code that shares its overlap, never less than the
    cheapest code overall, and its reported cost must be the cost of its bits;
  - on the real 16-bit trellis: targets that are themselves decoded weights of
    a random code are encoded at zero cost and decode back exactly; the
    reported cost is the squared error of the decoded code; it is bounded below
    by per-weight nearest-value rounding and above by another code with the
    same overlap; the squared error falls as K grows.
"""
import itertools

import numpy as np
import pytest

import oracle


def windows(bits, T, L, K):
    """States of a cyclic bit string (MSB first): weight i's state is the L bits
    ending at position iK + K."""
    n = T * K
    out = []
    for i in range(T):
        s = 0
        for j in range(L):
            s = (s << 1) | bits[(i * K + K - L + j) % n]
        out.append(s)
    return out


def chunk_bits(chunks, K):
    return [(int(c) >> (K - 1 - j)) & 1 for c in chunks for j in range(K)]


@pytest.mark.parametrize("L,K,T,seed", [(8, 1, 10, 0), (8, 2, 8, 1), (8, 2, 6, 2), (8, 3, 6, 3),
                                        (8, 4, 4, 4), (6, 2, 5, 5), (8, 2, 8, 6), (8, 1, 12, 7)])
def test_encoder_matches_exhaustive_search_on_a_small_trellis(L, K, T, seed):
    rng = np.random.default_rng(seed)
    cb = rng.standard_normal(1 << L).astype(np.float32)
    target = rng.standard_normal(T).astype(np.float32)
    chunks, cost, o = oracle.encode_seq(target, L, K, cb)
    mask = (1 << (L - K)) - 1
    tg, cb64 = target.astype(np.float64), cb.astype(np.float64)

    def cost_of(bits):
        st = windows(bits, T, L, K)
        return float(sum((tg[i] - cb64[s]) ** 2 for i, s in enumerate(st))), st

    # the encoder's own bits: consistent tail-biting path, cost as reported
    mine, st = cost_of(chunk_bits(chunks, K))
    assert st[-1] & mask == o and (st[0] >> K) == o
    assert [s & ((1 << K) - 1) for s in st] == [int(c) for c in chunks]
    assert abs(mine - cost) <= 1e-5 * max(1.0, mine)
    # exhaustive: best overall, best among codes with the same overlap
    best_all, best_o = np.inf, np.inf
    for bits in itertools.product((0, 1), repeat=T * K):
        c, s2 = cost_of(bits)
        best_all = min(best_all, c)
        if s2[-1] & mask == o:
            best_o = min(best_o, c)
    assert abs(mine - best_o) <= 1e-5 * max(1.0, best_o)
    assert mine >= best_all - 1e-5 * max(1.0, best_all)


def test_encoder_free_start_pass_bounds_the_closed_code():
    # the closed code can cost more than the best open path only through the
    # wrap: with a constant cost table every code costs the same
    L, K, T = 8, 2, 8
    cb = np.full(1 << L, 0.5, dtype=np.float32)
    target = np.linspace(-1, 1, T).astype(np.float32)
    _, cost, o = oracle.encode_seq(target, L, K, cb)
    assert o == 0  # all ends tie: the smallest overlap
    assert abs(cost - float(((target.astype(np.float64) - 0.5) ** 2).sum())) < 1e-5


@pytest.mark.parametrize("K", [1, 2, 3, 4, 5, 6, 7, 8])
def test_decodable_targets_round_trip_at_zero_cost(K):
    rng = np.random.default_rng(100 + K)
    k, n = 16, 32
    tr = rng.integers(0, 65536, size=(k // 16, n // 16, 16 * K), dtype=np.uint16)
    w = oracle.half_to_double(oracle.decode_tiles(tr, k, n, K)).astype(np.float32)
    enc, cost = oracle.encode(w, K)
    assert (cost == 0).all()
    back = oracle.decode_tiles(enc, k, n, K)
    assert np.array_equal(back, oracle.decode_tiles(tr, k, n, K))


def _tile_sse(w, dec):
    k, n = w.shape
    d = (dec - w.astype(np.float64)) ** 2
    return d.reshape(k // 16, 16, n // 16, 16).sum(axis=(1, 3))


@pytest.mark.parametrize("K", [2, 3, 4])
def test_encoded_cost_is_the_decoded_error_and_within_bounds(K):
    rng = np.random.default_rng(200 + K)
    k, n = 16, 48
    w = rng.standard_normal((k, n)).astype(np.float32)
    enc, cost = oracle.encode(w, K)
    dec = oracle.half_to_double(oracle.decode_tiles(enc, k, n, K))
    sse = _tile_sse(w, dec)
    assert np.allclose(sse, cost, rtol=1e-5, atol=1e-6)
    # lower bound: every weight rounded to its nearest codebook value, ignoring
    # the trellis
    values = np.unique(oracle.half_to_double(oracle.codebook_table()))
    idx = np.clip(np.searchsorted(values, w.astype(np.float64)), 1, values.size - 1)
    near = np.minimum(np.abs(values[idx] - w), np.abs(values[idx - 1] - w))
    assert (cost >= _tile_sse(w, w - near) * (1 - 1e-6)).all()
    # upper bound: the closed code is the cheapest code with its overlap (the
    # stream's last 16 - K bits), so it costs no more than the code that is all
    # zero bits except for that overlap
    other = np.zeros_like(enc)
    for tk in range(k // 16):
        for tn in range(n // 16):
            bits = np.unpackbits(enc[tk, tn].astype(">u2").view(np.uint8))
            keep = np.zeros_like(bits)
            keep[-(16 - K):] = bits[-(16 - K):]
            other[tk, tn] = np.packbits(keep).view(">u2").astype(np.uint16)
    odec = oracle.half_to_double(oracle.decode_tiles(other, k, n, K))
    assert (cost <= _tile_sse(w, odec) * (1 + 1e-6) + 1e-6).all()


def test_squared_error_falls_with_K():
    rng = np.random.default_rng(300)
    k, n = 16, 64
    w = (1.2 * rng.standard_normal((k, n))).astype(np.float32)
    mse = []
    for K in range(1, 9):
        _, cost = oracle.encode(w, K, threads=oracle.threads_available())
        mse.append(float(cost.sum()) / w.size)
    assert all(a > b for a, b in zip(mse, mse[1:])), mse
    assert mse[-1] < 1e-3 * mse[0]
