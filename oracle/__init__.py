"""fp64 CPU oracle for the EXL3 trellis-decoded matmul -- TEST INFRASTRUCTURE.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never does, and shares no code with it.

The arithmetic lives in ``exl3_oracle.c`` (plain C, fp64); this module loads it
with ctypes and converts numpy arrays.  ``recurrence.py`` holds a second,
independent pure-Python formulation of the trellis states used to pin the C
code.  Every function states which passage of the pages it follows in the C
source; the readings of open points are listed there too.

Parity status: every oracle function is pinned by a test under tests/
(test_oracle_*.py) against closed forms, library routines, brute force or
hand-worked fixtures.
"""
import ctypes

import numpy as np

from . import build as _build

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        u16p = ctypes.POINTER(ctypes.c_uint16)
        f64p = ctypes.POINTER(ctypes.c_double)
        i64 = ctypes.c_int64
        lib.oracle_half_to_double.argtypes = [ctypes.c_uint16]
        lib.oracle_half_to_double.restype = ctypes.c_double
        lib.oracle_double_to_half.argtypes = [ctypes.c_double]
        lib.oracle_double_to_half.restype = ctypes.c_uint16
        lib.oracle_codebook.argtypes = [ctypes.c_uint16]
        lib.oracle_codebook.restype = ctypes.c_uint16
        lib.oracle_state.argtypes = [u16p, ctypes.c_int, ctypes.c_int]
        lib.oracle_state.restype = ctypes.c_uint16
        lib.oracle_states.argtypes = [u16p, i64, i64, ctypes.c_int, u16p]
        lib.oracle_states.restype = None
        lib.oracle_decode_tiles.argtypes = [u16p, i64, i64, ctypes.c_int, u16p]
        lib.oracle_decode_tiles.restype = None
        lib.oracle_hadamard.argtypes = [f64p, f64p, i64, i64, f64p, f64p]
        lib.oracle_hadamard.restype = None
        lib.oracle_linear.argtypes = [u16p, u16p, u16p, u16p, i64, i64, i64, ctypes.c_int,
                                      i64, i64, f64p, ctypes.c_int]
        lib.oracle_linear.restype = None
        f32p = ctypes.POINTER(ctypes.c_float)
        u8p = ctypes.POINTER(ctypes.c_uint8)
        lib.oracle_encode_seq.argtypes = [f32p, ctypes.c_int, ctypes.c_int, ctypes.c_int, f32p, u8p, f32p,
                                          ctypes.POINTER(ctypes.c_int)]
        lib.oracle_encode_seq.restype = ctypes.c_int
        lib.oracle_encode.argtypes = [f32p, i64, i64, ctypes.c_int, u16p, f32p, ctypes.c_int]
        lib.oracle_encode.restype = ctypes.c_int
        lib.oracle_threads_available.argtypes = []
        lib.oracle_threads_available.restype = ctypes.c_int
        _lib = lib
    return _lib


def _u16(a):
    a = np.ascontiguousarray(a)
    if a.dtype == np.float16:
        a = a.view(np.uint16)
    assert a.dtype == np.uint16, a.dtype
    return a


def _ptr(a, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def half_to_double(bits):
    """fp16 bit patterns (uint16 array) -> float64 array, via the oracle's own decoder."""
    lib = _load()
    flat = _u16(bits).ravel()
    out = np.array([lib.oracle_half_to_double(int(b)) for b in flat], dtype=np.float64)
    return out.reshape(np.shape(bits))


def double_to_half(values):
    """float64 array -> fp16 bit patterns (uint16), round-to-nearest-even."""
    lib = _load()
    flat = np.ascontiguousarray(values, dtype=np.float64).ravel()
    out = np.array([lib.oracle_double_to_half(float(v)) for v in flat], dtype=np.uint16)
    return out.reshape(np.shape(values))


def codebook_table():
    """fp16 bits of the codebook value of every 16-bit state (65536 entries)."""
    lib = _load()
    return np.array([lib.oracle_codebook(s) for s in range(65536)], dtype=np.uint16)


def codebook(state):
    return int(_load().oracle_codebook(int(state)))


def state(tile_words, K, i):
    words = _u16(tile_words)
    assert words.size == 16 * K
    return int(_load().oracle_state(_ptr(words, ctypes.c_uint16), int(K), int(i)))


def states(trellis, k, n, K):
    """States of every weight: array [k/16, n/16, 256] (weight index i = 16 r + c)."""
    t = _u16(trellis)
    assert t.size == (k // 16) * (n // 16) * 16 * K
    out = np.empty((k // 16, n // 16, 256), dtype=np.uint16)
    _load().oracle_states(_ptr(t, ctypes.c_uint16), k, n, K, _ptr(out, ctypes.c_uint16))
    return out


def decode_tiles(trellis, k, n, K):
    """Decoded weights W_hat as k x n fp16 bit patterns (uint16)."""
    t = _u16(trellis)
    assert t.size == (k // 16) * (n // 16) * 16 * K
    out = np.empty((k, n), dtype=np.uint16)
    _load().oracle_decode_tiles(_ptr(t, ctypes.c_uint16), k, n, K, _ptr(out, ctypes.c_uint16))
    return out


def hadamard(x, pre=None, post=None):
    """Blockwise 128-point Hadamard of a rows x cols float64 array (cols % 128 == 0)."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    rows, cols = x.shape
    assert cols % 128 == 0
    y = np.empty_like(x)
    pre_a = None if pre is None else np.ascontiguousarray(pre, dtype=np.float64)
    post_a = None if post is None else np.ascontiguousarray(post, dtype=np.float64)
    _load().oracle_hadamard(_ptr(x, ctypes.c_double), _ptr(y, ctypes.c_double), rows, cols,
                            None if pre_a is None else _ptr(pre_a, ctypes.c_double),
                            None if post_a is None else _ptr(post_a, ctypes.c_double))
    return y


def linear(x, trellis, suh, svh, K, col_blocks=None, threads=1):
    """y = svh .* H(H(x .* suh) W_hat) in fp64 for the 128-column blocks
    [nb0, nb1) (default: all).  x: m x k fp16, suh: k fp16, svh: n fp16."""
    xb = _u16(x)
    m, k = xb.shape
    sv = _u16(svh)
    n = sv.size
    t = _u16(trellis)
    assert t.size == (k // 16) * (n // 16) * 16 * K
    nb0, nb1 = (0, n // 128) if col_blocks is None else col_blocks
    y = np.empty((m, (nb1 - nb0) * 128), dtype=np.float64)
    _load().oracle_linear(_ptr(xb, ctypes.c_uint16), _ptr(t, ctypes.c_uint16),
                          _ptr(_u16(suh), ctypes.c_uint16), _ptr(sv, ctypes.c_uint16),
                          m, k, n, int(K), nb0, nb1, _ptr(y, ctypes.c_double), int(threads))
    return y


def encode_seq(target, L, K, cb):
    """Tail-biting Viterbi encoding of one sequence on an L-bit trellis with K
    bits per weight and state values cb (2^L floats).  Returns (chunks, cost,
    overlap): each weight's K new bits, the fp32 squared-error sum of the
    closed path, and the overlap (low L-K bits of the last state)."""
    t = np.ascontiguousarray(target, dtype=np.float32)
    c = np.ascontiguousarray(cb, dtype=np.float32)
    assert c.size == 1 << L and 2 * K <= L
    chunks = np.empty(t.size, dtype=np.uint8)
    cost = ctypes.c_float()
    o = ctypes.c_int()
    rc = _load().oracle_encode_seq(_ptr(t, ctypes.c_float), int(t.size), int(L), int(K), _ptr(c, ctypes.c_float),
                                   _ptr(chunks, ctypes.c_uint8), ctypes.byref(cost), ctypes.byref(o))
    assert rc == 0
    return chunks, float(cost.value), int(o.value)


def encode(w, K, threads=1):
    """Encodes a k x n float32 matrix into the trellis layout [k/16][n/16][16K]
    (uint16).  Returns (trellis, cost): cost[tk, tn] is the tile's fp32
    squared-error sum."""
    a = np.ascontiguousarray(w, dtype=np.float32)
    k, n = a.shape
    assert k % 16 == 0 and n % 16 == 0
    trellis = np.empty((k // 16, n // 16, 16 * K), dtype=np.uint16)
    cost = np.empty((k // 16, n // 16), dtype=np.float32)
    rc = _load().oracle_encode(_ptr(a, ctypes.c_float), k, n, int(K), _ptr(trellis, ctypes.c_uint16),
                               _ptr(cost, ctypes.c_float), int(threads))
    assert rc == 0
    return trellis, cost


def threads_available():
    return int(_load().oracle_threads_available())


__all__ = ["half_to_double", "double_to_half", "codebook_table", "codebook", "state", "states",
           "decode_tiles", "hadamard", "linear", "encode_seq", "encode", "threads_available"]
