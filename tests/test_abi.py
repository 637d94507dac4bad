"""CPU-side checks of the C-ABI library: it builds, loads, exports every symbol
the public headers declare, and rejects bad arguments before launching
anything (no compute call is made here)."""
import ctypes
import glob
import os
import re

import pytest

from conftest import ROOT
from trellis_coded_bit_b200 import exl3

HEADERS = sorted(glob.glob(os.path.join(ROOT, "include", "*.h")))


def declared_functions():
    names = []
    for h in HEADERS:
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"\b(exl3_\w+)\s*\(", text)
    return sorted(set(names))


def test_headers_declare_the_four_calls():
    names = declared_functions()
    for fn in ("exl3_hadamard", "exl3_decode_tiles", "exl3_gemv", "exl3_gemm"):
        assert fn in names


def test_library_exports_every_declared_symbol():
    lib = exl3.load()
    names = declared_functions()
    assert set(names) == set(exl3.EXPORTED)
    for name in names:
        assert hasattr(lib, name), name  # ctypes raises AttributeError if not exported
    assert exl3.library_path().startswith(os.path.join(ROOT, "trellis_coded_bit_b200"))


def test_status_strings_and_version():
    for code in range(6):
        assert exl3.status_string(code).startswith("EXL3_")
    assert "sm_100a" in exl3.version()


def test_wait_limit_hook_roundtrip():
    exl3.exl3_debug_set_wait_limit_ns(12345)
    assert exl3.exl3_debug_wait_limit_ns() == 12345
    exl3.exl3_debug_set_wait_limit_ns(0)
    assert exl3.exl3_debug_wait_limit_ns() == 1_000_000_000


# Fake, never-dereferenced device addresses: argument checks run before any
# CUDA call, so these calls return without touching a GPU.
A = 1 << 20        # 16-byte aligned
B = 2 << 20
C = 3 << 20
D = 4 << 20
E = 5 << 20
MIS = A + 8        # misaligned


def _gemv(fn, x=A, t=B, suh=C, svh=D, y=E, m=1, k=256, n=256, K=4, ws=None, wsb=1 << 20):
    lib = exl3.load()
    return getattr(lib, fn)(x, t, suh, svh, y, m, k, n, K, ws, wsb, None)


@pytest.mark.parametrize("fn", ["exl3_gemv", "exl3_gemm", "exl3_matmul"])
def test_linear_argument_errors(fn):
    inv = exl3.EXL3_ERR_INVALID_ARG
    assert _gemv(fn, x=None) == inv
    assert _gemv(fn, y=MIS) == inv
    assert _gemv(fn, t=MIS) == inv
    assert _gemv(fn, k=200) == inv          # not a multiple of 128
    assert _gemv(fn, n=0) == inv
    assert _gemv(fn, K=0) == inv
    assert _gemv(fn, K=9) == inv
    assert _gemv(fn, m=0) == inv
    assert _gemv(fn, x=A, y=A) == inv       # y overlaps x


def test_gemv_rejects_large_m_and_missing_workspace():
    assert _gemv("exl3_gemv", m=17) == exl3.EXL3_ERR_UNSUPPORTED
    assert _gemv("exl3_gemv", ws=None) == exl3.EXL3_ERR_WORKSPACE
    assert _gemv("exl3_gemv", ws=A, wsb=16) == exl3.EXL3_ERR_WORKSPACE
    assert _gemv("exl3_gemv", ws=MIS) == exl3.EXL3_ERR_WORKSPACE


def test_workspace_sizes():
    lib = exl3.load()
    assert lib.exl3_gemv_workspace_size(1, 4096, 4096, 4) >= 256
    assert lib.exl3_gemv_workspace_size(17, 4096, 4096, 4) == 0
    assert lib.exl3_gemv_workspace_size(1, 100, 4096, 4) == 0
    assert lib.exl3_gemm_workspace_size(2048, 8192, 28672, 3) >= 2048 * 8192 * 2


def test_matmul_dispatch_and_gemm_tail_sizes():
    # exl3_matmul picks the GEMV for m <= 16 and the GEMM above: its workspace
    # size is that of the path m selects, and its workspace errors are that
    # path's
    lib = exl3.load()
    for m in (1, 9, 16):
        assert lib.exl3_matmul_workspace_size(m, 4096, 1024, 4) == lib.exl3_gemv_workspace_size(m, 4096, 1024, 4)
    for m in (17, 32, 2048):
        assert lib.exl3_matmul_workspace_size(m, 4096, 1024, 4) == lib.exl3_gemm_workspace_size(m, 4096, 1024, 4)
    assert _gemv("exl3_matmul", m=16, ws=None) == exl3.EXL3_ERR_WORKSPACE
    assert _gemv("exl3_matmul", m=32, ws=None) == exl3.EXL3_ERR_WORKSPACE
    assert _gemv("exl3_matmul", m=32, ws=A, wsb=16) == exl3.EXL3_ERR_WORKSPACE
    # the GEMM takes n = 256j + 128 (a half-width last tile)
    for n in (128, 384, 1152):
        assert lib.exl3_gemm_workspace_size(32, 1024, n, 3) > 0
    assert lib.exl3_gemm_workspace_size(32, 1024, 200, 3) == 0
    assert _gemv("exl3_gemm", m=32, n=384, ws=A, wsb=16) == exl3.EXL3_ERR_WORKSPACE  # not UNSUPPORTED


def test_hadamard_and_decode_argument_errors():
    lib = exl3.load()
    inv = exl3.EXL3_ERR_INVALID_ARG
    assert lib.exl3_hadamard(A, B, 4, 100, None, None, None) == inv
    assert lib.exl3_hadamard(MIS, B, 4, 128, None, None, None) == inv
    assert lib.exl3_hadamard(A, A + 64, 4, 128, None, None, None) == inv  # partial overlap
    assert lib.exl3_hadamard(None, None, 0, 128, None, None, None) == exl3.EXL3_OK  # empty
    assert lib.exl3_decode_tiles(A, B, 16, 16, 0, None) == inv
    assert lib.exl3_decode_tiles(A, B, 24, 16, 4, None) == inv
    assert lib.exl3_decode_tiles(None, B, 16, 16, 4, None) == inv
    assert lib.exl3_workspace_status(None, 0, 0, None) == exl3.EXL3_ERR_WORKSPACE


def _multi(descs, m=1, ws=None, wsb=1 << 30):
    lib = exl3.load()
    arr = (exl3.Exl3Linear * max(1, len(descs)))(*[exl3.Exl3Linear(*d) for d in descs])
    return lib.exl3_gemv_multi(arr, len(descs), m, ws, wsb, None)


def test_gemv_multi_argument_errors_and_sizes():
    lib = exl3.load()
    good = (A, B, C, D, E, 256, 256, 4)
    inv = exl3.EXL3_ERR_INVALID_ARG
    assert _multi([]) == inv                                  # no layers
    assert _multi([good, (A, B, C, D, E, 200, 256, 4)]) == inv  # one bad layer: nothing runs
    assert _multi([good, (A, B, C, D, MIS, 256, 256, 4)]) == inv
    assert _multi([good], m=17) == exl3.EXL3_ERR_UNSUPPORTED
    assert _multi([good], ws=None) == exl3.EXL3_ERR_WORKSPACE
    assert _multi([good], ws=A, wsb=16) == exl3.EXL3_ERR_WORKSPACE

    def size(descs, m=1):
        arr = (exl3.Exl3Linear * len(descs))(*[exl3.Exl3Linear(*d) for d in descs])
        return lib.exl3_gemv_multi_workspace_size(arr, len(descs), m)

    one = size([good])
    assert 256 <= one <= lib.exl3_gemv_workspace_size(1, 256, 256, 4)
    # layers of any mix of K share one launch: one region holding both layers'
    # activation blocks (k/16 x 512 bytes each) besides the status word
    other = (A, B, C, D, E, 512, 1024, 2)
    two_k = size([good, other])
    assert two_k >= 256 + (256 // 16 + 512 // 16) * 512
    # more than 32 layers need a second launch, with a region of its own after
    # the first launch's
    many = [good] * 33
    assert size(many) >= size([good] * 32) + size([good])
    assert size([(A, B, C, D, E, 200, 256, 4)]) == 0


def _gemm_multi(descs, m=32, ws=None, wsb=1 << 30, fn="exl3_gemm_multi"):
    lib = exl3.load()
    arr = (exl3.Exl3Linear * max(1, len(descs)))(*[exl3.Exl3Linear(*d) for d in descs])
    return getattr(lib, fn)(arr, len(descs), m, ws, wsb, None)


def test_gemm_multi_argument_errors_and_sizes():
    lib = exl3.load()
    good = (A, B, C, D, E, 256, 256, 4)
    inv, uns = exl3.EXL3_ERR_INVALID_ARG, exl3.EXL3_ERR_UNSUPPORTED
    assert _gemm_multi([]) == inv                                       # no layers
    assert _gemm_multi([good, (A, B, C, D, E, 200, 256, 4)]) == inv     # one bad layer
    assert _gemm_multi([good, (A, B, C, D, E, 512, 256, 4)]) == uns     # k differs
    assert _gemm_multi([good, (A, B, C, D, E, 256, 256, 3)]) == uns     # K differs
    assert _gemm_multi([good]) == exl3.EXL3_ERR_WORKSPACE               # no workspace
    assert _gemm_multi([good], ws=A, wsb=16) == exl3.EXL3_ERR_WORKSPACE

    def size(descs, m=32, kind="gemm"):
        arr = (exl3.Exl3Linear * len(descs))(*[exl3.Exl3Linear(*d) for d in descs])
        return getattr(lib, "exl3_%s_multi_workspace_size" % kind)(arr, len(descs), m)

    one = size([good])
    assert one == lib.exl3_gemm_workspace_size(32, 256, 256, 4)
    # one tiled x' per layer of a launch: a second layer needs at least one more
    wide = (A, B, C, D, E, 256, 1152, 4)
    assert size([good, wide]) >= one + 32 * 256 * 2
    # more than 8 layers run as several launches on the same workspace: the
    # size is the largest launch's
    assert size([good] * 9) == size([good] * 8)
    assert size([good, (A, B, C, D, E, 256, 256, 5)]) == 0
    # the matmul multi call picks by m
    assert size([good], m=16, kind="matmul") == size([good], m=16, kind="gemv")
    assert size([good], m=17, kind="matmul") == size([good], m=17, kind="gemm")
    assert _gemm_multi([good, (A, B, C, D, E, 512, 256, 2)], m=8, fn="exl3_matmul_multi") == \
        exl3.EXL3_ERR_WORKSPACE  # GEMV multi: any mix of k and K, only the workspace is missing
    assert _gemm_multi([good, (A, B, C, D, E, 512, 256, 2)], m=40, fn="exl3_matmul_multi") == uns


def test_encode_argument_errors_and_sizes():
    lib = exl3.load()
    inv = exl3.EXL3_ERR_INVALID_ARG
    ws = 1 << 24

    def enc(w=A, t=B, cost=C, k=64, n=64, K=4, wsp=ws, wsb=1 << 40):
        return lib.exl3_encode(w, t, cost, k, n, K, wsp, wsb, None)

    assert enc(w=None) == inv
    assert enc(t=MIS) == inv
    assert enc(cost=A + 2) == inv            # fp32 costs need 4-byte alignment
    assert enc(k=24) == inv                  # not a multiple of 16
    assert enc(K=0) == inv and enc(K=9) == inv
    assert enc(w=A, t=A) == inv              # trellis overlaps w
    assert enc(cost=A + 64) == inv           # cost overlaps w
    assert enc(cost=B) == inv                # cost overlaps trellis
    assert enc(wsp=None) == exl3.EXL3_ERR_WORKSPACE
    assert enc(wsb=16) == exl3.EXL3_ERR_WORKSPACE
    # per CTA in flight: 256 x 2^(16-K) bytes of recorded choices (plus the
    # cost vectors for K = 1); never more CTAs than tiles
    for K in range(1, 9):
        one = lib.exl3_encode_workspace_size(16, 16, K)
        extra = 2 * 4 * (1 << 15) if K == 1 else 0
        assert one == 256 + 256 * (1 << (16 - K)) + extra
        assert lib.exl3_encode_workspace_size(4096, 4096, K) <= 256 + (1 << 30)
    assert lib.exl3_encode_workspace_size(24, 16, 4) == 0


def test_udu_and_ldlq_argument_errors_and_sizes():
    lib = exl3.load()
    inv = exl3.EXL3_ERR_INVALID_ARG
    assert lib.exl3_udu(None, B, 32, C, 1 << 20, None) == inv
    assert lib.exl3_udu(A, B, 24, C, 1 << 20, None) == inv          # not a multiple of 16
    assert lib.exl3_udu(A, A + 64, 32, C, 1 << 20, None) == inv     # overlapping, not equal
    assert lib.exl3_udu(A, B, 32, None, 0, None) == exl3.EXL3_ERR_WORKSPACE
    assert lib.exl3_udu_workspace_size(32) == 256 + 16 * 16 * 8 + 32 * 16 * 8
    assert lib.exl3_udu_workspace_size(24) == 0

    def ldlq(w=A, h=B, t=C, wh=None, k=64, n=64, K=4, ws=D, wsb=1 << 40):
        return lib.exl3_ldlq(w, h, t, wh, k, n, K, ws, wsb, None)

    assert ldlq(w=None) == inv
    assert ldlq(h=MIS) == inv
    assert ldlq(K=9) == inv
    assert ldlq(n=40) == inv
    assert ldlq(wh=A) == inv                                         # w_hat overlaps w
    assert ldlq(ws=None) == exl3.EXL3_ERR_WORKSPACE
    # the factor and the errors in fp64, plus the encoder's workspace for 16 x n
    need = lib.exl3_ldlq_workspace_size(64, 128, 4)
    assert need >= 64 * 64 * 8 + 64 * 128 * 8 + lib.exl3_encode_workspace_size(16, 128, 4)
    assert lib.exl3_ldlq_workspace_size(64, 40, 4) == 0


def test_binding_checks_tensor_sizes_before_the_call():
    # the binding compares every tensor with (m, k, n, K) before anything
    # reaches the C ABI (CPU tensors suffice: the check comes first)
    import torch
    m, k, n, K = 2, 256, 128, 3
    x = torch.zeros((m, k), dtype=torch.float16)
    t = torch.zeros((k // 16, n // 16, 16 * K), dtype=torch.uint16)
    suh = torch.ones(k, dtype=torch.float16)
    svh = torch.ones(n, dtype=torch.float16)
    y = torch.empty((m, n), dtype=torch.float16)
    bad = [
        dict(trellis=t[:-1]),
        dict(suh=suh[:-1]),
        dict(y=torch.empty((m, n - 1), dtype=torch.float16)),
        dict(K=K + 1),
    ]
    for change in bad:
        a = dict(x=x, trellis=t, suh=suh, svh=svh, K=K, y=y)
        a.update(change)
        for fn in (exl3.exl3_gemv, exl3.exl3_gemm):
            with pytest.raises(ValueError):
                fn(a["x"], a["trellis"], a["suh"], a["svh"], a["K"], y=a["y"], workspace=torch.zeros(256, dtype=torch.uint8))
        with pytest.raises(ValueError):
            exl3.exl3_gemv_noalloc(a["x"], a["trellis"], a["suh"], a["svh"], a["K"], y=a["y"])
