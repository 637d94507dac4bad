"""Thin ctypes binding of the EXL3 B200 C ABI (include/exl3.h).

Argument marshalling only: every step of the computation runs in the CUDA
kernels of libexl3_b200.so.  PyTorch supplies device memory and streams.
There is no CPU fallback: if the library cannot be built or loaded, or no
CUDA device is present, these functions raise.
"""
import ctypes
import os
import threading

import torch

from . import build as _build

EXL3_OK = 0
EXL3_ERR_INVALID_ARG = 1
EXL3_ERR_UNSUPPORTED = 2
EXL3_ERR_WORKSPACE = 3
EXL3_ERR_CUDA = 4
EXL3_ERR_TIMEOUT = 5

# Every symbol the public headers declare.
EXPORTED = ["exl3_status_string", "exl3_version", "exl3_hadamard", "exl3_decode_tiles",
            "exl3_gemv_workspace_size", "exl3_gemv", "exl3_gemv_multi_workspace_size", "exl3_gemv_multi",
            "exl3_gemv_noalloc_max_scratch",
            "exl3_gemv_noalloc", "exl3_gemm_workspace_size", "exl3_gemm",
            "exl3_matmul_workspace_size", "exl3_matmul",
            "exl3_gemm_multi_workspace_size", "exl3_gemm_multi",
            "exl3_matmul_multi_workspace_size", "exl3_matmul_multi",
            "exl3_encode_workspace_size", "exl3_encode", "exl3_udu_workspace_size", "exl3_udu",
            "exl3_ldlq_workspace_size", "exl3_ldlq",
            "exl3_workspace_status", "exl3_set_launch_flags", "exl3_launch_flags",
            "exl3_debug_set_wait_limit_ns", "exl3_debug_wait_limit_ns"]

EXL3_LAUNCH_PDL = 1

_lib = None
_lock = threading.Lock()


class Exl3Linear(ctypes.Structure):
    """The C struct exl3_linear: one layer of an exl3_gemv_multi call."""
    _fields_ = [("x", ctypes.c_void_p), ("trellis", ctypes.c_void_p), ("suh", ctypes.c_void_p),
                ("svh", ctypes.c_void_p), ("y", ctypes.c_void_p), ("k", ctypes.c_int64),
                ("n", ctypes.c_int64), ("K", ctypes.c_int)]


class Exl3Error(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__("%s: %s" % (where, status_string(status)))


def library_path():
    return _build.LIB


def load(build_if_needed=True):
    """Load (building first if the sources are newer) the shared library."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        path = _build.build() if build_if_needed else _build.LIB
        if not os.path.exists(path):
            raise RuntimeError("EXL3 CUDA library not found at %s" % path)
        lib = ctypes.CDLL(path)
        vp, i64, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t
        ci = ctypes.c_int
        lib.exl3_status_string.argtypes = [ci]
        lib.exl3_status_string.restype = ctypes.c_char_p
        lib.exl3_version.argtypes = []
        lib.exl3_version.restype = ctypes.c_char_p
        lib.exl3_hadamard.argtypes = [vp, vp, i64, i64, vp, vp, vp]
        lib.exl3_hadamard.restype = ci
        lib.exl3_decode_tiles.argtypes = [vp, vp, i64, i64, ci, vp]
        lib.exl3_decode_tiles.restype = ci
        for name in ("exl3_gemv_workspace_size", "exl3_gemm_workspace_size", "exl3_matmul_workspace_size"):
            getattr(lib, name).argtypes = [i64, i64, i64, ci]
            getattr(lib, name).restype = sz
        for name in ("exl3_gemv", "exl3_gemm", "exl3_matmul"):
            getattr(lib, name).argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, ci, vp, sz, vp]
            getattr(lib, name).restype = ci
        for kind in ("gemv", "gemm", "matmul"):
            getattr(lib, "exl3_%s_multi_workspace_size" % kind).argtypes = [ctypes.POINTER(Exl3Linear), ci, i64]
            getattr(lib, "exl3_%s_multi_workspace_size" % kind).restype = sz
            getattr(lib, "exl3_%s_multi" % kind).argtypes = [ctypes.POINTER(Exl3Linear), ci, i64, vp, sz, vp]
            getattr(lib, "exl3_%s_multi" % kind).restype = ci
        lib.exl3_gemv_noalloc_max_scratch.argtypes = []
        lib.exl3_gemv_noalloc_max_scratch.restype = sz
        lib.exl3_gemv_noalloc.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, ci, vp]
        lib.exl3_gemv_noalloc.restype = ci
        lib.exl3_encode_workspace_size.argtypes = [i64, i64, ci]
        lib.exl3_encode_workspace_size.restype = sz
        lib.exl3_encode.argtypes = [vp, vp, vp, i64, i64, ci, vp, sz, vp]
        lib.exl3_encode.restype = ci
        lib.exl3_udu_workspace_size.argtypes = [i64]
        lib.exl3_udu_workspace_size.restype = sz
        lib.exl3_udu.argtypes = [vp, vp, i64, vp, sz, vp]
        lib.exl3_udu.restype = ci
        lib.exl3_ldlq_workspace_size.argtypes = [i64, i64, ci]
        lib.exl3_ldlq_workspace_size.restype = sz
        lib.exl3_ldlq.argtypes = [vp, vp, vp, vp, i64, i64, ci, vp, sz, vp]
        lib.exl3_ldlq.restype = ci
        lib.exl3_workspace_status.argtypes = [vp, sz, ci, vp]
        lib.exl3_workspace_status.restype = ci
        lib.exl3_set_launch_flags.argtypes = [ctypes.c_uint]
        lib.exl3_set_launch_flags.restype = None
        lib.exl3_launch_flags.argtypes = []
        lib.exl3_launch_flags.restype = ctypes.c_uint
        lib.exl3_debug_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
        lib.exl3_debug_set_wait_limit_ns.restype = None
        lib.exl3_debug_wait_limit_ns.argtypes = []
        lib.exl3_debug_wait_limit_ns.restype = ctypes.c_uint64
        _lib = lib
        return lib


def status_string(status):
    return load().exl3_status_string(int(status)).decode()


def version():
    return load().exl3_version().decode()


def _check(status, where):
    if status != EXL3_OK:
        raise Exl3Error(status, where)


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dev(t, dtype, name):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError("%s must be a CUDA tensor" % name)
    if t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    return ctypes.c_void_p(t.data_ptr())


def _ptr_or_none(t, dtype, name):
    return None if t is None else _dev(t, dtype, name)


def _check_layer_shapes(x, trellis, suh, svh, K, y):
    """Sizes of a layer's tensors against (m, k, n, K), checked before the C
    call so that an undersized tensor never reaches a kernel."""
    if x.dim() != 2:
        raise ValueError("x must be m x k")
    m, k = x.shape
    n = svh.numel()
    if suh.numel() != k:
        raise ValueError("suh must have k = %d elements, has %d" % (k, suh.numel()))
    if k % 16 or n % 16 or trellis.numel() != (k // 16) * (n // 16) * 16 * int(K):
        raise ValueError("trellis must have (k/16)(n/16)16K = %d words for k=%d, n=%d, K=%d, has %d"
                         % ((k // 16) * (n // 16) * 16 * int(K), k, n, int(K), trellis.numel()))
    if y is not None and tuple(y.shape) != (m, n):
        raise ValueError("y must be m x n = %d x %d, is %s" % (m, n, tuple(y.shape)))
    return m, k, n


# ----------------------------------------------------------------- calls ---

def exl3_hadamard(x, y=None, pre=None, post=None, stream=None):
    """y = H128(x .* pre)/sqrt(128) .* post, blockwise over the last dimension."""
    rows, cols = x.shape
    if y is None:
        y = torch.empty_like(x)
    _check(load().exl3_hadamard(_dev(x, torch.float16, "x"), _dev(y, torch.float16, "y"), rows, cols,
                                _ptr_or_none(pre, torch.float16, "pre"),
                                _ptr_or_none(post, torch.float16, "post"), _stream(stream)),
           "exl3_hadamard")
    return y


def exl3_decode_tiles(trellis, k, n, K, w=None, stream=None):
    """Dense k x n fp16 weights decoded from a [k/16, n/16, 16K] uint16 trellis."""
    if w is None:
        w = torch.empty((k, n), dtype=torch.float16, device=trellis.device)
    _check(load().exl3_decode_tiles(_dev(trellis, torch.uint16, "trellis"), _dev(w, torch.float16, "w"),
                                    k, n, K, _stream(stream)), "exl3_decode_tiles")
    return w


def exl3_gemv_workspace_size(m, k, n, K):
    return int(load().exl3_gemv_workspace_size(m, k, n, K))


def exl3_gemm_workspace_size(m, k, n, K):
    return int(load().exl3_gemm_workspace_size(m, k, n, K))


def exl3_matmul_workspace_size(m, k, n, K):
    return int(load().exl3_matmul_workspace_size(m, k, n, K))


def new_workspace(nbytes, device=None):
    """Zero-filled workspace buffer (uint8) of at least nbytes, 256-byte aligned."""
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8,
                       device=device if device is not None else "cuda")


def _linear(fn, name, x, trellis, suh, svh, K, y, workspace, stream):
    m, k, n = _check_layer_shapes(x, trellis, suh, svh, K, y)
    if y is None:
        y = torch.empty((m, n), dtype=torch.float16, device=x.device)
    if workspace is None:
        raise ValueError("%s needs a workspace (see new_workspace / *_workspace_size)" % name)
    _check(fn(_dev(x, torch.float16, "x"), _dev(trellis, torch.uint16, "trellis"),
              _dev(suh, torch.float16, "suh"), _dev(svh, torch.float16, "svh"),
              _dev(y, torch.float16, "y"), m, k, n, int(K), _dev(workspace, torch.uint8, "workspace"),
              workspace.numel(), _stream(stream)), name)
    return y


def exl3_gemv(x, trellis, suh, svh, K, y=None, workspace=None, stream=None):
    """y = svh .* H(H(x .* suh) W_hat) for 1 <= m <= 16 (memory-bound path)."""
    return _linear(load().exl3_gemv, "exl3_gemv", x, trellis, suh, svh, K, y, workspace, stream)


def _linear_array(layers, m):
    """layers: sequence of (x, trellis, suh, svh, K, y) CUDA tensors (y may be None)."""
    arr = (Exl3Linear * len(layers))()
    ys = []
    for i, (x, trellis, suh, svh, K, y) in enumerate(layers):
        if x.shape[0] != m:
            raise ValueError("every layer of a multi call has the same batch size m")
        _, k, n = _check_layer_shapes(x, trellis, suh, svh, K, y)
        if y is None:
            y = torch.empty((m, n), dtype=torch.float16, device=x.device)
        arr[i] = Exl3Linear(_dev(x, torch.float16, "x"), _dev(trellis, torch.uint16, "trellis"),
                            _dev(suh, torch.float16, "suh"), _dev(svh, torch.float16, "svh"),
                            _dev(y, torch.float16, "y"), k, n, int(K))
        ys.append(y)
    return arr, ys


def _multi_workspace_size(kind, layers, m):
    arr, _ = _linear_array(layers, m)
    return int(getattr(load(), "exl3_%s_multi_workspace_size" % kind)(arr, len(layers), m))


def _multi(kind, layers, workspace, stream):
    m = layers[0][0].shape[0]
    arr, ys = _linear_array(layers, m)
    name = "exl3_%s_multi" % kind
    if workspace is None:
        raise ValueError("%s needs a workspace (%s_workspace_size)" % (name, name))
    _check(getattr(load(), name)(arr, len(layers), m, _dev(workspace, torch.uint8, "workspace"),
                                 workspace.numel(), _stream(stream)), name)
    return ys


def exl3_gemv_multi_workspace_size(layers, m):
    """Workspace bytes for exl3_gemv_multi over `layers` (see exl3_gemv_multi)."""
    return _multi_workspace_size("gemv", layers, m)


def exl3_gemv_multi(layers, workspace=None, stream=None):
    """Several independent layers (same m <= 16) in one call: each entry is
    (x, trellis, suh, svh, K, y-or-None); returns the list of y."""
    return _multi("gemv", layers, workspace, stream)


def exl3_gemm_multi_workspace_size(layers, m):
    """Workspace bytes for exl3_gemm_multi over `layers` (see exl3_gemm_multi)."""
    return _multi_workspace_size("gemm", layers, m)


def exl3_gemm_multi(layers, workspace=None, stream=None):
    """Several layers with the same m, k and K through the GEMM in one call
    (entries as for exl3_gemv_multi); returns the list of y."""
    return _multi("gemm", layers, workspace, stream)


def exl3_matmul_multi_workspace_size(layers, m):
    """Workspace bytes for exl3_matmul_multi over `layers`."""
    return _multi_workspace_size("matmul", layers, m)


def exl3_matmul_multi(layers, workspace=None, stream=None):
    """Several layers with the same m, the kernel chosen by m (GEMV multi for
    m <= 16, GEMM multi above); returns the list of y."""
    return _multi("matmul", layers, workspace, stream)


class MultiCall:
    """A prepared multi-layer call (`kind` "gemv", "gemm" or "matmul"): the
    descriptor array is built once, so repeated calls (a decode loop) cost
    only the C call.  `layers` as for exl3_gemv_multi; the tensors must stay
    alive and in place."""

    kind = "matmul"

    def __init__(self, layers, kind=None):
        if kind is not None:
            self.kind = kind
        self.m = layers[0][0].shape[0]
        self.count = len(layers)
        self._arr, self.ys = _linear_array(layers, self.m)
        self._name = "exl3_%s_multi" % self.kind
        self.workspace_size = int(getattr(load(), self._name + "_workspace_size")(self._arr, self.count, self.m))

    def __call__(self, workspace, stream=None):
        _check(getattr(load(), self._name)(self._arr, self.count, self.m, _dev(workspace, torch.uint8, "workspace"),
                                           workspace.numel(), _stream(stream)), self._name)
        return self.ys


class GemvMulti(MultiCall):
    """A prepared exl3_gemv_multi call (see MultiCall)."""

    kind = "gemv"


def exl3_gemv_noalloc_max_scratch():
    return int(load().exl3_gemv_noalloc_max_scratch())


def exl3_gemv_noalloc(x, trellis, suh, svh, K, y, stream=None):
    """exl3_gemv without a workspace: the library's own fixed scratch array is
    used, for callers that cannot allocate device memory (y must be given)."""
    m, k, n = _check_layer_shapes(x, trellis, suh, svh, K, y)
    _check(load().exl3_gemv_noalloc(_dev(x, torch.float16, "x"), _dev(trellis, torch.uint16, "trellis"),
                                    _dev(suh, torch.float16, "suh"), _dev(svh, torch.float16, "svh"),
                                    _dev(y, torch.float16, "y"), m, k, n, int(K), _stream(stream)),
           "exl3_gemv_noalloc")
    return y


def exl3_gemm(x, trellis, suh, svh, K, y=None, workspace=None, stream=None):
    """The same layer on the tensor cores, any m (tuned for m >= 64)."""
    return _linear(load().exl3_gemm, "exl3_gemm", x, trellis, suh, svh, K, y, workspace, stream)


def exl3_matmul(x, trellis, suh, svh, K, y=None, workspace=None, stream=None):
    """The layer for any m, the kernel chosen by the library (GEMV for m <= 16,
    tensor-core GEMM above)."""
    return _linear(load().exl3_matmul, "exl3_matmul", x, trellis, suh, svh, K, y, workspace, stream)


def exl3_encode_workspace_size(k, n, K):
    return int(load().exl3_encode_workspace_size(k, n, K))


def exl3_encode(w, K, trellis=None, cost=None, workspace=None, stream=None):
    """Tail-biting trellis encoding of a k x n fp32 matrix into a [k/16, n/16, 16K]
    uint16 trellis.  Returns (trellis, cost): cost[tk, tn] is the tile's fp32
    squared-error sum."""
    k, n = w.shape
    if trellis is None:
        trellis = torch.empty((k // 16, n // 16, 16 * K), dtype=torch.uint16, device=w.device)
    if cost is None:
        cost = torch.empty((k // 16, n // 16), dtype=torch.float32, device=w.device)
    if workspace is None:
        raise ValueError("exl3_encode needs a workspace (see new_workspace / exl3_encode_workspace_size)")
    _check(load().exl3_encode(_dev(w, torch.float32, "w"), _dev(trellis, torch.uint16, "trellis"),
                              _dev(cost, torch.float32, "cost"), k, n, int(K),
                              _dev(workspace, torch.uint8, "workspace"), workspace.numel(), _stream(stream)),
           "exl3_encode")
    return trellis, cost


def exl3_udu(h, ud=None, stream=None):
    """Block factorisation H = U D U^T (fp64, 16 x 16 blocks) of a k x k CUDA
    tensor: returns ud with D in the diagonal blocks, U above them, zeros below."""
    k = h.shape[0]
    if ud is None:
        ud = torch.empty_like(h)
    ws = new_workspace(load().exl3_udu_workspace_size(k), device=h.device)
    _check(load().exl3_udu(_dev(h, torch.float64, "h"), _dev(ud, torch.float64, "ud"), k,
                           _dev(ws, torch.uint8, "workspace"), ws.numel(), _stream(stream)), "exl3_udu")
    return ud


def exl3_ldlq_workspace_size(k, n, K):
    return int(load().exl3_ldlq_workspace_size(k, n, K))


def exl3_ldlq(w, h, K, trellis=None, w_hat=None, workspace=None, stream=None):
    """LDLQ of a k x n fp32 layer against the k x k fp64 Hessian h with the
    K-bit trellis encoder.  Returns (trellis, w_hat)."""
    k, n = w.shape
    if trellis is None:
        trellis = torch.empty((k // 16, n // 16, 16 * K), dtype=torch.uint16, device=w.device)
    if w_hat is None:
        w_hat = torch.empty((k, n), dtype=torch.float32, device=w.device)
    if workspace is None:
        raise ValueError("exl3_ldlq needs a workspace (see new_workspace / exl3_ldlq_workspace_size)")
    _check(load().exl3_ldlq(_dev(w, torch.float32, "w"), _dev(h, torch.float64, "h"),
                            _dev(trellis, torch.uint16, "trellis"), _dev(w_hat, torch.float32, "w_hat"), k, n,
                            int(K), _dev(workspace, torch.uint8, "workspace"), workspace.numel(), _stream(stream)),
           "exl3_ldlq")
    return trellis, w_hat


def exl3_workspace_status(workspace, clear=False, stream=None):
    """Status word of a gemv/gemm workspace (synchronises the stream)."""
    return int(load().exl3_workspace_status(_dev(workspace, torch.uint8, "workspace"), workspace.numel(),
                                            1 if clear else 0, _stream(stream)))


def exl3_set_launch_flags(flags):
    """EXL3_LAUNCH_PDL: programmatic dependent launch (weights must be immutable)."""
    load().exl3_set_launch_flags(int(flags))


def exl3_launch_flags():
    return int(load().exl3_launch_flags())


def exl3_debug_set_wait_limit_ns(ns):
    load().exl3_debug_set_wait_limit_ns(int(ns))


def exl3_debug_wait_limit_ns():
    return int(load().exl3_debug_wait_limit_ns())
