"""The Llama-3.1-70B decoder-layer linear stack through the C ABI.

q 8192x8192, k/v 8192x1024, o 8192x8192 at K = 4; gate/up 8192x28672 and
down 28672x8192 at K = 2; lm_head 8192x128256 at K = 3 -- at m = 1 (the
GEMV) and m = 32 (the tensor-core GEMM).  Every layer runs in full on the
GPU; the fp64 oracle checks sampled 128-column blocks (first, middle, last)
within max|y - y_ref| <= 1e-2 rms(y_ref) + 1e-3.
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


@pytest.mark.parametrize("case", range(len(workloads.LAYER_STACK)))
def test_layer_stack_sampled(case):
    name, m, k, n, K, outl = workloads.LAYER_STACK[case]
    layer = inputs.make_layer(m, k, n, K, inputs.seed_for(4, case), outl)
    args = (dev(layer.x), dev(layer.trellis), dev(layer.suh), dev(layer.svh), K)
    if m <= 16:
        ws = exl3.new_workspace(exl3.exl3_gemv_workspace_size(m, k, n, K))
        y = exl3.exl3_gemv(*args, workspace=ws)
    else:
        ws = exl3.new_workspace(exl3.exl3_gemm_workspace_size(m, k, n, K))
        y = exl3.exl3_gemm(*args, workspace=ws)
    torch.cuda.synchronize()
    assert exl3.exl3_workspace_status(ws) == exl3.EXL3_OK
    y = y.cpu().numpy().astype(np.float64)
    assert np.isfinite(y).all()
    nb = n // 128
    for c in sorted({0, nb // 2, nb - 1}):
        ref = oracle.linear(layer.x, layer.trellis, layer.suh, layer.svh, K, col_blocks=(c, c + 1))
        ok, err, bound = within_tolerance(y[:, c * 128:(c + 1) * 128], ref)
        assert ok, "%s block %d: max err %.4g > bound %.4g" % (name, c, err, bound)
