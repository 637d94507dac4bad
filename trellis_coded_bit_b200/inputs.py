"""Seeded synthetic inputs for the EXL3 linear layer.

This module only draws random numbers: it holds none of the method's
arithmetic, so both the CUDA path and the fp64 oracle can consume the same
bytes.  Recipe (numpy PCG64, seed = 1000 + 100 * workload_index + case_index):

  trellis  uniform uint16 words, shape [k/16, n/16, 16*K] -- every bit string is
           a valid tail-biting code, so uniform words are valid weights;
  suh      +-1 per input channel (fp16);
  svh      +-1 * U(0.01, 0.05) per output channel (fp16);
  x        N(0, 1) as fp16, shape [m, k]; with ``outliers`` 1% of the input
           channels (chosen without replacement) are scaled by 20 before the
           fp16 cast.

These follow the shapes and value distributions of the Llama-3.1 8B / 70B
linear layers the pages discuss; no model weights are involved.
"""
from dataclasses import dataclass

import numpy as np


def seed_for(workload_index: int, case_index: int) -> int:
    return 1000 + 100 * int(workload_index) + int(case_index)


@dataclass
class Layer:
    m: int
    k: int
    n: int
    K: int
    x: np.ndarray        # [m, k] float16
    trellis: np.ndarray  # [k/16, n/16, 16K] uint16
    suh: np.ndarray      # [k] float16
    svh: np.ndarray      # [n] float16

    @property
    def trellis_bytes(self) -> int:
        return self.trellis.nbytes


def make_trellis(rng, k, n, K):
    return rng.integers(0, 65536, size=(k // 16, n // 16, 16 * K), dtype=np.uint16)


def make_x(rng, m, k, outliers=False):
    x = rng.standard_normal((m, k))
    if outliers and k >= 100:
        ch = rng.choice(k, k // 100, replace=False)
        x[:, ch] *= 20.0
    return x.astype(np.float16)


def make_layer(m, k, n, K, seed, outliers=False) -> Layer:
    rng = np.random.Generator(np.random.PCG64(seed))
    trellis = make_trellis(rng, k, n, K)
    suh = rng.choice(np.array([-1.0, 1.0]), k).astype(np.float16)
    svh = (rng.choice(np.array([-1.0, 1.0]), n) * rng.uniform(0.01, 0.05, n)).astype(np.float16)
    x = make_x(rng, m, k, outliers)
    return Layer(m, k, n, K, x, trellis, suh, svh)
