"""LDLQ with the trellis encoder -- TEST INFRASTRUCTURE (plain numpy, fp64).

Follows the page "ExLlamaV3推理快的秘密: EXL3 GEMM内核与融合Viterbi编码CUDA实现剖析",
section Viterbi编码内核剖析: before the trellis kernel runs, ldlq() performs a
block-wise LDLQ decomposition of each layer, and quantize_tiles() encodes the
16x16 tiles.  (The overview page "为什么ExLlamaV3值得关注" adds that the
Hessian is computed on the fly during conversion.)

What is computed (readings of what the pages leave open):
  - the proxy loss of a quantised layer is tr(E^T H E), E = W_hat - W, with
    W the k x n weight in the x . W orientation (rows = input channels) and H
    the k x k input Hessian;
  - H = U D U^T, U unit block-upper-triangular and D block-diagonal, with
    16 x 16 blocks (one block per tile row of 16 input channels);
  - the tile rows are quantised in order b = 0, 1, ...; row block b's target
    is T_b = W_b - sum_{c<b} U_{c,b}^T (W_hat_c - W_c), rounded to fp32, and
    W_hat_b is the trellis encoder's code for T_b (oracle.encode), decoded.
    Then tr(E^T H E) = sum_b tr(F_b^T D_b F_b) with F_b = W_hat_b - T_b:
    each block's own quantisation error, weighted by D_b, is all that is
    left of the loss.
The matrix products are numpy's (a library primitive); the factorisation is
the textbook block recursion, written out.
"""
import numpy as np

from . import decode_tiles, encode, half_to_double

BLOCK = 16


def udu(h):
    """Block factorisation H = U D U^T (fp64): U unit block-upper-triangular,
    D block-diagonal, 16 x 16 blocks.  Bottom-up: for b = B-1 .. 0,
    D_b = H_bb - sum_{c>b} U_bc D_c U_bc^T and, for a < b,
    U_ab = (H_ab - sum_{c>b} U_ac D_c U_bc^T) D_b^-1."""
    h = np.asarray(h, dtype=np.float64)
    k = h.shape[0]
    assert h.shape == (k, k) and k % BLOCK == 0
    nb = k // BLOCK
    U = np.eye(k)
    D = np.zeros((k, k))

    def blk(m, a, b):
        return m[a * BLOCK:(a + 1) * BLOCK, b * BLOCK:(b + 1) * BLOCK]

    for b in range(nb - 1, -1, -1):
        d = blk(h, b, b).copy()
        for c in range(b + 1, nb):
            d -= blk(U, b, c) @ blk(D, c, c) @ blk(U, b, c).T
        blk(D, b, b)[:] = d
        dinv = np.linalg.inv(d)
        for a in range(b):
            s = blk(h, a, b).copy()
            for c in range(b + 1, nb):
                s -= blk(U, a, c) @ blk(D, c, c) @ blk(U, b, c).T
            blk(U, a, b)[:] = s @ dinv
    return U, D


def ldlq(w, h, K, threads=1):
    """LDLQ of a k x n fp32 weight matrix against the k x k Hessian h with the
    K-bit trellis encoder.  Returns (trellis [k/16][n/16][16K] uint16,
    W_hat k x n fp64, targets k x n fp32, U, D)."""
    w = np.asarray(w, dtype=np.float32)
    k, n = w.shape
    U, D = udu(h)
    w64 = w.astype(np.float64)
    err = np.zeros((k, n))
    what = np.zeros((k, n))
    targets = np.zeros((k, n), dtype=np.float32)
    trellis = np.zeros((k // BLOCK, n // BLOCK, BLOCK * K), dtype=np.uint16)
    for b in range(k // BLOCK):
        r0, r1 = b * BLOCK, (b + 1) * BLOCK
        t = w64[r0:r1] - U[:r0, r0:r1].T @ err[:r0]
        t32 = t.astype(np.float32)
        code, _ = encode(t32, K, threads=threads)
        dec = half_to_double(decode_tiles(code, BLOCK, n, K))
        trellis[b] = code[0]
        targets[r0:r1] = t32
        what[r0:r1] = dec
        err[r0:r1] = dec - w64[r0:r1]
    return trellis, what, targets, U, D


def proxy_loss(w_hat, w, h):
    e = np.asarray(w_hat, dtype=np.float64) - np.asarray(w, dtype=np.float64)
    return float(np.trace(e.T @ np.asarray(h, dtype=np.float64) @ e))
