"""W4A8: INT4 group-wise weights with dynamic INT8 activations.

Test infrastructure only (see ``oracle/__init__.py``).

"Low Bit ARM kernels" measures 4-bit weights with dynamic INT8 activations
(group size 32): the inner loop multiplies int8 activations with the unpacked
weight codes as integers (the SMMLA int8 matrix multiply), accumulates in
int32, and applies the group scales afterwards. The weights are the INT4
format of ``oracle.int4`` (symmetric (q - 8) s or asymmetric (q - zp) s).

Readings taken where the page is silent:

* The activations are quantised per row in blocks of 32 consecutive k (the
  page's group size), symmetric: s = amax / 127 in IEEE FP32 (amax the block's
  largest |x|), xq = clamp(rint(x / s), -127, 127) with the division in FP32;
  an all-zero block has s = 0 and xq = 0. The scale stays FP32 (it is computed
  at run time and never stored in a format).
* Per 32-k block b and column n the integer sum  I = sum xq q - z sum xq  is
  exact (z = 8 for SYM, the zero point for ASYM); the result is
  y[m][n] = sum_b s_x[m][b] s_w[g(b)][n] I[m][b][n], i.e. exactly the product of
  the dequantised activations xq s_x with the dequantised weight.
"""

import numpy as np

F32 = np.float32
BLOCK = 32


def quantize_activations(X):
    """X [M, K] (float32 values of FP16/BF16 inputs) -> (xq int8 [M, K],
    s float32 [M, K/32])."""
    X = np.asarray(X)
    if X.dtype != np.float32:
        raise TypeError("X must be float32 (the exact values of the FP16/BF16 inputs)")
    M, K = X.shape
    if K % BLOCK:
        raise ValueError("K must be a multiple of 32")
    Xb = X.reshape(M, K // BLOCK, BLOCK)
    amax = np.abs(Xb).max(axis=2)
    s = (amax / F32(127.0)).astype(np.float32)
    safe = np.where(s == 0, F32(1.0), s)
    xq = np.clip(np.rint(Xb / safe[:, :, None]), -127, 127)
    xq = np.where(s[:, :, None] == 0, F32(0.0), xq)
    return xq.astype(np.int8).reshape(M, K), s


def dequant_activations(xq, s):
    """Exact xq * s as float64 [M, K]."""
    xq = np.asarray(xq).astype(np.float64)
    s = np.asarray(s, dtype=np.float32).astype(np.float64)
    return xq * np.repeat(s, BLOCK, axis=1)


def block_integer_sums(xq, q, z, group):
    """I[m][b][n] = sum over block b of xq (q - z) as int64; z [K/group, N]
    (int) or the scalar 8 for SYM."""
    xq = np.asarray(xq).astype(np.int64)
    q = np.asarray(q).astype(np.int64)
    M, K = xq.shape
    N = q.shape[1]
    zk = np.repeat(np.broadcast_to(np.asarray(z, dtype=np.int64), (K // group, N)), group, axis=0)
    w = q - zk
    nb = K // BLOCK
    return np.einsum("mbk,bkn->mbn", xq.reshape(M, nb, BLOCK), w.reshape(nb, BLOCK, N))


def matmul(xq, sx, q, sw, zp, group):
    """y = sum_b s_x s_w I in FP64 from the exact integer block sums; zp None
    means SYM (z = 8)."""
    I = block_integer_sums(xq, q, 8 if zp is None else zp, group).astype(np.float64)
    K = np.asarray(q).shape[0]
    swb = np.repeat(np.asarray(sw, dtype=np.float16).astype(np.float64), group // BLOCK, axis=0)  # [K/32, N]
    sxb = np.asarray(sx, dtype=np.float32).astype(np.float64)  # [M, K/32]
    assert swb.shape[0] == K // BLOCK
    return np.einsum("mb,bn,mbn->mn", sxb, swb, I)
