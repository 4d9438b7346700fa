"""Generic b-bit affine group-wise weights (b = 1..8): quantisation, canonical
bit-stream packing and exact dequantisation.

Test infrastructure only (see ``oracle/__init__.py``).

"Low Bit ARM kernels" keeps one kernel per bit width in a bit-width x tile table
(its ``kernels[8][3]`` lookup with an ``unpack`` routine per width of 1..8 bits)
and notes that 3-bit weights often match 4-bit accuracy; the group-wise section
gives the affine form: an FP16 scale and an int8 zero point per group of 32, 64
or 128 consecutive k of a column. The value of code q is (q - zp) * s.

Readings taken where the pages are silent (the 4-bit case is exactly the
asymmetric INT4 form of ``oracle.int4``):

* L = 2^b - 1 levels above zero: s = fp16((max w - min w) / L) over the group,
  computed in FP32 and rounded to nearest even; zp = clamp(rint(-min w / s),
  -128, 127) with the stored scale widened to FP32; q = clamp(rint(w / s) + zp,
  0, L). A group whose stored scale is 0 gets zp = 0 and q = 0.
* Canonical packing: per column n, the K codes form one little-endian bit
  stream, code k in bits [b k, b k + b); byte j of column n's stream is
  packed[j, n], so the canonical array is uint8 [K b / 8, N]. For b = 4 this is
  two codes per byte with the low nibble the even k, the INT4 canonical layout.
"""

import numpy as np

F32 = np.float32


def levels(bits):
    if not 1 <= bits <= 8:
        raise ValueError("bits must be 1..8")
    return (1 << bits) - 1


def quantize(W, group, bits):
    """Asymmetric b-bit codes with an FP16 scale and int8 zero point per group.
    Returns (q uint8 [K, N], scale float16 [K/group, N], zp int8 [K/group, N])."""
    L = F32(levels(bits))
    W = np.asarray(W)
    if W.dtype != np.float32:
        raise TypeError("W must be float32")
    K, N = W.shape
    if group <= 0 or K % group:
        raise ValueError("K must be a positive multiple of group")
    Wg = W.reshape(K // group, group, N)
    lo = Wg.min(axis=1)
    hi = Wg.max(axis=1)
    s16 = ((hi - lo) / L).astype(np.float16)
    s = s16.astype(np.float32)
    safe = np.where(s == 0, F32(1.0), s)
    zp = np.where(s == 0, F32(0.0), np.clip(np.rint(-lo / safe), -128, 127))
    q = np.clip(np.rint(Wg / safe[:, None, :]) + zp[:, None, :], 0, L)
    q = np.where(s[:, None, :] == 0, F32(0.0), q)
    return q.astype(np.uint8).reshape(K, N), s16, zp.astype(np.int8)


def pack(q, bits):
    """Canonical bit streams: code k of column n at bits [b k, b k + b) of that
    column's little-endian stream; returns uint8 [K b / 8, N]."""
    q = np.asarray(q, dtype=np.uint8)
    K, N = q.shape
    if (K * bits) % 8:
        raise ValueError("K * bits must be a whole number of bytes")
    if np.any(q > levels(bits)):
        raise ValueError("codes out of range")
    out = np.zeros((K * bits // 8, N), dtype=np.uint8)
    for k in range(K):
        for i in range(bits):
            bit = bits * k + i
            out[bit // 8] |= (((q[k] >> i) & 1) << (bit % 8)).astype(np.uint8)
    return out


def unpack(packed, bits, K):
    """Inverse of :func:`pack`: uint8 [K b / 8, N] -> codes uint8 [K, N]."""
    packed = np.asarray(packed, dtype=np.uint8)
    N = packed.shape[1]
    q = np.zeros((K, N), dtype=np.uint8)
    for k in range(K):
        for i in range(bits):
            bit = bits * k + i
            q[k] |= (((packed[bit // 8] >> (bit % 8)) & 1) << i).astype(np.uint8)
    return q


def dequant(q, scale16, group, zp):
    """Exact values (q - zp) * s as float64 [K, N]."""
    q = np.asarray(q).astype(np.float64)
    K, N = q.shape
    s = np.asarray(scale16, dtype=np.float16).astype(np.float64)
    z = np.asarray(zp, dtype=np.int8).astype(np.float64)
    if s.shape != (K // group, N) or z.shape != s.shape:
        raise ValueError("scale and zp must be [K/group, N]")
    return (q - np.repeat(z, group, axis=0)) * np.repeat(s, group, axis=0)


def algorithmic_bytes(K, N, group, bits):
    """K N b / 8 code bytes + 3 bytes (FP16 scale, int8 zero point) per group."""
    return K * N * bits // 8 + (K // group) * N * 3
