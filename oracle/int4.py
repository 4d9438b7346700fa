"""INT4 group-wise quantisation, canonical packing and exact dequantisation.

Test infrastructure only (see ``oracle/__init__.py``).

Logical weight layout: W is [K, N] and Y = X . W, as in the problem statement of
"Low Bit Metal Kernels" (INT4 dequant + matmul listing: X is M x K, W_tile is
indexed [k][n]). Groups run along K: one FP16 scale (and, for the asymmetric
form, one int8 zero point) per (group of ``group`` consecutive k, column n);
"Low Bit ARM kernels", group-wise scale section (group size 32, 64 or 128).

Readings taken where the pages are silent:

* The scale is computed in FP32 and stored as FP16 (round to nearest even);
  the codes are computed by dividing by the *stored* scale widened back to FP32,
  so that dequantisation reproduces exactly the value the codes were fitted to.
* Rounding of w/s (and of -min/s) is round-half-to-even (``rint``).
* Asymmetric: lo = min(w), hi = max(w) over the group (zero is not forced into
  the range); s = fp16((hi - lo) / 15); zp = clamp(rint(-lo / s), -128, 127).
* A group whose stored scale is 0 (all zeros, or hi == lo, or an FP16
  underflow) gets q = 8 (symmetric) or zp = 0, q = 0 (asymmetric): it
  dequantises to 0.
"""

import numpy as np

F32 = np.float32


def _grouped(W, group):
    """View W [K, N] as [K/group, group, N] (groups along K)."""
    W = np.asarray(W)
    if W.dtype != np.float32:
        raise TypeError("W must be float32")
    K, N = W.shape
    if group <= 0 or K % group != 0:
        raise ValueError("K must be a positive multiple of group")
    return W.reshape(K // group, group, N)


def quantize_sym(W, group):
    """Symmetric INT4: s = fp16(max|w| / 7); q = clamp(rint(w/s) + 8, 0, 15).

    Follows "Low Bit Metal Kernels" (the dequant lines of the INT4 listing
    subtract 8 from each nibble before multiplying by the group scale) and
    "Low Bit ARM kernels" (symmetric = scale only, zero point fixed).
    Returns (q uint8 [K, N], scale float16 [K/group, N]).
    """
    Wg = _grouped(W, group)
    amax = np.max(np.abs(Wg), axis=1)                      # [G, N], exact in FP32
    s16 = (amax / F32(7.0)).astype(np.float16)             # FP32 divide, RN to FP16
    s = s16.astype(np.float32)[:, None, :]                 # the stored scale, widened
    safe = np.where(s == 0, F32(1.0), s)
    r = np.rint(Wg / safe)                                 # FP32 divide, half-to-even
    q = np.clip(r + F32(8.0), 0, 15)
    q = np.where(s == 0, F32(8.0), q)
    K, N = np.asarray(W).shape
    return q.astype(np.uint8).reshape(K, N), s16


def quantize_asym(W, group):
    """Asymmetric INT4 with an int8 zero point (min/max fit).

    "Low Bit ARM kernels", group-wise scale section: asymmetric = an FP16 scale
    plus an int8 zero point per group. With lo/hi the group's min/max:
    s = fp16((hi - lo) / 15), zp = clamp(rint(-lo/s), -128, 127),
    q = clamp(rint(w/s) + zp, 0, 15); dequantised value (q - zp) * s.
    Returns (q uint8 [K, N], scale float16 [K/group, N], zp int8 [K/group, N]).
    """
    Wg = _grouped(W, group)
    lo = np.min(Wg, axis=1)
    hi = np.max(Wg, axis=1)
    s16 = ((hi - lo) / F32(15.0)).astype(np.float16)      # FP32 subtract + divide, RN to FP16
    s = s16.astype(np.float32)
    safe = np.where(s == 0, F32(1.0), s)
    zp = np.clip(np.rint(-lo / safe), -128, 127)
    zp = np.where(s == 0, F32(0.0), zp)
    r = np.rint(Wg / safe[:, None, :])
    q = np.clip(r + zp[:, None, :], 0, 15)
    q = np.where(s[:, None, :] == 0, F32(0.0), q)
    K, N = np.asarray(W).shape
    return q.astype(np.uint8).reshape(K, N), s16, zp.astype(np.int8)


def pack_nibbles(q):
    """Canonical packing: two codes per byte, low nibble = even k.

    "Low Bit Metal Kernels", INT4 listing: ``packed & 0x0F`` feeds W_tile row
    2*i and ``packed >> 4`` feeds row 2*i+1 of the same column. So
    byte[j, n] = q[2j, n] | q[2j+1, n] << 4, giving uint8 [K/2, N].
    """
    q = np.asarray(q, dtype=np.uint8)
    if q.shape[0] % 2:
        raise ValueError("K must be even")
    if np.any(q > 15):
        raise ValueError("codes must be 0..15")
    return (q[0::2] | (q[1::2] << 4)).astype(np.uint8)


def unpack_nibbles(packed):
    """Inverse of :func:`pack_nibbles`: uint8 [K/2, N] -> codes uint8 [K, N]."""
    packed = np.asarray(packed, dtype=np.uint8)
    K2, N = packed.shape
    q = np.empty((2 * K2, N), dtype=np.uint8)
    q[0::2] = packed & 0x0F
    q[1::2] = packed >> 4
    return q


def dequant(q, scale16, group, zp=None):
    """Exact dequantisation (q - zp) * s, returned as float64 [K, N].

    zp=None means the symmetric form, whose zero point is 8 ("Low Bit Metal
    Kernels": ``((int)(packed & 0x0F) - 8) * scales[group]``). The product of a
    small integer and an FP16 value is exact in FP32 and in FP64.
    """
    q = np.asarray(q).astype(np.float64)
    K, N = q.shape
    s = np.asarray(scale16, dtype=np.float16).astype(np.float64)
    if s.shape != (K // group, N):
        raise ValueError("scale must be [K/group, N]")
    z = np.full_like(s, 8.0) if zp is None else np.asarray(zp, dtype=np.int8).astype(np.float64)
    s_k = np.repeat(s, group, axis=0)
    z_k = np.repeat(z, group, axis=0)
    return (q - z_k) * s_k


def quantize(W, group, mode):
    """Dispatch on mode ('sym' or 'asym'); returns (q, scale16, zp or None)."""
    if mode == "sym":
        q, s = quantize_sym(W, group)
        return q, s, None
    if mode == "asym":
        return quantize_asym(W, group)
    raise ValueError(mode)


def algorithmic_bytes(K, N, group, mode):
    """Bytes the format must hold: K*N/2 nibble bytes + 2 bytes of scale per
    group (+ 1 byte of zero point per group in the asymmetric form)."""
    per_group = 2 + (1 if mode == "asym" else 0)
    return K * N // 2 + (K // group) * N * per_group
