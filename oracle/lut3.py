"""The 3-bit LUT weight format: exact decode and the canonical index stream.

Test infrastructure only (see ``oracle/__init__.py``).

Source: the vLLM PR 62759 write-up ("LUT-B MoE with MXFP8 activations"),
format section: each weight is a 3-bit index into an 8-entry E4M3 codebook;
one codebook is shared by a tile of 8 output channels x 64 K, and each tile
carries one UE8M0 exponent (about 3.14 bits per weight). The exponent keeps
small tiles out of the E4M3 subnormal range, so a weight's value is
codebook[idx] * 2^(E - 127). E4M3 and UE8M0 are the OCP Microscaling (MX)
element and scale types that page links to.

Readings taken where the page is silent:

* E4M3 is the "fn" variant: bias 7, subnormals, max 448, 0x7F / 0xFF are NaN.
* UE8M0 has bias 127 and 0xFF is NaN.
* Tiles are ordered [K/64][N/8]; codebooks are [K/64][N/8][8] bytes and
  exponents [K/64][N/8] bytes.
* Canonical index stream: per tile and per output channel, the 64 indices
  (k = 64*kt + i) form a little-endian 192-bit stream, index i in bits
  [3i, 3i + 3): 24 bytes per channel, 192 bytes per tile.
"""

import numpy as np

TILE_K = 64
TILE_N = 8


def e4m3_value(byte):
    """Value of one E4M3 ("fn") byte as a Python float (NaN for 0x7F/0xFF).

    Sign bit 7, exponent bits 6..3 (bias 7), mantissa bits 2..0. Exponent 0
    encodes subnormals m/8 * 2^-6.
    """
    b = int(byte) & 0xFF
    sign = -1.0 if b & 0x80 else 1.0
    e = (b >> 3) & 0xF
    m = b & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return sign * (m / 8.0) * 2.0 ** -6
    return sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)


E4M3_TABLE = np.array([e4m3_value(b) for b in range(256)], dtype=np.float64)


def ue8m0_value(byte):
    """Value of one UE8M0 byte: 2^(E - 127); 0xFF is NaN."""
    e = int(byte) & 0xFF
    if e == 0xFF:
        return float("nan")
    return float(np.ldexp(1.0, e - 127))


def check_tiles(K, N):
    if K % TILE_K or N % TILE_N or K <= 0 or N <= 0:
        raise ValueError("LUT3 needs K % 64 == 0 and N % 8 == 0")


def dequant(idx, codebooks, exponents):
    """Exact decode: W[k, n] = E4M3(cb[k//64, n//8, idx[k, n]]) * 2^(E[k//64, n//8] - 127).

    idx uint8 [K, N] (0..7), codebooks uint8 [K/64, N/8, 8], exponents uint8
    [K/64, N/8]. Returns float64 [K, N]. NaN codebook entries or exponents are
    rejected.
    """
    idx = np.asarray(idx, dtype=np.uint8)
    K, N = idx.shape
    check_tiles(K, N)
    cb = np.asarray(codebooks, dtype=np.uint8)
    ex = np.asarray(exponents, dtype=np.uint8)
    if cb.shape != (K // TILE_K, N // TILE_N, 8) or ex.shape != (K // TILE_K, N // TILE_N):
        raise ValueError("codebook / exponent shapes do not match the tile grid")
    if np.any(idx > 7):
        raise ValueError("indices must be 0..7")
    if np.any((cb & 0x7F) == 0x7F) or np.any(ex == 0xFF):
        raise ValueError("NaN codebook entry or exponent")
    cb_val = E4M3_TABLE[cb]                                        # [KT, NT, 8]
    scale = np.ldexp(1.0, ex.astype(np.int64) - 127)               # [KT, NT]
    kt = np.arange(K)[:, None] // TILE_K
    nt = np.arange(N)[None, :] // TILE_N
    return cb_val[kt, nt, idx] * scale[kt, nt]


def pack_indices(idx):
    """Canonical index stream: uint8 [K, N] (0..7) -> uint8 [K/64, N/8, 8, 24].

    Output [kt, nt, c, :] holds the 64 indices of channel n = 8*nt + c for
    k = 64*kt .. 64*kt + 63, index i occupying bits [3i, 3i+3) of a
    little-endian 192-bit string.
    """
    idx = np.asarray(idx, dtype=np.uint8)
    K, N = idx.shape
    check_tiles(K, N)
    if np.any(idx > 7):
        raise ValueError("indices must be 0..7")
    KT, NT = K // TILE_K, N // TILE_N
    # t[kt, nt, c, i] = idx[64 kt + i, 8 nt + c]
    t = idx.reshape(KT, TILE_K, NT, TILE_N).transpose(0, 2, 3, 1).astype(np.uint64)
    out = np.zeros((KT, NT, TILE_N, 24), dtype=np.uint8)
    for i in range(TILE_K):
        bit = 3 * i
        for b in range(3):
            pos = bit + b
            out[..., pos // 8] |= (((t[..., i] >> np.uint64(b)) & np.uint64(1)) << np.uint64(pos % 8)).astype(np.uint8)
    return out


def unpack_indices(packed):
    """Inverse of :func:`pack_indices`: uint8 [K/64, N/8, 8, 24] -> idx [K, N]."""
    p = np.asarray(packed, dtype=np.uint8)
    KT, NT, C, B = p.shape
    if C != TILE_N or B != 24:
        raise ValueError("packed indices must be [K/64, N/8, 8, 24]")
    t = np.zeros((KT, NT, TILE_N, TILE_K), dtype=np.uint8)
    for i in range(TILE_K):
        v = np.zeros((KT, NT, TILE_N), dtype=np.uint8)
        for b in range(3):
            pos = 3 * i + b
            v |= ((p[..., pos // 8] >> (pos % 8)) & 1) << b
        t[..., i] = v
    return t.transpose(0, 3, 1, 2).reshape(KT * TILE_K, NT * TILE_N)


def algorithmic_bytes(K, N):
    """Index bytes (3 bits per weight) + 8 codebook bytes + 1 exponent byte per tile."""
    check_tiles(K, N)
    tiles = (K // TILE_K) * (N // TILE_N)
    return K * N * 3 // 8 + tiles * (8 + 1)
