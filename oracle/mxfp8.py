"""MXFP8 activations: E4M3 elements with one UE8M0 scale per 32 consecutive k.

Test infrastructure only (see ``oracle/__init__.py``).

Source: the vLLM PR 62759 write-up ("LUT-B MoE with MXFP8 activations"). The
Rubin kernel there takes the activations as MXFP8 -- E4M3 elements with one
UE8M0 scale per 1 x 32 block -- because its LUT-decompressing MMA accepts only
FP8/FP6/FP4 for the other operand; its emulation path quantises the
activations to MXFP8 and back before each GEMM, so both paths compute
Y = dequant_mx(X) . W. The page points to the OCP Microscaling Formats (MX)
v1.0 specification for the element and scale types.

Readings taken where the page is silent (the plainest reading of the MX
scheme it links):

* A block is 32 consecutive k of one activation row: k = 32 b .. 32 b + 31.
* The block's shared scale is 2^(floor(log2(amax)) - 8), amax being the
  block's largest |x| and 8 the exponent of E4M3's largest binade
  (448 = 1.75 * 2^8). It is stored as the UE8M0 byte
  floor(log2(amax)) - 8 + 127, clamped to [0, 254]; a block of zeros stores
  127 (scale 1).
* Each element is x / scale rounded to the nearest E4M3 value, ties to even,
  saturating at +-448 (x / scale < 512 always, so only [448, 512) clamps).
  Elements too small for E4M3's subnormals round to +-0 (sign kept).
"""

import math

import numpy as np

from . import lut3

BLOCK = 32
E4M3_EMAX = 8        # 448 = 1.75 * 2^8
E4M3_MAX = 448.0
E4M3_MIN_EXP = -6    # smallest normal binade; subnormals are m * 2^-9


def round_e4m3(v):
    """Nearest E4M3 value of a real v (ties to even), saturating at +-448."""
    v = float(v)
    if math.isnan(v):
        raise ValueError("NaN activation")
    a = abs(v)
    if a >= E4M3_MAX:
        r = E4M3_MAX
    elif a == 0.0:
        r = 0.0
    else:
        e = max(math.floor(math.log2(a)), E4M3_MIN_EXP)
        # floor(log2) of a float can be off by one at binade edges: fix it exactly
        if e > E4M3_MIN_EXP and math.ldexp(1.0, e) > a:
            e -= 1
        elif math.ldexp(1.0, e + 1) <= a:
            e += 1
        quantum = math.ldexp(1.0, e - 3)           # 3 mantissa bits (subnormals: 2^-9)
        r = round(a / quantum) * quantum            # Python round(): ties to even, exact here
        r = min(r, E4M3_MAX)
    return math.copysign(r, v)


# value -> byte for every finite E4M3 value (0x00 for +0, 0x80 for -0)
_E4M3_BYTE = {}
for _b in range(256):
    _v = lut3.E4M3_TABLE[_b]
    if not math.isnan(_v):
        _E4M3_BYTE.setdefault((_v, math.copysign(1.0, _v) if _v == 0 else 0.0), _b)


def e4m3_byte(value):
    """Byte of an exactly representable E4M3 value."""
    key = (value, math.copysign(1.0, value) if value == 0 else 0.0)
    return _E4M3_BYTE[key]


def block_scale_byte(amax):
    """UE8M0 byte of a block whose largest |x| is amax."""
    if amax == 0.0:
        return 127
    e = math.floor(math.log2(amax))
    if math.ldexp(1.0, e) > amax:
        e -= 1
    elif math.ldexp(1.0, e + 1) <= amax:
        e += 1
    return int(min(max(e - E4M3_EMAX + 127, 0), 254))


def quantize(X):
    """X [M, K] (real values, K % 32 == 0) -> (codes uint8 [M, K] E4M3,
    scales uint8 [M, K/32] UE8M0)."""
    X = np.asarray(X, dtype=np.float64)
    M, K = X.shape
    if K % BLOCK:
        raise ValueError("K must be a multiple of 32")
    codes = np.zeros((M, K), dtype=np.uint8)
    scales = np.zeros((M, K // BLOCK), dtype=np.uint8)
    for m in range(M):
        for b in range(K // BLOCK):
            blk = X[m, BLOCK * b:BLOCK * (b + 1)]
            sb = block_scale_byte(float(np.max(np.abs(blk))))
            scales[m, b] = sb
            inv = math.ldexp(1.0, 127 - sb)  # exact power of two
            for i, x in enumerate(blk):
                codes[m, BLOCK * b + i] = e4m3_byte(round_e4m3(float(x) * inv))
    return codes, scales


def dequant(codes, scales):
    """Exact values: E4M3(code) * 2^(scale - 127), float64 [M, K]."""
    codes = np.asarray(codes, dtype=np.uint8)
    scales = np.asarray(scales, dtype=np.uint8)
    M, K = codes.shape
    if scales.shape != (M, K // BLOCK):
        raise ValueError("scales must be [M, K/32]")
    if np.any((codes & 0x7F) == 0x7F) or np.any(scales == 0xFF):
        raise ValueError("NaN element or scale")
    blk = np.arange(K) // BLOCK
    return lut3.E4M3_TABLE[codes] * np.ldexp(1.0, scales.astype(np.int64)[:, blk] - 127)


def lut3_matmul(X, idx, codebooks, exponents):
    """Y = dequant_mx(quantize(X)) . decode(W) with FP64 accumulation, the
    result of both of the page's LUT3 x MXFP8 paths. Every product is exact
    in FP64 (two 4-bit significands and powers of two)."""
    codes, scales = quantize(X)
    Xq = dequant(codes, scales)
    W = lut3.dequant(idx, codebooks, exponents)
    return Xq @ W
