"""Generic b-bit affine parity on the GPU, b = 1..8: the image's canonical bit
streams, scales and zero points bit-exact against ``oracle.affine``; GEMV
outputs within |y - y_ref| <= 4e-3*S + ulp16(|y_ref|) of the FP64 product with
the oracle's exact dequantised weight."""

import numpy as np
import pytest

import workloads
from helpers import check_outputs, sample_columns
from oracle import affine

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch():
    import torch
    assert torch.cuda.is_available(), "these tests need a CUDA device"
    return torch


@pytest.fixture(scope="module")
def lbq():
    import bit_weight_only_pack_b200 as lbq
    return lbq


def oracle_affine(W, group, bits):
    q, s, zp = affine.quantize(W, group, bits)
    return dict(q=q, s=s, zp=zp, packed=affine.pack(q, bits), deq=affine.dequant(q, s, group, zp))


def _special_groups(W, group):
    """Plant the degenerate and one-sided groups the quantiser has to handle."""
    K, N = W.shape
    if N >= 4 and K >= 2 * group:
        W[:group, 0] = 0.0                                   # all-zero group (scale 0)
        W[group:2 * group, 1] = 0.37                         # constant group (scale 0)
        W[:group, 2] = np.abs(W[:group, 2]) + 0.01           # all-positive group
        W[group:2 * group, 3] = -np.abs(W[group:2 * group, 3]) - 0.5  # all-negative, zp clamps
    return W


def _pack_and_compare(torch, lbq, W, group, bits):
    K, N = W.shape
    ref = oracle_affine(W, group, bits)
    img = lbq.pack_affine(torch.from_numpy(W).cuda(), group, bits)
    q, s, z = lbq.unpack_affine_canonical(img, K, N, group, bits)
    assert np.array_equal(q.cpu().numpy(), ref["packed"])
    assert np.array_equal(s.cpu().view(torch.int16).numpy(), ref["s"].view(np.int16))
    assert np.array_equal(z.cpu().numpy(), ref["zp"])
    return img, ref


BITS = list(range(1, 9))
SHAPES = [
    (32, 1, 32),        # one chunk, one column
    (96, 8, 32),        # three chunks
    (256, 40, 64),
    (1024, 139, 128),   # one full warp of chunks, N ragged for every row block
    (4096, 77, 32),     # four warps
]


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("K,N,group", SHAPES)
def test_pack_bit_exact(torch, lbq, bits, K, N, group):
    W = _special_groups(workloads.weights_host(100 + 7 * bits + K + N, K, N), group)
    _pack_and_compare(torch, lbq, W, group, bits)


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("xdt", ["f16", "bf16"])
@pytest.mark.parametrize("K,N,group", [(1024, 139, 64), (4096, 77, 32), (96, 8, 32)])
def test_gemv_parity(torch, lbq, bits, xdt, K, N, group):
    W = _special_groups(workloads.weights_host(200 + bits + K, K, N), group)
    img, ref = _pack_and_compare(torch, lbq, W, group, bits)
    for M in (1, 2, 3, 4, 6, 16):   # every batch tile, a ragged tile, several launches
        X = workloads.activations_host(300 + M + bits, M, K, xdt)
        for ydt in ("f16", "bf16"):
            Y = lbq.affine_gemv(X.cuda(), img, N, group, bits, y_dtype=ydt)
            torch.cuda.synchronize()
            check_outputs(Y.cpu(), X, ref["deq"])
    lbq.device_status()


@pytest.mark.parametrize("bits", [1, 3, 8])
def test_gemv_longest_k(torch, lbq, bits):
    """K = 16384: sixteen warps per CTA, the kernel's limit."""
    K, N, group = 16384, 24, 128
    W = workloads.weights_host(400 + bits, K, N)
    img, ref = _pack_and_compare(torch, lbq, W, group, bits)
    for xdt in ("f16", "bf16"):
        X = workloads.activations_host(401, 1, K, xdt)
        Y = lbq.affine_gemv(X.cuda(), img, N, group, bits)
        torch.cuda.synchronize()
        check_outputs(Y.cpu(), X, ref["deq"])


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_decode_shape_full_size_sampled(torch, lbq, bits):
    """The gate/up projection shape at batch 1 (K=4096, N=14336, g64): codes of
    sampled columns bit-exact, outputs of the same columns within the bound."""
    K, N, group = 4096, 14336, 64
    W = workloads.weights_host(500 + bits, K, N)
    Wd = torch.from_numpy(W).cuda()
    img = lbq.pack_affine(Wd, group, bits)
    del Wd
    cols = sample_columns(N, 256, seed=bits)
    ref = oracle_affine(np.ascontiguousarray(W[:, cols]), group, bits)
    q, s, z = lbq.unpack_affine_canonical(img, K, N, group, bits)
    assert np.array_equal(q.cpu().numpy()[:, cols], ref["packed"])
    assert np.array_equal(s.cpu().view(torch.int16).numpy()[:, cols], ref["s"].view(np.int16))
    assert np.array_equal(z.cpu().numpy()[:, cols], ref["zp"])
    for xdt in ("f16", "bf16"):
        X = workloads.activations_host(501, 1, K, xdt)
        Y = lbq.affine_gemv(X.cuda(), img, N, group, bits)
        torch.cuda.synchronize()
        check_outputs(Y.cpu(), X, ref["deq"], cols)


def test_large_activation_magnitudes(torch, lbq):
    K, N, group = 2048, 64, 32
    for bits in (1, 5, 8):
        W = workloads.weights_host(600 + bits, K, N)
        img, ref = _pack_and_compare(torch, lbq, W, group, bits)
        for xdt in ("f16", "bf16"):
            X = (workloads.activations_host(601, 2, K, xdt).float() * 100).to(
                torch.float16 if xdt == "f16" else torch.bfloat16)
            Y = lbq.affine_gemv(X.cuda(), img, N, group, bits)
            torch.cuda.synchronize()
            check_outputs(Y.cpu(), X, ref["deq"])


def test_four_bits_match_the_int4_path(torch, lbq):
    """bits = 4 is the asymmetric INT4 format: the two libraries' images
    dequantise to the same weight, so both GEMVs meet the same oracle."""
    K, N, group = 1024, 64, 32
    W = workloads.weights_host(700, K, N)
    img_a, ref = _pack_and_compare(torch, lbq, W, group, 4)
    img_i = lbq.pack(torch.from_numpy(W).cuda(), group, "asym")
    deq_i = lbq.dequant(img_i, K, N, group, "asym").cpu().numpy().astype(np.float64)
    assert np.array_equal(deq_i, ref["deq"])
    X = workloads.activations_host(701, 1, K, "f16")
    check_outputs(lbq.affine_gemv(X.cuda(), img_a, N, group, 4).cpu(), X, ref["deq"])
    check_outputs(lbq.gemv(X.cuda(), img_i, N, group, "asym").cpu(), X, ref["deq"])


def test_argument_and_header_errors(torch, lbq):
    W = workloads.weights_host(800, 64, 8)
    img = lbq.pack_affine(torch.from_numpy(W).cuda(), 32, 3)
    with pytest.raises(lbq.LbqError):
        lbq.unpack_affine_canonical(img, 64, 8, 32, 2)      # bits do not match the image
    with pytest.raises(lbq.LbqError):
        lbq.unpack_affine_canonical(img, 64, 8, 64, 3)      # group does not match
    X = workloads.activations_host(800, 17, 64, "f16").cuda()
    with pytest.raises(lbq.LbqError):
        lbq.affine_gemv(X, img, 8, 32, 3)                   # M = 17 > 16
    with pytest.raises(lbq.LbqError):
        lbq.affine_gemv(X[:1], img, 8, 32, 9)               # bits out of range
    lbq.device_status()
