"""W4A8 parity on the GPU: the dynamic INT8 activation quantiser bit-exact
against ``oracle.w4a8``; the W4A8 GEMV (INT4 image x the quantiser's INT8
activations) against the oracle's exact integer block sums,
both within the library's acceptance bound and within the much tighter bound
that exact integer sums leave (FP32 rounding of the block terms plus the
output's own rounding)."""

import numpy as np
import pytest

import workloads
from helpers import sample_columns
from oracle import int4, matmul, w4a8

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


def _tdt(torch, xdt):
    return torch.float16 if xdt == "f16" else torch.bfloat16


def _quant_compare(torch, lbq, X):
    Xf = X.float().numpy()
    ref_q, ref_s = w4a8.quantize_activations(Xf)
    xq, sx = lbq.quantize_int8(X.cuda())
    torch.cuda.synchronize()
    assert np.array_equal(xq.cpu().numpy(), ref_q)
    assert np.array_equal(sx.cpu().numpy().view(np.uint32), ref_s.view(np.uint32))
    return ref_q, ref_s


def test_quantize_int8_golden(torch, lbq, golden):
    g = golden("w4a8_block_1x64.json")
    for xdt in ("f16", "bf16"):
        X = torch.tensor(g["x"], dtype=_tdt(torch, xdt))
        assert np.array_equal(X.double().numpy(), np.array(g["x"]))   # exact in both types
        q, s = _quant_compare(torch, lbq, X)
        assert q.tolist() == g["xq"] and s.tolist() == g["s"]


def _planted(torch, xdt, M, K, seed, extreme=True):
    """Seeded activations with planted blocks; `extreme` adds the format's
    largest and smallest magnitudes (the GEMV tests keep outputs in FP16 range)."""
    X = workloads.activations_host(seed, M, K, xdt).clone()
    tiny = 6e-8 if xdt == "f16" else (1e-38 if extreme else 1e-30)
    huge = 6e4 if (xdt == "f16" or not extreme) else 1e38
    if K >= 256:
        X[0, 0:32] = 0.0                                   # zero block: s = 0
        X[0, 32:64] = tiny                                 # smallest magnitudes (FP32 subnormal s for BF16)
        X[0, 64:96] = 0.0
        X[0, 70] = -huge                                   # one huge element
        X[0, 96:128] = torch.arange(32) * 0.03125 - 0.5    # exact scale 1/16: every other x/s is a tie
        X[0, 96] = 7.9375
        X[0, 128:160] = X[0, 128:160] * 1e-3
    return X


@pytest.mark.parametrize("xdt", ["f16", "bf16"])
@pytest.mark.parametrize("M,K", [(1, 32), (3, 4096), (16, 1024), (5, 14336)])
def test_quantize_int8_bit_exact(torch, lbq, xdt, M, K):
    _quant_compare(torch, lbq, _planted(torch, xdt, M, K, 31 + M + K))


def _ulp_out(v, dt):
    a = np.abs(v)
    out = np.full(a.shape, 2.0 ** (-24 if dt == "f16" else -133))
    big = a >= (2.0 ** -14 if dt == "f16" else 2.0 ** -126)
    out[big] = np.exp2(np.floor(np.log2(a[big])) - (10 if dt == "f16" else 7))
    return out


def _check(Y_gpu, xq, sx, q, s, zp, group, ydt, cols=None):
    """Acceptance bound and the tight bound of exact integer sums."""
    Y = matmul.as_f64(Y_gpu)
    if cols is not None:
        Y = Y[:, cols]
    y_ref = w4a8.matmul(xq, sx, q, s, zp, group)
    Xe = w4a8.dequant_activations(xq, sx)
    S = matmul.abs_scale(Xe, int4.dequant(q, s, group, zp))
    ok, worst = matmul.check(Y, y_ref, S)
    assert ok, f"max error ratio {worst:.3g} > 1"
    tight = 2e-5 * S + _ulp_out(y_ref, ydt)
    assert np.all(np.abs(Y - y_ref) <= tight), float(np.max(np.abs(Y - y_ref) / tight))


SHAPES = [
    (96, 8, 32, "sym"),        # three blocks
    (1024, 139, 64, "asym"),   # a full warp of blocks, N ragged for every row block
    (4096, 77, 32, "asym"),
    (4096, 64, 128, "sym"),
    (14336, 40, 32, "asym"),   # fourteen warps
    (16384, 24, 128, "asym"),  # sixteen warps, the kernel's limit
]


@pytest.mark.parametrize("K,N,group,mode", SHAPES)
@pytest.mark.parametrize("xdt", ["f16", "bf16"])
def test_w4a8_gemv_parity(torch, lbq, K, N, group, mode, xdt):
    """Batch 1 on the staged kernel (and on the tiled one through the test
    hook), batches 2..16 on the tiled kernel."""
    W = workloads.weights_host(900 + K + N, K, N)
    q, s, zp = int4.quantize(W, group, mode)
    img = lbq.pack(torch.from_numpy(W).cuda(), group, mode)
    for M, tiled in ((1, False), (1, True), (2, False), (3, False), (4, False), (5, False), (16, False)):
        X = _planted(torch, xdt, M, K, 910 + M, extreme=False)
        xq, sx = _quant_compare(torch, lbq, X)
        dxq, dsx = lbq.quantize_int8(X.cuda())
        lbq.lbq_debug_w4a8_tiled(tiled)
        try:
            for ydt in ("f16", "bf16"):
                Y = lbq.w4a8_gemv(dxq, dsx, img, N, group, mode, y_dtype=ydt)
                torch.cuda.synchronize()
                _check(Y.cpu(), xq, sx, q, s, zp if mode == "asym" else None, group, ydt)
        finally:
            lbq.lbq_debug_w4a8_tiled(False)
    lbq.device_status()


@pytest.mark.parametrize("variant", [-1, 2, 3, 4])
def test_w4a8_staged_depths_and_grouped_launch(torch, lbq, variant):
    """q/k/v-shaped items sharing X in one launch, every staging depth; each
    item equals the oracle and the single-GEMV call bit for bit."""
    K, group, mode = 4096, 32, "asym"
    Ns = (4096, 1024, 1000)
    Ws = [workloads.weights_host(960 + i, K, n) for i, n in enumerate(Ns)]
    imgs = [lbq.pack(torch.from_numpy(W).cuda(), group, mode) for W in Ws]
    X = _planted(torch, "f16", 1, K, 961, extreme=False)
    xq, sx = _quant_compare(torch, lbq, X)
    dxq, dsx = lbq.quantize_int8(X.cuda())
    lbq.lbq_debug_direct_variant(variant)
    try:
        Ys = lbq.w4a8_gemv_grouped([(dxq, dsx, img, n) for img, n in zip(imgs, Ns)], group, mode)
        singles = [lbq.w4a8_gemv(dxq, dsx, img, n, group, mode) for img, n in zip(imgs, Ns)]
        torch.cuda.synchronize()
    finally:
        lbq.lbq_debug_direct_variant(-1)
    for W, Y, Y1 in zip(Ws, Ys, singles):
        q, s, zp = int4.quantize(W, group, mode)
        _check(Y.cpu(), xq, sx, q, s, zp, group, "f16")
        assert torch.equal(Y, Y1)
    lbq.device_status()


def test_w4a8_decode_step_shapes_sampled(torch, lbq):
    """The four launch shapes of the Llama-3-8B decode step (asym g32, batch 1),
    full size, outputs on sampled columns."""
    for p, (name, K, N) in enumerate(workloads.LLAMA3_8B_PROJ):
        seed = workloads.c2_seed(0, p)
        W = workloads.weights_host(seed, K, N)
        img = lbq.pack(torch.from_numpy(W).cuda(), 32, "asym")
        cols = sample_columns(N, 192, seed=p)
        q, s, zp = int4.quantize(np.ascontiguousarray(W[:, cols]), 32, "asym")
        X = workloads.activations_host(seed, 1, K, "f16")
        xq, sx = w4a8.quantize_activations(X.float().numpy())
        dxq, dsx = lbq.quantize_int8(X.cuda())
        Y = lbq.w4a8_gemv(dxq, dsx, img, N, 32, "asym")
        torch.cuda.synchronize()
        _check(Y.cpu(), xq, sx, q, s, zp, 32, "f16", cols)


def test_w4a8_errors(torch, lbq):
    W = workloads.weights_host(950, 64, 8)
    img = lbq.pack(torch.from_numpy(W).cuda(), 32, "sym")
    X = workloads.activations_host(950, 17, 64, "f16").cuda()
    xq, sx = lbq.quantize_int8(X)
    with pytest.raises(lbq.LbqError):
        lbq.w4a8_gemv(xq, sx, img, 8, 32, "sym")                  # M = 17 > 16
    with pytest.raises(lbq.LbqError):
        lbq.w4a8_gemv(xq[:1], sx[:1], img, 8, 32, "lut3")         # not an INT4 mode
    with pytest.raises(lbq.LbqError):
        lbq.quantize_int8(X[:, :48].contiguous())                 # K not a multiple of 32
    lbq.device_status()
