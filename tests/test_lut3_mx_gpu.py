"""LUT3 weights x MXFP8 activations on the block-scaled FP8 tensor path,
against the oracle (exact MXFP8 and LUT3 decodes, FP64 product), within
|y - y_ref| <= 4e-3*S + ulp16(|y_ref|)."""

import numpy as np
import pytest

import workloads
from oracle import lut3, matmul, mxfp8

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


def _check(Y_gpu, Xq, W):
    Y = matmul.as_f64(Y_gpu)
    ok, worst = matmul.check(Y, matmul.matmul_f64(Xq, W), matmul.abs_scale(Xq, W))
    assert ok, f"max error ratio {worst:.3g} > 1"
    return worst


def _run(torch, lbq, codes, scales, idx, cb, ex, ydt):
    K, N = idx.shape
    img = lbq.pack_lut3(torch.from_numpy(idx).cuda(), torch.from_numpy(cb).cuda(), torch.from_numpy(ex).cuda())
    Y = lbq.lut3_mx_gemm(torch.from_numpy(codes).cuda(), torch.from_numpy(scales).cuda(), img, N, y_dtype=ydt)
    torch.cuda.synchronize()
    lbq.device_status()
    return Y.cpu()


@pytest.mark.parametrize("M,K,N", [
    (256, 512, 128),     # one tile, one 512-k scale row
    (300, 1024, 136),    # ragged tokens and channels (a partial channel tile of one group)
    (17, 512, 264),      # fewer tokens than a tile, three channel tiles
    (512, 2048, 256),    # several token tiles and k-blocks
])
@pytest.mark.parametrize("ydt", ["bf16", "f16"])
def test_mx_gemm_parity(torch, lbq, M, K, N, ydt):
    codes, scales = workloads.mx_activations_host(400 + M + K, M, K)
    idx, cb, ex = workloads.lut3_host(401 + N, K, N)
    Y = _run(torch, lbq, codes, scales, idx, cb, ex, ydt)
    _check(Y, mxfp8.dequant(codes, scales), lut3.dequant(idx, cb, ex))


@pytest.mark.parametrize("M,K,N", [
    (300, 1024, 10000),  # 158 tiles: the tail wave's tiles cut along K, ragged tokens
    (1100, 1024, 4104),  # 165 tiles, a partial channel tile
])
def test_mx_gemm_stream_k(torch, lbq, M, K, N):
    """With the workspace the last waves' tiles are cut between neighbouring
    CTAs (the parked part added in a fixed order): both schedules match the
    oracle, repeated calls on one workspace are identical and every flag is
    back at zero after each call."""
    codes, scales = workloads.mx_activations_host(430 + M, M, K)
    idx, cb, ex = workloads.lut3_host(431 + N, K, N)
    img = lbq.pack_lut3(torch.from_numpy(idx).cuda(), torch.from_numpy(cb).cuda(), torch.from_numpy(ex).cuda())
    cd, sd = torch.from_numpy(codes).cuda(), torch.from_numpy(scales).cuda()
    ws = lbq.workspace(2, M, K, N, 0, "lut3")
    assert ws is not None
    grid = lbq.lbq_debug_gemm_schedule(M, K, N, 1, 0)[0]
    Ys = [lbq.lut3_mx_gemm(cd, sd, img, N, ws=ws) for _ in range(3)]
    torch.cuda.synchronize()
    lbq.device_status()
    assert all(torch.equal(Ys[0], Y) for Y in Ys[1:])
    assert int(ws[:grid * 4].view(torch.int32).abs().sum()) == 0
    Xq, W = mxfp8.dequant(codes, scales), lut3.dequant(idx, cb, ex)
    _check(Ys[0].cpu(), Xq, W)
    lbq.lbq_debug_gemm_stream_k(0)
    try:
        Y0 = lbq.lut3_mx_gemm(cd, sd, img, N, ws=ws)
        torch.cuda.synchronize()
    finally:
        lbq.lbq_debug_gemm_stream_k(1)
    _check(Y0.cpu(), Xq, W)


def test_mx_gemm_stream_k_wait_runs_out_and_is_reported(torch, lbq):
    """A withheld flag (test hook) ends each earlier part's wait after a short
    bound: LBQ_ERR_DEVICE is reported, and the next call on the same workspace
    matches the oracle."""
    M, K, N = 300, 1024, 10000
    codes, scales = workloads.mx_activations_host(440, M, K)
    idx, cb, ex = workloads.lut3_host(441, K, N)
    img = lbq.pack_lut3(torch.from_numpy(idx).cuda(), torch.from_numpy(cb).cuda(), torch.from_numpy(ex).cuda())
    cd, sd = torch.from_numpy(codes).cuda(), torch.from_numpy(scales).cuda()
    ws = lbq.workspace(2, M, K, N, 0, "lut3")
    lbq.device_status()
    lbq.lbq_debug_gemm_hold(2000)
    try:
        lbq.lut3_mx_gemm(cd, sd, img, N, ws=ws)
        with pytest.raises(lbq.LbqError) as err:
            lbq.device_status()
        assert err.value.status == 4  # LBQ_ERR_DEVICE
    finally:
        lbq.lbq_debug_gemm_hold(0)
    lbq.device_status()
    Y = lbq.lut3_mx_gemm(cd, sd, img, N, ws=ws)
    torch.cuda.synchronize()
    lbq.device_status()
    _check(Y.cpu(), mxfp8.dequant(codes, scales), lut3.dequant(idx, cb, ex))


def test_mx_gemm_scale_extremes(torch, lbq):
    """Exponents and scale bytes at the ends of a wide range (weights down to
    2^-117 x E4M3, activations 2^-24..2^+8): the block scales enter the
    product exactly."""
    M, K, N = 64, 512, 128
    codes, scales = workloads.mx_activations_host(410, M, K, scale_lo=103, scale_hi=135)
    idx, cb, ex = workloads.lut3_host(411, K, N)
    rng = np.random.default_rng(412)
    ex = rng.integers(40, 201, size=ex.shape, dtype=np.uint8)  # products stay inside FP32
    Y = _run(torch, lbq, codes, scales, idx, cb, ex, "bf16")
    _check(Y, mxfp8.dequant(codes, scales), lut3.dequant(idx, cb, ex))


def test_mx_gemm_after_gpu_quantiser_matches_the_oracle_end_to_end(torch, lbq):
    """BF16 activations -> lbq_quantize_mxfp8 -> the block-scaled GEMM, against
    oracle.mxfp8.lut3_matmul (the oracle's own quantiser and decode)."""
    M, K, N = 40, 512, 128
    X = workloads.activations_host(420, M, K, "bf16")
    idx, cb, ex = workloads.lut3_host(421, K, N)
    codes, scales = lbq.quantize_mxfp8(X.cuda())
    img = lbq.pack_lut3(torch.from_numpy(idx).cuda(), torch.from_numpy(cb).cuda(), torch.from_numpy(ex).cuda())
    Y = lbq.lut3_mx_gemm(codes, scales, img, N)
    torch.cuda.synchronize()
    lbq.device_status()
    Y_ref = mxfp8.lut3_matmul(matmul.as_f64(X), idx, cb, ex)
    oc, osc = mxfp8.quantize(matmul.as_f64(X))
    S = matmul.abs_scale(mxfp8.dequant(oc, osc), lut3.dequant(idx, cb, ex))
    ok, worst = matmul.check(matmul.as_f64(Y.cpu()), Y_ref, S)
    assert ok, f"max error ratio {worst:.3g} > 1"


def test_mx_gemm_full_size_sampled(torch, lbq):
    """The LUT3 prefill shape at M=2048 (K=4096, N=14336), 48 sampled
    channel groups of 8 against the oracle."""
    M, K, N = 2048, 4096, 14336
    codes, scales = workloads.mx_activations_host(430, M, K)
    idx, cb, ex = workloads.lut3_host(5, K, N)
    Y = _run(torch, lbq, codes, scales, idx, cb, ex, "bf16")
    rng = np.random.default_rng(431)
    groups = np.sort(rng.choice(N // 8, size=48, replace=False))
    cols = (groups[:, None] * 8 + np.arange(8)[None, :]).reshape(-1)
    W = lut3.dequant(np.ascontiguousarray(idx[:, cols]), np.ascontiguousarray(cb[:, groups]),
                     np.ascontiguousarray(ex[:, groups]))
    _check(Y[:, cols], mxfp8.dequant(codes, scales), W)


def test_mx_gemm_rejects_bad_arguments(torch, lbq):
    idx, cb, ex = workloads.lut3_host(440, 256, 128)
    img = lbq.pack_lut3(torch.from_numpy(idx).cuda(), torch.from_numpy(cb).cuda(), torch.from_numpy(ex).cuda())
    codes = torch.zeros((8, 256), dtype=torch.uint8, device="cuda")
    scales = torch.zeros((8, 8), dtype=torch.uint8, device="cuda")
    with pytest.raises(lbq.LbqError):  # K % 512 != 0
        lbq.lut3_mx_gemm(codes, scales, img, 128)
