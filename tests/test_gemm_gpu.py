"""Prefill GEMM (tcgen05) parity on the GPU: outputs within
|y - y_ref| <= 4e-3*S + ulp16(|y_ref|) of the oracle's FP64 product."""

import numpy as np
import pytest

import workloads
from helpers import check_outputs, oracle_int4, sample_columns

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


GEMM_SHAPES = [
    # M, K, N, group, mode, x dtype
    (128, 256, 256, 128, "asym", "bf16"),      # one tile
    (300, 1024, 520, 128, "asym", "bf16"),     # ragged M and N
    (17, 512, 264, 64, "sym", "f16"),          # N % 256 != 0, smallest M routed to the GEMM
    (256, 4096, 512, 128, "asym", "bf16"),     # the prefill K, two N tiles
    (130, 96, 36, 32, "asym", "f16"),          # K < one k-block, N % 8 != 0
    (384, 2048, 768, 32, "sym", "bf16"),
    (2500, 256, 520, 128, "asym", "bf16"),    # 10 token tiles: a full band of 8 and a ragged band of 2
]


@pytest.mark.parametrize("M,K,N,group,mode,xdt", GEMM_SHAPES)
@pytest.mark.parametrize("path", [0, 1])  # 0: weights in tensor memory, 1: weights in shared memory
def test_gemm_parity(torch, lbq, M, K, N, group, mode, xdt, path):
    W = workloads.weights_host(500 + K + N, K, N)
    ref = oracle_int4(W, group, mode)
    img = lbq.pack(torch.from_numpy(W).cuda(), group, mode)
    X = workloads.activations_host(500 + M, M, K, xdt)
    lbq.lbq_debug_gemm_path(path)
    try:
        for ydt in ("bf16", "f16"):
            Y = lbq.gemm(X.cuda(), img, N, group, mode, y_dtype=ydt)
            torch.cuda.synchronize()
            check_outputs(Y.cpu(), X, ref["deq"])
    finally:
        lbq.lbq_debug_gemm_path(0)
    lbq.device_status()


@pytest.mark.parametrize("M", [1, 5, 16])
def test_gemm_kernel_at_decode_batch(torch, lbq, M):
    """The tcgen05 kernel itself at M <= 16 (normally routed to the GEMV)."""
    K, N = 1024, 512
    W = workloads.weights_host(600, K, N)
    ref = oracle_int4(W, 128, "asym")
    img = lbq.pack(torch.from_numpy(W).cuda(), 128, "asym")
    X = workloads.activations_host(600 + M, M, K, "bf16")
    lbq.lbq_debug_force_tc(1)
    try:
        Y = lbq.gemm(X.cuda(), img, N, 128, "asym")
        torch.cuda.synchronize()
    finally:
        lbq.lbq_debug_force_tc(0)
    check_outputs(Y.cpu(), X, ref["deq"])


def test_gemm_is_deterministic(torch, lbq):
    K, N, M = 2048, 768, 640
    W = workloads.weights_host(700, K, N)
    img = lbq.pack(torch.from_numpy(W).cuda(), 128, "asym")
    X = workloads.activations_host(700, M, K, "bf16").cuda()
    Ys = [lbq.gemm(X, img, N, 128, "asym") for _ in range(3)]
    torch.cuda.synchronize()
    assert all(torch.equal(Ys[0], Y) for Y in Ys[1:])


@pytest.mark.parametrize("M", [512, 2048, 8192])
def test_prefill_full_size_sampled(torch, lbq, M):
    """K=4096, N=14336, asymmetric group 128, BF16 X and Y: every row, sampled columns."""
    K, N = 4096, 14336
    W = workloads.weights_host(4, K, N)
    img = lbq.pack(torch.from_numpy(W).cuda(), 128, "asym")
    cols = sample_columns(N, 256, seed=M)
    ref = oracle_int4(np.ascontiguousarray(W[:, cols]), 128, "asym")
    X = workloads.activations_host(4, M, K, "bf16")
    Y = lbq.gemm(X.cuda(), img, N, 128, "asym", y_dtype="bf16")
    torch.cuda.synchronize()
    check_outputs(Y.cpu(), X, ref["deq"], cols)


SK_SHAPES = [
    # more tiles than SMs with a part-filled last wave: the prefill cuts tiles (stream-K)
    (300, 1024, 10000, 128, "asym", "bf16"),   # 158 tiles, ragged M and N, 8 k-blocks
    (520, 2048, 9000, 64, "sym", "f16"),       # 213 tiles, 16 k-blocks
    (700, 1056, 5000, 32, "asym", "bf16"),     # 120 tiles (no cut) ... and K ending inside a block
    (1100, 1056, 4100, 32, "sym", "bf16"),     # 165 tiles, 9 k-blocks (the last part-filled), N % 8 != 0
]


@pytest.mark.parametrize("M,K,N,group,mode,xdt", SK_SHAPES)
def test_gemm_stream_k_parity(torch, lbq, M, K, N, group, mode, xdt):
    """With the workspace the last waves' tiles are cut by k-block; both
    schedules match the oracle, repeated calls on one workspace are identical
    and every flag is back at zero after each call."""
    W = workloads.weights_host(800 + K + N, K, N)
    ref = oracle_int4(W, group, mode)
    img = lbq.pack(torch.from_numpy(W).cuda(), group, mode)
    X = workloads.activations_host(800 + M, M, K, xdt).cuda()
    ws = lbq.workspace(1, M, K, N, group, mode)
    grid = lbq.lbq_debug_gemm_schedule(M, K, N, 1, 0)[0]
    cut = ws is not None
    assert cut == ((M, N) != (700, 5000))
    Ys = [lbq.gemm(X, img, N, group, mode, ws=ws) for _ in range(3)]
    torch.cuda.synchronize()
    lbq.device_status()
    assert all(torch.equal(Ys[0], Y) for Y in Ys[1:])
    if cut:
        assert int(ws[:grid * 4].view(torch.int32).abs().sum()) == 0
    check_outputs(Ys[0].cpu(), X.cpu(), ref["deq"])
    lbq.lbq_debug_gemm_stream_k(0)
    try:
        Y0 = lbq.gemm(X, img, N, group, mode, ws=ws)
        torch.cuda.synchronize()
    finally:
        lbq.lbq_debug_gemm_stream_k(1)
    check_outputs(Y0.cpu(), X.cpu(), ref["deq"])


def test_gemm_stream_k_wait_runs_out_and_is_reported(torch, lbq):
    """Failure detection without a GPU fault: with the later parts' flags
    withheld (test hook), every earlier part's wait gives up after a short
    bound, its tile is not written, the device flag is reported as
    LBQ_ERR_DEVICE, and the next call on the same workspace passes parity."""
    M, K, N, group, mode = 300, 1024, 10000, 128, "asym"
    W = workloads.weights_host(810, K, N)
    ref = oracle_int4(W, group, mode)
    img = lbq.pack(torch.from_numpy(W).cuda(), group, mode)
    X = workloads.activations_host(811, M, K, "bf16").cuda()
    ws = lbq.workspace(1, M, K, N, group, mode)
    assert ws is not None
    lbq.device_status()  # nothing pending
    lbq.lbq_debug_gemm_hold(2000)
    try:
        lbq.gemm(X, img, N, group, mode, ws=ws)
        with pytest.raises(lbq.LbqError) as err:
            lbq.device_status()
        assert err.value.status == 4  # LBQ_ERR_DEVICE
    finally:
        lbq.lbq_debug_gemm_hold(0)
    lbq.device_status()  # the flag was cleared by the report
    Y = lbq.gemm(X, img, N, group, mode, ws=ws)
    torch.cuda.synchronize()
    lbq.device_status()
    check_outputs(Y.cpu(), X.cpu(), ref["deq"])
