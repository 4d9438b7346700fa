"""lbq_gemv_noalloc: the GEMV with the library's fixed scratch instead of a
caller workspace. Called through the C ABI and compared, on two calls in a
row, with lbq_gemv (and with the oracle) under the parity tolerance
|y - y_ref| <= 4e-3*S + ulp16(|y_ref|). Collected last on purpose: it has to
pass after the other GPU tests as well as alone in a fresh process."""

import numpy as np
import pytest

import workloads
from helpers import check_outputs, oracle_int4
from oracle import matmul

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


def _noalloc(torch, lbq, X, img, N, group, mode):
    M, K = X.shape
    Y = torch.full((M, N), float("nan"), dtype=X.dtype, device=X.device)
    dt = lbq.DTYPES["bf16" if X.dtype == torch.bfloat16 else "f16"]
    lbq.lbq_gemv_noalloc(X.data_ptr(), dt, M, K, N, group, lbq.MODES[mode], img.data_ptr(), Y.data_ptr(), dt,
                         torch.cuda.current_stream().cuda_stream)
    return Y


# Ordered so that consecutive calls place their tile counters at different
# offsets of the one scratch array (over partial sums the call before left).
CASES = [
    # K, N, group, mode, M, x dtype, forced M=1 splits
    (14336, 4096, 32, "asym", 1, "f16", 4),   # M=1 split-K partials and counters
    (4096, 1024, 128, "sym", 4, "bf16", 0),   # tensor-core GEMV
    (14336, 264, 64, "asym", 16, "bf16", 0),  # stream-K: row tiles shared by many CTAs
    (4096, 4096, 32, "asym", 1, "f16", 3),
    (8192, 520, 32, "sym", 9, "f16", 0),
]


def test_noalloc_matches_gemv_twice_in_a_row(torch, lbq):
    for K, N, group, mode, M, xdt, splits in CASES:
        W = workloads.weights_host(800 + K + N, K, N)
        ref = oracle_int4(W, group, mode)
        img = lbq.pack(torch.from_numpy(W).cuda(), group, mode)
        X = workloads.activations_host(800 + M, M, K, xdt)
        Xd = X.cuda()
        lbq.lbq_debug_force_splits(splits)
        try:
            Y_ws = lbq.gemv(Xd, img, N, group, mode)
            Ys = [_noalloc(torch, lbq, Xd, img, N, group, mode) for _ in range(2)]
            torch.cuda.synchronize()
        finally:
            lbq.lbq_debug_force_splits(0)
        lbq.device_status()
        check_outputs(Y_ws.cpu(), X, ref["deq"])
        S = matmul.abs_scale(matmul.as_f64(X), ref["deq"])
        for Y in Ys:
            check_outputs(Y.cpu(), X, ref["deq"])
            ok, worst = matmul.check(matmul.as_f64(Y.cpu()), matmul.as_f64(Y_ws.cpu()), S)
            assert ok, f"{(K, N, M)}: differs from lbq_gemv by {worst:.3g} of the tolerance"


def test_noalloc_rejects_shapes_beyond_its_scratch(torch, lbq):
    """M=16 over a 128256-wide output needs about 16 MB of partial sums, twice
    the fixed 8 MiB: refused up front, nothing launched, Y untouched."""
    K, N, M = 4096, 128256, 16
    g = torch.Generator(device="cuda")
    g.manual_seed(7)
    W = torch.randn((K, N), generator=g, device="cuda") * 0.02
    img = lbq.pack(W, 128, "sym")
    del W
    X = workloads.activations_host(7, M, K, "bf16").cuda()
    Y = torch.zeros((M, N), dtype=torch.bfloat16, device="cuda")
    torch.cuda.synchronize()
    before = lbq.lbq_launch_count()
    with pytest.raises(lbq.LbqError) as err:
        lbq.lbq_gemv_noalloc(X.data_ptr(), lbq.DTYPES["bf16"], M, K, N, 128, lbq.MODES["sym"],
                             img.data_ptr(), Y.data_ptr(), lbq.DTYPES["bf16"], torch.cuda.current_stream().cuda_stream)
    assert "scratch" in str(err.value)
    assert lbq.lbq_launch_count() == before
    torch.cuda.synchronize()
    assert int(torch.count_nonzero(Y)) == 0
    assert np.isfinite(Y.float().cpu().numpy()).all()
