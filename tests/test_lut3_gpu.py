"""3-bit LUT parity on the GPU: the packed image's indices, codebooks and
exponents recovered bit-exactly, the decode exact against the oracle, and the
GEMV / GEMM outputs within |y - y_ref| <= 4e-3*S + ulp16(|y_ref|)."""

import numpy as np
import pytest

import workloads
from helpers import check_outputs, sample_columns
from oracle import lut3

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


def _inputs(seed, K, N):
    idx, cb, ex = workloads.lut3_host(seed, K, N)
    if K >= 128 and N >= 16:
        # planted edge cases: a tile whose codebook holds the E4M3 extremes
        # (+-448, +-smallest subnormal, +-0, +-1), every entry in use; a tile
        # whose indices are all 7; a tile with a tiny and one with a large
        # exponent (kept small enough that FP16 outputs stay finite)
        idx[:64, :8] = np.arange(64)[:, None] % 8
        cb[0, 0] = [0x7E, 0xFE, 0x01, 0x81, 0x00, 0x80, 0x38, 0xB8]
        idx[64:128, :8] = 7
        ex[1, 0] = 127 - 60
        ex[0, 1] = 127 + 4
    return idx, cb, ex


def _image(torch, lbq, idx, cb, ex):
    return lbq.pack_lut3(*(torch.from_numpy(np.ascontiguousarray(a)).cuda() for a in (idx, cb, ex)))


PACK_SHAPES = [
    (4096, 14336),   # the 3-bit LUT workload
    (64, 8),         # one tile
    (320, 200),      # K not a multiple of 256, N not a multiple of 128
    (1024, 136),
]


@pytest.mark.parametrize("K,N", PACK_SHAPES)
def test_pack_unpack_and_decode_bit_exact(torch, lbq, K, N):
    idx, cb, ex = _inputs(40 + K + N, K, N)
    img = _image(torch, lbq, idx, cb, ex)
    stream, cb_out, ex_out = lbq.unpack_lut3_canonical(img, K, N)
    if K * N > 1 << 22:  # full size: compare the canonical stream on a slice of tiles
        kt = slice(0, 4)
        assert np.array_equal(stream.cpu().numpy()[kt], lut3.pack_indices(idx[:256]))
        assert np.array_equal(lut3.unpack_indices(stream.cpu().numpy()), idx)
    else:
        assert np.array_equal(stream.cpu().numpy(), lut3.pack_indices(idx))
    assert np.array_equal(cb_out.cpu().numpy(), cb)
    assert np.array_equal(ex_out.cpu().numpy(), ex)
    cols = sample_columns(N // 8, 64, seed=K) if K * N > 1 << 22 else np.arange(N // 8)
    ch = (cols[:, None] * 8 + np.arange(8)[None, :]).reshape(-1)
    W = lbq.dequant(img, K, N, 0, "lut3").cpu().numpy()[:, ch]
    ref = lut3.dequant(idx[:, ch], cb[:, cols], ex[:, cols])
    assert np.array_equal(W.astype(np.float64), ref)
    _check_tables(torch, img, K, N, cb, ex)


def _check_tables(torch, img, K, N, cb, ex):
    """The image's per-tile decode tables (what the GEMV / GEMM kernels read):
    the tile's 8 weights e4m3(cb) * 2^(E-127) as BF16, low bytes then high bytes."""
    raw = img.cpu().numpy()
    off3 = int(raw[56:64].view(np.uint64)[0])
    T = raw[off3:off3 + (K // 64) * (N // 8) * 16].reshape(K // 64, N // 8, 16)
    got = T[..., :8].astype(np.uint16) | (T[..., 8:].astype(np.uint16) << 8)
    vals = lut3.E4M3_TABLE[cb] * np.ldexp(1.0, ex.astype(np.int64) - 127)[..., None]
    want = torch.from_numpy(vals.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(vals.astype(np.float32).astype(np.float64), vals)  # exact in FP32, hence in BF16
    assert np.array_equal(got, want)


def _check_gemm(torch, lbq, idx, cb, ex, img, X, groups=None, y_dtype=None):
    """Run lut3_gemm and check it against the oracle on the 8-channel groups given (all by default)."""
    K, N = idx.shape
    Y = lbq.lut3_gemm(X.cuda(), img, N, y_dtype=y_dtype)
    torch.cuda.synchronize()
    if groups is None:
        groups = np.arange(N // 8)
    ch = (groups[:, None] * 8 + np.arange(8)[None, :]).reshape(-1)
    deq = lut3.dequant(np.ascontiguousarray(idx[:, ch]), cb[:, groups], ex[:, groups])
    return check_outputs(Y.cpu(), X, deq, ch), Y


SKINNY_SHAPES = [
    (4096, 1024),    # whole 256-k stages, whole 128-channel tiles
    (320, 200),      # a 64-k tail stage, ragged last tile
    (64, 8),         # one tile
    (14336, 264),    # long K over few tiles: stream-K shares tiles between CTAs
]


@pytest.mark.parametrize("M", [1, 2, 3, 8, 9, 12, 16])
@pytest.mark.parametrize("K,N", SKINNY_SHAPES)
# 0: library's choice (the TMA-fed warp-MMA kernel at M = 1 for K <= 8192),
# 2: the skinny warp-MMA kernel
@pytest.mark.parametrize("path", [0, 2])
def test_lut3_gemv_parity(torch, lbq, M, K, N, path):
    idx, cb, ex = _inputs(70 + K + N, K, N)
    img = _image(torch, lbq, idx, cb, ex)
    X = workloads.activations_host(70 + M, M, K, "bf16")
    lbq.lbq_debug_gemv_path(path)
    try:
        for ydt in ("bf16", "f16"):
            _check_gemm(torch, lbq, idx, cb, ex, img, X, y_dtype=ydt)
    finally:
        lbq.lbq_debug_gemv_path(0)
    lbq.device_status()


@pytest.mark.parametrize("M", [17, 130, 300, 2500])  # 2500: a band of 8 token tiles and a ragged band of 2
@pytest.mark.parametrize("K,N", [(1024, 512), (320, 264), (4096, 1032)])
@pytest.mark.parametrize("path", [0, 1])  # 0: weights in tensor memory, 1: weights in shared memory
def test_lut3_gemm_parity(torch, lbq, M, K, N, path):
    idx, cb, ex = _inputs(90 + K + N, K, N)
    img = _image(torch, lbq, idx, cb, ex)
    X = workloads.activations_host(90 + M, M, K, "bf16")
    lbq.lbq_debug_gemm_path(path)
    try:
        _check_gemm(torch, lbq, idx, cb, ex, img, X, y_dtype="bf16")
    finally:
        lbq.lbq_debug_gemm_path(0)
    lbq.device_status()


@pytest.mark.parametrize("M", [1, 5, 16])
def test_lut3_tcgen05_kernel_at_decode_batch(torch, lbq, M):
    """The tcgen05 kernel itself at M <= 16 (normally routed to the GEMV)."""
    K, N = 1024, 264
    idx, cb, ex = _inputs(95, K, N)
    img = _image(torch, lbq, idx, cb, ex)
    X = workloads.activations_host(95 + M, M, K, "bf16")
    lbq.lbq_debug_force_tc(1)
    try:
        _check_gemm(torch, lbq, idx, cb, ex, img, X)
    finally:
        lbq.lbq_debug_force_tc(0)


@pytest.mark.parametrize("M,K,N", [(300, 1024, 10000), (1100, 1024, 4104)])
def test_lut3_gemm_stream_k(torch, lbq, M, K, N):
    """The LUT3 prefill with cut tiles (158 / 165 tiles on the SMs): against
    the oracle, identical over repeated calls on one workspace, flags reset."""
    idx, cb, ex = _inputs(98 + K + N, K, N)
    img = _image(torch, lbq, idx, cb, ex)
    X = workloads.activations_host(98 + M, M, K, "bf16").cuda()
    ws = lbq.workspace(2, M, K, N, 0, "lut3")
    assert ws is not None
    grid = lbq.lbq_debug_gemm_schedule(M, K, N, 1, 0)[0]
    Ys = [lbq.lut3_gemm(X, img, N, ws=ws) for _ in range(3)]
    torch.cuda.synchronize()
    lbq.device_status()
    assert all(torch.equal(Ys[0], Y) for Y in Ys[1:])
    assert int(ws[:grid * 4].view(torch.int32).abs().sum()) == 0
    ch = np.arange(N)
    check_outputs(Ys[0].cpu(), X.cpu(), lut3.dequant(idx, cb, ex), ch)


def test_lut3_repeat_calls_identical(torch, lbq):
    """Three calls on one workspace (shared tiles, so the counters must reset)."""
    K, N, M = 14336, 264, 4
    idx, cb, ex = _inputs(97, K, N)
    img = _image(torch, lbq, idx, cb, ex)
    X = workloads.activations_host(97, M, K, "bf16").cuda()
    ws = lbq.workspace(2, M, K, N, 0, "lut3")
    Ys = [lbq.lut3_gemm(X, img, N, ws=ws) for _ in range(3)]
    torch.cuda.synchronize()
    assert all(torch.equal(Ys[0], Y) for Y in Ys[1:])


@pytest.mark.parametrize("M", [1, 16, 2048])
def test_lut3_full_size_sampled(torch, lbq, M):
    """K=4096, N=14336 (the 3-bit LUT workload): every row, sampled 8-channel groups."""
    K, N = 4096, 14336
    idx, cb, ex = workloads.lut3_host(5, K, N)
    img = _image(torch, lbq, idx, cb, ex)
    X = workloads.activations_host(5 + M, M, K, "bf16")
    _check_gemm(torch, lbq, idx, cb, ex, img, X, groups=sample_columns(N // 8, 48, seed=M))


def test_lut3_rejects_fp16_activations(torch, lbq):
    K, N = 128, 16
    idx, cb, ex = _inputs(99, K, N)
    img = _image(torch, lbq, idx, cb, ex)
    X = workloads.activations_host(99, 1, K, "f16").cuda()
    with pytest.raises(lbq.LbqError):
        lbq.lut3_gemm(X, img, N)


@pytest.mark.parametrize("K,N", [(16384, 72), (16448, 40)])
def test_lut3_m1_direct_kernel_k_limit(torch, lbq, K, N):
    """Batch 1 at the longest K the direct LUT3 kernel takes (256 tiles) and
    one tile past it (the warp-MMA kernel), every channel."""
    idx, cb, ex = _inputs(60 + K, K, N)
    img = _image(torch, lbq, idx, cb, ex)
    X = workloads.activations_host(60 + K, 1, K, "bf16")
    for ydt in ("bf16", "f16"):
        _check_gemm(torch, lbq, idx, cb, ex, img, X, y_dtype=ydt)
    lbq.device_status()


M1_SHAPES = SKINNY_SHAPES + [
    (16384, 72),     # the direct kernel's longest K (the TMA kernel takes K <= 8192)
    (1024, 8),       # one codebook group: a one-CTA grid
    (8192, 40),      # the TMA kernel's longest K: 8 tiles per lane quad
    (4160, 16),      # past 4096: the two-group form with idle tiles in the last warp
    (4096, 14336),   # the 3-bit LUT workload: 13 groups on the busiest CTAs
]


@pytest.mark.parametrize("K,N", M1_SHAPES)
# (gemv path, ring stages): the library's choice; the TMA-fed kernel with a
# one-stage ring (every unit waits for the previous one's release) and with
# its longest ring; the register-pipelined direct kernel
@pytest.mark.parametrize("path,stages", [(0, 0), (0, 1), (0, 16), (4, 0)])
def test_lut3_m1_kernels(torch, lbq, K, N, path, stages):
    """Batch 1 on the TMA-fed warp-MMA kernel (the default for K <= 8192, at
    several ring lengths) and on the register-pipelined direct kernel, within
    the oracle's tolerance (full size: on sampled channels), and the same bits
    on a repeated call."""
    if K * N > 1 << 24:
        idx, cb, ex = workloads.lut3_host(5, K, N)
        cols = sample_columns(N, 96, seed=K)
    else:
        idx, cb, ex = _inputs(80 + K + N, K, N)
        cols = None
    img = _image(torch, lbq, idx, cb, ex)
    X = workloads.activations_host(80 + K, 1, K, "bf16")
    lbq.lbq_debug_gemv_path(path)
    lbq.lbq_debug_lut3_stages(stages)
    try:
        if cols is None:
            _, Y = _check_gemm(torch, lbq, idx, cb, ex, img, X)
        else:
            Y = lbq.lut3_gemm(X.cuda(), img, N)
            torch.cuda.synchronize()
            groups = np.unique(cols // 8)
            ch = (groups[:, None] * 8 + np.arange(8)[None, :]).reshape(-1)
            deq = lut3.dequant(np.ascontiguousarray(idx[:, ch]), cb[:, groups], ex[:, groups])
            check_outputs(Y.cpu(), X, deq, ch)
        Y0 = lbq.lut3_gemm(X.cuda(), img, N)
        torch.cuda.synchronize()
        assert torch.equal(Y, Y0)
    finally:
        lbq.lbq_debug_gemv_path(0)
        lbq.lbq_debug_lut3_stages(0)
    lbq.device_status()


# the batch-1 kernel; the batch kernel (16-row units, batch on the columns) with one and two blocks of 8 rows
@pytest.mark.parametrize("M", [1, 4, 16])
def test_lut3_m1_bounded_wait_runs_out_and_is_reported(torch, lbq, M):
    """Failure detection without a GPU fault on the TMA-fed LUT3 kernels: with
    the producer's copies withheld (test hook) on a one-CTA launch, every
    consumer wait gives up after a short spin limit (the batch kernel's warps
    keep their named-barrier sequence), Y is not written, the device flag reads
    LBQ_ERR_DEVICE and is cleared, and the next call passes parity."""
    K, N = 1024, 8
    idx, cb, ex = _inputs(360, K, N)
    img = _image(torch, lbq, idx, cb, ex)
    X = workloads.activations_host(361, M, K, "bf16")
    sentinel = torch.full((M, N), 7.0, dtype=torch.bfloat16, device="cuda")
    lbq.device_status()  # nothing pending
    lbq.lbq_debug_drop_copies(1)
    try:
        lbq.lut3_gemm(X.cuda(), img, N, Y=sentinel)
        with pytest.raises(lbq.LbqError) as err:
            lbq.device_status()
        assert err.value.status == 4  # LBQ_ERR_DEVICE
    finally:
        lbq.lbq_debug_drop_copies(0)
    assert torch.equal(sentinel.cpu(), torch.full((M, N), 7.0, dtype=torch.bfloat16))  # Y untouched
    lbq.device_status()  # the flag was cleared
    _check_gemm(torch, lbq, idx, cb, ex, img, X)
    lbq.device_status()


def test_tables_exact_at_the_exponent_range_ends(torch, lbq):
    """The BF16 decode tables hold every weight e4m3(b) * 2^(E-127) exactly for
    3 <= E <= 246 (E4M3 magnitudes run from 2^-9 to 448; BF16 from 2^-133 to
    just under 2^128): tiles at E = 3, 4, 245 and 246 with the E4M3 extremes
    in their codebooks decode bit-exactly, and the dequantised image equals the
    oracle's exact decode."""
    K, N = 256, 32
    idx, cb, ex = workloads.lut3_host(701, K, N)
    extremes = [0x7E, 0xFE, 0x01, 0x81, 0x00, 0x80, 0x08, 0xF8]  # +-448, +-2^-9, +-0, +-2^-6, -240
    for kt, e in enumerate((3, 4, 245, 246)):
        cb[kt, :] = extremes
        ex[kt, :] = e
        idx[64 * kt:64 * kt + 64, :] = np.arange(64)[:, None] % 8
    img = _image(torch, lbq, idx, cb, ex)
    _check_tables(torch, img, K, N, cb, ex)
    W = lbq.dequant(img, K, N, 0, "lut3").cpu().numpy()
    assert np.array_equal(W.astype(np.float64), lut3.dequant(idx, cb, ex))
    lbq.device_status()


@pytest.mark.parametrize("M", [1, 4, 16])  # the batch-1 kernel; the batch kernel (one and two row blocks)
def test_lut3_m1_pdl_graph(torch, lbq, M):
    """The TMA-fed LUT3 kernels with programmatic dependent launch inside a
    CUDA graph: three back-to-back launches, each reading the previous one's
    output as its activation (the weights stream before the wait, X only
    after it)."""
    K = N = 4096
    idx, cb, ex = workloads.lut3_host(342, K, N)
    img = _image(torch, lbq, idx, cb, ex)
    deq = lut3.dequant(idx, cb, ex)
    X0 = workloads.activations_host(343, M, K, "bf16").cuda()
    bufs = [X0] + [torch.empty((M, N), dtype=torch.bfloat16, device="cuda") for _ in range(3)]
    ws = lbq.workspace(2, M, K, N, 0, "lut3")
    lbq.lbq_set_option(lbq.LBQ_OPT_PDL, 1)
    try:
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            for i in range(3):
                lbq.lut3_gemm(bufs[i], img, N, ws=ws, Y=bufs[i + 1])
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(3):
                lbq.lut3_gemm(bufs[i], img, N, ws=ws, Y=bufs[i + 1])
        for b in bufs[1:]:
            b.zero_()
        g.replay()
        torch.cuda.synchronize()
    finally:
        lbq.lbq_set_option(lbq.LBQ_OPT_PDL, 0)
    lbq.device_status()
    # each stage against the oracle applied to the previous stage's GPU output
    for i in range(3):
        check_outputs(bufs[i + 1].cpu(), bufs[i].cpu(), deq)


@pytest.mark.parametrize("off", [0, 1])  # the TMA-fed batch kernel; the skinny kernel
@pytest.mark.parametrize("M", [4, 16])
def test_lut3_batch_full_size_sampled(torch, lbq, off, M):
    """The 3-bit LUT workload at batches 4 and 16 (K=4096, N=14336), sampled
    channel groups, on the batch kernel and on the skinny kernel."""
    K, N = 4096, 14336
    idx, cb, ex = workloads.lut3_host(5, K, N)
    img = _image(torch, lbq, idx, cb, ex)
    X = workloads.activations_host(344, M, K, "bf16")
    groups = np.unique(sample_columns(N, 96, seed=344) // 8)
    lbq.lbq_debug_lut3_batch_off(off)
    try:
        _check_gemm(torch, lbq, idx, cb, ex, img, X, groups=groups)
    finally:
        lbq.lbq_debug_lut3_batch_off(0)
    lbq.device_status()
