"""INT4 parity on the GPU: packing and dequantisation bit-exact against the
oracle, GEMV outputs within |y - y_ref| <= 4e-3*S + ulp16(|y_ref|)."""

import numpy as np
import pytest

import workloads
from helpers import check_outputs, oracle_int4, sample_columns
from oracle import int4

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


def _special_groups(W, group):
    """Plant the degenerate and one-sided groups the quantiser has to handle."""
    K, N = W.shape
    if N >= 4 and K >= 2 * group:
        W[:group, 0] = 0.0                                   # all-zero group
        W[group:2 * group, 1] = 0.37                         # constant group
        W[:group, 2] = np.abs(W[:group, 2]) + 0.01           # all-positive group
        W[group:2 * group, 3] = -np.abs(W[group:2 * group, 3]) - 0.5  # all-negative, far from 0
    return W


def _pack_and_compare(torch, lbq, W, group, mode):
    K, N = W.shape
    ref = oracle_int4(W, group, mode)
    img = lbq.pack(torch.from_numpy(W).cuda(), group, mode)
    q, s, z = lbq.unpack_canonical(img, K, N, group, mode)
    assert np.array_equal(q.cpu().numpy(), ref["packed"])
    assert np.array_equal(s.cpu().view(torch.int16).numpy(), ref["s"].view(np.int16))
    if mode == "asym":
        assert np.array_equal(z.cpu().numpy(), ref["zp"])
    deq = lbq.dequant(img, K, N, group, mode).cpu().numpy()
    assert np.array_equal(deq.astype(np.float64), ref["deq"])
    return img, ref


SHAPES = [
    (4096, 4096, 32, "sym"),     # the single-GEMV workload
    (4096, 1024, 32, "asym"),    # k/v projection of the decode step
    (14336, 64, 32, "asym"),     # down projection, a column slice
    (96, 40, 32, "asym"),        # three chunks, ragged N
    (128, 8, 64, "sym"),
    (256, 24, 128, "asym"),
    (32, 1, 32, "sym"),          # one chunk, one column
]


@pytest.mark.parametrize("K,N,group,mode", SHAPES)
def test_pack_and_dequant_bit_exact(torch, lbq, K, N, group, mode):
    W = _special_groups(workloads.weights_host(11 + K + N, K, N), group)
    _pack_and_compare(torch, lbq, W, group, mode)


def test_pack_outliers_bit_exact(torch, lbq):
    W = workloads.weights_host(3, 1024, 512, outlier_frac=1e-3, outlier_mult=20.0)
    for group in (64, 128):
        _pack_and_compare(torch, lbq, W, group, "sym")


PATHS = {"auto": 0, "cudacore_m1": 1, "warp_mma": 2, "tcgen05": 3, "direct_m1": 4}


class gemv_path:
    """Route lbq_gemv to one kernel for the duration of a block (test hook)."""

    def __init__(self, lbq, name):
        self.lbq, self.path = lbq, PATHS[name]

    def __enter__(self):
        self.lbq.lbq_debug_gemv_path(self.path)

    def __exit__(self, *exc):
        self.lbq.lbq_debug_gemv_path(0)


@pytest.mark.parametrize("K,N,group,mode", SHAPES)
@pytest.mark.parametrize("xdt", ["f16", "bf16"])
@pytest.mark.parametrize("path", ["auto", "cudacore_m1", "warp_mma", "tcgen05"])
def test_gemv_m1_parity(torch, lbq, K, N, group, mode, xdt, path):
    W = _special_groups(workloads.weights_host(11 + K + N, K, N), group)
    img, ref = _pack_and_compare(torch, lbq, W, group, mode)
    X = workloads.activations_host(5 + K, 1, K, xdt)
    with gemv_path(lbq, path):
        for ydt in ("f16", "bf16"):
            Y = lbq.gemv(X.cuda(), img, N, group, mode, y_dtype=ydt)
            torch.cuda.synchronize()
            check_outputs(Y.cpu(), X, ref["deq"])
    lbq.device_status()


@pytest.mark.parametrize("splits", [2, 3, 4, 7])
def test_gemv_m1_forced_split_k(torch, lbq, splits):
    K, N, group, mode = 14336, 1000, 32, "asym"   # K-slices start on 2048-k boundaries
    W = workloads.weights_host(77, K, N)
    img, ref = _pack_and_compare(torch, lbq, W, group, mode)
    X = workloads.activations_host(77, 1, K, "f16")
    lbq.lbq_debug_force_splits(splits)
    try:
        ws = lbq.workspace(0, 1, K, N, group, mode)
        assert ws is not None and int(ws.count_nonzero()) == 0
        Ys = [lbq.gemv(X.cuda(), img, N, group, mode, ws=ws) for _ in range(3)]
        torch.cuda.synchronize()
        counters_at = -(-splits * N * 4 // 256) * 256
        assert int(ws[counters_at:].count_nonzero()) == 0  # tile counters left zeroed
        for Y in Ys:
            check_outputs(Y.cpu(), X, ref["deq"])
        assert all(torch.equal(Ys[0], Y) for Y in Ys[1:])  # deterministic, workspace reusable
    finally:
        lbq.lbq_debug_force_splits(0)


def test_decode_step_layer_shapes(torch, lbq):
    """One Llama-3-8B-shaped layer of the decode step, full size, every column."""
    for p, (name, K, N) in enumerate(workloads.LLAMA3_8B_PROJ):
        seed = workloads.c2_seed(0, p)
        W = workloads.weights_host(seed, K, N)
        ref = oracle_int4(W, 32, "asym")
        img = lbq.pack(torch.from_numpy(W).cuda(), 32, "asym")
        X = workloads.activations_host(seed, 1, K, "f16")
        Y = lbq.gemv(X.cuda(), img, N, 32, "asym")
        torch.cuda.synchronize()
        check_outputs(Y.cpu(), X, ref["deq"])


@pytest.mark.parametrize("group", [64, 128])
def test_batch_sweep_full_size_sampled(torch, lbq, group):
    """K=8192, N=28672 with 0.1% x20 outliers, BF16 X, M in {1,2,4,8,16}; outputs
    checked on sampled columns, codes on the same columns bit-exactly."""
    K, N = 8192, 28672
    W = workloads.weights_host(3, K, N, outlier_frac=1e-3, outlier_mult=20.0)
    Wd = torch.from_numpy(W).cuda()
    img = lbq.pack(Wd, group, "sym")
    del Wd
    cols = sample_columns(N, 384, seed=group)
    ref = oracle_int4(np.ascontiguousarray(W[:, cols]), group, "sym")
    q, s, _ = lbq.unpack_canonical(img, K, N, group, "sym")
    assert np.array_equal(q.cpu().numpy()[:, cols], ref["packed"])
    assert np.array_equal(s.cpu().view(torch.int16).numpy()[:, cols], ref["s"].view(np.int16))
    for M in (1, 2, 4, 8, 16):
        X = workloads.activations_host(3, M, K, "bf16")
        Y = lbq.gemv(X.cuda(), img, N, group, "sym")
        torch.cuda.synchronize()
        check_outputs(Y.cpu(), X, ref["deq"], cols)


def test_large_activation_magnitudes(torch, lbq):
    K, N = 2048, 256
    W = workloads.weights_host(5, K, N)
    ref = oracle_int4(W, 32, "asym")
    img = lbq.pack(torch.from_numpy(W).cuda(), 32, "asym")
    X = (workloads.activations_host(5, 1, K, "f16").float() * 100).half()
    Y = lbq.gemv(X.cuda(), img, N, 32, "asym")
    torch.cuda.synchronize()
    check_outputs(Y.cpu(), X, ref["deq"])


def test_wrong_header_is_reported_by_debug_calls(torch, lbq):
    W = workloads.weights_host(1, 64, 8)
    img = lbq.pack(torch.from_numpy(W).cuda(), 32, "sym")
    with pytest.raises(lbq.LbqError):
        lbq.unpack_canonical(img, 64, 16, 32, "sym")   # N does not match the image
    with pytest.raises(lbq.LbqError):
        lbq.dequant(img, 64, 8, 32, "asym")             # mode does not match


def test_pdl_back_to_back_graph(torch, lbq):
    """Programmatic dependent launch: a graph of GEMVs where each X is the
    previous GEMV's output (a real dependency), results equal to the oracle."""
    K = N = 1024
    Ws = [workloads.weights_host(40 + i, K, N) for i in range(4)]
    refs = [oracle_int4(W, 64, "sym") for W in Ws]
    imgs = [lbq.pack(torch.from_numpy(W).cuda(), 64, "sym") for W in Ws]
    X0 = workloads.activations_host(40, 1, K, "f16").cuda()
    lbq.lbq_set_option(lbq.LBQ_OPT_PDL, 1)
    try:
        bufs = [X0] + [torch.empty((1, N), dtype=torch.float16, device="cuda") for _ in imgs]
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            for i, img in enumerate(imgs):
                lbq.gemv(bufs[i], img, N, 64, "sym", Y=bufs[i + 1])
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        eager = [b.clone() for b in bufs[1:]]
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i, img in enumerate(imgs):
                lbq.gemv(bufs[i], img, N, 64, "sym", Y=bufs[i + 1])
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        lbq.device_status()
    finally:
        lbq.lbq_set_option(lbq.LBQ_OPT_PDL, 0)
    for i in range(len(imgs)):
        assert torch.equal(eager[i], bufs[i + 1])
        check_outputs(bufs[i + 1].cpu(), bufs[i].cpu(), refs[i]["deq"])


SKINNY_SHAPES = [
    (4096, 1000, 32, "asym", "f16"),
    (512, 72, 64, "sym", "bf16"),
    (1024, 130, 128, "asym", "bf16"),
    (96, 40, 32, "sym", "f16"),       # K below one 256-k stage, ragged N
    (8320, 64, 128, "sym", "f16"),    # K not a multiple of 256
]


@pytest.mark.parametrize("M", [2, 3, 8, 9, 16])
@pytest.mark.parametrize("K,N,group,mode,xdt", SKINNY_SHAPES)
@pytest.mark.parametrize("path", ["auto", "tcgen05"])
def test_skinny_parity(torch, lbq, M, K, N, group, mode, xdt, path):
    W = _special_groups(workloads.weights_host(300 + K + N, K, N), group)
    ref = oracle_int4(W, group, mode)
    img = lbq.pack(torch.from_numpy(W).cuda(), group, mode)
    X = workloads.activations_host(300 + M, M, K, xdt)
    with gemv_path(lbq, path):
        for ydt in ("f16", "bf16"):
            Y = lbq.gemv(X.cuda(), img, N, group, mode, y_dtype=ydt)
            torch.cuda.synchronize()
            check_outputs(Y.cpu(), X, ref["deq"])
    lbq.device_status()


@pytest.mark.parametrize("K,N,M", [(4096, 520, 5), (14336, 1000, 16), (8192, 128, 3), (14336, 264, 1)])
@pytest.mark.parametrize("path", ["warp_mma", "tcgen05"])
def test_skinny_stream_k_shared_tiles(torch, lbq, K, N, M, path):
    """Few row tiles over many CTAs: row tiles are shared between CTAs and
    finished by the last one; three calls on one workspace give identical,
    correct results (so the tile counters are reset after every call)."""
    W = workloads.weights_host(91 + K, K, N)
    ref = oracle_int4(W, 64, "asym")
    img = lbq.pack(torch.from_numpy(W).cuda(), 64, "asym")
    X = workloads.activations_host(91, M, K, "bf16")
    with gemv_path(lbq, path):
        ws = lbq.workspace(0, M, K, N, 64, "asym")
        assert ws is not None
        Ys = [lbq.gemv(X.cuda(), img, N, 64, "asym", ws=ws) for _ in range(3)]
        torch.cuda.synchronize()
    lbq.device_status()
    for Y in Ys:
        check_outputs(Y.cpu(), X, ref["deq"])
    assert all(torch.equal(Ys[0], Y) for Y in Ys[1:])


def test_m1_through_the_skinny_kernel(torch, lbq):
    K, N = 4096, 1024
    W = workloads.weights_host(93, K, N)
    ref = oracle_int4(W, 32, "asym")
    img = lbq.pack(torch.from_numpy(W).cuda(), 32, "asym")
    X = workloads.activations_host(93, 1, K, "f16")
    lbq.lbq_debug_force_skinny(1)
    try:
        Y = lbq.gemv(X.cuda(), img, N, 32, "asym")
        torch.cuda.synchronize()
    finally:
        lbq.lbq_debug_force_skinny(0)
    check_outputs(Y.cpu(), X, ref["deq"])


@pytest.mark.parametrize("shared_x", [True, False])
@pytest.mark.parametrize("xdt,mode,group", [("f16", "asym", 32), ("bf16", "sym", 128)])
def test_gemv_grouped_matches_single_calls(torch, lbq, shared_x, xdt, mode, group):
    """Three GEMVs in one launch (q/k/v-like widths, one ragged): each output
    equals the single-GEMV output bit for bit and passes the oracle check."""
    K, Ns = 1024, (512, 128, 72)
    Ws = [workloads.weights_host(950 + i, K, N) for i, N in enumerate(Ns)]
    refs = [oracle_int4(W, group, mode) for W in Ws]
    imgs = [lbq.pack(torch.from_numpy(W).cuda(), group, mode) for W in Ws]
    Xs = [workloads.activations_host(960 + (0 if shared_x else i), 1, K, xdt) for i in range(len(Ns))]
    Xd = [X.cuda() for X in Xs]
    Ys = lbq.gemv_grouped([(Xd[i], imgs[i], N) for i, N in enumerate(Ns)], group, mode)
    singles = [lbq.gemv(Xd[i], imgs[i], N, group, mode) for i, N in enumerate(Ns)]
    torch.cuda.synchronize()
    lbq.device_status()
    for i in range(len(Ns)):
        assert torch.equal(Ys[i], singles[i])
        check_outputs(Ys[i].cpu(), Xs[i], refs[i]["deq"])


def test_gemv_grouped_rejects_bad_groups(torch, lbq):
    W = workloads.weights_host(970, 256, 64)
    img = lbq.pack(torch.from_numpy(W).cuda(), 32, "sym")
    X = workloads.activations_host(970, 1, 256, "f16").cuda()
    with pytest.raises(lbq.LbqError):
        lbq.gemv_grouped([(X, img, 64)] * 5, 32, "sym")   # more than 4 items
    Y = torch.empty((1, 64), dtype=torch.float16, device="cuda")
    items = lbq.make_gemv_items([(X.data_ptr(), img.data_ptr(), Y.data_ptr(), 64)])
    with pytest.raises(lbq.LbqError):
        lbq.lbq_gemv_grouped(items, 1, 32768, 32, 0, 0, 0, None)  # K beyond the direct kernel


@pytest.mark.parametrize("K,N,group,mode", [
    (16384, 9, 32, "sym"),       # the longest K the direct kernel takes, one partial row block
    (16416, 200, 32, "asym"),    # one chunk past it: the TMA batch-1 kernel
    (28672, 136, 128, "asym"),   # long K (a 70B-class down projection), ragged N
    (4096, 3, 128, "asym"),      # fewer columns than one row block
])
@pytest.mark.parametrize("xdt", ["f16", "bf16"])
def test_m1_dispatch_boundaries(torch, lbq, K, N, group, mode, xdt):
    """Batch 1 through the library's own kernel choice on both sides of the
    K limit of the direct kernel, every column."""
    W = _special_groups(workloads.weights_host(90 + K + N, K, N), group)
    img, ref = _pack_and_compare(torch, lbq, W, group, mode)
    X = workloads.activations_host(90 + K, 1, K, xdt)
    for ydt in ("f16", "bf16"):
        Y = lbq.gemv(X.cuda(), img, N, group, mode, y_dtype=ydt)
        torch.cuda.synchronize()
        check_outputs(Y.cpu(), X, ref["deq"])
    lbq.device_status()


def test_m1_long_k_many_weights_sampled(torch, lbq):
    """K=16512, N=8200: past the direct kernel's K limit and over 2^27 weights,
    where batch 1 goes to the warp-MMA kernel; sampled columns."""
    K, N, group = 16512, 8200, 128
    W = workloads.weights_host(31, K, N)
    Wd = torch.from_numpy(W).cuda()
    img = lbq.pack(Wd, group, "asym")
    del Wd
    cols = sample_columns(N, 256, seed=31)
    ref = oracle_int4(np.ascontiguousarray(W[:, cols]), group, "asym")
    del W
    X = workloads.activations_host(31, 1, K, "bf16")
    Y = lbq.gemv(X.cuda(), img, N, group, "asym")
    torch.cuda.synchronize()
    check_outputs(Y.cpu(), X, ref["deq"], cols)
    lbq.device_status()


class direct_variant:
    """Route the batch-1 direct GEMV to one of its variants for a block (test hook):
    0 = weights pipelined through registers; 2..4 = that many row blocks
    staged through shared memory."""

    def __init__(self, lbq, variant):
        self.lbq, self.variant = lbq, variant

    def __enter__(self):
        self.lbq.lbq_debug_direct_variant(self.variant, 0)

    def __exit__(self, *exc):
        self.lbq.lbq_debug_direct_variant(-1, 0)


@pytest.mark.parametrize("K,N,group,mode", SHAPES + [(14336, 136, 128, "asym"), (16384, 40, 64, "sym"),
                                                     (1056, 24, 32, "asym"), (2080, 17, 32, "sym")])
@pytest.mark.parametrize("xdt", ["f16", "bf16"])
@pytest.mark.parametrize("variant", [0, 2, 3, 4])
def test_gemv_m1_direct_variants(torch, lbq, K, N, group, mode, xdt, variant):
    W = _special_groups(workloads.weights_host(11 + K + N, K, N), group)
    img, ref = _pack_and_compare(torch, lbq, W, group, mode)
    X = workloads.activations_host(5 + K, 1, K, xdt)
    with gemv_path(lbq, "direct_m1"), direct_variant(lbq, variant):
        for ydt in ("f16", "bf16"):
            Y = lbq.gemv(X.cuda(), img, N, group, mode, y_dtype=ydt)
            torch.cuda.synchronize()
            check_outputs(Y.cpu(), X, ref["deq"])
    lbq.device_status()


@pytest.mark.parametrize("variant", [0, 2, 3, 4])
@pytest.mark.parametrize("shared_x", [True, False])
def test_gemv_grouped_direct_variants(torch, lbq, variant, shared_x):
    """Grouped launches (distinct or shared X) on each direct-kernel variant
    match single calls on the same variant bit for bit, and the oracle."""
    K, group, mode = 4096, 32, "asym"
    Ns = (4096, 1024, 1000)
    imgs, refs = [], []
    for i, N in enumerate(Ns):
        W = workloads.weights_host(200 + i, K, N)
        img, ref = _pack_and_compare(torch, lbq, W, group, mode)
        imgs.append(img)
        refs.append(ref)
    Xs = [workloads.activations_host(300 + (0 if shared_x else i), 1, K, "f16") for i in range(len(Ns))]
    Xd = [Xs[0].cuda()] * len(Ns) if shared_x else [X.cuda() for X in Xs]  # shared: one device vector
    with direct_variant(lbq, variant):
        singles = [lbq.gemv(X, img, N, group, mode) for X, img, N in zip(Xd, imgs, Ns)]
        grouped = lbq.gemv_grouped([(X, img, N) for X, img, N in zip(Xd, imgs, Ns)], group, mode)
        torch.cuda.synchronize()
    for Ys, Yg, X, ref in zip(singles, grouped, Xs, refs):
        assert torch.equal(Ys, Yg)
        check_outputs(Yg.cpu(), X, ref["deq"])
    lbq.device_status()
