"""Batch-1 INT4 GEMV on the TMA-fed warp-MMA kernel against the oracle.

Every K split the kernel plans (1, 2 or 4 K-ranges), FP16 and BF16
activations, symmetric and asymmetric codes at groups 32/64/128, ragged N,
several GEMVs per launch, determinism and the workspace contract (tile
counters back at zero after each call)."""

import numpy as np
import pytest

import workloads
from helpers import check_outputs, oracle_int4, sample_columns

pytestmark = pytest.mark.gpu

TMMA = 5


@pytest.fixture(scope="module")
def torch():
    import torch
    assert torch.cuda.is_available(), "these tests need a CUDA device"
    return torch


@pytest.fixture(scope="module")
def lbq():
    import bit_weight_only_pack_b200 as lbq
    return lbq


class tmma:
    """Route batch-1 GEMVs to the TMA-fed kernel, optionally with a forced K split."""

    def __init__(self, lbq, split=0):
        self.lbq, self.split = lbq, split

    def __enter__(self):
        self.lbq.lbq_debug_gemv_path(TMMA)
        self.lbq.lbq_debug_tmma_default(1)
        self.lbq.lbq_debug_tmma_split(self.split)

    def __exit__(self, *exc):
        self.lbq.lbq_debug_gemv_path(0)
        self.lbq.lbq_debug_tmma_default(-1)
        self.lbq.lbq_debug_tmma_split(0)


def _planted(W, group):
    K, N = W.shape
    if N >= 4 and K >= 2 * group:
        W[:group, 0] = 0.0
        W[group:2 * group, 1] = 0.37
        W[:group, 2] = np.abs(W[:group, 2]) + 0.01
        W[group:2 * group, 3] = -np.abs(W[group:2 * group, 3]) - 0.5
    return W


SHAPES = [
    (4096, 4096, 32, "asym"),    # o projection of the decode step
    (4096, 1024, 32, "asym"),    # k / v projection
    (4096, 4096, 32, "sym"),     # the single-GEMV workload
    (14336, 136, 32, "asym"),    # down projection, a ragged column slice
    (8192, 40, 128, "sym"),      # batch-sweep K, ragged N
    (16384, 24, 64, "asym"),     # longest K the kernel takes
    (256, 16, 32, "sym"),        # one slice, one row tile
    (768, 300, 64, "asym"),      # three slices: a K-range of 2 or 4 with empty slices
    (1280, 17, 128, "sym"),      # one row of a second row tile
]


@pytest.mark.parametrize("K,N,group,mode", SHAPES)
@pytest.mark.parametrize("xdt", ["f16", "bf16"])
@pytest.mark.parametrize("split", [0, 1, 2, 4])
def test_tmma_parity(torch, lbq, K, N, group, mode, xdt, split):
    if split and (K // 256 + split - 1) // split > 16:
        pytest.skip("a K-range holds at most 16 slices")
    if split > 1 and (split - 1) * ((K // 32 + 8 * split - 1) // (8 * split)) * 8 >= K // 32:
        pytest.skip("the split would leave a K-range empty")
    W = _planted(workloads.weights_host(300 + K + N, K, N), group)
    ref = oracle_int4(W, group, mode)
    img = lbq.pack(torch.from_numpy(W).cuda(), group, mode)
    X = workloads.activations_host(301 + K, 1, K, xdt)
    with tmma(lbq, split):
        ws = lbq.workspace(0, 1, K, N, group, mode)
        for ydt in ("f16", "bf16"):
            Y = lbq.gemv(X.cuda(), img, N, group, mode, y_dtype=ydt, ws=ws)
            torch.cuda.synchronize()
            check_outputs(Y.cpu(), X, ref["deq"])
        if ws is not None and split > 1:
            cnt_off = -(-split * N * 4 // 256) * 256
            assert int(ws[cnt_off:].count_nonzero()) == 0  # tile counters left at zero
    lbq.device_status()


@pytest.mark.parametrize("split", [1, 2, 4])
def test_tmma_deterministic_and_workspace_reusable(torch, lbq, split):
    K, N, group, mode = 4096, 2000, 32, "asym"
    W = workloads.weights_host(310, K, N)
    ref = oracle_int4(W, group, mode)
    img = lbq.pack(torch.from_numpy(W).cuda(), group, mode)
    X = workloads.activations_host(311, 1, K, "f16").cuda()
    with tmma(lbq, split):
        ws = lbq.workspace(0, 1, K, N, group, mode)
        assert (ws is None) == (split == 1)
        Ys = [lbq.gemv(X, img, N, group, mode, ws=ws) for _ in range(4)]
        torch.cuda.synchronize()
    lbq.device_status()
    for Y in Ys:
        check_outputs(Y.cpu(), X.cpu(), ref["deq"])
    assert all(torch.equal(Ys[0], Y) for Y in Ys[1:])


@pytest.mark.parametrize("shared_x", [True, False])
@pytest.mark.parametrize("xdt,mode,group", [("f16", "asym", 32), ("bf16", "sym", 128), ("f16", "sym", 64)])
def test_tmma_grouped(torch, lbq, shared_x, xdt, mode, group):
    """q/k/v-like widths (one ragged) in one launch: each output equals the
    single call with the same (unsplit) K range bit for bit, and the oracle."""
    K, Ns = 4096, (1024, 256, 72)
    Ws = [workloads.weights_host(320 + i, K, N) for i, N in enumerate(Ns)]
    refs = [oracle_int4(W, group, mode) for W in Ws]
    imgs = [lbq.pack(torch.from_numpy(W).cuda(), group, mode) for W in Ws]
    Xs = [workloads.activations_host(330 + (0 if shared_x else i), 1, K, xdt) for i in range(len(Ns))]
    Xd = [X.cuda() for X in Xs]
    with tmma(lbq, 1):
        Ys = lbq.gemv_grouped([(Xd[i], imgs[i], N) for i, N in enumerate(Ns)], group, mode)
        singles = [lbq.gemv(Xd[i], imgs[i], N, group, mode) for i, N in enumerate(Ns)]
        torch.cuda.synchronize()
    lbq.device_status()
    for i in range(len(Ns)):
        assert torch.equal(Ys[i], singles[i])
        check_outputs(Ys[i].cpu(), Xs[i], refs[i]["deq"])


def test_tmma_decode_layer_full_size(torch, lbq):
    """One layer of the decode step at full size through the kernel, grouped as
    in the step (q/k/v, o, gate/up, down), every column against the oracle."""
    proj = workloads.LLAMA3_8B_PROJ
    groups = ((0, 1, 2), (3,), (4, 5), (6,))
    with tmma(lbq):
        for grp in groups:
            K = proj[grp[0]][1]
            seed_x = workloads.c2_seed(0, grp[0])
            X = workloads.activations_host(seed_x, 1, K, "f16")
            Xd = X.cuda()
            items, refs = [], []
            for p in grp:
                _, Kp, N = proj[p]
                W = workloads.weights_host(workloads.c2_seed(0, p), Kp, N)
                refs.append(oracle_int4(W, 32, "asym")["deq"])
                items.append((Xd, lbq.pack(torch.from_numpy(W).cuda(), 32, "asym"), N))
                del W
            if len(items) > 1:
                Ys = lbq.gemv_grouped(items, 32, "asym")
            else:
                Ys = [lbq.gemv(Xd, items[0][1], items[0][2], 32, "asym")]
            torch.cuda.synchronize()
            for Y, deq in zip(Ys, refs):
                check_outputs(Y.cpu(), X, deq)
    lbq.device_status()


def test_tmma_pdl_graph(torch, lbq):
    """Back-to-back launches with programmatic dependent launch inside a CUDA
    graph, each reading the previous one's output as its activation."""
    K = N = 4096
    W = workloads.weights_host(340, K, N)
    ref = oracle_int4(W, 32, "sym")
    img = lbq.pack(torch.from_numpy(W).cuda(), 32, "sym")
    X0 = workloads.activations_host(341, 1, K, "f16").cuda()
    bufs = [X0] + [torch.empty((1, N), dtype=torch.float16, device="cuda") for _ in range(3)]
    with tmma(lbq):
        ws = [lbq.workspace(0, 1, K, N, 32, "sym") for _ in range(3)]
        lbq.lbq_set_option(lbq.LBQ_OPT_PDL, 1)
        try:
            s = torch.cuda.Stream()
            s.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(s):
                for i in range(3):
                    lbq.gemv(bufs[i], img, N, 32, "sym", ws=ws[i], Y=bufs[i + 1])
            torch.cuda.current_stream().wait_stream(s)
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                for i in range(3):
                    lbq.gemv(bufs[i], img, N, 32, "sym", ws=ws[i], Y=bufs[i + 1])
            for b in bufs[1:]:
                b.zero_()
            g.replay()
            torch.cuda.synchronize()
        finally:
            lbq.lbq_set_option(lbq.LBQ_OPT_PDL, 0)
    lbq.device_status()
    # each stage against the oracle applied to the previous stage's GPU output
    for i in range(3):
        check_outputs(bufs[i + 1].cpu(), bufs[i].cpu(), ref["deq"])


def test_tmma_large_sampled(torch, lbq):
    """K=8192, N=28672 sym g128 BF16 (the batch-sweep shape), sampled columns."""
    K, N, group = 8192, 28672, 128
    W = workloads.weights_host(3, K, N, outlier_frac=1e-3, outlier_mult=20.0)
    img = lbq.pack(torch.from_numpy(W).cuda(), group, "sym")
    cols = sample_columns(N, 384, seed=5)
    ref = oracle_int4(np.ascontiguousarray(W[:, cols]), group, "sym")
    del W
    X = workloads.activations_host(3, 1, K, "bf16")
    with tmma(lbq):
        Y = lbq.gemv(X.cuda(), img, N, group, "sym")
        torch.cuda.synchronize()
    lbq.device_status()
    check_outputs(Y.cpu(), X, ref["deq"], cols=cols)


def test_bounded_wait_runs_out_and_is_reported(torch, lbq):
    """Failure detection without a GPU fault: with the producer's copies
    withheld (test hook) on a one-CTA launch, every consumer wait gives up
    after a short spin limit, the kernel returns without writing Y, the device
    flag is reported as LBQ_ERR_DEVICE and cleared, and the next call on the
    same context passes parity."""
    K, N, group, mode = 1024, 16, 32, "sym"   # one row tile: a one-CTA grid
    W = workloads.weights_host(350, K, N)
    ref = oracle_int4(W, group, mode)
    img = lbq.pack(torch.from_numpy(W).cuda(), group, mode)
    X = workloads.activations_host(351, 1, K, "f16")
    sentinel = torch.full((1, N), 7.0, dtype=torch.float16, device="cuda")
    with tmma(lbq, 1):
        lbq.device_status()  # nothing pending
        lbq.lbq_debug_drop_copies(1)
        try:
            lbq.gemv(X.cuda(), img, N, group, mode, Y=sentinel)
            with pytest.raises(lbq.LbqError) as err:
                lbq.device_status()
            assert err.value.status == 4  # LBQ_ERR_DEVICE
        finally:
            lbq.lbq_debug_drop_copies(0)
        assert torch.equal(sentinel.cpu(), torch.full((1, N), 7.0, dtype=torch.float16))  # Y untouched
        lbq.device_status()  # the flag was cleared
        Y = lbq.gemv(X.cuda(), img, N, group, mode)
        torch.cuda.synchronize()
    lbq.device_status()
    check_outputs(Y.cpu(), X, ref["deq"])
