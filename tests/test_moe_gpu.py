"""Grouped MoE GEMM of LUT3 experts with MXFP8 activations on the GPU.

The device alignment is checked against ``oracle.moe.align`` (what is unique:
the total, the experts of the blocks, each expert's set of pairs and where the
padding sits; the order of pairs inside an expert's run is free). The GEMM's
output rows are checked against the oracle's pair-by-pair routing definition
(``oracle.moe.routed_matmul``), within |y - y_ref| <= 4e-3*S + ulp16(|y_ref|)."""

import numpy as np
import pytest

import workloads
from oracle import lut3, matmul, moe, mxfp8

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


def _routing(seed, T, top_k, E):
    """Each token picks top_k distinct experts (seeded)."""
    rng = np.random.default_rng(seed)
    return np.stack([rng.choice(E, size=top_k, replace=False) for _ in range(T)]).astype(np.int32)


def _check_align(torch, lbq, ids, E, emap=None, block=128):
    P = ids.size
    s, e, t = lbq.moe_align(torch.from_numpy(ids).cuda(), E,
                            torch.from_numpy(emap).cuda() if emap is not None else None, block)
    torch.cuda.synchronize()
    s, e, total = s.cpu().numpy(), e.cpu().numpy(), int(t.item())
    rs, re, rtotal = moe.align(ids, E, block)
    assert total == rtotal and s.size == moe.max_padded(P, E, block)
    mapped = re if emap is None else emap[re]
    assert np.array_equal(e[:total // block], mapped) and np.all(e[total // block:] == -1)
    assert np.all(s[total:] == P)
    b = 0
    while b < total // block:  # one expert's run at a time
        b1 = b
        while b1 < total // block and re[b1] == re[b]:
            b1 += 1
        run, rrun = s[b * block:b1 * block], rs[b * block:b1 * block]
        n = int(np.sum(rrun < P))
        assert sorted(run[:n].tolist()) == rrun[:n].tolist()  # the expert's pairs, padding after them
        assert np.all(run[n:] == P)
        b = b1
    return s, e, total


# the last two: more experts than the kernel's 1024 threads (each thread scans a range of experts)
@pytest.mark.parametrize("T,top_k,E", [(1, 8, 256), (16, 8, 256), (256, 8, 64), (37, 2, 8), (300, 1, 3),
                                       (300, 4, 1500), (5, 2, 2048)])
def test_align_matches_the_oracle(torch, lbq, T, top_k, E):
    _check_align(torch, lbq, _routing(70 + T, T, top_k, E), E)


def test_align_with_expert_map_and_small_block(torch, lbq):
    ids = _routing(71, 50, 4, 12)
    emap = np.array([0, -1, 1, 2, -1, 3, 4, 5, -1, 6, 7, 8], dtype=np.int32)
    _check_align(torch, lbq, ids, 12, emap)
    _check_align(torch, lbq, ids, 12, None, block=16)


def _experts(seed, E, K, N):
    return [workloads.lut3_host(seed + i, K, N) for i in range(E)]


def _run_case(torch, lbq, T, top_k, E, K, N, ydt="bf16", emap=None, seed=80):
    ids = _routing(seed, T, top_k, E)
    codes, scales = workloads.mx_activations_host(seed + 1, T, K)
    experts = _experts(seed + 2, E, K, N)
    local = experts if emap is None else [experts[i] for i in range(E) if emap[i] >= 0]
    dev = [tuple(torch.from_numpy(a).cuda() for a in ex) for ex in local]
    images, stride = lbq.pack_lut3_experts(dev)
    aligned = lbq.moe_align(torch.from_numpy(ids).cuda(), E, torch.from_numpy(emap).cuda() if emap is not None else None)
    Y = lbq.moe_lut3_mx_gemm(torch.from_numpy(codes).cuda(), torch.from_numpy(scales).cuda(), top_k, aligned, images,
                             stride, len(local), N, y_dtype=ydt)
    torch.cuda.synchronize()
    lbq.device_status()
    # oracle: the pair-by-pair routing definition, and the size of each row's terms
    lmap = None
    if emap is not None:
        lmap = np.full(E, -1)
        lmap[emap >= 0] = np.arange(int(np.sum(emap >= 0)))
    y_ref = moe.routed_matmul(codes, scales, ids, local, lmap)
    Xq = np.abs(mxfp8.dequant(codes, scales))
    S = np.zeros_like(y_ref)
    Wabs = {}
    for p, e in enumerate(ids.reshape(-1)):
        le = e if lmap is None else lmap[e]
        if le < 0:
            continue
        if le not in Wabs:
            Wabs[le] = np.abs(lut3.dequant(*local[le]))
        S[p] = Xq[p // top_k] @ Wabs[le]
    ok, worst = matmul.check(matmul.as_f64(Y.cpu()), y_ref, S)
    assert ok, f"max error ratio {worst:.3g} > 1"
    return Y, y_ref


@pytest.mark.parametrize("T,top_k,E,K,N", [
    (37, 2, 4, 256, 136),      # ragged channel tile, several experts per block boundary
    (5, 3, 8, 128, 64),        # fewer rows than a block for every expert, one k-block
    (64, 8, 16, 2048, 256),    # the MoE layer's gate/up K, two channel tiles
    (200, 2, 2, 512, 128),     # experts with several blocks each
    (1, 8, 32, 2048, 1024),    # one token over 8 of 32 experts at the layer's gate/up shape
    (16, 8, 64, 512, 2056),    # 16 tokens, some experts with several pairs; a ragged last channel tile
])
@pytest.mark.parametrize("ydt", ["bf16", "f16"])
def test_grouped_gemm_matches_the_routing_definition(torch, lbq, T, top_k, E, K, N, ydt):
    _run_case(torch, lbq, T, top_k, E, K, N, ydt)


def test_non_local_experts_write_zero_rows(torch, lbq):
    E = 6
    emap = np.array([0, -1, 1, -1, 2, 3], dtype=np.int32)
    Y, y_ref = _run_case(torch, lbq, 40, 2, E, 256, 64, emap=emap, seed=90)
    ids = _routing(90, 40, 2, E).reshape(-1)
    remote = np.isin(ids, [1, 3])
    assert remote.any() and np.all(Y.cpu().float().numpy()[remote] == 0)


def test_grouped_gemm_errors(torch, lbq):
    ids = torch.zeros((4, 2), dtype=torch.int32, device="cuda")
    with pytest.raises(lbq.LbqError):
        lbq.moe_align(ids, 0)                                            # no experts
    aligned = lbq.moe_align(ids, 2)
    codes = torch.zeros((4, 192), dtype=torch.uint8, device="cuda")     # K % 128 != 0
    scales = torch.zeros((4, 6), dtype=torch.uint8, device="cuda")
    with pytest.raises(lbq.LbqError):
        lbq.moe_lut3_mx_gemm(codes, scales, 2, aligned, torch.zeros(1 << 16, dtype=torch.uint8, device="cuda"),
                             1 << 15, 2, 64)
    lbq.device_status()
