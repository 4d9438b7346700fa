"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every symbol include/lbq.h declares, sizes its images as the format says, and
rejects bad arguments before touching a device."""

import ctypes
import os
import re

import pytest

from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "lbq.h")


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\S.*?\b(lbq_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_boundary():
    names = declared_symbols()
    for required in ("lbq_pack", "lbq_gemv", "lbq_gemm", "lbq_lut3_gemm", "lbq_pack_lut3", "lbq_packed_size",
                     "lbq_workspace_size", "lbq_unpack_canonical", "lbq_dequant", "lbq_last_error"):
        assert required in names


def test_library_exports_every_declared_symbol():
    import bit_weight_only_pack_b200.binding as b
    lib = ctypes.CDLL(b.LIB_PATH)
    for name in declared_symbols():
        assert hasattr(lib, name), name
    for name in b.exported_symbols():
        assert hasattr(lib, name), name


def test_packed_size_matches_the_format():
    import bit_weight_only_pack_b200 as lbq
    from oracle import int4, lut3
    for K, N, g, mode in [(4096, 4096, 32, "sym"), (4096, 14336, 128, "asym"), (8192, 28672, 64, "sym"),
                          (96, 40, 32, "asym")]:
        size = lbq.lbq_packed_size(K, N, g, lbq.MODES[mode])
        payload = int4.algorithmic_bytes(K, N, g, mode)
        # header + region alignment + scale / zero-point rows padded to 16 bytes
        assert payload <= size <= payload + 256 * 4 + N * 30
    size = lbq.lbq_packed_size(4096, 14336, 0, lbq.MODES["lut3"])
    # the payload plus the per-tile BF16 decode tables (16 bytes per 8 channels x 64 k)
    tables = (4096 // 64) * (14336 // 8) * 16
    assert lut3.algorithmic_bytes(4096, 14336) <= size <= lut3.algorithmic_bytes(4096, 14336) + tables + 1024


@pytest.mark.parametrize("args,status", [
    ((4096, 4096, 48, 0), 2),     # group not in {32, 64, 128}
    ((4100, 4096, 32, 0), 1),     # K not a multiple of the group
    ((4096, 0, 32, 0), 1),        # empty N
    ((4096, 4096, 32, 7), 2),     # unknown mode
    ((100, 8, 0, 2), 1),          # LUT3 K not a multiple of 64
    ((128, 12, 0, 2), 1),         # LUT3 N not a multiple of 8
])
def test_bad_shapes_are_rejected(args, status):
    import bit_weight_only_pack_b200 as lbq
    with pytest.raises(lbq.LbqError) as e:
        lbq.lbq_packed_size(*args)
    assert e.value.status == status
    assert lbq.lbq_last_error()


def test_null_and_misaligned_pointers_are_rejected_on_the_host():
    import bit_weight_only_pack_b200 as lbq
    before = lbq.lbq_launch_count()
    with pytest.raises(lbq.LbqError) as e:
        lbq.lbq_pack(None, 64, 8, 32, 0, None, 1 << 20, None)
    assert e.value.status == lbq.binding.LBQ_ERR_INVALID_ARG
    with pytest.raises(lbq.LbqError) as e:
        lbq.lbq_gemv(8, 0, 1, 64, 8, 32, 0, 16, 32, 0, None, 0, None)  # misaligned X
    assert e.value.status == lbq.binding.LBQ_ERR_INVALID_ARG
    with pytest.raises(lbq.LbqError) as e:
        lbq.lbq_gemv(16, 0, 0, 64, 8, 32, 0, 16, 32, 0, None, 0, None)  # M = 0
    assert e.value.status == lbq.binding.LBQ_ERR_INVALID_ARG
    with pytest.raises(lbq.LbqError) as e:
        lbq.lbq_gemv(16, 3, 1, 64, 8, 32, 0, 16, 32, 0, None, 0, None)  # bad dtype
    assert e.value.status == lbq.binding.LBQ_ERR_UNSUPPORTED
    with pytest.raises(lbq.LbqError) as e:
        lbq.lbq_pack(16, 64, 8, 32, 0, 32, 16, None)  # image buffer too small
    assert e.value.status == lbq.binding.LBQ_ERR_INVALID_ARG
    assert lbq.lbq_launch_count() == before


def test_workspace_query_is_host_only():
    import bit_weight_only_pack_b200 as lbq
    assert lbq.lbq_workspace_size(0, 1, 4096, 4096, 32, 0) >= 0
    with pytest.raises(lbq.LbqError):
        lbq.lbq_workspace_size(9, 1, 4096, 4096, 32, 0)


def test_grouped_noalloc_and_lut3_calls_reject_bad_arguments_on_the_host():
    """Argument checks of the grouped, no-alloc and LUT3 calls run before any
    device work: each bad call returns its status and launches nothing."""
    import bit_weight_only_pack_b200 as lbq
    b = lbq.binding
    before = lbq.lbq_launch_count()
    good = [(16, 32, 48, 64)]  # X, image, Y (16-byte aligned fake addresses), N
    cases = [
        (lambda: lbq.lbq_gemv_grouped(None, 1, 64, 32, 0, 0, 0, None), b.LBQ_ERR_INVALID_ARG),          # no items
        (lambda: lbq.lbq_gemv_grouped(lbq.make_gemv_items(good), 0, 64, 32, 0, 0, 0, None), b.LBQ_ERR_INVALID_ARG),
        (lambda: lbq.lbq_gemv_grouped(lbq.make_gemv_items(good * 5), 5, 64, 32, 0, 0, 0, None), b.LBQ_ERR_INVALID_ARG),
        (lambda: lbq.lbq_gemv_grouped(lbq.make_gemv_items(good), 1, 32768, 32, 0, 0, 0, None), b.LBQ_ERR_UNSUPPORTED),
        (lambda: lbq.lbq_gemv_grouped(lbq.make_gemv_items(good), 1, 64, 48, 0, 0, 0, None), b.LBQ_ERR_UNSUPPORTED),
        (lambda: lbq.lbq_gemv_grouped(lbq.make_gemv_items([(8, 32, 48, 64)]), 1, 64, 32, 0, 0, 0, None),
         b.LBQ_ERR_INVALID_ARG),                                                                        # misaligned X
        (lambda: lbq.lbq_gemv_grouped(lbq.make_gemv_items(good), 1, 64, 32, 0, 2, 0, None), b.LBQ_ERR_UNSUPPORTED),
        (lambda: lbq.lbq_gemv_noalloc(16, 0, 17, 64, 8, 32, 0, 32, 48, 0, None), b.LBQ_ERR_UNSUPPORTED),  # M > 16
        (lambda: lbq.lbq_gemv_noalloc(16, 0, 1, 60, 8, 32, 0, 32, 48, 0, None), b.LBQ_ERR_INVALID_ARG),   # K % group
        (lambda: lbq.lbq_lut3_gemm(16, 1, 1, 96, 8, 32, 48, 1, None, 0, None), b.LBQ_ERR_INVALID_ARG),    # K % 64
        (lambda: lbq.lbq_lut3_gemm(16, 1, 1, 128, 12, 32, 48, 1, None, 0, None), b.LBQ_ERR_INVALID_ARG),  # N % 8
        (lambda: lbq.lbq_lut3_gemm(16, 0, 1, 128, 8, 32, 48, 1, None, 0, None), b.LBQ_ERR_UNSUPPORTED),   # FP16 X
    ]
    for call, status in cases:
        with pytest.raises(lbq.LbqError) as e:
            call()
        assert e.value.status == status, lbq.lbq_last_error()
        assert lbq.lbq_last_error()
    assert lbq.lbq_launch_count() == before
