"""Thin ctypes binding of liblbq.so: the C ABI of include/lbq.h, same names.

Argument marshalling only. Every step of the computation runs in the CUDA
kernels of liblbq.so; there is no CPU or Python fallback. If the library has
not been built, importing this module raises.

Two layers:
* ``lbq_*`` functions mirror the C calls one to one (integers and raw
  pointers; a non-OK status raises :class:`LbqError`).
* Small torch helpers (``pack``, ``gemv``, ``gemm``, ...) take CUDA tensors,
  pass their data pointers and the current stream, and allocate outputs with
  torch (the library itself never allocates).
"""

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "liblbq.so")

LBQ_OK, LBQ_ERR_INVALID_ARG, LBQ_ERR_UNSUPPORTED, LBQ_ERR_CUDA, LBQ_ERR_DEVICE = range(5)
MODES = {"sym": 0, "asym": 1, "lut3": 2, "affine": 3}
DTYPES = {"f16": 0, "bf16": 1}
STATUS_NAMES = {0: "LBQ_OK", 1: "LBQ_ERR_INVALID_ARG", 2: "LBQ_ERR_UNSUPPORTED", 3: "LBQ_ERR_CUDA",
                4: "LBQ_ERR_DEVICE"}


class LbqError(RuntimeError):
    def __init__(self, status, message):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python bit_weight_only_pack_b200/build.py` "
                      "(the CUDA library is required; there is no fallback)")

_lib = ctypes.CDLL(LIB_PATH)

_c_int, _c_size, _vp, _u64 = ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_uint64

class lbq_gemv_item(ctypes.Structure):
    """One GEMV of lbq_gemv_grouped (include/lbq.h)."""
    _fields_ = [("X", ctypes.c_void_p), ("image", ctypes.c_void_p), ("Y", ctypes.c_void_p), ("N", ctypes.c_int)]


class lbq_w4a8_item(ctypes.Structure):
    """One GEMV of lbq_w4a8_gemv_grouped (include/lbq.h)."""
    _fields_ = [("xq", ctypes.c_void_p), ("sx", ctypes.c_void_p), ("image", ctypes.c_void_p), ("Y", ctypes.c_void_p),
                ("N", ctypes.c_int)]


_SIGS = {
    "lbq_last_error": ([], ctypes.c_char_p),
    "lbq_version": ([], _c_int),
    "lbq_launch_count": ([], _u64),
    "lbq_packed_size": ([_c_int, _c_int, _c_int, _c_int, ctypes.POINTER(_c_size)], _c_int),
    "lbq_pack": ([_vp, _c_int, _c_int, _c_int, _c_int, _vp, _c_size, _vp], _c_int),
    "lbq_pack_lut3": ([_vp, _vp, _vp, _c_int, _c_int, _vp, _c_size, _vp], _c_int),
    "lbq_workspace_size": ([_c_int, _c_int, _c_int, _c_int, _c_int, _c_int, ctypes.POINTER(_c_size)], _c_int),
    "lbq_gemv": ([_vp, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _vp, _vp, _c_int, _vp, _c_size, _vp], _c_int),
    "lbq_gemm": ([_vp, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _vp, _vp, _c_int, _vp, _c_size, _vp], _c_int),
    "lbq_lut3_gemm": ([_vp, _c_int, _c_int, _c_int, _c_int, _vp, _vp, _c_int, _vp, _c_size, _vp], _c_int),
    "lbq_unpack_canonical": ([_vp, _c_int, _c_int, _c_int, _c_int, _vp, _vp, _vp, _vp], _c_int),
    "lbq_unpack_lut3_canonical": ([_vp, _c_int, _c_int, _vp, _vp, _vp, _vp], _c_int),
    "lbq_dequant": ([_vp, _c_int, _c_int, _c_int, _c_int, _vp, _vp], _c_int),
    "lbq_device_status": ([_vp], _c_int),
    "lbq_set_option": ([_c_int, _c_int], _c_int),
    "lbq_gemv_noalloc": ([_vp, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _vp, _vp, _c_int, _vp], _c_int),
    "lbq_gemv_grouped": ([ctypes.POINTER(lbq_gemv_item), _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _vp], _c_int),
    "lbq_quantize_mxfp8": ([_vp, _c_int, _c_int, _c_int, _vp, _vp, _vp], _c_int),
    "lbq_lut3_mx_gemm": ([_vp, _vp, _c_int, _c_int, _c_int, _vp, _vp, _c_int, _vp, _c_size, _vp], _c_int),
    "lbq_affine_packed_size": ([_c_int, _c_int, _c_int, _c_int, ctypes.POINTER(_c_size)], _c_int),
    "lbq_pack_affine": ([_vp, _c_int, _c_int, _c_int, _c_int, _vp, _c_size, _vp], _c_int),
    "lbq_affine_gemv": ([_vp, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _vp, _vp, _c_int, _vp], _c_int),
    "lbq_unpack_affine_canonical": ([_vp, _c_int, _c_int, _c_int, _c_int, _vp, _vp, _vp, _vp], _c_int),
    "lbq_quantize_int8": ([_vp, _c_int, _c_int, _c_int, _vp, _vp, _vp], _c_int),
    "lbq_w4a8_gemv": ([_vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int, _vp, _vp, _c_int, _vp], _c_int),
    "lbq_w4a8_gemv_grouped": ([ctypes.POINTER(lbq_w4a8_item), _c_int, _c_int, _c_int, _c_int, _c_int, _vp],
                              _c_int),
    "lbq_debug_w4a8_tiled": ([_c_int], None),
    "lbq_debug_lut3_stages": ([_c_int], None),
    "lbq_debug_lut3_batch_off": ([_c_int], None),
    "lbq_debug_gemm_stream_k": ([_c_int], None),
    "lbq_debug_gemm_hold": ([_c_int], None),
    "lbq_debug_tile_coords": ([_c_int, _c_int, _c_int, ctypes.POINTER(_c_int), ctypes.POINTER(_c_int)], None),
    "lbq_debug_gemm_schedule": ([_c_int, _c_int, _c_int, _c_int, _c_int, ctypes.POINTER(_c_int),
                                 ctypes.POINTER(_c_int), ctypes.POINTER(_c_int), _c_int], _c_int),
    "lbq_moe_max_padded": ([_c_int, _c_int, _c_int, ctypes.POINTER(_c_int)], _c_int),
    "lbq_moe_align": ([_vp, _c_int, _c_int, _c_int, _vp, _vp, _vp, _vp, _c_int, _vp], _c_int),
    "lbq_moe_lut3_mx_gemm": ([_vp, _vp, _c_int, _c_int, _c_int, _c_int, _vp, _vp, _vp, _c_int, _vp, _c_size, _c_int,
                              _vp, _c_int, _vp], _c_int),
    "lbq_debug_force_splits": ([_c_int], None),
    "lbq_debug_force_skinny": ([_c_int], None),
    "lbq_debug_force_tc": ([_c_int], None),
    "lbq_debug_gemv_path": ([_c_int], None),
    "lbq_debug_gemm_path": ([_c_int], None),
    "lbq_debug_direct_variant": ([_c_int, _c_int], None),
    "lbq_debug_tmma_default": ([_c_int], None),
    "lbq_debug_tmma_split": ([_c_int], None),
    "lbq_debug_drop_copies": ([_c_int], None),
}
for _name, (_args, _res) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.argtypes = _args
    _f.restype = _res


def exported_symbols():
    """Names this binding binds (each must be exported by liblbq.so)."""
    return sorted(_SIGS)


def _check(status):
    if status != LBQ_OK:
        raise LbqError(status, _lib.lbq_last_error().decode())


def lbq_last_error():
    return _lib.lbq_last_error().decode()


def lbq_version():
    return _lib.lbq_version()


def lbq_launch_count():
    return int(_lib.lbq_launch_count())


def lbq_packed_size(K, N, group, mode):
    out = _c_size(0)
    _check(_lib.lbq_packed_size(K, N, group, mode, ctypes.byref(out)))
    return out.value


def lbq_workspace_size(op, M, K, N, group, mode):
    out = _c_size(0)
    _check(_lib.lbq_workspace_size(op, M, K, N, group, mode, ctypes.byref(out)))
    return out.value


def lbq_pack(W, K, N, group, mode, image, image_bytes, stream):
    _check(_lib.lbq_pack(W, K, N, group, mode, image, image_bytes, stream))


def lbq_pack_lut3(idx, codebooks, exponents, K, N, image, image_bytes, stream):
    _check(_lib.lbq_pack_lut3(idx, codebooks, exponents, K, N, image, image_bytes, stream))


def lbq_gemv(X, x_dtype, M, K, N, group, mode, image, Y, y_dtype, ws, ws_bytes, stream):
    _check(_lib.lbq_gemv(X, x_dtype, M, K, N, group, mode, image, Y, y_dtype, ws, ws_bytes, stream))


def lbq_gemm(X, x_dtype, M, K, N, group, mode, image, Y, y_dtype, ws, ws_bytes, stream):
    _check(_lib.lbq_gemm(X, x_dtype, M, K, N, group, mode, image, Y, y_dtype, ws, ws_bytes, stream))


def lbq_lut3_gemm(X, x_dtype, M, K, N, image, Y, y_dtype, ws, ws_bytes, stream):
    _check(_lib.lbq_lut3_gemm(X, x_dtype, M, K, N, image, Y, y_dtype, ws, ws_bytes, stream))


def lbq_unpack_canonical(image, K, N, group, mode, q_packed, scales, zp, stream):
    _check(_lib.lbq_unpack_canonical(image, K, N, group, mode, q_packed, scales, zp, stream))


def lbq_unpack_lut3_canonical(image, K, N, idx_stream, codebooks, exponents, stream):
    _check(_lib.lbq_unpack_lut3_canonical(image, K, N, idx_stream, codebooks, exponents, stream))


def lbq_dequant(image, K, N, group, mode, W_out, stream):
    _check(_lib.lbq_dequant(image, K, N, group, mode, W_out, stream))


def lbq_device_status(stream):
    _check(_lib.lbq_device_status(stream))


def lbq_gemv_grouped(items, count, K, group, mode, x_dtype, y_dtype, stream):
    """items: a ctypes array of lbq_gemv_item (host memory)."""
    _check(_lib.lbq_gemv_grouped(items, count, K, group, mode, x_dtype, y_dtype, stream))


def make_gemv_items(triples):
    """[(X ptr, image ptr, Y ptr, N), ...] -> ctypes array for lbq_gemv_grouped."""
    arr = (lbq_gemv_item * len(triples))()
    for i, (x, img, y, n) in enumerate(triples):
        arr[i] = lbq_gemv_item(x, img, y, n)
    return arr


def lbq_gemv_noalloc(X, x_dtype, M, K, N, group, mode, image, Y, y_dtype, stream):
    _check(_lib.lbq_gemv_noalloc(X, x_dtype, M, K, N, group, mode, image, Y, y_dtype, stream))


LBQ_OPT_PDL = 1


def lbq_quantize_mxfp8(X, x_dtype, M, K, codes, scales, stream):
    _check(_lib.lbq_quantize_mxfp8(X, x_dtype, M, K, codes, scales, stream))


def quantize_mxfp8(X):
    """MXFP8 activations: X [M, K] FP16/BF16 -> (codes uint8 [M, K] E4M3, scales uint8 [M, K/32] UE8M0)."""
    torch = _torch()
    _need_cuda(X)
    M, K = X.shape
    codes = torch.empty((M, K), dtype=torch.uint8, device=X.device)
    scales = torch.empty((M, K // 32), dtype=torch.uint8, device=X.device)
    lbq_quantize_mxfp8(X.data_ptr(), _dt(X), M, K, codes.data_ptr(), scales.data_ptr(), _stream())
    return codes, scales


def lbq_lut3_mx_gemm(codes, scales, M, K, N, image, Y, y_dtype, ws, ws_bytes, stream):
    _check(_lib.lbq_lut3_mx_gemm(codes, scales, M, K, N, image, Y, y_dtype, ws, ws_bytes, stream))


def lut3_mx_gemm(codes, scales, image, N, y_dtype="bf16", Y=None, ws=None):
    """Y[M, N] = MXFP8 activations (codes uint8 [M, K], scales uint8 [M, K/32]) . LUT3 weights."""
    torch = _torch()
    _need_cuda(codes, scales, image, Y, ws)
    M, K = codes.shape
    if Y is None:
        Y = torch.empty((M, N), dtype={"f16": torch.float16, "bf16": torch.bfloat16}[y_dtype], device=codes.device)
    if ws is None and M > 16:
        ws = workspace(2, M, K, N, 0, "lut3", codes.device)
    lbq_lut3_mx_gemm(codes.data_ptr(), scales.data_ptr(), M, K, N, image.data_ptr(), Y.data_ptr(), _dt(Y),
                     ws.data_ptr() if ws is not None else None, ws.numel() if ws is not None else 0, _stream())
    return Y


def lbq_affine_packed_size(K, N, group, bits):
    n = _c_size(0)
    _check(_lib.lbq_affine_packed_size(K, N, group, bits, ctypes.byref(n)))
    return n.value


def lbq_pack_affine(W, K, N, group, bits, image, image_bytes, stream):
    _check(_lib.lbq_pack_affine(W, K, N, group, bits, image, image_bytes, stream))


def lbq_affine_gemv(X, x_dtype, M, K, N, group, bits, image, Y, y_dtype, stream):
    _check(_lib.lbq_affine_gemv(X, x_dtype, M, K, N, group, bits, image, Y, y_dtype, stream))


def lbq_unpack_affine_canonical(image, K, N, group, bits, q_stream, scales, zp, stream):
    _check(_lib.lbq_unpack_affine_canonical(image, K, N, group, bits, q_stream, scales, zp, stream))


def lbq_quantize_int8(X, x_dtype, M, K, xq, sx, stream):
    _check(_lib.lbq_quantize_int8(X, x_dtype, M, K, xq, sx, stream))


def lbq_w4a8_gemv(xq, sx, M, K, N, group, mode, image, Y, y_dtype, stream):
    _check(_lib.lbq_w4a8_gemv(xq, sx, M, K, N, group, mode, image, Y, y_dtype, stream))


def lbq_w4a8_gemv_grouped(items, count, K, group, mode, y_dtype, stream):
    _check(_lib.lbq_w4a8_gemv_grouped(items, count, K, group, mode, y_dtype, stream))


def make_w4a8_items(rows):
    """ctypes array of lbq_w4a8_item from (xq_ptr, sx_ptr, image_ptr, Y_ptr, N) tuples."""
    arr = (lbq_w4a8_item * len(rows))()
    for i, (xq, sx, img, Y, N) in enumerate(rows):
        arr[i].xq, arr[i].sx, arr[i].image, arr[i].Y, arr[i].N = xq, sx, img, Y, N
    return arr


def lbq_debug_w4a8_tiled(on):
    """Test hook: batch-1 W4A8 on the tiled kernel instead of the staged one."""
    _lib.lbq_debug_w4a8_tiled(1 if on else 0)


def lbq_debug_lut3_stages(stages):
    """Test hook: ring stages of the TMA-fed LUT3 batch-1 kernel (0 = the plan's choice)."""
    _lib.lbq_debug_lut3_stages(int(stages))


def lbq_debug_lut3_batch_off(on):
    """Test hook: LUT3 at M = 2..8 on the skinny kernel instead of the TMA-fed batch kernel."""
    _lib.lbq_debug_lut3_batch_off(1 if on else 0)


def lbq_debug_gemm_stream_k(on):
    """Test hook: prefill stream-K on (the library's choice) or off (whole tiles only)."""
    _lib.lbq_debug_gemm_stream_k(1 if on else 0)


def lbq_debug_gemm_hold(polls):
    """Test hook: with polls > 0 the prefill's parked parts are never flagged and the wait gives up after polls."""
    _lib.lbq_debug_gemm_hold(int(polls))


def lbq_debug_gemm_schedule(M, K, N, stream_k, cta):
    """Test hook: (grid, k_blocks, [(tile, kb0, kb1, part), ...]) of one prefill CTA, as the kernel walks it."""
    grid, nkb = _c_int(0), _c_int(0)
    n = _lib.lbq_debug_gemm_schedule(M, K, N, 1 if stream_k else 0, cta, ctypes.byref(grid), ctypes.byref(nkb), None, 0)
    buf = (_c_int * max(4 * n, 4))()
    _lib.lbq_debug_gemm_schedule(M, K, N, 1 if stream_k else 0, cta, ctypes.byref(grid), ctypes.byref(nkb), buf, n)
    return grid.value, nkb.value, [tuple(buf[4 * i:4 * i + 4]) for i in range(n)]


def lbq_debug_tile_coords(tile, n_tiles, m_tiles):
    """Test hook: (channel tile, token tile) of a prefill tile index in the kernel's banded order."""
    nt, mt = _c_int(0), _c_int(0)
    _lib.lbq_debug_tile_coords(tile, n_tiles, m_tiles, ctypes.byref(nt), ctypes.byref(mt))
    return nt.value, mt.value


def lbq_moe_max_padded(num_pairs, num_experts, block):
    n = _c_int(0)
    _check(_lib.lbq_moe_max_padded(num_pairs, num_experts, block, ctypes.byref(n)))
    return n.value


def lbq_moe_align(topk_ids, num_pairs, num_experts, block, expert_map, sorted_ids, expert_ids, total, max_padded,
                  stream):
    _check(_lib.lbq_moe_align(topk_ids, num_pairs, num_experts, block, expert_map, sorted_ids, expert_ids, total,
                              max_padded, stream))


def lbq_moe_lut3_mx_gemm(codes, scales, T, top_k, K, N, sorted_ids, expert_ids, total, max_padded, images,
                         image_stride, num_local_experts, Y, y_dtype, stream):
    _check(_lib.lbq_moe_lut3_mx_gemm(codes, scales, T, top_k, K, N, sorted_ids, expert_ids, total, max_padded, images,
                                     image_stride, num_local_experts, Y, y_dtype, stream))


def lbq_set_option(option, value):
    _check(_lib.lbq_set_option(option, value))


def lbq_debug_force_splits(splits):
    _lib.lbq_debug_force_splits(splits)


def lbq_debug_force_tc(on):
    _lib.lbq_debug_force_tc(1 if on else 0)


def lbq_debug_gemv_path(path):
    """Test hook: GEMV kernel for M <= 16 (0 auto, 1 CUDA-core M=1, 2 warp MMA, 3 tcgen05,
    4 direct-load CUDA-core M=1, 5 TMA-fed warp-MMA M=1)."""
    _lib.lbq_debug_gemv_path(path)


def lbq_debug_tmma_default(mode):
    """Test hook: when the TMA-fed warp-MMA kernel is the batch-1 choice (0 never, 1 always,
    2 launches of >= 4 16-row tiles per SM with K <= 4096)."""
    _lib.lbq_debug_tmma_default(int(mode))


def lbq_debug_drop_copies(on):
    """Test hook: TMA-fed GEMV launches issue no copies, so their bounded waits run out."""
    _lib.lbq_debug_drop_copies(1 if on else 0)


def lbq_debug_tmma_split(r):
    """Test hook: force the TMA-fed kernel's K split into r in {1, 2, 4} ranges (0 = its own choice)."""
    _lib.lbq_debug_tmma_split(r)


def lbq_debug_direct_variant(variant, ctas_per_sm=0):
    """Test hook: batch-1 direct kernel variant (-1 library's choice, 0 registers, 2..4 staged copies,
    1 / 5 tensor cores with exact / offset-form operands) and a CTAs-per-SM cap."""
    _lib.lbq_debug_direct_variant(variant, ctas_per_sm)


def lbq_debug_gemm_path(path):
    """Test hook: prefill kernel (0 weights in tensor memory, 1 weights dequantised into shared memory)."""
    _lib.lbq_debug_gemm_path(path)


def lbq_debug_force_skinny(on):
    _lib.lbq_debug_force_skinny(1 if on else 0)


# ----------------------------------------------------------------------------- torch helpers

def _torch():
    import torch
    return torch


def _stream():
    return _torch().cuda.current_stream().cuda_stream


def _mode(mode):
    return MODES[mode] if isinstance(mode, str) else int(mode)


def _dt(t):
    torch = _torch()
    if t.dtype == torch.float16:
        return DTYPES["f16"]
    if t.dtype == torch.bfloat16:
        return DTYPES["bf16"]
    raise TypeError(f"unsupported dtype {t.dtype}")


def _need_cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("tensors must be contiguous CUDA tensors")


def pack(W, group, mode):
    """Quantise + repack a float32 [K, N] CUDA tensor; returns the uint8 image."""
    torch = _torch()
    _need_cuda(W)
    K, N = W.shape
    m = _mode(mode)
    img = torch.empty(lbq_packed_size(K, N, group, m), dtype=torch.uint8, device=W.device)
    lbq_pack(W.data_ptr(), K, N, group, m, img.data_ptr(), img.numel(), _stream())
    return img


def pack_lut3(idx, codebooks, exponents):
    """Build a LUT3 image from idx uint8 [K, N], codebooks uint8 [K/64, N/8, 8], exponents uint8 [K/64, N/8]."""
    torch = _torch()
    _need_cuda(idx, codebooks, exponents)
    K, N = idx.shape
    img = torch.empty(lbq_packed_size(K, N, 0, MODES["lut3"]), dtype=torch.uint8, device=idx.device)
    lbq_pack_lut3(idx.data_ptr(), codebooks.data_ptr(), exponents.data_ptr(), K, N, img.data_ptr(), img.numel(),
                  _stream())
    return img


def workspace(op, M, K, N, group, mode, device="cuda"):
    """A zero-filled workspace of the size the call needs (None when it needs none)."""
    torch = _torch()
    n = lbq_workspace_size(op, M, K, N, group, _mode(mode))
    return torch.zeros(n, dtype=torch.uint8, device=device) if n else None


def _out(X, N, y_dtype):
    torch = _torch()
    dt = {None: X.dtype, "f16": torch.float16, "bf16": torch.bfloat16}[y_dtype] if not hasattr(y_dtype, "is_floating_point") else y_dtype
    return torch.empty((X.shape[0], N), dtype=dt, device=X.device)


def _out_dt(M, N, y_dtype, device):
    torch = _torch()
    return torch.empty((M, N), dtype={"f16": torch.float16, "bf16": torch.bfloat16}[y_dtype], device=device)


def gemv(X, image, N, group, mode, y_dtype=None, ws=None, Y=None):
    """Y[M, N] = X[M, K] . dequant(image) for 1 <= M <= 16 (INT4 image)."""
    _need_cuda(X, image, ws, Y)
    M, K = X.shape
    m = _mode(mode)
    if ws is None:
        ws = workspace(0, M, K, N, group, m, X.device)
    Y = _out(X, N, y_dtype) if Y is None else Y
    lbq_gemv(X.data_ptr(), _dt(X), M, K, N, group, m, image.data_ptr(), Y.data_ptr(), _dt(Y),
             ws.data_ptr() if ws is not None else None, ws.numel() if ws is not None else 0, _stream())
    return Y


def gemm(X, image, N, group, mode, y_dtype=None, ws=None, Y=None):
    """Y[M, N] = X[M, K] . dequant(image) for any M (INT4 image)."""
    _need_cuda(X, image, ws, Y)
    M, K = X.shape
    m = _mode(mode)
    if ws is None:
        ws = workspace(1, M, K, N, group, m, X.device)
    Y = _out(X, N, y_dtype) if Y is None else Y
    lbq_gemm(X.data_ptr(), _dt(X), M, K, N, group, m, image.data_ptr(), Y.data_ptr(), _dt(Y),
             ws.data_ptr() if ws is not None else None, ws.numel() if ws is not None else 0, _stream())
    return Y


def lut3_gemm(X, image, N, y_dtype=None, ws=None, Y=None):
    """Y[M, N] = X[M, K] . decode(image) for a LUT3 image, any M."""
    _need_cuda(X, image, ws, Y)
    M, K = X.shape
    if ws is None:
        ws = workspace(2, M, K, N, 0, MODES["lut3"], X.device)
    Y = _out(X, N, y_dtype) if Y is None else Y
    lbq_lut3_gemm(X.data_ptr(), _dt(X), M, K, N, image.data_ptr(), Y.data_ptr(), _dt(Y),
                  ws.data_ptr() if ws is not None else None, ws.numel() if ws is not None else 0, _stream())
    return Y


def unpack_canonical(image, K, N, group, mode):
    """(q_packed uint8 [K/2, N], scale fp16 [K/group, N], zp int8 [K/group, N] or None)."""
    torch = _torch()
    m = _mode(mode)
    q = torch.empty((K // 2, N), dtype=torch.uint8, device=image.device)
    s = torch.empty((K // group, N), dtype=torch.int16, device=image.device)
    z = torch.empty((K // group, N), dtype=torch.int8, device=image.device) if m == MODES["asym"] else None
    lbq_unpack_canonical(image.data_ptr(), K, N, group, m, q.data_ptr(), s.data_ptr(),
                         z.data_ptr() if z is not None else None, _stream())
    return q, s.view(torch.float16), z


def unpack_lut3_canonical(image, K, N):
    torch = _torch()
    idx = torch.empty((K // 64, N // 8, 8, 24), dtype=torch.uint8, device=image.device)
    cb = torch.empty((K // 64, N // 8, 8), dtype=torch.uint8, device=image.device)
    ex = torch.empty((K // 64, N // 8), dtype=torch.uint8, device=image.device)
    lbq_unpack_lut3_canonical(image.data_ptr(), K, N, idx.data_ptr(), cb.data_ptr(), ex.data_ptr(), _stream())
    return idx, cb, ex


def dequant(image, K, N, group, mode):
    """Exact FP32 [K, N] dequantisation of an image (debug / parity)."""
    torch = _torch()
    W = torch.empty((K, N), dtype=torch.float32, device=image.device)
    lbq_dequant(image.data_ptr(), K, N, group, _mode(mode), W.data_ptr(), _stream())
    return W


def gemv_grouped(problems, group, mode, y_dtype=None):
    """Batch-1 GEMVs in one launch. problems: [(X [1, K], image, N), ...] with a
    common K; returns the list of Y [1, N]."""
    torch = _torch()
    K = problems[0][0].shape[1]
    Ys = []
    rows = []
    for X, img, N in problems:
        _need_cuda(X, img)
        if X.shape != (1, K) or X.dtype != problems[0][0].dtype:
            raise ValueError("grouped GEMVs need X [1, K] of one K and dtype")
        Y = _out(X, N, y_dtype)
        Ys.append(Y)
        rows.append((X.data_ptr(), img.data_ptr(), Y.data_ptr(), N))
    lbq_gemv_grouped(make_gemv_items(rows), len(rows), K, group, _mode(mode), _dt(problems[0][0]), _dt(Ys[0]),
                     _stream())
    return Ys


def gemv_noalloc(X, image, N, group, mode, y_dtype=None, Y=None):
    """lbq_gemv with the library's fixed scratch instead of a workspace."""
    _need_cuda(X, image, Y)
    M, K = X.shape
    Y = _out(X, N, y_dtype) if Y is None else Y
    lbq_gemv_noalloc(X.data_ptr(), _dt(X), M, K, N, group, _mode(mode), image.data_ptr(), Y.data_ptr(), _dt(Y),
                     _stream())
    return Y


def pack_affine(W, group, bits):
    """Quantise + repack a float32 [K, N] CUDA tensor to b-bit affine codes; returns the uint8 image."""
    torch = _torch()
    _need_cuda(W)
    K, N = W.shape
    img = torch.empty(lbq_affine_packed_size(K, N, group, bits), dtype=torch.uint8, device=W.device)
    lbq_pack_affine(W.data_ptr(), K, N, group, bits, img.data_ptr(), img.numel(), _stream())
    return img


def affine_gemv(X, image, N, group, bits, y_dtype=None, Y=None):
    """Y[M, N] = X[M, K] . dequant(image) for a b-bit affine image, 1 <= M <= 16."""
    _need_cuda(X, image, Y)
    M, K = X.shape
    Y = _out(X, N, y_dtype) if Y is None else Y
    lbq_affine_gemv(X.data_ptr(), _dt(X), M, K, N, group, bits, image.data_ptr(), Y.data_ptr(), _dt(Y), _stream())
    return Y


def unpack_affine_canonical(image, K, N, group, bits):
    """(q_stream uint8 [K*bits/8, N], scale fp16 [K/group, N], zp int8 [K/group, N])."""
    torch = _torch()
    q = torch.empty((K * bits // 8, N), dtype=torch.uint8, device=image.device)
    s = torch.empty((K // group, N), dtype=torch.int16, device=image.device)
    z = torch.empty((K // group, N), dtype=torch.int8, device=image.device)
    lbq_unpack_affine_canonical(image.data_ptr(), K, N, group, bits, q.data_ptr(), s.data_ptr(), z.data_ptr(),
                                _stream())
    return q, s.view(torch.float16), z


def quantize_int8(X):
    """Dynamic INT8 activations of X [M, K]: (xq int8 [M, K], sx float32 [M, K/32])."""
    torch = _torch()
    _need_cuda(X)
    M, K = X.shape
    xq = torch.empty((M, K), dtype=torch.int8, device=X.device)
    sx = torch.empty((M, K // 32), dtype=torch.float32, device=X.device)
    lbq_quantize_int8(X.data_ptr(), _dt(X), M, K, xq.data_ptr(), sx.data_ptr(), _stream())
    return xq, sx


def w4a8_gemv(xq, sx, image, N, group, mode, y_dtype="f16", Y=None):
    """Y[M, N] = dequant(xq, sx) . dequant(image) for an INT4 image, 1 <= M <= 16
    (xq, sx from :func:`quantize_int8`)."""
    _need_cuda(xq, sx, image, Y)
    M, K = xq.shape
    Y = _out_dt(M, N, y_dtype, xq.device) if Y is None else Y
    lbq_w4a8_gemv(xq.data_ptr(), sx.data_ptr(), M, K, N, group, _mode(mode), image.data_ptr(), Y.data_ptr(), _dt(Y),
                  _stream())
    return Y


def w4a8_gemv_grouped(problems, group, mode, y_dtype="f16"):
    """Batch-1 W4A8 GEMVs in one launch. problems: [(xq [1, K], sx [1, K/32],
    image, N), ...] with a common K; returns the list of Y [1, N]."""
    K = problems[0][0].shape[1]
    Ys, rows = [], []
    for xq, sx, img, N in problems:
        _need_cuda(xq, sx, img)
        if xq.shape != (1, K):
            raise ValueError("grouped GEMVs need xq [1, K] of one K")
        Y = _out_dt(1, N, y_dtype, xq.device)
        Ys.append(Y)
        rows.append((xq.data_ptr(), sx.data_ptr(), img.data_ptr(), Y.data_ptr(), N))
    lbq_w4a8_gemv_grouped(make_w4a8_items(rows), len(rows), K, group, _mode(mode), _dt(Ys[0]), _stream())
    return Ys


MOE_BLOCK = 128  # rows per tile of the grouped GEMM = the alignment block


def moe_align(topk_ids, num_experts, expert_map=None, block=MOE_BLOCK):
    """(sorted_ids int32 [max_padded], expert_ids int32 [max_padded / block],
    total int32 [1]) on the device for topk_ids int32 [T, top_k]."""
    torch = _torch()
    _need_cuda(topk_ids, expert_map)
    P = topk_ids.numel()
    mp = lbq_moe_max_padded(P, num_experts, block)
    s = torch.empty(mp, dtype=torch.int32, device=topk_ids.device)
    e = torch.empty(mp // block, dtype=torch.int32, device=topk_ids.device)
    t = torch.empty(1, dtype=torch.int32, device=topk_ids.device)
    lbq_moe_align(topk_ids.data_ptr(), P, num_experts, block, expert_map.data_ptr() if expert_map is not None else None,
                  s.data_ptr(), e.data_ptr(), t.data_ptr(), mp, _stream())
    return s, e, t


def pack_lut3_experts(experts):
    """One uint8 buffer holding every expert's LUT3 image at a fixed stride:
    experts = [(idx, codebooks, exponents), ...] (CUDA tensors, one K, N).
    Returns (images, stride)."""
    torch = _torch()
    K, N = experts[0][0].shape
    size = lbq_packed_size(K, N, 0, MODES["lut3"])
    stride = -(-size // 256) * 256
    buf = torch.empty(stride * len(experts), dtype=torch.uint8, device=experts[0][0].device)
    for i, (idx, cb, ex) in enumerate(experts):
        _need_cuda(idx, cb, ex)
        lbq_pack_lut3(idx.data_ptr(), cb.data_ptr(), ex.data_ptr(), K, N, buf.data_ptr() + i * stride, stride,
                      _stream())
    return buf, stride


def moe_lut3_mx_gemm(codes, scales, top_k, aligned, images, stride, num_local_experts, N, y_dtype="bf16", Y=None):
    """Y [T * top_k, N] of the grouped GEMM; aligned = moe_align(...) with block 128."""
    torch = _torch()
    sorted_ids, expert_ids, total = aligned
    _need_cuda(codes, scales, sorted_ids, expert_ids, total, images, Y)
    T, K = codes.shape
    Y = _out_dt(T * top_k, N, y_dtype, codes.device) if Y is None else Y
    lbq_moe_lut3_mx_gemm(codes.data_ptr(), scales.data_ptr(), T, top_k, K, N, sorted_ids.data_ptr(),
                         expert_ids.data_ptr(), total.data_ptr(), sorted_ids.numel(), images.data_ptr(), stride,
                         num_local_experts, Y.data_ptr(), _dt(Y), _stream())
    return Y


def device_status():
    lbq_device_status(_stream())
