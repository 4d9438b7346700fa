"""bit_weight_only_pack_b200: fused low-bit weight dequantize + matmul on B200.

Y[M, N] = X[M, K] . dequant(Wq)[K, N] for INT4 (group-wise FP16 scales,
symmetric or asymmetric with an int8 zero point) and 3-bit LUT weights
(E4M3 codebook per 8 x 64 tile, UE8M0 exponent), as a decode GEMV / skinny
GEMM and as a tcgen05 prefill GEMM; LUT3 weights with MXFP8 activations on the
block-scaled FP8 tensor path; generic 1..8-bit affine weights as a decode GEMV;
INT4 weights with dynamic INT8 activations (W4A8) as a decode GEMV; a grouped
MoE GEMM of LUT3 experts with MXFP8 activations gathered by expert.
The work is done by liblbq.so (C ABI in include/lbq.h); this package is its
thin Python binding.
"""

from .binding import (  # noqa: F401
    DTYPES, MODES, LbqError, dequant, device_status, gemm, gemv, gemv_grouped, gemv_noalloc, make_gemv_items, lut3_gemm, lut3_mx_gemm, pack, pack_lut3, quantize_mxfp8,
    unpack_canonical, unpack_lut3_canonical, workspace,
    lbq_debug_force_splits, lbq_debug_force_skinny, lbq_debug_force_tc, lbq_debug_gemv_path, lbq_debug_gemm_path, lbq_debug_direct_variant, lbq_debug_tmma_default, lbq_debug_tmma_split, lbq_debug_drop_copies, lbq_dequant, lbq_device_status, lbq_gemm, lbq_gemv, lbq_gemv_grouped, lbq_gemv_noalloc, lbq_last_error,
    lbq_launch_count, lbq_lut3_gemm, lbq_pack, lbq_set_option, LBQ_OPT_PDL, lbq_pack_lut3, lbq_packed_size, lbq_unpack_canonical,
    lbq_unpack_lut3_canonical, lbq_version, lbq_workspace_size, lbq_quantize_mxfp8, lbq_lut3_mx_gemm,
    affine_gemv, pack_affine, unpack_affine_canonical, lbq_affine_gemv, lbq_affine_packed_size, lbq_pack_affine,
    lbq_unpack_affine_canonical, quantize_int8, w4a8_gemv, lbq_quantize_int8, lbq_w4a8_gemv,
    w4a8_gemv_grouped, lbq_w4a8_gemv_grouped, lbq_debug_w4a8_tiled, lbq_debug_lut3_stages, lbq_debug_lut3_batch_off, lbq_debug_gemm_stream_k, lbq_debug_gemm_hold, lbq_debug_gemm_schedule, lbq_debug_tile_coords, make_w4a8_items,
    MOE_BLOCK, moe_align, moe_lut3_mx_gemm, pack_lut3_experts, lbq_moe_align, lbq_moe_lut3_mx_gemm, lbq_moe_max_padded,
)
