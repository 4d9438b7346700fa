"""Plain CPU oracle for the fused low-bit weight dequantize + matmul.

TEST INFRASTRUCTURE ONLY. Nothing in the product package imports, calls or
links anything here; only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may use it.

What it computes, and where each step comes from:

* ``oracle.int4``   -- group-wise INT4 quantisation (symmetric ``(q-8)*s`` and
  asymmetric ``(q-zp)*s`` with an int8 zero point), the canonical two-nibbles-
  per-byte packing (low nibble = even k) and the exact FP32 dequantisation.
  Sources: "Low Bit Metal Kernels" (INT4 dequant + matmul listing) and
  "Low Bit ARM kernels" (group-wise scale section).
* ``oracle.lut3``   -- the 3-bit LUT format: a 3-bit index into an 8-entry E4M3
  codebook shared by a tile of 8 output channels x 64 K, scaled by one UE8M0
  exponent per tile; its canonical index bit stream and its exact decode.
  Source: vLLM PR 62759 write-up (format section; tile and memory budget).
* ``oracle.mxfp8``  -- MXFP8 activations (E4M3 elements, one UE8M0 scale per
  32 k) and the LUT3 x MXFP8 product: the activation format of the same page's
  native and emulated LUT-B paths (the next row after the BF16 LUT3 path).
* ``oracle.affine`` -- generic b-bit (1..8) affine group-wise weights: the
  quantiser, the canonical per-column little-endian bit stream and the exact
  dequantisation ("Low Bit ARM kernels": one kernel per bit width in a
  bit-width x tile table; group-wise scale and zero point).
* ``oracle.w4a8``   -- dynamic INT8 activations (symmetric, one FP32 scale per
  32-k block of a row) and the W4A8 product from exact integer block sums
  ("Low Bit ARM kernels": 4-bit weights with dynamic INT8 activations, group
  32, integer inner loop, group scales applied after it).
* ``oracle.moe``    -- the grouped MoE GEMM of LUT3 experts with MXFP8
  activations: moe_align_block_size (expert-sorted, block-padded pair lists)
  and the gathered product with zero rows for non-local experts (vLLM PR
  62759 write-up, gather and expert-parallelism sections).
* ``oracle.matmul`` -- Y = X . W accumulated in FP64, the error scale
  S = |X| . |W|, and the acceptance test |y - y_ref| <= 4e-3*S + ulp16(|y_ref|).

Everything is plain numpy in FP64 (FP32 where the pages fix a quantity that
decides an integer code, so that both sides take that decision in the same
precision). The oracle shares no code with the CUDA path.

Parity status: every function here is pinned by ``tests/test_oracle.py``
(hand examples in ``tests/golden/``, exact rational brute force, library
decoders, nearest-level characterisation of the quantiser). Quantisation
*quality* (MSE, task accuracy) is not modelled: parity unpinned for that,
and it is out of scope.
"""

from . import affine, int4, lut3, matmul, moe, mxfp8, w4a8  # noqa: F401
