/*
 * lbq.h -- low-bit weight-only GEMV / GEMM for NVIDIA B200 (sm_100a).
 *
 * The operation (problem statement of "Low Bit Metal Kernels", INT4 dequant +
 * matmul listing):  Y[M, N] = X[M, K] . dequant(Wq)[K, N],
 * X and Y row-major FP16 or BF16, FP32 accumulation, Y rounded to nearest.
 *
 * Two weight formats:
 *  - INT4, two codes per byte, one FP16 scale per group of `group` (32, 64,
 *    128) consecutive k of a column, symmetric value (q - 8) * s or asymmetric
 *    value (q - zp) * s with an int8 zero point ("Low Bit Metal Kernels",
 *    dequant lines of the INT4 listing; "Low Bit ARM kernels", group-wise
 *    scale section).
 *  - LUT3: a 3-bit index into an 8-entry E4M3 codebook shared by a tile of 8
 *    output channels x 64 k, times one UE8M0 exponent 2^(E-127) per tile
 *    (vLLM PR 62759 write-up, format section).
 *
 * Conventions for every call:
 *  - Pointers marked (device) are CUDA device pointers, (host) host pointers.
 *    The caller owns and allocates every buffer; the library never allocates
 *    device memory and keeps no pointer after a call returns.
 *  - Calls that take a `stream` only enqueue work on it (cudaStream_t passed as
 *    void*, 0 = legacy default stream) and return without synchronising. They
 *    are safe to capture in a CUDA graph.
 *  - Every call returns an lbq_status. On failure nothing is enqueued and
 *    lbq_last_error() (thread-local) describes the cause. The library never
 *    throws, aborts or exits.
 *  - Compute calls trust that K, N, group and mode match the image (checking
 *    the device header would cost a dependent memory round trip per launch);
 *    the debug calls (unpack / dequant) do read and check the header.
 *  - A kernel that detects a problem on the device (a pipeline wait that ran
 *    past its bound) abandons its work and raises a flag that
 *    lbq_device_status() reports; no kernel waits without a bound.
 *  - Device pointers must be 16-byte aligned; K, N, M must be > 0 unless stated.
 *
 * The device image (what lbq_pack / lbq_pack_lut3 write) is an opaque blob of
 * lbq_packed_size() bytes: a 256-byte header followed by the repacked codes,
 * scales and zero points (or LUT3 indices, codebooks and exponents). Its
 * layout is fixed by this library version; lbq_unpack_canonical /
 * lbq_unpack_lut3_canonical recover the canonical arrays from it bit-exactly.
 */
#ifndef LBQ_H
#define LBQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  LBQ_OK = 0,
  LBQ_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, bad size, buffer too small */
  LBQ_ERR_UNSUPPORTED = 2,  /* a combination this version does not implement */
  LBQ_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed */
  LBQ_ERR_DEVICE = 4        /* a kernel reported a problem (lbq_device_status) */
} lbq_status;

typedef enum { LBQ_MODE_SYM = 0, LBQ_MODE_ASYM = 1, LBQ_MODE_LUT3 = 2, LBQ_MODE_AFFINE = 3 } lbq_mode;
typedef enum { LBQ_DTYPE_F16 = 0, LBQ_DTYPE_BF16 = 1 } lbq_dtype;

/* Human-readable description of the last failure on the calling thread. */
const char* lbq_last_error(void);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int lbq_version(void);

/*
 * Size in bytes of the device image for a K x N weight in `mode`.
 * INT4 (SYM/ASYM): group in {32, 64, 128}, K % group == 0, N >= 1. The
 *   format holds two codes per byte ("Low Bit Metal Kernels", INT4 listing:
 *   one byte = two nibbles) plus one FP16 scale, and for ASYM one int8 zero
 *   point, per group of a column ("Low Bit ARM kernels", group-wise scale
 *   section): K*N/2 + (K/group)*N*(2 or 3) bytes. The image adds a 256-byte
 *   header, 256-byte region alignment and the scales / zero points padded to
 *   128-channel tiles.
 * LUT3: group is ignored (pass 0), K % 64 == 0, N % 8 == 0. The format is a
 *   3-bit index per weight, 8 E4M3 codebook bytes and one UE8M0 exponent per
 *   8-channel x 64-k tile: 3 + 72/512 = 3.140625 bits per weight, the write-up's
 *   "about 3.14 bits/weight", with 6144 index bytes per 128 x 128 block (vLLM
 *   PR 62759 write-up, format section and its tile / memory budget). The image
 *   adds the header, a 16-byte BF16 table per tile and alignment.
 * Writes *bytes (host). No device work. Errors: LBQ_ERR_UNSUPPORTED for an
 * unknown mode or group, LBQ_ERR_INVALID_ARG for sizes the format cannot hold
 * or a null `bytes`.
 */
lbq_status lbq_packed_size(int K, int N, int group, int mode, size_t* bytes);

/*
 * Quantise and repack an FP32 weight into the device image (INT4 only).
 *   W      (device) float32 [K, N] row-major, the logical weight of Y = X . W.
 *   image  (device) lbq_packed_size() bytes, written entirely.
 * Quantisation ("Low Bit ARM kernels", group-wise scale section; formulas of
 * the INT4 listing in "Low Bit Metal Kernels"), per group of `group` k of a
 * column n, all in IEEE FP32 with round-half-to-even:
 *   SYM : s = fp16(max|w| / 7);           q = clamp(rint(w / s) + 8, 0, 15)
 *   ASYM: s = fp16((max w - min w) / 15); zp = clamp(rint(-min w / s), -128, 127);
 *         q = clamp(rint(w / s) + zp, 0, 15)
 * where s in the divisions is the stored FP16 scale widened to FP32; a group
 * whose stored scale is 0 gets q = 8 (SYM) or zp = 0, q = 0 (ASYM).
 * W must be finite. Asynchronous on `stream`.
 */
lbq_status lbq_pack(const float* W, int K, int N, int group, int mode,
                    void* image, size_t image_bytes, void* stream);

/*
 * Build a LUT3 device image from the format's canonical arrays (vLLM PR 62759
 * write-up, format section).
 *   idx        (device) uint8 [K, N], values 0..7 (weight (k, n)'s index)
 *   codebooks  (device) uint8 [K/64, N/8, 8]  E4M3 ("fn") bytes per tile
 *   exponents  (device) uint8 [K/64, N/8]     UE8M0 bytes per tile (bias 127)
 * Weight value = e4m3(codebooks[k/64][n/8][idx[k][n]]) * 2^(exponents[k/64][n/8] - 127).
 * Indices > 7 are taken modulo 8; NaN codebook bytes (0x7F/0xFF) and NaN
 * exponents (0xFF) are the caller's responsibility (they decode to NaN).
 * The BF16-activation kernels (lbq_lut3_gemm) decode through a per-tile BF16
 * table that holds every weight exactly for 3 <= exponent <= 246 (E4M3
 * magnitudes 2^-9 .. 448 times 2^(E-127) inside BF16's 2^-133 .. 2^128);
 * outside that range its entries are the weights rounded to BF16 (down to 0,
 * up to infinity at the extremes). The MXFP8 kernels read the format's own
 * bytes and are exact for every exponent. Asynchronous on `stream`.
 */
lbq_status lbq_pack_lut3(const uint8_t* idx, const uint8_t* codebooks, const uint8_t* exponents,
                         int K, int N, void* image, size_t image_bytes, void* stream);

/*
 * Workspace needed by lbq_gemv / lbq_gemm / lbq_lut3_gemm for this shape:
 * the split-K partial sums and tile counters of the dispatch the library
 * would pick. Decode at batch 1 is a GEMV whose rows are split over many
 * lanes and reduced ("Low Bit ARM kernels": decode is a GEMV; "BaseRT",
 * kernel-selection section: SIMD groups share one weight row); when the rows
 * alone cannot fill the 148 SMs the K range is split as well, and the slices'
 * FP32 partial sums meet here. op: 0 = lbq_gemv, 1 = lbq_gemm, 2 = lbq_lut3_gemm.
 * Writes *bytes (host); 0 means the call needs no workspace (ws may be null).
 * The workspace's tile counters must be zero when a call starts: zero-fill a
 * new workspace before its first use; every call that completes returns its
 * counters to zero (its partial sums are left behind), so one buffer can be
 * reused by consecutive calls of the same shape on one stream (not by calls
 * running concurrently). Reusing it for another shape needs a new zero fill.
 */
lbq_status lbq_workspace_size(int op, int M, int K, int N, int group, int mode, size_t* bytes);

/*
 * Decode GEMV / skinny GEMM on INT4 weights, 1 <= M <= 16.
 *   X      (device) [M, K] row-major, x_dtype (LBQ_DTYPE_F16 / BF16)
 *   image  (device) from lbq_pack with the same K, N, group, mode
 *   Y      (device) [M, N] row-major, y_dtype, fully overwritten
 *   ws     (device) >= lbq_workspace_size(0, ...) bytes, zero-filled (see above)
 * y[m][n] = sum_k x[m][k] * (q[k][n] - z) * s[k/group][n], accumulated in FP32
 * ("Low Bit ARM kernels": decode at batch 1 is a GEMV; the page's Metal
 * kernel does the dequantisation inside the inner loop). Asynchronous.
 */
lbq_status lbq_gemv(const void* X, int x_dtype, int M, int K, int N, int group, int mode,
                    const void* image, void* Y, int y_dtype, void* ws, size_t ws_bytes,
                    void* stream);

/*
 * Several batch-1 INT4 GEMVs in one launch, e.g. the projections of a decoder
 * layer that read the same activation vector (q, k, v; gate, up). Item i:
 *   X      (device) [1, K], x_dtype
 *   image  (device) from lbq_pack with K, items[i].N, group, mode
 *   Y      (device) [1, items[i].N], y_dtype, fully overwritten
 * items is a host array of 1..4 entries; all share K (<= 16384), group, mode
 * and the dtypes. No workspace. The result of each item equals that of
 * lbq_gemv with M = 1 on it. Asynchronous on `stream`.
 */
typedef struct {
  const void* X;
  const void* image;
  void* Y;
  int N;
} lbq_gemv_item;
lbq_status lbq_gemv_grouped(const lbq_gemv_item* items, int count, int K, int group, int mode,
                            int x_dtype, int y_dtype, void* stream);

/*
 * Prefill GEMM on INT4 weights, any M >= 1 (M <= 16 is routed to lbq_gemv's
 * kernels). Same arguments and result as lbq_gemv; X may be FP16 or BF16.
 * For M > 16 the weights are dequantised into the activation type ((q - z)
 * formed exactly, the product with the scale rounded once) straight into
 * tensor memory and multiplied on the tcgen05 tensor cores with FP32
 * accumulation ("Low Bit Metal Kernels": dequantise just before the
 * multiply). For M > 16 the workspace is optional: where the 128-channel x
 * 256-token output tiles leave the SMs' last wave part-filled,
 * lbq_workspace_size(1, ...) is non-zero, and with a workspace of that size
 * the last two waves' tiles are cut along K between neighbouring CTAs (one
 * FP32 tile and one flag per CTA; the two parts are added in a fixed order,
 * so results do not depend on timing). With ws null or smaller every tile is
 * computed whole. A part that waits about 4 s for its partner gives up and
 * raises LBQ_ERR_DEVICE (lbq_device_status); zero-fill the workspace again
 * after that. Asynchronous.
 */
lbq_status lbq_gemm(const void* X, int x_dtype, int M, int K, int N, int group, int mode,
                    const void* image, void* Y, int y_dtype, void* ws, size_t ws_bytes,
                    void* stream);

/*
 * GEMV / GEMM on LUT3 weights (image from lbq_pack_lut3), any M >= 1.
 * X must be BF16. y[m][n] = sum_k x[m][k] * w[k][n] with w the decoded
 * LUT3 value (exact in BF16 for the exponents the format's workloads use).
 * ws: lbq_workspace_size(2, ...) bytes, zero-filled; required by the
 * skinny kernel's split-K (M <= 16), optional for M > 16 (the prefill's
 * cut tiles, as lbq_gemm).
 */
lbq_status lbq_lut3_gemm(const void* X, int x_dtype, int M, int K, int N,
                         const void* image, void* Y, int y_dtype, void* ws, size_t ws_bytes,
                         void* stream);

/*
 * Debug / parity: recover the canonical arrays from an INT4 image, the exact
 * inverse of the repack: two codes per byte with the low nibble the even k
 * ("Low Bit Metal Kernels", INT4 listing: the low nibble is taken first), the
 * FP16 scale and int8 zero point per group ("Low Bit ARM kernels", group-wise
 * scale section). Reads and checks the image header (synchronous 64-byte copy);
 * LBQ_ERR_INVALID_ARG if it does not match K, N, group, mode.
 *   q_packed (device) uint8 [K/2, N]: byte[j][n] = q[2j][n] | q[2j+1][n] << 4
 *   scales   (device) uint16 [K/group, N]: FP16 bit patterns
 *   zp       (device) int8 [K/group, N] (ASYM; may be null, ignored for SYM)
 */
lbq_status lbq_unpack_canonical(const void* image, int K, int N, int group, int mode,
                                uint8_t* q_packed, uint16_t* scales, int8_t* zp, void* stream);

/*
 * Debug / parity: recover the canonical LUT3 arrays from a LUT3 image (the
 * format of the vLLM PR 62759 write-up, format section: 3-bit indices, 8 E4M3
 * codebook bytes and one UE8M0 exponent per 8-channel x 64-k tile). Reads and
 * checks the image header; LBQ_ERR_INVALID_ARG if it does not match K, N.
 *   idx_stream (device) uint8 [K/64, N/8, 8, 24]: per tile and channel, the 64
 *              indices as a little-endian 192-bit string, index i in bits [3i, 3i+3)
 *   codebooks  (device) uint8 [K/64, N/8, 8];  exponents (device) uint8 [K/64, N/8]
 */
lbq_status lbq_unpack_lut3_canonical(const void* image, int K, int N, uint8_t* idx_stream,
                                     uint8_t* codebooks, uint8_t* exponents, void* stream);

/*
 * Debug / parity: the exact dequantised weight, W_out (device) float32 [K, N].
 * INT4: (q - z) * s ("Low Bit Metal Kernels", INT4 listing: (nibble - 8) *
 * scale; "Low Bit ARM kernels": (q - zp) * s with a zero point);
 * LUT3: e4m3(cb) * 2^(E-127) (vLLM PR 62759 write-up, format section).
 * Both are exact in FP32. Reads and checks the image header.
 */
lbq_status lbq_dequant(const void* image, int K, int N, int group, int mode,
                       float* W_out, void* stream);

/*
 * Synchronise `stream` and report (then clear) the device-side error flag the
 * kernels raise on this device: LBQ_OK, or LBQ_ERR_DEVICE with the reason in
 * lbq_last_error().
 */
lbq_status lbq_device_status(void* stream);

/*
 * Process-wide launch options.
 *   LBQ_OPT_PDL (value 0/1, default 0): launch the GEMV kernels with
 *   programmatic dependent launch. A kernel may then start, and stream its
 *   weight image, while the previous kernel in the stream is still running;
 *   it reads X and writes Y only after that kernel has completed. Enable it
 *   only when no preceding kernel in the stream writes the image (images are
 *   normally written once by lbq_pack and then only read), e.g. for the
 *   back-to-back projections of a decode step.
 */
typedef enum { LBQ_OPT_PDL = 1 } lbq_option;
lbq_status lbq_set_option(int option, int value);

/*
 * lbq_gemv without a caller-provided workspace: same arguments (minus ws,
 * ws_bytes), same kernels, same result. The pages describe no such call; it
 * serves callers that cannot give the library device memory (a plain C
 * program without a device allocator, or a process whose device memory is
 * partitioned once at start-up). Nothing is allocated or freed, ever.
 *   Scratch: one fixed module-level device array of 8 MiB per device, placed
 *   by the CUDA runtime when it loads the library's module. A call whose
 *   dispatch needs more (roughly (296 + 2 * ceil(N/128)) * M * 512 bytes for
 *   2 <= M <= 16) fails with LBQ_ERR_UNSUPPORTED and launches nothing; use
 *   lbq_gemv with a workspace for it.
 *   Zero state: nothing has to be zero beforehand; each call clears the tile
 *   counters it will use (one memset on `stream`) before its kernel.
 *   Address: outside stream capture every call looks the array's device
 *   address up (cheap once loaded; a module reloaded after cudaDeviceReset
 *   is found at its new place). Under capture the address of the last
 *   uncaptured call on the device is used, so the first call on each device
 *   must come before any capture (LBQ_ERR_INVALID_ARG otherwise), and a
 *   cudaDeviceReset must be followed by an uncaptured call before capturing.
 *   Concurrency: all calls on one device share the one array, so two calls
 *   whose work can overlap (different streams, or host threads racing on one
 *   stream) corrupt each other's partial sums. Serialise them.
 * Asynchronous on `stream`.
 */
lbq_status lbq_gemv_noalloc(const void* X, int x_dtype, int M, int K, int N, int group, int mode,
                            const void* image, void* Y, int y_dtype, void* stream);

/*
 * MXFP8 quantisation of activations (vLLM PR 62759 write-up: MXFP8
 * activations = E4M3 elements with one UE8M0 scale per 1 x 32 block; OCP MX
 * element and scale types): the activation side of a LUT3 x MXFP8 product.
 *   X      (device) [M, K] row-major FP16 / BF16 (x_dtype), finite, 16-byte aligned
 *   K      a multiple of 32; block b of row m is k = 32 b .. 32 b + 31
 *   codes  (device) uint8 [M, K], E4M3 bytes, 16-byte aligned
 *   scales (device) uint8 [M, K/32], UE8M0 bytes
 * Per block: scale byte = floor(log2 amax) - 8 + 127 clamped to [0, 254]
 * (127 for an all-zero block), amax its largest |x|; each element is
 * x * 2^(127 - byte) rounded to nearest E4M3, ties to even, saturating at
 * +-448 (zeros keep their sign). Bit-identical to the CPU reference.
 * Asynchronous on `stream`; argument errors are reported before any launch.
 */
lbq_status lbq_quantize_mxfp8(const void* X, int x_dtype, int M, int K, uint8_t* codes, uint8_t* scales,
                              void* stream);

/*
 * LUT3 weights x MXFP8 activations on the block-scaled FP8 tensor path (vLLM
 * PR 62759 write-up: LUT-B weights with MXFP8 activations, E4M3 elements and
 * one UE8M0 scale per 1 x 32 block; its format section: the tile's UE8M0
 * exponent maps onto the weight operand's per-32-k block scale). The decoded
 * weight of a LUT3 index is its codebook's E4M3 byte, the tile exponent its
 * block scale, so the product runs as tcgen05.mma.kind::mxf8f6f4.block_scale
 * with every product exact and FP32 accumulation:
 *   y[m][n] = sum_k e4m3(codes[m][k]) 2^(scales[m][k/32] - 127)
 *                   * e4m3(cb[k/64][n/8][idx[k][n]]) 2^(E[k/64][n/8] - 127)
 *   codes  (device) uint8 [M, K], E4M3 bytes (e.g. from lbq_quantize_mxfp8)
 *   scales (device) uint8 [M, K/32], UE8M0 bytes
 *   image  (device) from lbq_pack_lut3 with this K, N
 *   Y      (device) [M, N] row-major, y_dtype, fully overwritten
 *   ws     (device) optional, lbq_workspace_size(2, M, K, N, 0, LBQ_MODE_LUT3)
 *          bytes, zero-filled (see lbq_workspace_size): with it the tail
 *          wave's tiles are cut along K as in lbq_gemm; null (or smaller)
 *          computes every tile whole
 * K % 512 == 0 (the block scales are read 16 bytes, 512 k, at a time), N % 8
 * == 0, M >= 1; every pointer 16-byte aligned. NaN codes (0x7F / 0xFF) or scale
 * bytes (0xFF) give NaN outputs. Errors: LBQ_ERR_INVALID_ARG for null or
 * misaligned pointers or bad sizes, LBQ_ERR_UNSUPPORTED for K % 512 != 0 or an
 * unknown y_dtype, before any launch. Asynchronous on `stream`.
 */
lbq_status lbq_lut3_mx_gemm(const uint8_t* codes, const uint8_t* scales, int M, int K, int N, const void* image,
                            void* Y, int y_dtype, void* ws, size_t ws_bytes, void* stream);

/*
 * Generic b-bit affine weights, b = 1..8 ("Low Bit ARM kernels": one GEMV
 * micro-kernel and one unpack routine per bit width 1..8 in a bit-width x tile
 * table; 3-bit weights as an accuracy point between 2 and 4 bits; the
 * group-wise scale section for the affine form). A weight is a code q in
 * 0 .. 2^bits - 1 with value (q - zp) * s, one FP16 scale s and one int8 zero
 * point zp per group of `group` (32, 64, 128) consecutive k of a column.
 * bits = 4 is the asymmetric INT4 format in another image layout.
 *
 * lbq_affine_packed_size: size of the device image, K*N*bits/8 code bytes
 *   plus the scales and zero points padded to 128-channel tiles, a 256-byte
 *   header and 256-byte region alignment. Writes *bytes (host); no device work.
 *   Errors: LBQ_ERR_UNSUPPORTED for bits outside 1..8 or group outside
 *   {32, 64, 128}; LBQ_ERR_INVALID_ARG for K % group != 0, K or N <= 0, or a
 *   null `bytes`.
 */
lbq_status lbq_affine_packed_size(int K, int N, int group, int bits, size_t* bytes);

/*
 * Quantise and repack an FP32 weight into a b-bit affine image.
 *   W      (device) float32 [K, N] row-major, finite, 16-byte aligned
 *   image  (device) lbq_affine_packed_size() bytes, written entirely
 * Per group of a column, in IEEE FP32 with round-half-to-even, L = 2^bits - 1:
 *   s = fp16((max w - min w) / L); zp = clamp(rint(-min w / s), -128, 127);
 *   q = clamp(rint(w / s) + zp, 0, L)
 * (s in the divisions is the stored FP16 scale widened to FP32; a group whose
 * stored scale is 0 gets zp = 0, q = 0). Asynchronous on `stream`.
 */
lbq_status lbq_pack_affine(const float* W, int K, int N, int group, int bits, void* image, size_t image_bytes,
                           void* stream);

/*
 * Decode GEMV on b-bit affine weights, 1 <= M <= 16:
 *   Y[m][n] = sum_k X[m][k] (q[k][n] - zp) s, FP32 accumulation, Y rounded to
 *   nearest in y_dtype.
 *   X      (device) [M, K] row-major, x_dtype (LBQ_DTYPE_F16 / BF16), finite
 *   image  (device) from lbq_pack_affine with this K, N, group, bits
 *   Y      (device) [M, N] row-major, y_dtype, fully overwritten
 * K <= 16384. X is read in tiles of up to 4 rows (one launch per tile; each
 * launch streams the whole weight once). No workspace. Errors:
 * LBQ_ERR_INVALID_ARG / LBQ_ERR_UNSUPPORTED before any launch, as above, and
 * LBQ_ERR_UNSUPPORTED for M > 16 or K > 16384. Asynchronous on `stream`.
 */
lbq_status lbq_affine_gemv(const void* X, int x_dtype, int M, int K, int N, int group, int bits, const void* image,
                           void* Y, int y_dtype, void* stream);

/*
 * Recover the canonical arrays of a b-bit affine image bit-exactly (debug /
 * parity). Reads and checks the image header (a synchronous 64-byte copy).
 *   q_stream (device) uint8 [K*bits/8, N]: per column n one little-endian bit
 *            stream, code k at bits [bits*k, bits*k + bits); byte j of column
 *            n's stream at q_stream[j][n]
 *   scales   (device) uint16 [K/group, N] FP16 bits
 *   zp       (device) int8 [K/group, N]
 * Errors: LBQ_ERR_INVALID_ARG for null pointers or a header that does not
 * match the call. The copy-out kernels run asynchronously on `stream`.
 */
lbq_status lbq_unpack_affine_canonical(const void* image, int K, int N, int group, int bits, uint8_t* q_stream,
                                       uint16_t* scales, int8_t* zp, void* stream);

/*
 * Dynamic INT8 activations for W4A8 ("Low Bit ARM kernels": 4-bit weights
 * with dynamic INT8 activations, group size 32, an integer inner loop with
 * int32 accumulation and the group scales applied after it). Each row of X is
 * quantised in blocks of 32 consecutive k, symmetric, in IEEE FP32:
 *   s = amax / 127 (amax the block's largest |x|);
 *   xq = clamp(rint(x / s), -127, 127), ties to even; an all-zero block has
 *   s = 0 and xq = 0.
 *   X   (device) [M, K] row-major, x_dtype (LBQ_DTYPE_F16 / BF16), finite
 *   xq  (device) int8 [M, K], 16-byte aligned
 *   sx  (device) float32 [M, K/32]
 * K % 32 == 0. Bit-identical to the CPU reference. Errors: LBQ_ERR_INVALID_ARG
 * for null or misaligned pointers or bad sizes, LBQ_ERR_UNSUPPORTED for an
 * unknown x_dtype, before any launch. Asynchronous on `stream`.
 */
lbq_status lbq_quantize_int8(const void* X, int x_dtype, int M, int K, int8_t* xq, float* sx, void* stream);

/*
 * W4A8 decode GEMV, 1 <= M <= 16: INT4 weights (an lbq_pack image, SYM or
 * ASYM) times INT8 activations from lbq_quantize_int8 ("Low Bit ARM kernels":
 * the integer inner loop with int32 accumulation, group scales after it). Per
 * 32-k block b of row m and column n the integer sum
 * I = sum xq q - z sum xq is exact (z = 8 for SYM, the zero point for ASYM), and
 *   Y[m][n] = sum_b sx[m][b] s_w[group of b][n] I[m][b][n]
 * accumulated in FP32, rounded to nearest in y_dtype.
 *   xq     (device) int8 [M, K], 16-byte aligned
 *   sx     (device) float32 [M, K/32]
 *   image  (device) from lbq_pack with this K, N, group, mode
 *   Y      (device) [M, N] row-major, y_dtype, fully overwritten
 * K <= 16384. M = 1 runs as the staged batch-1 kernel; larger M in tiles of
 * up to 4 rows (one launch per tile; each launch streams the whole weight
 * once). No workspace. Errors: LBQ_ERR_INVALID_ARG / LBQ_ERR_UNSUPPORTED for
 * bad pointers, sizes or modes, M > 16 or K > 16384, before any launch.
 * Asynchronous on `stream`.
 */
lbq_status lbq_w4a8_gemv(const int8_t* xq, const float* sx, int M, int K, int N, int group, int mode,
                         const void* image, void* Y, int y_dtype, void* stream);

/*
 * Several batch-1 W4A8 GEMVs in one launch (the projections of a decoder
 * layer that read the same activation vector, quantised once). Item i:
 *   xq, sx (device) [1, K] INT8 codes and [1, K/32] scales (lbq_quantize_int8)
 *   image  (device) from lbq_pack with K, items[i].N, group, mode
 *   Y      (device) [1, items[i].N], y_dtype, fully overwritten
 * items is a host array of 1..4 entries sharing K (<= 16384), group and mode;
 * each item's result equals lbq_w4a8_gemv with M = 1 on it. No workspace.
 * Errors as lbq_w4a8_gemv, before any launch. Asynchronous on `stream`.
 */
typedef struct {
  const int8_t* xq;
  const float* sx;
  const void* image;
  void* Y;
  int N;
} lbq_w4a8_item;
lbq_status lbq_w4a8_gemv_grouped(const lbq_w4a8_item* items, int count, int K, int group, int mode, int y_dtype,
                                 void* stream);

/*
 * Grouped MoE GEMM of LUT3 expert weights with MXFP8 activations (vLLM PR
 * 62759 write-up: the native grouped GEMM gathers token rows through
 * sorted_token_ids from moe_align_block_size, takes one expert per M block,
 * zero-fills the A rows of padding entries through the copy's source size,
 * and writes zeros for the rows of a block whose expert is not on this rank).
 *
 * Pairs: pair p = t * top_k + j is token t's j-th choice, routed to expert
 * topk_ids[p]; P = T * top_k pairs.
 *
 * lbq_moe_max_padded: *max_padded = the largest `total` lbq_moe_align can
 *   produce, (P + min(P, E) (block - 1)) rounded down to a multiple of block:
 *   the length to allocate for sorted_ids (and max_padded / block for
 *   expert_ids). Host only. Errors: LBQ_ERR_INVALID_ARG for non-positive
 *   arguments or a list longer than 2^30.
 */
lbq_status lbq_moe_max_padded(int num_pairs, int num_experts, int block, int* max_padded);

/*
 * moe_align_block_size on the device (one CTA):
 *   topk_ids    (device) int32 [num_pairs], expert of each pair, 0 <= id < num_experts
 *               (other ids are left out of the lists; their output rows are not written)
 *   expert_map  (device) int32 [num_experts] global -> local expert (negative: not on
 *               this rank), or null for the identity
 *   sorted_ids  (device) int32 [max_padded]: each expert's pair ids contiguous (experts in
 *               ascending id, the pairs of one expert in no fixed order), each run padded
 *               to a multiple of `block` with the id num_pairs, which also fills the
 *               entries past the total
 *   expert_ids  (device) int32 [max_padded / block]: the (mapped) expert of each block,
 *               -1 past the total
 *   total       (device) int32 scalar: entries in use
 * num_experts <= 2048; max_padded >= lbq_moe_max_padded(). Errors before any
 * launch: LBQ_ERR_INVALID_ARG. Asynchronous on `stream`.
 */
lbq_status lbq_moe_align(const int32_t* topk_ids, int num_pairs, int num_experts, int block, const int32_t* expert_map,
                         int32_t* sorted_ids, int32_t* expert_ids, int32_t* total, int max_padded, void* stream);

/*
 * The grouped GEMM, tile of 128 sorted rows (lbq_moe_align with block = 128):
 *   Y[p][n] = sum_k e4m3(codes[p / top_k][k]) 2^(scales[p / top_k][k/32] - 127) * W_e[k][n]
 * for every pair p listed in a block whose local expert e is in
 * 0 .. num_local_experts - 1 (W_e the LUT3 decode of expert e's image, every
 * product exact, FP32 accumulation); Y[p][:] = 0 for pairs of a block with a
 * negative (or too large) expert id. Rows of pairs that are not listed are not written.
 *   codes, scales (device) uint8 [T, K] E4M3 and [T, K/32] UE8M0 (lbq_quantize_mxfp8)
 *   sorted_ids, expert_ids, total (device) from lbq_moe_align(block = 128)
 *   images  (device) local expert e's lbq_pack_lut3 image (K, N) at images + e * image_stride
 *   Y       (device) [T * top_k, N] row-major, y_dtype
 * K % 128 == 0, K <= 8192, N % 8 == 0; max_padded the value the lists were sized with
 * (a multiple of 128); pointers and image_stride 16-byte aligned. Errors
 * before any launch: LBQ_ERR_INVALID_ARG / LBQ_ERR_UNSUPPORTED. Asynchronous
 * on `stream`.
 */
lbq_status lbq_moe_lut3_mx_gemm(const uint8_t* codes, const uint8_t* scales, int T, int top_k, int K, int N,
                                const int32_t* sorted_ids, const int32_t* expert_ids, const int32_t* total,
                                int max_padded, const void* images, size_t image_stride, int num_local_experts,
                                void* Y, int y_dtype, void* stream);

/* Number of kernel launches the library has enqueued so far in this process. */
uint64_t lbq_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* LBQ_H */
