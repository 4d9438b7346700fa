// Shared definitions of the lbq device library: image layout, launch
// bookkeeping and the small PTX wrappers the kernels use.
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <stddef.h>

#include "lbq.h"

namespace lbq {

// Device-side error word: kernels OR a code into it; lbq_device_status()
// reads and clears it.
__device__ unsigned int g_device_error;

// ----------------------------------------------------------------------------
// Device image layout
//
// [0, 256)           header (ImageHeader, zero padded)
// INT4 (SYM / ASYM):
//   Q region         N rows of K/2 bytes. Row n holds column n of the logical
//                    [K, N] weight, k ascending, in 16-byte chunks of 32 k.
//                    Chunk c = four little-endian 32-bit words; word w holds
//                    k = 32c + 8w + i (i = 0..7) with code i in nibble slot
//                    kSlot[i] (bits 4*slot .. 4*slot+3). The slot order puts
//                    (k, k+1) pairs in the two 16-bit halves of the same mask,
//                    so one AND/OR turns two codes into a half2/bf16x2.
//   S region         FP16 scales tiled by 128 output channels: the scale of
//                    (channel n, group gi) is element ((n/128)*G + gi)*128 + n%128
//                    (G = K/group; N padded to a multiple of 128 with zeros), so
//                    the scales of one 128-channel tile for a run of groups are
//                    one contiguous block.
//   Z region (ASYM)  int8 zero points, same tiling.
// LUT3:
//   I region         indices, tile-major: [K/64][N][24 bytes] (the 64 indices
//                    of channel n in 64-k tile kt, in the order of lut3.cuh).
//   C region         codebooks, N/8 rows of K/64 x 8 E4M3 bytes (stride padded to 16).
//   E region         exponents, N/8 rows of K/64 UE8M0 bytes (stride padded to 16).
//   T region         per tile, the 8 decoded weights e4m3(cb[j]) * 2^(E-127) as
//                    BF16 in a byte-planar 16 bytes (low bytes of entries 0..7,
//                    then high bytes), [K/64][N/8][16]: what the kernels read.
//                    C and E keep the format's own bytes for exact recovery.
// AFFINE (b-bit codes, b = 1..8, in the header's `bits`):
//   Q region         N rows of K*b/8 bytes, chunks of 32 k of b 32-bit words
//                    each (layout in affine.cuh).
//   S, Z regions     FP16 scales and int8 zero points, tiled as for INT4.
// Every region starts on a 256-byte boundary.
// ----------------------------------------------------------------------------

constexpr uint32_t kMagicInt4 = 0x3451424Cu;  // "LBQ4"
constexpr uint32_t kMagicLut3 = 0x3351424Cu;  // "LBQ3"
constexpr uint32_t kMagicAffine = 0x4151424Cu;  // "LBQA"
constexpr uint32_t kImageVersion = 1;
constexpr size_t kHeaderBytes = 256;
constexpr size_t kRegionAlign = 256;

// nibble slot of the i-th k of an 8-k word: pairs (k0,k1) (k2,k3) (k4,k5) (k6,k7)
// sit in slots (0,4) (1,5) (2,6) (3,7).
__host__ __device__ constexpr int slot_of(int i) { return (i >> 1) + ((i & 1) << 2); }

struct ImageHeader {
  uint32_t magic;
  uint32_t version;
  int32_t K, N, group, mode;
  uint64_t off0, off1, off2;  // INT4: Q, S, Z   LUT3: I, C, E
  uint64_t total;
  uint64_t off3;              // LUT3: T
  int32_t bits;               // AFFINE: code width (0 for the other formats)
};
static_assert(sizeof(ImageHeader) <= kHeaderBytes, "header too large");

__host__ __device__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Element index of (channel n, group gi) in the 128-channel-tiled S / Z regions.
__host__ __device__ inline size_t meta_index(int n, int gi, int G) {
  return ((size_t)(n >> 7) * G + gi) * 128 + (n & 127);
}

struct Layout {
  int K, N, group, mode, bits;
  size_t off0, off1, off2, off3, total;
  size_t bytes0, bytes1, bytes2, bytes3;
  size_t s_stride, z_stride;  // LUT3: padded row strides (bytes) of the C and E regions
};

inline Layout make_layout(int K, int N, int group, int mode, int bits = 0) {
  Layout L{};
  L.K = K; L.N = N; L.group = group; L.mode = mode;
  L.bits = mode == LBQ_MODE_AFFINE ? bits : 0;
  if (mode == LBQ_MODE_AFFINE) {
    const size_t tiles128 = (size_t)(N + 127) / 128;
    L.bytes0 = (size_t)N * (size_t)(K / 32) * 4 * (size_t)bits;
    L.bytes1 = tiles128 * (size_t)(K / group) * 128 * 2;
    L.bytes2 = tiles128 * (size_t)(K / group) * 128;
  } else if (mode == LBQ_MODE_LUT3) {
    L.s_stride = align_up((size_t)(K / 64) * 8, 16);  // codebook row stride
    L.z_stride = align_up((size_t)(K / 64), 16);      // exponent row stride
    L.bytes0 = (size_t)N * (size_t)(K / 64) * 24;
    L.bytes1 = (size_t)(N / 8) * L.s_stride;
    L.bytes2 = (size_t)(N / 8) * L.z_stride;
    L.bytes3 = (size_t)(K / 64) * (size_t)(N / 8) * 16;
  } else {
    const size_t tiles128 = (size_t)(N + 127) / 128;
    L.bytes0 = (size_t)N * (size_t)(K / 2);
    L.bytes1 = tiles128 * (size_t)(K / group) * 128 * 2;
    L.bytes2 = mode == LBQ_MODE_ASYM ? tiles128 * (size_t)(K / group) * 128 : 0;
  }
  L.off0 = kHeaderBytes;
  L.off1 = align_up(L.off0 + L.bytes0, kRegionAlign);
  L.off2 = align_up(L.off1 + L.bytes1, kRegionAlign);
  L.off3 = align_up(L.off2 + L.bytes2, kRegionAlign);
  L.total = align_up(L.off3 + L.bytes3, kRegionAlign);
  return L;
}

inline ImageHeader make_header(const Layout& L) {
  ImageHeader h{};
  h.magic = L.mode == LBQ_MODE_LUT3 ? kMagicLut3 : L.mode == LBQ_MODE_AFFINE ? kMagicAffine : kMagicInt4;
  h.bits = L.bits;
  h.version = kImageVersion;
  h.K = L.K; h.N = L.N; h.group = L.group; h.mode = L.mode;
  h.off0 = L.off0; h.off1 = L.off1; h.off2 = L.off2; h.total = L.total; h.off3 = L.off3;
  return h;
}

// ----------------------------------------------------------------------------
// PTX wrappers
// ----------------------------------------------------------------------------

// 16-byte streaming load through the non-coherent path, no L1 allocation.
__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

// Per-thread asynchronous global -> shared copies (completion tracked per
// thread with commit/wait groups; no barrier is involved).
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;"
               :: "r"((uint32_t)__cvta_generic_to_shared(smem)), "l"(gmem), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async8(void* smem, const void* gmem) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;"
               :: "r"((uint32_t)__cvta_generic_to_shared(smem)), "l"(gmem) : "memory");
}
__device__ __forceinline__ uint2 lds64(uint32_t smem) {
  uint2 r;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(r.x), "=r"(r.y) : "r"(smem) : "memory");
  return r;
}

// The same copies with a 32-bit shared-memory address.
__device__ __forceinline__ void cp_async16_s(uint32_t smem, const void* gmem, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" :: "r"(smem), "l"(gmem), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async8_s(uint32_t smem, const void* gmem) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" :: "r"(smem), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" :: "n"(N) : "memory"); }

__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

// (a & b) | c in one LOP3.
__device__ __forceinline__ uint32_t and_or(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// acc += x.lo * w.lo + x.hi * w.hi with FP16 (or BF16) products accumulated in
// FP32 (mixed-precision FMA; the FP16 x FP16 product is exact in FP32).
__device__ __forceinline__ float fma2_f16_f32(uint32_t x2, uint32_t w2, float acc) {
  asm("{\n\t.reg .b16 xl, xh, wl, wh;\n\t"
      "mov.b32 {xl, xh}, %1;\n\t"
      "mov.b32 {wl, wh}, %2;\n\t"
      "fma.rn.f32.f16 %0, xl, wl, %0;\n\t"
      "fma.rn.f32.f16 %0, xh, wh, %0;\n\t}"
      : "+f"(acc) : "r"(x2), "r"(w2));
  return acc;
}

__device__ __forceinline__ float fma2_bf16_f32(uint32_t x2, uint32_t w2, float acc) {
  asm("{\n\t.reg .b16 xl, xh, wl, wh;\n\t"
      "mov.b32 {xl, xh}, %1;\n\t"
      "mov.b32 {wl, wh}, %2;\n\t"
      "fma.rn.f32.bf16 %0, xl, wl, %0;\n\t"
      "fma.rn.f32.bf16 %0, xh, wh, %0;\n\t}"
      : "+f"(acc) : "r"(x2), "r"(w2));
  return acc;
}

__device__ __forceinline__ float h2f_bits(uint16_t h) { return __half2float(__ushort_as_half(h)); }
__device__ __forceinline__ float bf2f_bits(uint16_t h) { return __uint_as_float(((uint32_t)h) << 16); }

template <bool BF16>
__device__ __forceinline__ float x2f(uint16_t h) { return BF16 ? bf2f_bits(h) : h2f_bits(h); }

__device__ __forceinline__ void store_out(void* Y, size_t i, float v, bool bf16) {
  if (bf16) reinterpret_cast<__nv_bfloat16*>(Y)[i] = __float2bfloat16_rn(v);
  else reinterpret_cast<__half*>(Y)[i] = __float2half_rn(v);
}

}  // namespace lbq
