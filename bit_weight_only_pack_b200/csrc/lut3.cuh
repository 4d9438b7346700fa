// The 3-bit LUT weight format: packing into the device image, the debug
// inverses, and the decode used by the LUT3 kernels.
//
// Format (vLLM PR 62759 write-up, format section): a 3-bit index per weight
// into an 8-entry E4M3 codebook shared by a tile of 8 output channels x 64 k,
// times one UE8M0 exponent 2^(E-127) per tile.
//
// Device image (after the 256-byte header):
//   I region  tile-major [K/64][N][24 bytes]: per 64-k tile and output channel
//             24 bytes, so the indices of a block of channels for one tile are
//             contiguous. A tile's 64 indices are two 32-index chunks of
//             three 32-bit words
//             {A, B, C}; index i of a chunk (k = 32c + i) is stored as
//               low 2 bits: A bits [4i, 4i+2)        for i in 0..7
//                           A bits [4(i-8)+2, +2)    for i in 8..15
//                           B bits [4(i-16), +2)     for i in 16..23
//                           B bits [4(i-24)+2, +2)   for i in 24..31
//               high bit:   C bit 4(i%8) + {2, 3, 1, 0}[i/8]
//             so the 8 indices k = 32c + 8t .. 8t+7 become a byte-permute
//             selector (one index per nibble, bit 3 clear) in two or three
//             AND/OR/shift operations.
//   C region  codebooks, N/8 rows of K/64 x 8 E4M3 bytes, row stride padded to 16.
//   E region  exponents, N/8 rows of K/64 UE8M0 bytes, row stride padded to 16.
//   T region  [K/64][N/8][16 bytes]: the tile's 8 weights e4m3(cb[j]) * 2^(E-127)
//             rounded to BF16 (exact while inside BF16's normal range, which
//             covers every E4M3 value times 2^-117 .. 2^119), low bytes of
//             entries 0..7 then high bytes: two byte-permute tables.
#pragma once

#include "common.cuh"

namespace lbq {

__host__ __device__ inline size_t lut3_c_stride(int K) { return align_up((size_t)(K / 64) * 8, 16); }
__host__ __device__ inline size_t lut3_e_stride(int K) { return align_up((size_t)(K / 64), 16); }

// position of index i's high bit in the chunk's C word
__host__ __device__ constexpr int lut3_hi_pos(int i) {
  return 4 * (i & 7) + ((i >> 3) == 0 ? 2 : (i >> 3) == 1 ? 3 : (i >> 3) == 2 ? 1 : 0);
}

// position of index i's two low bits in the chunk's A (i < 16) or B word
__host__ __device__ constexpr int lut3_lo_pos(int i) { return 4 * (i & 7) + (((i >> 3) & 1) ? 2 : 0); }

__device__ inline float e4m3_to_float(uint32_t b);

// BF16 bit pattern of e4m3(b) * 2^(e - 127). The product has at most four
// significant bits, so while it is a normal FP32 number its FP32 pattern ends in
// 16 zero bits and its top half is the exact BF16 pattern; outside that range
// (|value| below 2^-126 or NaN) the value is rounded to nearest even.
__device__ inline uint32_t lut3_table_entry(uint32_t b, uint32_t e) {
  if (e == 255u) return 0x7FC0u;
  const uint32_t f = __float_as_uint(ldexpf(e4m3_to_float(b), (int)e - 127));
  if ((f & 0xFFFFu) == 0u) return f >> 16;
  const __nv_bfloat16 h = __float2bfloat16_rn(__uint_as_float(f));
  return (uint32_t)__bfloat16_as_ushort(h);
}

// One thread per (channel n, 64-k tile kt).

__global__ void __launch_bounds__(256) pack_lut3_kernel(const uint8_t* __restrict__ idx, const uint8_t* __restrict__ cb,
                                                        const uint8_t* __restrict__ ex, int K, int N,
                                                        uint8_t* __restrict__ i_region, uint8_t* __restrict__ c_region,
                                                        uint8_t* __restrict__ e_region, uint8_t* __restrict__ t_region) {
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const int KT = K / 64;
  if (t >= (long long)KT * N) return;
  const int n = (int)(t % N);
  const int kt = (int)(t / N);
  uint32_t w[6] = {0, 0, 0, 0, 0, 0};
  for (int c = 0; c < 2; ++c) {
    for (int i = 0; i < 32; ++i) {
      const uint32_t v = idx[(size_t)(kt * 64 + c * 32 + i) * N + n] & 7u;
      w[3 * c + (i < 16 ? 0 : 1)] |= (v & 3u) << lut3_lo_pos(i);
      w[3 * c + 2] |= (v >> 2) << lut3_hi_pos(i);
    }
  }
  uint32_t* dst = reinterpret_cast<uint32_t*>(i_region + ((size_t)kt * N + n) * 24);
  for (int j = 0; j < 6; ++j) dst[j] = w[j];
  if ((n & 7) == 0) {
    const int grp = n >> 3;
    const uint8_t e = ex[(size_t)kt * (N / 8) + grp];
    uint32_t lo[2] = {0u, 0u}, hi[2] = {0u, 0u};
    for (int j = 0; j < 8; ++j) {
      const uint8_t b = cb[((size_t)kt * (N / 8) + grp) * 8 + j];
      c_region[(size_t)grp * lut3_c_stride(K) + kt * 8 + j] = b;
      const uint32_t bits = lut3_table_entry(b, e);
      lo[j >> 2] |= (bits & 0xFFu) << (8 * (j & 3));
      hi[j >> 2] |= (bits >> 8) << (8 * (j & 3));
    }
    *reinterpret_cast<uint4*>(t_region + ((size_t)kt * (N / 8) + grp) * 16) = make_uint4(lo[0], lo[1], hi[0], hi[1]);
    e_region[(size_t)grp * lut3_e_stride(K) + kt] = e;
  }
}

__device__ __forceinline__ uint32_t lut3_image_index(const uint8_t* i_region, int N, int k, int n) {
  const int kt = k >> 6, c = (k >> 5) & 1, i = k & 31;
  const uint32_t* w = reinterpret_cast<const uint32_t*>(i_region + ((size_t)kt * N + n) * 24) + 3 * c;
  const uint32_t lo = (w[i < 16 ? 0 : 1] >> lut3_lo_pos(i)) & 3u;
  const uint32_t hi = (w[2] >> lut3_hi_pos(i)) & 1u;
  return lo | (hi << 2);
}

// Canonical index stream [K/64][N/8][8][24]: per tile and channel the 64
// indices as a little-endian 192-bit string, index i in bits [3i, 3i+3).
// One thread per (tile, channel).
__global__ void __launch_bounds__(256) unpack_lut3_kernel(const uint8_t* __restrict__ i_region,
                                                          const uint8_t* __restrict__ c_region,
                                                          const uint8_t* __restrict__ e_region, int K, int N,
                                                          uint8_t* __restrict__ idx_stream, uint8_t* __restrict__ cb,
                                                          uint8_t* __restrict__ ex) {
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const int KT = K / 64;
  if (t >= (long long)KT * N) return;
  const int n = (int)(t % N);
  const int kt = (int)(t / N);
  uint8_t out[24];
  for (int b = 0; b < 24; ++b) out[b] = 0;
  for (int i = 0; i < 64; ++i) {
    const uint32_t v = lut3_image_index(i_region, N, kt * 64 + i, n);
    for (int b = 0; b < 3; ++b) {
      const int pos = 3 * i + b;
      out[pos >> 3] |= (uint8_t)(((v >> b) & 1u) << (pos & 7));
    }
  }
  const int grp = n >> 3, ch = n & 7;
  uint8_t* dst = idx_stream + (((size_t)kt * (N / 8) + grp) * 8 + ch) * 24;
  for (int b = 0; b < 24; ++b) dst[b] = out[b];
  if (ch == 0) {
    for (int j = 0; j < 8; ++j) cb[((size_t)kt * (N / 8) + grp) * 8 + j] = c_region[(size_t)grp * lut3_c_stride(K) + kt * 8 + j];
    ex[(size_t)kt * (N / 8) + grp] = e_region[(size_t)grp * lut3_e_stride(K) + kt];
  }
}

// E4M3 ("fn") byte -> float (exact). NaN for 0x7F / 0xFF.
__device__ inline float e4m3_to_float(uint32_t b) {
  const uint32_t e = (b >> 3) & 0xFu, m = b & 7u;
  float v;
  if (e == 15u && m == 7u) v = __int_as_float(0x7FC00000);
  else if (e == 0u) v = (float)m * 0.001953125f;  // m/8 * 2^-6
  else v = __int_as_float((int)(((e + 120u) << 23) | (m << 20)));
  return (b & 0x80u) ? -v : v;
}

// Exact decode: W[k][n] = e4m3(cb) * 2^(E - 127) (exact in FP32 while the
// product stays in the normal range).
__global__ void __launch_bounds__(256) dequant_lut3_kernel(const uint8_t* __restrict__ i_region,
                                                           const uint8_t* __restrict__ c_region,
                                                           const uint8_t* __restrict__ e_region, int K, int N,
                                                           float* __restrict__ W_out) {
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= (long long)K * N) return;
  const int n = (int)(t % N);
  const int k = (int)(t / N);
  const int kt = k >> 6, grp = n >> 3;
  const uint32_t v = lut3_image_index(i_region, N, k, n);
  const uint32_t b = c_region[(size_t)grp * lut3_c_stride(K) + kt * 8 + v];
  const int E = (int)e_region[(size_t)grp * lut3_e_stride(K) + kt];
  W_out[t] = E == 255 ? __int_as_float(0x7FC00000) : ldexpf(e4m3_to_float(b), E - 127);
}

}  // namespace lbq
