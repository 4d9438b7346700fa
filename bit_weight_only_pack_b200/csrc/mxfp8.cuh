// MXFP8 quantisation of activations: E4M3 elements with one UE8M0 scale per
// 32 consecutive k of a row (the activation format of the LUT-B MoE kernels
// in the vLLM PR 62759 write-up; MX element and scale types of the OCP
// Microscaling specification it links).
//
// One thread per 32-element block: it reads the block's 64 bytes, takes the
// largest magnitude amax, stores the scale byte floor(log2 amax) - 8 + 127
// (clamped to [0, 254]; 127 for an all-zero block) and writes the 32 elements
// x * 2^(127 - byte) rounded to nearest E4M3, ties to even, saturating at
// +-448. Consecutive threads take consecutive blocks, so a warp reads 2 KB
// and writes 1 KB + 32 B contiguously.
#pragma once

#include "common.cuh"

namespace lbq {

// floor(log2 |a|) of a finite non-zero float (subnormals included)
__device__ __forceinline__ int floor_log2_abs(float a) {
  const uint32_t b = __float_as_uint(a) & 0x7FFFFFFFu;
  const int e = (int)(b >> 23);
  if (e != 0) return e - 127;
  return (31 - __clz((int)b)) - 149;  // subnormal: value = mantissa * 2^-149
}

// two floats -> two E4M3 bytes (lo in bits 0..7, hi in bits 8..15)
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  uint16_t d;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(hi), "f"(lo));
  return (uint32_t)d;
}

template <bool BF16>
__global__ void quantize_mxfp8_kernel(const uint16_t* __restrict__ X, uint8_t* __restrict__ codes,
                                      uint8_t* __restrict__ scales, long long blocks) {
  const long long b = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= blocks) return;
  const uint4* src = reinterpret_cast<const uint4*>(X + b * 32);
  float v[32];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 u = ld_nc_v4(src + q);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[8 * q + 2 * i] = x2f<BF16>((uint16_t)(w[i] & 0xFFFFu));
      v[8 * q + 2 * i + 1] = x2f<BF16>((uint16_t)(w[i] >> 16));
    }
  }
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
  int byte = 127;
  if (amax > 0.0f) byte = min(max(floor_log2_abs(amax) - 8 + 127, 0), 254);
  // 2^(127 - byte), built exactly from its bits (byte <= 253 for finite inputs, so it is normal)
  const float mul = __uint_as_float((uint32_t)(254 - byte) << 23);
  uint32_t out[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t a = e4m3x2(v[4 * i] * mul, v[4 * i + 1] * mul);
    const uint32_t c = e4m3x2(v[4 * i + 2] * mul, v[4 * i + 3] * mul);
    out[i] = a | (c << 16);
  }
  uint4* dst = reinterpret_cast<uint4*>(codes + b * 32);
  dst[0] = make_uint4(out[0], out[1], out[2], out[3]);
  dst[1] = make_uint4(out[4], out[5], out[6], out[7]);
  scales[b] = (uint8_t)byte;
}

}  // namespace lbq
