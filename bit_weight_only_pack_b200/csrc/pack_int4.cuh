// INT4 quantise + repack, and the debug inverses (canonical unpack, exact
// dequantisation).
//
// Quantisation follows "Low Bit ARM kernels" (group-wise scale section: one
// FP16 scale per group along K, symmetric or asymmetric with an int8 zero
// point) with the symmetric formula of the INT4 listing in "Low Bit Metal
// Kernels" ((nibble - 8) * scale). Every step that decides a code is done in
// IEEE FP32 with explicit round-to-nearest intrinsics, so the codes are
// bit-identical to any other IEEE FP32 implementation of the same steps.
#pragma once

#include "common.cuh"

namespace lbq {

// One thread per (group gi, column n). Threads of a warp take consecutive n,
// so every read of W is a coalesced row segment.
template <bool ASYM>
__global__ void __launch_bounds__(256) quantize_pack_int4_kernel(
    const float* __restrict__ W, int K, int N, int group,
    uint8_t* __restrict__ q_region, uint8_t* __restrict__ s_region, uint8_t* __restrict__ z_region) {
  const int G = K / group;
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= (long long)G * N) return;
  const int n = (int)(t % N);
  const int gi = (int)(t / N);
  const float* w = W + (size_t)gi * group * N + n;

  float s;
  float zp = 8.0f;
  __half s16;
  if (!ASYM) {
    float amax = 0.0f;
    for (int i = 0; i < group; ++i) amax = fmaxf(amax, fabsf(w[(size_t)i * N]));
    s16 = __float2half_rn(__fdiv_rn(amax, 7.0f));
    s = __half2float(s16);
  } else {
    float lo = w[0], hi = w[0];
    for (int i = 1; i < group; ++i) {
      const float v = w[(size_t)i * N];
      lo = fminf(lo, v);
      hi = fmaxf(hi, v);
    }
    s16 = __float2half_rn(__fdiv_rn(__fsub_rn(hi, lo), 15.0f));
    s = __half2float(s16);
    zp = (s == 0.0f) ? 0.0f : fminf(fmaxf(rintf(__fdiv_rn(-lo, s)), -128.0f), 127.0f);
  }
  const bool degenerate = (s == 0.0f);
  const float q_degenerate = ASYM ? 0.0f : 8.0f;

  uint8_t* row = q_region + (size_t)n * (K / 2);
  const int c0 = gi * group / 32;
  for (int c = 0; c < group / 32; ++c) {
    uint32_t words[4];
#pragma unroll
    for (int wd = 0; wd < 4; ++wd) {
      uint32_t word = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int k = c * 32 + wd * 8 + i;  // k within the group
        float q;
        if (degenerate) {
          q = q_degenerate;
        } else {
          const float r = rintf(__fdiv_rn(w[(size_t)k * N], s));
          q = fminf(fmaxf(__fadd_rn(r, zp), 0.0f), 15.0f);
        }
        word |= ((uint32_t)q) << (4 * slot_of(i));
      }
      words[wd] = word;
    }
    *reinterpret_cast<uint4*>(row + (size_t)(c0 + c) * 16) = make_uint4(words[0], words[1], words[2], words[3]);
  }
  reinterpret_cast<uint16_t*>(s_region)[meta_index(n, gi, G)] = __half_as_ushort(s16);
  if (ASYM) reinterpret_cast<int8_t*>(z_region)[meta_index(n, gi, G)] = (int8_t)(int)zp;
}

__device__ __forceinline__ uint32_t image_code(const uint8_t* q_region, int K, int k, int n) {
  const uint32_t word = *reinterpret_cast<const uint32_t*>(q_region + (size_t)n * (K / 2) + (k >> 5) * 16 + ((k >> 3) & 3) * 4);
  return (word >> (4 * slot_of(k & 7))) & 0xFu;
}

// Canonical bytes: q_packed[j][n] = q[2j][n] | q[2j+1][n] << 4; scales and
// zero points transposed back to [K/group][N].
__global__ void __launch_bounds__(256) unpack_int4_kernel(
    const uint8_t* __restrict__ q_region, const uint8_t* __restrict__ s_region,
    const uint8_t* __restrict__ z_region, int K, int N, int group,
    uint8_t* __restrict__ q_packed, uint16_t* __restrict__ s_out, int8_t* __restrict__ z_out) {
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long nbytes = (long long)(K / 2) * N;
  if (t < nbytes) {
    const int n = (int)(t % N);
    const int j = (int)(t / N);
    const uint32_t lo = image_code(q_region, K, 2 * j, n);
    const uint32_t hi = image_code(q_region, K, 2 * j + 1, n);
    q_packed[t] = (uint8_t)(lo | (hi << 4));
  }
  const int G = K / group;
  if (t < (long long)G * N) {
    const int n = (int)(t % N);
    const int gi = (int)(t / N);
    s_out[t] = reinterpret_cast<const uint16_t*>(s_region)[meta_index(n, gi, G)];
    if (z_out != nullptr && z_region != nullptr) z_out[t] = reinterpret_cast<const int8_t*>(z_region)[meta_index(n, gi, G)];
  }
}

// Exact dequantisation: W[k][n] = (q - z) * s (the integer difference and the
// FP16 scale multiply exactly in FP32).
__global__ void __launch_bounds__(256) dequant_int4_kernel(
    const uint8_t* __restrict__ q_region, const uint8_t* __restrict__ s_region,
    const uint8_t* __restrict__ z_region, int K, int N, int group, float* __restrict__ W_out) {
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= (long long)K * N) return;
  const int n = (int)(t % N);
  const int k = (int)(t / N);
  const int gi = k / group, G = K / group;
  const float s = h2f_bits(reinterpret_cast<const uint16_t*>(s_region)[meta_index(n, gi, G)]);
  const int z = z_region ? (int)reinterpret_cast<const int8_t*>(z_region)[meta_index(n, gi, G)] : 8;
  const int q = (int)image_code(q_region, K, k, n);
  W_out[t] = (float)(q - z) * s;
}

}  // namespace lbq
