// Decode GEMV at batch 1 on 3-bit LUT weights with plain vector loads:
// y[n] = sum_k x[k] * e4m3(cb[tile][idx[k][n]]) * 2^(E[tile] - 127).
//
// The image keeps a 64-k tile's indices for consecutive channels contiguous
// (24 bytes per channel) and one 16-byte BF16 decode table per 8 channels, so
// a block of 8 output rows (one codebook group) and one tile is 192 + 16
// contiguous bytes: lane l of warp w takes tile kt = 32w + l and loads them
// with thirteen 16-byte loads. The weights decode to exact BF16 values
// (selector from the index words, byte permutes through the table), and the
// products with x are accumulated in FP32. Row sums are reduced as in the
// INT4 direct kernel: a butterfly over the lanes, warp sums in shared memory,
// one barrier per CTA.
#pragma once

#include "common.cuh"
#include "gemv_m1.cuh"
#include "lut3_gemv.cuh"

namespace lbq {

constexpr int kLdMaxWarps = 8;  // K <= 64 * 32 * 8

struct Lut3DirectArgs {
  const uint16_t* X;        // [K] BF16 bits
  void* Y;                  // [N]
  const uint8_t* i_region;  // [K/64][N][24]
  const uint8_t* t_region;  // [K/64][N/8][16]
  int K, N;
  int row_blocks;           // N / 8
  int y_bf16;
};

// Dynamic shared memory: float [row blocks of this CTA][warps][8].
__global__ void __launch_bounds__(kLdMaxWarps * 32, 1) lut3_direct_kernel(const Lut3DirectArgs a) {
  extern __shared__ float red[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nw = blockDim.x >> 5;
  const int kt = warp * 32 + lane;
  const bool tok = kt < (a.K >> 6);

  uint32_t cur[48], nxt[48];  // 8 rows x 24 bytes of indices
  uint4 tab, tabn;
  auto load_block = [&](int rb, uint32_t (&w)[48], uint4& t) {
    if (!tok) {
#pragma unroll
      for (int i = 0; i < 48; ++i) w[i] = 0u;
      t = make_uint4(0u, 0u, 0u, 0u);
      return;
    }
    const uint8_t* base = a.i_region + ((size_t)kt * a.N + (size_t)rb * 8) * 24;
#pragma unroll
    for (int v = 0; v < 12; ++v) {
      const uint4 u = ld_stream_v4(base + 16 * v);
      w[4 * v + 0] = u.x; w[4 * v + 1] = u.y; w[4 * v + 2] = u.z; w[4 * v + 3] = u.w;
    }
    t = ld_nc_v4(a.t_region + ((size_t)kt * (a.N >> 3) + rb) * 16);
  };

  // The weights are only read, so the first row block is requested before
  // waiting for the previous kernel in the stream (which may write X).
  int rb = blockIdx.x;
  if (rb < a.row_blocks) load_block(rb, cur, tab);
  griddep_launch_dependents();
  griddep_wait();
  uint32_t xr[32];  // this tile's 64 activations as BF16 pairs
  if (tok) {
    const uint4* xp = reinterpret_cast<const uint4*>(a.X + (size_t)kt * 64);
#pragma unroll
    for (int v = 0; v < 8; ++v) {
      const uint4 u = ld_nc_v4(xp + v);
      xr[4 * v + 0] = u.x; xr[4 * v + 1] = u.y; xr[4 * v + 2] = u.z; xr[4 * v + 3] = u.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i) xr[i] = 0u;
  }

  int lb = 0;
  for (; rb < a.row_blocks; rb += gridDim.x, ++lb) {
    const int rbn = rb + gridDim.x;
    if (rbn < a.row_blocks) load_block(rbn, nxt, tabn);
    float part[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float acc = 0.0f;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t wa = cur[6 * i + 3 * h], wb = cur[6 * i + 3 * h + 1], wc = cur[6 * i + 3 * h + 2];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          uint32_t p[4];
          lut3_decode8(lut3_selector(t < 2 ? wa : wb, wc, t), tab, p);
#pragma unroll
          for (int e = 0; e < 4; ++e) acc = fma2_bf16_f32(xr[16 * h + 4 * t + e], p[e], acc);
        }
      }
      part[i] = acc;
    }
    const float total = butterfly8(part, lane);
    if ((lane & 3) == 0) red[(lb * nw + warp) * 8 + butterfly8_row(lane)] = total;
#pragma unroll
    for (int i = 0; i < 48; ++i) cur[i] = nxt[i];
    tab = tabn;
  }
  __syncthreads();
  for (int t = tid; t < lb * 8; t += blockDim.x) {
    const int l = t >> 3, row = t & 7;
    const int r = (blockIdx.x + l * gridDim.x) * 8 + row;
    float sum = 0.0f;
    for (int w = 0; w < nw; ++w) sum += red[(l * nw + w) * 8 + row];
    if (r < a.N) store_out(a.Y, (size_t)r, sum, a.y_bf16);
  }
}

}  // namespace lbq
