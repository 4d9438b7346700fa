// Decode GEMV / skinny GEMM (batch 1..16) on 3-bit LUT weights, BF16
// activations: Y^T[N, M] = W^T[N, K] . X^T[K, M] with W[k][n] =
// e4m3(cb[tile][idx]) * 2^(E - 127) (vLLM PR 62759 write-up, format section).
//
// Same structure as the INT4 skinny kernel (stream-K over (128-channel tile,
// 256-k stage) units, TMA/bulk-copy ring, 8 consumer warps, mma.sync with
// the weight rows on the MMA "M" side). The decode of one thread's 8 indices
// (k = 32c + 8t .. +7 of one row) is:
//   * a byte-permute selector with one index per nibble, from the chunk's
//     words: S = ((AB >> 2(t&1)) & 0x33333333) | (rotl(C, r_t) & 0x44444444);
//   * two table lookups per 4 indices (prmt over the tile's 8 low bytes and
//     8 high bytes of its BF16 weights, precomputed at pack time with the
//     tile exponent folded in; exact) and two byte-interleaves into BF16 pairs.
// The decoded weights are exact BF16 values, so the MMA sees the format's
// weights exactly and accumulates in FP32; there is no per-tile scaling.
#pragma once

#include "common.cuh"
#include "tma.cuh"
#include "lut3.cuh"
#include "skinny.cuh"

namespace lbq {

constexpr int kL3Stages = 4;
constexpr int kL3IBytes = 4 * kSkRows * 24;  // indices of 4 tiles x 128 channels
constexpr int kL3TBytes = 4 * (kSkRows / 8) * 16;  // tables of 4 tiles x 16 channel groups

struct Lut3SkinnyArgs {
  void* Y;
  float* partials;
  unsigned int* counters;
  const uint8_t* i_region;  // [K/64][N][24]
  const uint8_t* t_region;  // [K/64][N/8][16]
  int K, N, M;
  int stages_per_tile, row_tiles, max_slots;
  long long units;
  int y_bf16;
};

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// 8 indices (selector nibbles) -> 4 BF16 pairs via the byte-planar table.
__device__ __forceinline__ void lut3_decode8(uint32_t sel, const uint4 tab, uint32_t (&p)[4]) {
  const uint32_t l0 = prmt(tab.x, tab.y, sel), h0 = prmt(tab.z, tab.w, sel);
  const uint32_t s2 = sel >> 16;
  const uint32_t l1 = prmt(tab.x, tab.y, s2), h1 = prmt(tab.z, tab.w, s2);
  p[0] = prmt(l0, h0, 0x5140u);
  p[1] = prmt(l0, h0, 0x7362u);
  p[2] = prmt(l1, h1, 0x5140u);
  p[3] = prmt(l1, h1, 0x7362u);
}

// Selector of thread-quarter t (indices 8t .. 8t+7 of a 32-index chunk) from
// the chunk's words ab (A for t < 2, B otherwise) and c.
__device__ __forceinline__ uint32_t lut3_selector(uint32_t ab, uint32_t c, int t) {
  const uint32_t lo = (ab >> ((t & 1) * 2)) & 0x33333333u;
  const uint32_t rot = t == 0 ? 0u : t == 1 ? 31u : t == 2 ? 1u : 2u;
  const uint32_t hi = __funnelshift_l(c, c, rot) & 0x44444444u;
  return lo | hi;
}

template <int NT>
__global__ void __launch_bounds__(kSkThreads, 2) lut3_skinny_kernel(const __grid_constant__ CUtensorMap tx,
                                                                   const Lut3SkinnyArgs a) {
  constexpr int kXBox = NT * 1024;
  constexpr int kOffT = kL3IBytes;
  constexpr int kOffX = 13312;  // kL3IBytes + kL3TBytes rounded to 1024 (swizzled boxes)
  constexpr int kSlot = kOffX + 4 * kXBox;
  static_assert(kOffX >= kL3IBytes + kL3TBytes && kOffX % 1024 == 0, "slot layout");
  extern __shared__ uint8_t dsmem[];
  __shared__ __align__(8) uint64_t full_bar[kL3Stages];
  __shared__ __align__(8) uint64_t empty_bar[kL3Stages];
  __shared__ unsigned int s_last;
  uint8_t* ring = dsmem + ((1024u - (smem_u32(dsmem) & 1023u)) & 1023u);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int K = a.K, M = a.M, N = a.N;
  const int S_t = a.stages_per_tile;
  const long long u_begin = (long long)blockIdx.x * a.units / gridDim.x;
  const long long u_end = (long long)(blockIdx.x + 1) * a.units / gridDim.x;

  if (tid == 0) {
    for (int i = 0; i < kL3Stages; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], kSkWarps);
    }
    fence_barrier_init();
  }
  __syncthreads();
  asm volatile("griddepcontrol.launch_dependents;" :::);

  if (warp == kSkWarps) {
    if (lane == 0) {
      tma_prefetch_desc(&tx);
      asm volatile("griddepcontrol.wait;" ::: "memory");
      int it = 0;
      for (long long u = u_begin; u < u_end; ++u, ++it) {
        const int rt = (int)(u / S_t);
        const int st = (int)(u - (long long)rt * S_t);
        const int slot = it % kL3Stages;
        if (it >= kL3Stages && !mbar_wait(&empty_bar[slot], ((it / kL3Stages) & 1) ^ 1)) return;
        uint8_t* dst = ring + (size_t)slot * kSlot;
        const int rows = min(kSkRows, N - rt * kSkRows);        // a multiple of 8
        const int ntile = min(4, K / 64 - st * 4);              // 64-k tiles of the stage
        const int nxb = ntile;                                   // activation boxes (64 k each)
        mbar_arrive_expect_tx(&full_bar[slot], (uint32_t)(ntile * rows * 24 + ntile * (rows / 8) * 16 + nxb * M * 128));
        for (int j = 0; j < ntile; ++j) {
          const int kt = st * 4 + j;
          bulk_load(dst + j * kSkRows * 24, a.i_region + ((size_t)kt * N + rt * kSkRows) * 24, (uint32_t)(rows * 24),
                    &full_bar[slot]);
          bulk_load(dst + kOffT + j * (kSkRows / 8) * 16, a.t_region + ((size_t)kt * (N / 8) + rt * (kSkRows / 8)) * 16,
                    (uint32_t)((rows / 8) * 16), &full_bar[slot]);
        }
        for (int j = 0; j < nxb; ++j) tma_load_2d(dst + kOffX + j * kXBox, &tx, st * 256 + 64 * j, 0, &full_bar[slot]);
      }
    }
    return;
  }

  // ------------------------------------------------------------------ consumers
  const int g = lane >> 2, t = lane & 3;
  const int lrow = warp * 16 + g;  // rows lrow (group 2*warp) and lrow + 8 (group 2*warp + 1)
  uint32_t x_off[NT][2];
  bool x_ok[NT];
#pragma unroll
  for (int n = 0; n < NT; ++n) {
    x_ok[n] = (g + 8 * n) < M;
    x_off[n][0] = (uint32_t)(kOffX + sw128(g + 8 * n, t));
    x_off[n][1] = (uint32_t)(kOffX + sw128(g + 8 * n, 4 + t));
  }
  const int ab_word = t < 2 ? 0 : 4;

  int it = 0;
  bool ok = true;
  long long u = u_begin;
  while (u < u_end) {
    const int rt = (int)(u / S_t);
    const int st0 = (int)(u - (long long)rt * S_t);
    const int st1 = (int)min((long long)S_t, st0 + (u_end - u));
    float acc[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[n][i] = 0.0f;

    for (int st = st0; st < st1; ++st, ++it) {
      const int slot = it % kL3Stages;
      // after a timed-out wait the warp skips its work but keeps the same
      // sequence of named barriers as the other consumer warps
      if (ok && !mbar_wait(&full_bar[slot], (it / kL3Stages) & 1)) ok = false;
      if (!ok) continue;
      const uint8_t* sp = ring + (size_t)slot * kSlot;
      const int ntile = min(4, K / 64 - st * 4);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (j >= ntile) break;
        const uint4 ta = *reinterpret_cast<const uint4*>(sp + kOffT + (j * (kSkRows / 8) + 2 * warp) * 16);
        const uint4 tb = *reinterpret_cast<const uint4*>(sp + kOffT + (j * (kSkRows / 8) + 2 * warp + 1) * 16);
        const uint8_t* ra = sp + (j * kSkRows + lrow) * 24;
        const uint8_t* rb = ra + 8 * 24;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int ci = 2 * j + h;
          const uint32_t sa = lut3_selector(*reinterpret_cast<const uint32_t*>(ra + 12 * h + ab_word),
                                            *reinterpret_cast<const uint32_t*>(ra + 12 * h + 8), t);
          const uint32_t sbsel = lut3_selector(*reinterpret_cast<const uint32_t*>(rb + 12 * h + ab_word),
                                               *reinterpret_cast<const uint32_t*>(rb + 12 * h + 8), t);
          uint32_t pa[4], pb[4];
          lut3_decode8(sa, ta, pa);
          lut3_decode8(sbsel, tb, pb);
          const uint32_t a0[4] = {pa[0], pb[0], pa[1], pb[1]};
          const uint32_t a1[4] = {pa[2], pb[2], pa[3], pb[3]};
#pragma unroll
          for (int n = 0; n < NT; ++n) {
            uint4 xv = make_uint4(0u, 0u, 0u, 0u);
            if (x_ok[n]) xv = *reinterpret_cast<const uint4*>(sp + x_off[n][ci & 1] + (ci >> 1) * kXBox);
            mma_16816(acc[n], a0, xv.x, xv.y, true);
            mma_16816(acc[n], a1, xv.z, xv.w, true);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty_bar[slot]);
    }

    const int n0 = rt * kSkRows + lrow;
    const bool whole = (st0 == 0 && st1 == S_t);
    if (whole) {
#pragma unroll
      for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int m = 8 * n + 2 * t + (i & 1);
          const int nn = n0 + ((i & 2) ? 8 : 0);
          if (ok && m < M && nn < N) store_out(a.Y, (size_t)m * N + nn, acc[n][i], a.y_bf16);
        }
    } else {
      const long long tile_u0 = (long long)rt * S_t;
      const int first = sk_owner(tile_u0, a.units, gridDim.x);
      const int slot_id = blockIdx.x - first;
      float* base = a.partials + (size_t)rt * a.max_slots * M * kSkRows;
#pragma unroll
      for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int m = 8 * n + 2 * t + (i & 1);
          const int r = lrow + ((i & 2) ? 8 : 0);
          if (ok && m < M) base[((size_t)slot_id * M + m) * kSkRows + r] = acc[n][i];
        }
      __threadfence();
      asm volatile("bar.sync 1, %0;" :: "r"(kSkWarps * 32) : "memory");
      if (tid == 0) {
        s_last = 0u;
        if (ok) {
          const unsigned int add = (unsigned int)(st1 - st0);
          const unsigned int prev = atomicAdd(&a.counters[rt], add);
          s_last = (prev + add == (unsigned int)S_t);
        }
      }
      asm volatile("bar.sync 1, %0;" :: "r"(kSkWarps * 32) : "memory");
      if (s_last) {
        __threadfence();
        const int nslots = sk_owner(tile_u0 + S_t - 1, a.units, gridDim.x) - first + 1;
#pragma unroll
        for (int n = 0; n < NT; ++n)
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int m = 8 * n + 2 * t + (i & 1);
            const int r = lrow + ((i & 2) ? 8 : 0);
            const int nn = rt * kSkRows + r;
            if (m < M && nn < N) {
              float sum = 0.0f;
              for (int sl = 0; sl < nslots; ++sl) sum += __ldcg(base + ((size_t)sl * M + m) * kSkRows + r);
              store_out(a.Y, (size_t)m * N + nn, sum, a.y_bf16);
            }
          }
        if (tid == 0) a.counters[rt] = 0u;
      }
      asm volatile("bar.sync 1, %0;" :: "r"(kSkWarps * 32) : "memory");
    }
    u += st1 - st0;
  }
}

}  // namespace lbq
