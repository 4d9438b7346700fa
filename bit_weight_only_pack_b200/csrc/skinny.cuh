// Decode GEMV / skinny GEMM for batches 1..16 on INT4 weights (swap-AB on the
// tensor cores): Y^T[N, M] = dequant(W)^T[N, K] . X^T[K, M].
//
// The kernel is HBM-bound: at 4.1-4.75 bits per weight an SM must retire about
// 40 weights per clock, so the per-weight instruction budget is ~2 even at full
// issue rate. The tensor cores take every multiply-add (the FP32 FMAs of a
// CUDA-core GEMV grow with M; at M = 16 they alone would exceed the budget 8x),
// and the code-to-operand conversion is reduced to one AND/OR per two codes:
//
//  * OR-ing a nibble into the mantissa of 1024.0 (FP16) or 128.0 (BF16) gives
//    the operand value 1024 + q (or 1024 + 16 q for the upper nibble of a
//    byte) with no arithmetic. These offset-form operands go straight into the
//    MMA. The offsets and the zero point are removed by extra MMAs whose A
//    operand is the per-row constant -(1024 + z) (resp. -(1024 + 16 z),
//    -(128 + z)), exact in FP16/BF16, against the same activation fragment:
//    D = sum x (1024 + q) - (1024 + z) sum x = sum x (q - z), accumulated in
//    FP32 inside the tensor core. No weight is ever rounded.
//  * Per group, acc += s[row] * D (FP32 FMAs on the accumulator fragment);
//    FP16's upper-nibble class carries a factor 16, removed by using s/16.
//  * The weight rows are the MMA "M" side (16 output channels per
//    mma.m16n8k16) and the batch is the MMA "N" side (8 or 16 columns), so no
//    batch padding to 128 is streamed ("no swap-AB" is one of the reasons the
//    vLLM LUT-B kernel loses at small batch).
//  * Producer warp: per 256-k stage, TMA loads of a 128-row x 128-byte code
//    tile (128-byte swizzle), the 64-k activation boxes (128-byte swizzle) and
//    16-byte boxes of the rows' scales / zero points, completing on one
//    mbarrier; a ring of kSkStages stages feeds 8 consumer warps (16 rows
//    each). ldmatrix.x4 hands each thread the code words of rows r and r+8 for
//    two 32-k chunks; within a chunk the k order is permuted identically for A
//    and B so that thread t's MMA k-slots are exactly the 16 bytes of
//    activations it reads with one shared-memory load.
//  * Split-K: FP32 partials and a last-CTA reduction in slice order (the
//    workspace's counters are reset, so it is left zeroed).
#pragma once

#include "common.cuh"
#include "tma.cuh"

namespace lbq {

constexpr int kSkStages = 4;
constexpr int kSkWarps = 8;                 // consumer warps, 16 rows each
constexpr int kSkRows = kSkWarps * 16;      // rows of W per CTA tile
constexpr int kSkThreads = (kSkWarps + 1) * 32;
constexpr int kSkWBytes = kSkRows * 128;    // 16 KB of codes per 256-k stage
constexpr int kSkSBytes = kSkRows * 16;     // 16-byte scale box per row
constexpr int kSkZBytes = kSkRows * 16;     // 16-byte zero-point box per row

struct SkinnyArgs {
  void* Y;                   // [M][N]
  float* partials;           // [splits][M][N]
  unsigned int* counters;    // [row_tiles]
  int K, N, M;
  int stages_per_split, splits, row_tiles, total_tiles;
  int y_bf16;
};

__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1, bool bf16) {
  if (bf16)
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
                 "{%8, %9}, {%0, %1, %2, %3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  else
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
                 "{%8, %9}, {%0, %1, %2, %3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t hsub2_u32(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t hfma2_u32(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ uint32_t bsub2_u32(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ uint32_t pack_f16x2(float v) {
  const __half2 h = __float2half2_rn(v);
  return *reinterpret_cast<const uint32_t*>(&h);
}
__device__ __forceinline__ uint32_t pack_bf16x2(float v) {
  const __nv_bfloat162 h = __float2bfloat162_rn(v);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Exact (q - z) pairs in the activation type (used by the prefill GEMM):
//  FP16: c1 = (1024+z, 1024+z), c2 = -(64+z) pair;  BF16: c1 = (128+z, 128+z).
template <bool BF16>
__device__ __forceinline__ void zero_consts(int z, uint32_t& c1, uint32_t& c2) {
  if (!BF16) {
    c1 = pack_f16x2(1024.0f + (float)z);
    c2 = pack_f16x2(-(64.0f + (float)z));
  } else {
    c1 = pack_bf16x2(128.0f + (float)z);
    c2 = 0u;
  }
}

template <bool BF16, bool ASYM, int NT, int GC, bool KFULL>
__global__ void __launch_bounds__(kSkThreads, 2) skinny_kernel(
    const __grid_constant__ CUtensorMap tw, const __grid_constant__ CUtensorMap tx,
    const __grid_constant__ CUtensorMap ts, const __grid_constant__ CUtensorMap tz, const SkinnyArgs a) {
  constexpr int kXBox = NT * 1024;  // one 64-k activation box (8*NT rows x 128 B)
  constexpr int kOffX = kSkWBytes;
  constexpr int kOffS = kOffX + 4 * kXBox;
  constexpr int kOffZ = kOffS + kSkSBytes;
  constexpr int kSlot = kOffZ + (ASYM ? kSkZBytes : 0);
  extern __shared__ uint8_t dsmem[];
  __shared__ __align__(8) uint64_t full_bar[kSkStages];
  __shared__ __align__(8) uint64_t empty_bar[kSkStages];
  __shared__ unsigned int s_last;
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int K = a.K, M = a.M;
  const int total_stages = (K + 255) / 256;

  if (tid == 0) {
    for (int i = 0; i < kSkStages; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], kSkWarps);
    }
    fence_barrier_init();
  }
  __syncthreads();
  asm volatile("griddepcontrol.launch_dependents;" :::);

  if (warp == kSkWarps) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      tma_prefetch_desc(&tw);
      tma_prefetch_desc(&tx);
      tma_prefetch_desc(&ts);
      if (ASYM) tma_prefetch_desc(&tz);
      asm volatile("griddepcontrol.wait;" ::: "memory");  // X may come from the previous kernel
      int it = 0;
      for (int tile = blockIdx.x; tile < a.total_tiles; tile += gridDim.x) {
        const int split = tile / a.row_tiles;
        const int rt = tile - split * a.row_tiles;
        const int s0 = split * a.stages_per_split;
        const int s1 = min(s0 + a.stages_per_split, total_stages);
        for (int st = s0; st < s1; ++st, ++it) {
          const int slot = it % kSkStages;
          if (it >= kSkStages && !mbar_wait(&empty_bar[slot], ((it / kSkStages) & 1) ^ 1)) return;
          uint8_t* dst = ring + (size_t)slot * kSlot;
          const int gs0 = st * 8 / GC;  // first group of the stage
          const int nxb = KFULL ? 4 : min(4, (K - st * 256 + 63) / 64);  // activation boxes that start inside K
          mbar_arrive_expect_tx(&full_bar[slot],
                                (uint32_t)(kSkWBytes + nxb * M * 128 + kSkSBytes + (ASYM ? kSkZBytes : 0)));
          tma_load_2d(dst, &tw, st * 128, rt * kSkRows, &full_bar[slot]);
          for (int j = 0; j < nxb; ++j) tma_load_2d(dst + kOffX + j * kXBox, &tx, st * 256 + 64 * j, 0, &full_bar[slot]);
          tma_load_2d(dst + kOffS, &ts, (gs0 / 8) * 8, rt * kSkRows, &full_bar[slot]);
          if (ASYM) tma_load_2d(dst + kOffZ, &tz, (gs0 / 16) * 16, rt * kSkRows, &full_bar[slot]);
        }
      }
    }
    return;
  }

  // ------------------------------------------------------------------ consumers
  const int g = lane >> 2, t = lane & 3;
  const int lrow = warp * 16 + g;  // this thread's rows: lrow and lrow + 8
  // ldmatrix row address of this lane: matrix i = lane/8 -> rows +8*(i&1), chunk +(i>>1)
  const int lm_row = warp * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
  const uint32_t lm_off[4] = {sw128(lm_row, 0 + (lane >> 4)), sw128(lm_row, 2 + (lane >> 4)),
                              sw128(lm_row, 4 + (lane >> 4)), sw128(lm_row, 6 + (lane >> 4))};
  // activation fragment offsets of this thread: column m = g + 8n, chunk half (ci & 1)
  uint32_t x_off[NT][2];
  bool x_ok[NT];
#pragma unroll
  for (int n = 0; n < NT; ++n) {
    x_ok[n] = (g + 8 * n) < M;
    x_off[n][0] = (uint32_t)(kOffX + sw128(g + 8 * n, t));
    x_off[n][1] = (uint32_t)(kOffX + sw128(g + 8 * n, 4 + t));
  }
  const uint32_t s_off_r = (uint32_t)(kOffS + lrow * 16), s_off_r8 = s_off_r + 8 * 16;
  const uint32_t z_off_r = (uint32_t)(kOffZ + lrow * 16), z_off_r8 = z_off_r + 8 * 16;
  // constant A operands of the offset-removing MMAs (symmetric: z = 8)
  uint32_t ca_r = BF16 ? pack_bf16x2(-136.0f) : pack_f16x2(-1032.0f);
  uint32_t cb_r = BF16 ? 0u : pack_f16x2(-1152.0f);  // -(1024 + 16*8)
  uint32_t ca_r8 = ca_r, cb_r8 = cb_r;

  int it = 0;
  bool ok = true;
  for (int tile = blockIdx.x; tile < a.total_tiles && ok; tile += gridDim.x) {
    const int split = tile / a.row_tiles;
    const int rt = tile - split * a.row_tiles;
    const int s0 = split * a.stages_per_split;
    const int s1 = min(s0 + a.stages_per_split, total_stages);
    float acc[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[n][i] = 0.0f;
    float dA[NT][4], dB[NT][4];
    float s_r = 0.0f, s_r8 = 0.0f;

    for (int st = s0; st < s1; ++st, ++it) {
      const int slot = it % kSkStages;
      if (!mbar_wait(&full_bar[slot], (it / kSkStages) & 1)) { ok = false; break; }
      const uint32_t sb = smem_u32(ring + (size_t)slot * kSlot);
      const int k0 = st * 256;
      const int gs0 = st * 8 / GC;
      const int sx0 = (gs0 / 8) * 8, zx0 = (gs0 / 16) * 16;
#pragma unroll
      for (int cp = 0; cp < 4; ++cp) {
        if (!KFULL && k0 + 64 * cp >= K) continue;
        uint32_t wr[4];
        ldmatrix_x4(wr, sb + lm_off[cp]);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int ci = 2 * cp + h;
          if (!KFULL && k0 + 32 * ci >= K) continue;
          if (ci % GC == 0) {
            const int gl = gs0 + ci / GC;
            uint16_t b0, b1;
            asm volatile("ld.shared.u16 %0, [%1];" : "=h"(b0) : "r"(sb + s_off_r + (gl - sx0) * 2));
            asm volatile("ld.shared.u16 %0, [%1];" : "=h"(b1) : "r"(sb + s_off_r8 + (gl - sx0) * 2));
            s_r = h2f_bits(b0);
            s_r8 = h2f_bits(b1);
            if (ASYM) {
              int z0, z1;
              asm volatile("ld.shared.s8 %0, [%1];" : "=r"(z0) : "r"(sb + z_off_r + (gl - zx0)));
              asm volatile("ld.shared.s8 %0, [%1];" : "=r"(z1) : "r"(sb + z_off_r8 + (gl - zx0)));
              if (BF16) {
                ca_r = pack_bf16x2(-(128.0f + (float)z0));
                ca_r8 = pack_bf16x2(-(128.0f + (float)z1));
              } else {
                ca_r = pack_f16x2(-(1024.0f + (float)z0));
                ca_r8 = pack_f16x2(-(1024.0f + (float)z1));
                cb_r = pack_f16x2(-(1024.0f + 16.0f * (float)z0));
                cb_r8 = pack_f16x2(-(1024.0f + 16.0f * (float)z1));
              }
            }
#pragma unroll
            for (int n = 0; n < NT; ++n)
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                dA[n][i] = 0.0f;
                dB[n][i] = 0.0f;
              }
          }
          const uint32_t wa = wr[h ? 2 : 0], wb = wr[h ? 3 : 1];
          const uint32_t ca[4] = {ca_r, ca_r8, ca_r, ca_r8};
          if (!BF16) {
            // class A: (k0,k1) (k4,k5) = 1024+q;  class B: (k2,k3) (k6,k7) = 1024+16q
            const uint32_t ta = wa >> 8, tb = wb >> 8;
            const uint32_t aA[4] = {and_or(wa, 0x000F000Fu, 0x64006400u), and_or(wb, 0x000F000Fu, 0x64006400u),
                                    and_or(ta, 0x000F000Fu, 0x64006400u), and_or(tb, 0x000F000Fu, 0x64006400u)};
            const uint32_t aB[4] = {and_or(wa, 0x00F000F0u, 0x64006400u), and_or(wb, 0x00F000F0u, 0x64006400u),
                                    and_or(ta, 0x00F000F0u, 0x64006400u), and_or(tb, 0x00F000F0u, 0x64006400u)};
            const uint32_t cb[4] = {cb_r, cb_r8, cb_r, cb_r8};
#pragma unroll
            for (int n = 0; n < NT; ++n) {
              uint4 xv = make_uint4(0u, 0u, 0u, 0u);
              if (x_ok[n]) xv = lds128(sb + x_off[n][h] + (ci >> 1) * kXBox);
              mma_16816(dA[n], aA, xv.x, xv.z, false);
              mma_16816(dA[n], ca, xv.x, xv.z, false);
              mma_16816(dB[n], aB, xv.y, xv.w, false);
              mma_16816(dB[n], cb, xv.y, xv.w, false);
            }
          } else {
            const uint32_t a0[4] = {and_or(wa, 0x000F000Fu, 0x43004300u), and_or(wb, 0x000F000Fu, 0x43004300u),
                                    and_or(wa >> 4, 0x000F000Fu, 0x43004300u), and_or(wb >> 4, 0x000F000Fu, 0x43004300u)};
            const uint32_t a1[4] = {and_or(wa >> 8, 0x000F000Fu, 0x43004300u), and_or(wb >> 8, 0x000F000Fu, 0x43004300u),
                                    and_or(wa >> 12, 0x000F000Fu, 0x43004300u), and_or(wb >> 12, 0x000F000Fu, 0x43004300u)};
#pragma unroll
            for (int n = 0; n < NT; ++n) {
              uint4 xv = make_uint4(0u, 0u, 0u, 0u);
              if (x_ok[n]) xv = lds128(sb + x_off[n][h] + (ci >> 1) * kXBox);
              mma_16816(dA[n], a0, xv.x, xv.y, true);
              mma_16816(dA[n], ca, xv.x, xv.y, true);
              mma_16816(dA[n], a1, xv.z, xv.w, true);
              mma_16816(dA[n], ca, xv.z, xv.w, true);
            }
          }
          const bool group_end = (ci % GC == GC - 1) || (!KFULL && k0 + 32 * ci + 32 >= K);
          if (group_end) {
#pragma unroll
            for (int n = 0; n < NT; ++n) {
              acc[n][0] = fmaf(s_r, dA[n][0], acc[n][0]);
              acc[n][1] = fmaf(s_r, dA[n][1], acc[n][1]);
              acc[n][2] = fmaf(s_r8, dA[n][2], acc[n][2]);
              acc[n][3] = fmaf(s_r8, dA[n][3], acc[n][3]);
              if (!BF16) {
                acc[n][0] = fmaf(s_r * 0.0625f, dB[n][0], acc[n][0]);
                acc[n][1] = fmaf(s_r * 0.0625f, dB[n][1], acc[n][1]);
                acc[n][2] = fmaf(s_r8 * 0.0625f, dB[n][2], acc[n][2]);
                acc[n][3] = fmaf(s_r8 * 0.0625f, dB[n][3], acc[n][3]);
              }
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty_bar[slot]);
    }
    if (!ok) break;

    // ---------------------------------------------------------------- output
    const int n0 = rt * kSkRows + lrow;
#pragma unroll
    for (int n = 0; n < NT; ++n) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int m = 8 * n + 2 * t + (i & 1);
        const int nn = n0 + ((i & 2) ? 8 : 0);
        if (m < M && nn < a.N) {
          if (a.splits == 1) store_out(a.Y, (size_t)m * a.N + nn, acc[n][i], a.y_bf16);
          else a.partials[((size_t)split * M + m) * a.N + nn] = acc[n][i];
        }
      }
    }
    if (a.splits > 1) {
      __threadfence();
      asm volatile("bar.sync 1, %0;" :: "r"(kSkWarps * 32) : "memory");
      if (tid == 0) {
        const unsigned int prev = atomicAdd(&a.counters[rt], 1u);
        s_last = (prev == (unsigned int)(a.splits - 1));
      }
      asm volatile("bar.sync 1, %0;" :: "r"(kSkWarps * 32) : "memory");
      if (s_last) {
        __threadfence();
#pragma unroll
        for (int n = 0; n < NT; ++n) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int m = 8 * n + 2 * t + (i & 1);
            const int nn = n0 + ((i & 2) ? 8 : 0);
            if (m < M && nn < a.N) {
              float sum = 0.0f;
              for (int sp = 0; sp < a.splits; ++sp) sum += __ldcg(a.partials + ((size_t)sp * M + m) * a.N + nn);
              store_out(a.Y, (size_t)m * a.N + nn, sum, a.y_bf16);
            }
          }
        }
        if (tid == 0) a.counters[rt] = 0u;
      }
      asm volatile("bar.sync 1, %0;" :: "r"(kSkWarps * 32) : "memory");
    }
  }
}

}  // namespace lbq
