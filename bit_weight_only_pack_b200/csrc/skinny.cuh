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
//    FP16's upper-nibble class carries a factor 16, removed before scaling.
//  * The weight rows are the MMA "M" side (16 output channels per
//    mma.m16n8k16) and the batch is the MMA "N" side (8 or 16 columns), so no
//    batch padding to 128 is streamed ("no swap-AB" is one of the reasons the
//    vLLM LUT-B kernel loses at small batch).
//  * Producer warp: per 256-k stage, TMA loads of a 128-row x 128-byte code
//    tile (128-byte swizzle) and one box of the stage's activations (a 3-D
//    view of X: 32-k chunk x token x chunk, so chunk j of token m lands at
//    (j M + m) 64 bytes and a quarter-warp's two tokens fall in opposite bank
//    halves), and one bulk copy each of the tile's scales / zero points for
//    the stage's groups (contiguous in the 128-channel-tiled image), all
//    completing on one mbarrier; a ring of kSkStages stages feeds 8 consumer warps (16 rows
//    each). ldmatrix.x4 hands each thread the code words of rows r and r+8 for
//    two 32-k chunks; within a chunk the k order is permuted identically for A
//    and B so that thread t's MMA k-slots are exactly the 16 bytes of
//    activations it reads with one shared-memory load.
//  * Stream-K: every CTA takes an equal contiguous range of (row tile, stage)
//    units, so all SMs stream the same number of bytes whatever the shape;
//    shared row tiles are finished by the CTA completing their stage count
//    (FP32 partials added in slot order; counters reset, workspace left zeroed).
#pragma once

#include "common.cuh"
#include "tma.cuh"

namespace lbq {

constexpr int kSkStages = 4;
constexpr int kSkWarps = 8;                 // consumer warps, 16 rows each
constexpr int kSkRows = kSkWarps * 16;      // rows of W per CTA tile
constexpr int kSkThreads = (kSkWarps + 1) * 32;
constexpr int kSkWBytes = kSkRows * 128;    // 16 KB of codes per 256-k stage
constexpr int kSkSBytes = 8 * kSkRows * 2;  // scales of up to 8 groups for the tile's 128 rows
constexpr int kSkZBytes = 8 * kSkRows;      // zero points of up to 8 groups

// Stream-K work split: the (row tile, 256-k stage) units, row tile major,
// are divided into equal contiguous ranges, one per CTA, so every CTA streams
// the same number of bytes. A row tile covered by one CTA is written directly;
// a row tile shared by several CTAs gets FP32 partials in per-CTA slots, and
// the CTA that completes its stage count adds the slots in order.
struct SkinnyArgs {
  void* Y;                   // [M][N]
  float* partials;           // [row_tiles][max_slots][M][kSkRows]
  unsigned int* counters;    // [row_tiles]
  const uint8_t* s_region;   // 128-channel-tiled scales of the image
  const uint8_t* z_region;   // 128-channel-tiled zero points (ASYM)
  int K, N, M, G;
  int stages_per_tile, row_tiles, max_slots;
  long long units;           // row_tiles * stages_per_tile
  int y_bf16;
};

__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1, bool bf16) {
  if (bf16)
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
                 "{%8, %9}, {%0, %1, %2, %3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  else
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
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

// CTA that owns unit u when `units` units are split evenly over `grid` CTAs.
__device__ __forceinline__ int sk_owner(long long u, long long units, int grid) {
  return (int)(((u + 1) * grid - 1) / units);
}

__device__ __forceinline__ void mma_16816_zc(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1, bool bf16) {
  if (bf16)
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
                 "{%8, %9}, {%10, %10, %10, %10};"
                 : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(0.0f));
  else
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
                 "{%8, %9}, {%10, %10, %10, %10};"
                 : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(0.0f));
}

template <bool BF16, bool ASYM, int NT, int GC, bool KFULL>
__global__ void __launch_bounds__(kSkThreads, 2) skinny_kernel(
    const __grid_constant__ CUtensorMap tw, const __grid_constant__ CUtensorMap tx, const SkinnyArgs a) {
  constexpr int kXBytes = NT * 4096;  // the stage's activations: 8 chunks x up to 8*NT tokens x 64 B
  constexpr int kOffX = kSkWBytes;
  constexpr int kOffS = kOffX + kXBytes;
  constexpr int kOffZ = kOffS + kSkSBytes;
  constexpr int kSlot = kOffZ + (ASYM ? kSkZBytes : 0);
  extern __shared__ uint8_t dsmem[];
  __shared__ __align__(8) uint64_t full_bar[kSkStages];
  __shared__ __align__(8) uint64_t empty_bar[kSkStages];
  __shared__ unsigned int s_last;
  __shared__ uint2 zlut[ASYM ? 256 : 1];  // z + 128 -> zero-point constants {za, zb}
  // ring base: the first 1024-byte boundary of the dynamic shared memory
  uint8_t* ring = dsmem + ((1024u - (smem_u32(dsmem) & 1023u)) & 1023u);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int K = a.K, M = a.M;
  const int S_t = a.stages_per_tile;
  const long long u_begin = (long long)blockIdx.x * a.units / gridDim.x;
  const long long u_end = (long long)(blockIdx.x + 1) * a.units / gridDim.x;

  if (tid == 0) {
    for (int i = 0; i < kSkStages; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], kSkWarps);
    }
    fence_barrier_init();
  }
  if (ASYM) {
    for (int i = tid; i < 256; i += kSkThreads) {
      const float z = (float)(i - 128);
      zlut[i] = BF16 ? make_uint2(pack_bf16x2(128.0f + z), 0u)
                     : make_uint2(pack_f16x2(1024.0f + z), pack_f16x2(-(64.0f + z)));
    }
  }
  __syncthreads();
  asm volatile("griddepcontrol.launch_dependents;" :::);

  if (warp == kSkWarps) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      tma_prefetch_desc(&tw);
      tma_prefetch_desc(&tx);
      // The weights (codes, scales, zero points) are only read, so the first
      // ring slots are filled before waiting on the previous kernel; the
      // activations, which that kernel may write, are loaded after the wait.
      const int nfirst = (int)min((long long)kSkStages, u_end - u_begin);
      int it = 0;
      for (long long u = u_begin; u < u_end; ++u, ++it) {
        const int rt = (int)(u / S_t);
        const int st = (int)(u - (long long)rt * S_t);
        const int slot = it % kSkStages;
        if (it >= kSkStages && !mbar_wait(&empty_bar[slot], ((it / kSkStages) & 1) ^ 1)) return;
        uint8_t* dst = ring + (size_t)slot * kSlot;
        const int gs0 = st * 8 / GC;  // first group of the stage
        const int ng = min(8 / GC, a.G - gs0);  // groups of the stage
        // the activation box counts in full (chunks past K read as zeros)
        mbar_arrive_expect_tx(&full_bar[slot],
                              (uint32_t)(kSkWBytes + M * 512 + ng * kSkRows * (ASYM ? 3 : 2)));
        tma_load_2d(dst, &tw, st * 128, rt * kSkRows, &full_bar[slot]);
        const size_t meta0 = ((size_t)rt * a.G + gs0) * kSkRows;  // element index of (tile rt, group gs0, row 0)
        bulk_load(dst + kOffS, a.s_region + meta0 * 2, (uint32_t)(ng * kSkRows * 2), &full_bar[slot]);
        if (ASYM) bulk_load(dst + kOffZ, a.z_region + meta0, (uint32_t)(ng * kSkRows), &full_bar[slot]);
        if (it + 1 == nfirst) {
          asm volatile("griddepcontrol.wait;" ::: "memory");  // X may come from the previous kernel
          for (int i = 0; i <= it; ++i) {  // activations of the slots filled so far
            const long long ui = u_begin + i;
            const int sti = (int)(ui - (ui / S_t) * S_t);
            uint8_t* di = ring + (size_t)(i % kSkStages) * kSlot;
            tma_load_3d(di + kOffX, &tx, 0, 0, sti * 8, &full_bar[i % kSkStages]);
          }
        } else if (it >= nfirst) {
          tma_load_3d(dst + kOffX, &tx, 0, 0, st * 8, &full_bar[slot]);
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
  uint32_t lm_off[4];
#pragma unroll
  for (int cp = 0; cp < 4; ++cp) lm_off[cp] = sw128(lm_row, 2 * cp + (lane >> 4));
  // activation fragment offsets of this thread: column m = g + 8n, 16 bytes t
  // of each 32-k chunk ci at x_off[n] + ci * x_step
  uint32_t x_off[NT];
  bool x_ok[NT];
  const uint32_t x_step = (uint32_t)M * 64u;
#pragma unroll
  for (int n = 0; n < NT; ++n) {
    x_ok[n] = (g + 8 * n) < M;
    x_off[n] = (uint32_t)(kOffX + (g + 8 * n) * 64 + 16 * t);
  }
  const int s_off_r = kOffS + lrow * 2, s_off_r8 = s_off_r + 8 * 2;
  const int z_off_r = kOffZ + lrow, z_off_r8 = z_off_r + 8;
  // zero-point constants of rows lrow / lrow + 8 (symmetric: z = 8)
  //   FP16: za = (1024 + z) pair, zb = -(64 + z) pair;  BF16: za = (128 + z) pair
  uint32_t za_r = BF16 ? pack_bf16x2(136.0f) : pack_f16x2(1032.0f);
  uint32_t zb_r = BF16 ? 0u : pack_f16x2(-72.0f);
  uint32_t za_r8 = za_r, zb_r8 = zb_r;

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
    float d[NT][4];
    float s_r = 0.0f, s_r8 = 0.0f;

    for (int st = st0; st < st1; ++st, ++it) {
      const int slot = it % kSkStages;
      // after a timed-out wait the warp skips its work but keeps the same
      // sequence of named barriers as the other consumer warps
      if (ok && !mbar_wait(&full_bar[slot], (it / kSkStages) & 1)) ok = false;
      if (!ok) continue;
      const uint8_t* sp = ring + (size_t)slot * kSlot;
      const uint32_t sb = smem_u32(sp);
      const int k0 = st * 256;
      uint32_t wr[4][4];
#pragma unroll
      for (int cp = 0; cp < 4; ++cp) ldmatrix_x4(wr[cp], sb + lm_off[cp]);
#pragma unroll
      for (int ci = 0; ci < 8; ++ci) {
        if (!KFULL && k0 + 32 * ci >= K) continue;
        const bool group_start = (ci % GC == 0);
        if (group_start) {
          const int gl = ci / GC;  // group within the stage
          s_r = h2f_bits(*reinterpret_cast<const uint16_t*>(sp + s_off_r + gl * kSkRows * 2));
          s_r8 = h2f_bits(*reinterpret_cast<const uint16_t*>(sp + s_off_r8 + gl * kSkRows * 2));
          if (ASYM) {
            const int z0 = *reinterpret_cast<const int8_t*>(sp + z_off_r + gl * kSkRows);
            const int z1 = *reinterpret_cast<const int8_t*>(sp + z_off_r8 + gl * kSkRows);
            const uint2 c0 = zlut[z0 + 128], c1 = zlut[z1 + 128];
            za_r = c0.x; zb_r = c0.y;
            za_r8 = c1.x; zb_r8 = c1.y;
          }
        }
        const uint32_t wa = wr[ci >> 1][(ci & 1) ? 2 : 0], wb = wr[ci >> 1][(ci & 1) ? 3 : 1];
        uint32_t a0[4], a1[4];
        if (!BF16) {
          // (k0,k1) (k4,k5): 1024 + q minus (1024 + z);  (k2,k3) (k6,k7): (1024 + 16 q) / 16 - (64 + z)
          const uint32_t ta = wa >> 8, tb = wb >> 8;
          a0[0] = hsub2_u32(and_or(wa, 0x000F000Fu, 0x64006400u), za_r);
          a0[1] = hsub2_u32(and_or(wb, 0x000F000Fu, 0x64006400u), za_r8);
          a0[2] = hsub2_u32(and_or(ta, 0x000F000Fu, 0x64006400u), za_r);
          a0[3] = hsub2_u32(and_or(tb, 0x000F000Fu, 0x64006400u), za_r8);
          a1[0] = hfma2_u32(and_or(wa, 0x00F000F0u, 0x64006400u), 0x2C002C00u, zb_r);
          a1[1] = hfma2_u32(and_or(wb, 0x00F000F0u, 0x64006400u), 0x2C002C00u, zb_r8);
          a1[2] = hfma2_u32(and_or(ta, 0x00F000F0u, 0x64006400u), 0x2C002C00u, zb_r);
          a1[3] = hfma2_u32(and_or(tb, 0x00F000F0u, 0x64006400u), 0x2C002C00u, zb_r8);
        } else {
          // pairs (k0,k1) (k2,k3) | (k4,k5) (k6,k7): 128 + q minus (128 + z)
          a0[0] = bsub2_u32(and_or(wa, 0x000F000Fu, 0x43004300u), za_r);
          a0[1] = bsub2_u32(and_or(wb, 0x000F000Fu, 0x43004300u), za_r8);
          a0[2] = bsub2_u32(and_or(wa >> 4, 0x000F000Fu, 0x43004300u), za_r);
          a0[3] = bsub2_u32(and_or(wb >> 4, 0x000F000Fu, 0x43004300u), za_r8);
          a1[0] = bsub2_u32(and_or(wa >> 8, 0x000F000Fu, 0x43004300u), za_r);
          a1[1] = bsub2_u32(and_or(wb >> 8, 0x000F000Fu, 0x43004300u), za_r8);
          a1[2] = bsub2_u32(and_or(wa >> 12, 0x000F000Fu, 0x43004300u), za_r);
          a1[3] = bsub2_u32(and_or(wb >> 12, 0x000F000Fu, 0x43004300u), za_r8);
        }
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          uint4 xv = make_uint4(0u, 0u, 0u, 0u);
          if (x_ok[n]) xv = *reinterpret_cast<const uint4*>(sp + x_off[n] + ci * x_step);
          // FP16: a0 holds k-slots {0,1 | 4,5} of the 8-k word, a1 {2,3 | 6,7};
          // BF16: a0 {0,1 | 2,3}, a1 {4,5 | 6,7}
          const uint32_t b00 = xv.x, b01 = BF16 ? xv.y : xv.z, b10 = BF16 ? xv.z : xv.y, b11 = xv.w;
          if (group_start) mma_16816_zc(d[n], a0, b00, b01, BF16);
          else mma_16816(d[n], a0, b00, b01, BF16);
          mma_16816(d[n], a1, b10, b11, BF16);
        }
        const bool group_end = (ci % GC == GC - 1) || (!KFULL && k0 + 32 * ci + 32 >= K);
        if (group_end) {
#pragma unroll
          for (int n = 0; n < NT; ++n) {
            acc[n][0] = fmaf(s_r, d[n][0], acc[n][0]);
            acc[n][1] = fmaf(s_r, d[n][1], acc[n][1]);
            acc[n][2] = fmaf(s_r8, d[n][2], acc[n][2]);
            acc[n][3] = fmaf(s_r8, d[n][3], acc[n][3]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty_bar[slot]);
    }

    // ---------------------------------------------------------------- output
    const int n0 = rt * kSkRows + lrow;
    const bool whole = (st0 == 0 && st1 == S_t);
    if (whole) {
#pragma unroll
      for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int m = 8 * n + 2 * t + (i & 1);
          const int nn = n0 + ((i & 2) ? 8 : 0);
          if (ok && m < M && nn < a.N) store_out(a.Y, (size_t)m * a.N + nn, acc[n][i], a.y_bf16);
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
            if (m < M && nn < a.N) {
              float sum = 0.0f;
              for (int sl = 0; sl < nslots; ++sl) sum += __ldcg(base + ((size_t)sl * M + m) * kSkRows + r);
              store_out(a.Y, (size_t)m * a.N + nn, sum, a.y_bf16);
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
