// Prefill GEMM on the 5th-generation tensor cores: Y[M, N] = X[M, K] . dequant(W)[K, N].
//
// Prefill is a dense contraction (arithmetic intensity in the thousands of
// FLOP/byte), so it runs on tcgen05 with the accumulator in tensor memory.
// The weights stay packed in HBM and in the TMA pipeline; they are dequantised
// in shared memory right before the MMA reads them ("dequantise just before
// use" of "Low Bit Metal Kernels"; the weight tile is fetched in its kernel
// image with plain block copies, as the vLLM LUT-B kernel does).
//
// One persistent CTA per SM, tiles of BM = 128 tokens x BN = 256 outputs,
// k-blocks of 64. Warp roles:
//   warp 0      TMA producer: X tile (128 x 64, 128-byte swizzle), packed
//               code tile (256 rows x 32 bytes), and bulk copies of the
//               block's scales / zero points (contiguous per 128-channel tile);
//               one mbarrier per stage, ring of kTcStages.
//   warp 1      TMEM owner (alloc / dealloc of 512 columns) and MMA issuer:
//               one thread issues 4 x tcgen05.mma.kind::f16 (M=128, N=256,
//               K=16) per k-block into one of two TMEM accumulators and
//               commits to the stage / B-tile / accumulator barriers.
//   warps 2..9  dequantisers (one weight row each): codes -> BF16 (or FP16)
//               weights written straight into the K-major 128-byte-swizzled
//               layout the UMMA shared-memory descriptor describes;
//               fence.proxy.async, then arrive.
//   warps 10-13 epilogue: tcgen05.ld the finished accumulator (each warp its
//               32 TMEM lanes = 32 tokens), round to BF16/FP16, store to Y;
//               runs while the MMA fills the other accumulator.
//
// Dequantised value: w = (q - z) * s rounded once more to the activation
// type, as the Metal listing stores its dequantised weight in the activation
// type. (q - z) is formed exactly (magic-number AND/OR + subtract); the scale
// multiply rounds once (FP16: the scale is exact; BF16: the scale is first
// rounded to BF16), so each weight carries a relative error below 2^-7 for
// BF16 and 2^-11 for FP16.
#pragma once

#include "common.cuh"
#include "tma.cuh"
#include "lut3_gemv.cuh"

namespace lbq {

constexpr int kTcBM = 128, kTcBN = 256, kTcBK = 64;
constexpr int kTcStages = 4;                   // X + codes ring
constexpr int kTcBStages = 3;                  // dequantised weight tiles
constexpr int kTcDqWarps = 8, kTcEpWarps = 4;
constexpr int kTcDqRows = kTcBN / (kTcDqWarps * 32);  // weight rows per dequantiser thread
constexpr int kTcThreads = (2 + kTcDqWarps + kTcEpWarps) * 32;
constexpr int kTcABytes = kTcBM * kTcBK * 2;   // 16 KB
constexpr int kTcPBytes = kTcBN * kTcBK / 2;   // 8 KB of codes
constexpr int kTcSBytes = 1024;                // scales: 2 channel tiles x up to 2 groups x 128 x 2 B
constexpr int kTcZBytes = 1024;                // zero points: 2 x 2 x 128 x 1 B (padded)
constexpr int kTcStageBytes = kTcABytes + kTcPBytes + kTcSBytes + kTcZBytes;  // 26 KB, 1024-aligned
constexpr int kTcBBytes = kTcBN * kTcBK * 2;   // 32 KB
constexpr int kTcSmem = kTcStages * kTcStageBytes + kTcBStages * kTcBBytes + 1024;
constexpr uint32_t kTcTmemCols = 512;

struct GemmTcArgs {
  void* Y;
  const uint8_t* s_region;  // INT4: 128-channel-tiled scales; LUT3: I region (indices)
  const uint8_t* z_region;  // INT4: 128-channel-tiled zero points (ASYM); LUT3: T region (tables)
  int G, tiles128;          // groups per channel, 128-channel tiles
  int M, N, K, gshift64;   // gshift64: log2(group / 32)
  int m_tiles, n_tiles, k_blocks;
  int y_bf16;
};

// K-major operand tile with 128-byte swizzle: rows of 128 bytes, 8-row groups
// 1024 bytes apart (SBO), version 1, layout type 2.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t smem_addr) {
  return (uint64_t)((smem_addr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor of kind::f16: D = F32, A = B = BF16 (1) or F16 (0),
// both K-major, N = 256, M = 128.
__host__ __device__ constexpr uint32_t umma_idesc_f16(bool bf16) {
  return (1u << 4) | ((bf16 ? 1u : 0u) << 7) | ((bf16 ? 1u : 0u) << 10) | ((uint32_t)(kTcBN >> 3) << 17) |
         ((uint32_t)(kTcBM >> 4) << 24);
}

__device__ __forceinline__ void umma_f16(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t idesc, uint32_t acc) {
  asm volatile("{\n\t.reg .pred p;\n\t"
               "setp.ne.b32 p, %4, 0;\n\t"
               "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}"
               :: "r"(tmem_d), "l"(da), "l"(db), "r"(idesc), "r"(acc), "r"(0u), "r"(0u), "r"(0u), "r"(0u)
               : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               :: "r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 "
               "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
               "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
                 "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
                 "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
                 "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
                 "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
               : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// The same load without its wait: several loads may share one tmem_wait_ld().
__device__ __forceinline__ void tmem_ld32_nowait(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 "
               "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
               "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
                 "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
                 "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
                 "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
                 "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
               : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ uint32_t bmul2_u32(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t hmul2_u32(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// One 32-bit code word (8 consecutive k of one row) -> 8 weights (q - z) * s
// in k order, as four packed pairs.
template <bool BF16>
__device__ __forceinline__ uint4 dequant_scaled(uint32_t w, uint32_t c1, uint32_t c2, uint32_t s2) {
  uint4 o;
  if (!BF16) {
    const uint32_t t = w >> 8;
    o.x = hmul2_u32(hsub2_u32(and_or(w, 0x000F000Fu, 0x64006400u), c1), s2);
    o.y = hmul2_u32(hfma2_u32(and_or(w, 0x00F000F0u, 0x64006400u), 0x2C002C00u, c2), s2);
    o.z = hmul2_u32(hsub2_u32(and_or(t, 0x000F000Fu, 0x64006400u), c1), s2);
    o.w = hmul2_u32(hfma2_u32(and_or(t, 0x00F000F0u, 0x64006400u), 0x2C002C00u, c2), s2);
  } else {
    o.x = bmul2_u32(bsub2_u32(and_or(w, 0x000F000Fu, 0x43004300u), c1), s2);
    o.y = bmul2_u32(bsub2_u32(and_or(w >> 4, 0x000F000Fu, 0x43004300u), c1), s2);
    o.z = bmul2_u32(bsub2_u32(and_or(w >> 8, 0x000F000Fu, 0x43004300u), c1), s2);
    o.w = bmul2_u32(bsub2_u32(and_or(w >> 12, 0x000F000Fu, 0x43004300u), c1), s2);
  }
  return o;
}

template <bool BF16>
__device__ __forceinline__ uint32_t scale_pair(uint16_t s_bits) {
  if (!BF16) return (uint32_t)s_bits | ((uint32_t)s_bits << 16);
  const __nv_bfloat16 b = __float2bfloat16_rn(h2f_bits(s_bits));
  const uint16_t u = *reinterpret_cast<const uint16_t*>(&b);
  return (uint32_t)u | ((uint32_t)u << 16);
}

// LUT: false = INT4 image, true = LUT3 image (BF16 activations only).
template <bool BF16, bool ASYM, bool LUT>
__global__ void __launch_bounds__(kTcThreads, 1) gemm_tc_kernel(
    const __grid_constant__ CUtensorMap tx, const __grid_constant__ CUtensorMap tq, const GemmTcArgs a) {
  extern __shared__ uint8_t dsmem[];
  __shared__ __align__(8) uint64_t full_ap[kTcStages], empty_ap[kTcStages];
  __shared__ __align__(8) uint64_t full_b[kTcBStages], empty_b[kTcBStages];
  __shared__ __align__(8) uint64_t acc_full[2], acc_empty[2];
  __shared__ uint32_t tmem_base_sh;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem;
  uint8_t* btile = smem + kTcStages * kTcStageBytes;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int total_tiles = a.m_tiles * a.n_tiles;

  if (tid == 0) {
    for (int i = 0; i < kTcStages; ++i) {
      mbar_init(&full_ap[i], 1);
      mbar_init(&empty_ap[i], 1 + kTcDqWarps);
    }
    for (int i = 0; i < kTcBStages; ++i) {
      mbar_init(&full_b[i], kTcDqWarps);
      mbar_init(&empty_b[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], kTcEpWarps);
    }
    fence_barrier_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 :: "r"(smem_u32(&tmem_base_sh)), "r"(kTcTmemCols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_sh;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tx);
      tma_prefetch_desc(&tq);
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
        const int mb = tile % a.m_tiles, nb = tile / a.m_tiles;
        for (int kb = 0; kb < a.k_blocks; ++kb, ++it) {
          const int s = it % kTcStages;
          if (it >= kTcStages && !mbar_wait(&empty_ap[s], ((it / kTcStages) & 1) ^ 1)) { ok = false; break; }
          uint8_t* st = ring + s * kTcStageBytes;
          if (LUT) {
            // tile kb of the indices and tables of channels nb*256 .. (contiguous, tile-major)
            const int rows = min(kTcBN, a.N - nb * kTcBN);
            mbar_arrive_expect_tx(&full_ap[s], (uint32_t)(kTcABytes + rows * 24 + (rows / 8) * 16));
            tma_load_2d(st, &tx, kb * kTcBK, mb * kTcBM, &full_ap[s]);
            bulk_load(st + kTcABytes, a.s_region + ((size_t)kb * a.N + nb * kTcBN) * 24, (uint32_t)(rows * 24),
                      &full_ap[s]);
            bulk_load(st + kTcABytes + kTcPBytes, a.z_region + ((size_t)kb * (a.N / 8) + nb * (kTcBN / 8)) * 16,
                      (uint32_t)((rows / 8) * 16), &full_ap[s]);
            continue;
          }
          const int g0 = (kb * 2) >> a.gshift64;  // first group of the k-block
          const int ng = min(a.gshift64 == 0 ? 2 : 1, a.G - g0);  // groups of the k-block
          const int ntl = min(2, a.tiles128 - 2 * nb);  // 128-channel tiles of this 256-wide block
          mbar_arrive_expect_tx(&full_ap[s], (uint32_t)(kTcABytes + kTcPBytes + ntl * ng * 128 * (ASYM ? 3 : 2)));
          tma_load_2d(st, &tx, kb * kTcBK, mb * kTcBM, &full_ap[s]);
          tma_load_2d(st + kTcABytes, &tq, kb * (kTcBK / 2), nb * kTcBN, &full_ap[s]);
          for (int tl = 0; tl < ntl; ++tl) {
            const size_t meta0 = ((size_t)(2 * nb + tl) * a.G + g0) * 128;
            bulk_load(st + kTcABytes + kTcPBytes + tl * ng * 256, a.s_region + meta0 * 2, (uint32_t)(ng * 256), &full_ap[s]);
            if (ASYM)
              bulk_load(st + kTcABytes + kTcPBytes + kTcSBytes + tl * ng * 128, a.z_region + meta0, (uint32_t)(ng * 128),
                        &full_ap[s]);
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_f16(BF16);
      int it = 0, bit = 0, t_iter = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x, ++t_iter) {
        const int ab = t_iter & 1;
        if (t_iter >= 2 && !mbar_wait(&acc_empty[ab], ((t_iter >> 1) & 1) ^ 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t tmem_d = tmem_base + (uint32_t)(ab * kTcBN);
        for (int kb = 0; kb < a.k_blocks; ++kb, ++it, ++bit) {
          const int s = it % kTcStages;
          const int sb = bit % kTcBStages;
          if (!mbar_wait(&full_ap[s], (it / kTcStages) & 1)) { ok = false; break; }
          if (!mbar_wait(&full_b[sb], (bit / kTcBStages) & 1)) { ok = false; break; }
          tc_fence_after();
          const uint64_t da = umma_desc_sw128(smem_u32(ring + s * kTcStageBytes));
          const uint64_t db = umma_desc_sw128(smem_u32(btile + sb * kTcBBytes));
#pragma unroll
          for (int kk = 0; kk < kTcBK / 16; ++kk)
            umma_f16(tmem_d, da + (uint64_t)(kk * 2), db + (uint64_t)(kk * 2), idesc, (kb > 0 || kk > 0) ? 1u : 0u);
          umma_commit(&empty_ap[s]);
          umma_commit(&empty_b[sb]);
        }
        if (ok) umma_commit(&acc_full[ab]);
      }
    }
  } else if (warp < 2 + kTcDqWarps) {
    // ------------------------------------------------------------------ dequantisers
    const int dt = tid - 64;  // rows dt + kTcDqWarps * 32 * i of the weight tile
    int it = 0, bit = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
      const int nb = tile / a.m_tiles;
      for (int kb = 0; kb < a.k_blocks; ++kb, ++it, ++bit) {
        const int s = it % kTcStages;
        const int sb = bit % kTcBStages;
        if (!mbar_wait(&full_ap[s], (it / kTcStages) & 1)) { ok = false; break; }
        if (bit >= kTcBStages && !mbar_wait(&empty_b[sb], ((bit / kTcBStages) & 1) ^ 1)) { ok = false; break; }
        const uint32_t st = smem_u32(ring + s * kTcStageBytes);
        const uint32_t bt = smem_u32(btile + sb * kTcBBytes);
        if (LUT) {
#pragma unroll
          for (int hr = 0; hr < kTcDqRows; ++hr) {
            const int n = dt + kTcDqWarps * 32 * hr;
            if (nb * kTcBN + n >= a.N) continue;
            // 24 bytes of indices per channel: 8-byte aligned, so three 8-byte loads
            const uint8_t* ip = ring + s * kTcStageBytes + kTcABytes + n * 24;
            const uint2 p0 = *reinterpret_cast<const uint2*>(ip);
            const uint2 p1 = *reinterpret_cast<const uint2*>(ip + 8);
            const uint2 p2 = *reinterpret_cast<const uint2*>(ip + 16);
            const uint32_t w[6] = {p0.x, p0.y, p1.x, p1.y, p2.x, p2.y};
            const uint4 tab = lds128(st + kTcABytes + kTcPBytes + (n >> 3) * 16);
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
              for (int t = 0; t < 4; ++t) {
                uint32_t pr[4];
                lut3_decode8(lut3_selector(w[3 * h + (t < 2 ? 0 : 1)], w[3 * h + 2], t), tab, pr);
                const int c = 4 * h + t;
                asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};"
                             :: "r"(bt + (uint32_t)(n * 128 + ((c ^ (n & 7)) << 4))), "r"(pr[0]), "r"(pr[1]),
                                "r"(pr[2]), "r"(pr[3]) : "memory");
              }
          }
          fence_proxy_async();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(&full_b[sb]);
            mbar_arrive(&empty_ap[s]);
          }
          continue;
        }
        const int g0 = (kb * 2) >> a.gshift64;
        const int ng = min(a.gshift64 == 0 ? 2 : 1, a.G - g0);
#pragma unroll
        for (int h = 0; h < kTcDqRows; ++h) {
          const int n = dt + kTcDqWarps * 32 * h;
          const uint4 p0 = lds128(st + kTcABytes + n * 32);
          const uint4 p1 = lds128(st + kTcABytes + n * 32 + 16);
          const uint32_t words[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            // words 4*half .. 4*half+3 cover k = 32*half .. 32*half+31 of the k-block
            const int gi = (kb * 2 + half) >> a.gshift64;
            const int mi = ((n >> 7) * ng + (gi - g0)) * 128 + (n & 127);  // (tile, group, row) in the stage
            uint16_t sbits = 0;
            int z = 8;
            if (nb * kTcBN + n < a.N && gi - g0 < ng) {
              asm volatile("ld.shared.u16 %0, [%1];" : "=h"(sbits) : "r"(st + kTcABytes + kTcPBytes + mi * 2));
              if (ASYM) asm volatile("ld.shared.s8 %0, [%1];" : "=r"(z) : "r"(st + kTcABytes + kTcPBytes + kTcSBytes + mi));
            }
            uint32_t c1, c2;
            zero_consts<BF16>(z, c1, c2);
            const uint32_t s2 = scale_pair<BF16>(sbits);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int c = 4 * half + j;  // 16-byte chunk (8 k) of the 128-byte row
              const uint4 o = dequant_scaled<BF16>(words[c], c1, c2, s2);
              asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};"
                           :: "r"(bt + (uint32_t)(n * 128 + ((c ^ (n & 7)) << 4))), "r"(o.x), "r"(o.y), "r"(o.z),
                              "r"(o.w) : "memory");
            }
          }
        }
        fence_proxy_async();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&full_b[sb]);
          mbar_arrive(&empty_ap[s]);
        }
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue
    const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31
    int t_iter = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x, ++t_iter) {
      const int mb = tile % a.m_tiles, nb = tile / a.m_tiles;
      const int ab = t_iter & 1;
      if (!mbar_wait(&acc_full[ab], (t_iter >> 1) & 1)) { ok = false; break; }
      tc_fence_after();
      const int m = mb * kTcBM + quarter * 32 + lane;
      const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(ab * kTcBN);
#pragma unroll 1
      for (int j = 0; j < kTcBN / 32; ++j) {
        uint32_t r[32];
        tmem_ld32(taddr + (uint32_t)(j * 32), r);
        const int n0 = nb * kTcBN + j * 32;
        if (m < a.M) {
          uint8_t* yrow = static_cast<uint8_t*>(a.Y) + ((size_t)m * a.N + n0) * 2;
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint32_t pk[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float lo = __uint_as_float(r[8 * v + 2 * e]), hi = __uint_as_float(r[8 * v + 2 * e + 1]);
              if (a.y_bf16) {
                const __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
                pk[e] = *reinterpret_cast<const uint32_t*>(&b);
              } else {
                const __half2 b = __floats2half2_rn(lo, hi);
                pk[e] = *reinterpret_cast<const uint32_t*>(&b);
              }
            }
            const int n = n0 + 8 * v;
            if (n + 8 <= a.N && (a.N & 7) == 0) {
              *reinterpret_cast<uint4*>(yrow + v * 16) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            } else {
              for (int e = 0; e < 8 && n + e < a.N; ++e)
                reinterpret_cast<uint16_t*>(yrow + v * 16)[e] = (uint16_t)(pk[e >> 1] >> (16 * (e & 1)));
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[ab]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem_base), "r"(kTcTmemCols) : "memory");
  }
}

}  // namespace lbq
