// Prefill GEMM with the weights as the tcgen05 A operand in tensor memory:
// Y^T[N, M] = dequant(W)^T[N, K] . X^T[K, M], tiles of 128 output channels
// (the 128 TMEM lanes) x 256 tokens (the MMA's N).
//
// Putting the weights on the M side of the MMA makes every dequantised weight
// serve 256 tokens (twice the reuse of a 128-token tile) and keeps the
// dequantised operand out of shared memory: converter threads write it to
// tensor memory with tcgen05.st, so shared memory only carries the TMA'd
// activations (read once by the tensor core) and the packed codes.
//
//   warp 0      TMA producer: per 128-k block two activation boxes (256 tokens x
//               64 k, 128-byte swizzle = the K-major B-operand layout), the
//               channels' codes (128 rows x 64 bytes) and the block's scales /
//               zero points (INT4) or LUT3 indices and decode tables.
//   warp 1      TMEM owner and MMA issuer: 8 x tcgen05.mma (M = 128, N = 256,
//               K = 16, A from tensor memory) per k-block into one accumulator
//               (256 columns); commits free the A buffer and the stage. A
//               barrier wait costs a few hundred cycles on this GPU, so the
//               blocks are large enough that the waits hide behind the MMAs.
//   warps 2..9  converters: thread (quarter q, lane l) owns channel 32q + l and
//               two 32-k chunks of the k-block; INT4: w = (q - z) * s rounded once to the
//               activation type (nibble -> 1024 + q / 128 + q by AND/OR, an
//               exact packed subtract, one packed multiply); LUT3: the exact
//               BF16 weight from the tile's table (byte permutes). 16 pairs
//               per tcgen05.st. Four A buffers of 64 columns.
//   warps 10-17 epilogue, two per TMEM lane quarter, each taking half of the
//               tokens: tcgen05.ld the finished accumulator 64 tokens per
//               wait (thread = one channel), round and store the elements
//               (a warp's store of one token row is 64 contiguous bytes).
//               The accumulator is held only while it drains, so the fewer
//               the round trips, the less of each tile the converters (which
//               run at most three k-blocks ahead of the stalled MMAs) lose.
//
// Schedule: whole tiles strided over the grid in banded order (bands of 8
// token tiles), or stream-K over the last two waves when the tail wave leaves
// SMs idle (stream_k.cuh).
#pragma once

#include "common.cuh"
#include "tma.cuh"
#include "skinny.cuh"
#include "gemm_tc.cuh"
#include "tc_gemv.cuh"
#include "lut3_gemv.cuh"
#include "stream_k.cuh"

namespace lbq {

constexpr int kTsBN = 128;                 // channels per tile (TMEM lanes)
constexpr int kTsBM = 256;                 // tokens per tile (MMA N)
constexpr int kTsBK = 128;                 // k per block: 8 MMAs per pair of barrier waits
// TMA ring depth: three 74 KB stages, Y stored element by element by eight
// epilogue warps (measured on B200, K=4096 N=14336, LUT3 M=2048: 985-1066
// TFLOP/s against 935-944 with two stages and the output staged through
// shared memory for TMA stores; INT4 with two stages lost a fifth)
constexpr int kTsStages = 3;
constexpr int kTsABufs = 4;                // A (weights) buffers in tensor memory, 64 columns each
constexpr int kTsConvWarps = 8, kTsEpWarps = 8;
// the epilogue warps of one TMEM lane quarter split the tile's tokens
constexpr int kTsEpGroups = kTsEpWarps / 4;
constexpr int kTsEpPairs = kTsBM / 64 / kTsEpGroups;  // 64-token pairs of chunks per epilogue warp
// 32-k chunks per converter thread per block: the block's kTsBK / 32 chunks are
// split over the kTsConvWarps / 4 warps that share a TMEM lane quarter
constexpr int kTsChunksPerConv = (kTsBK / 32) / (kTsConvWarps / 4);
static_assert(kTsChunksPerConv >= 1 && kTsChunksPerConv * (kTsConvWarps / 4) * 32 == kTsBK, "converter split");
constexpr int kTsThreads = (2 + kTsConvWarps + kTsEpWarps) * 32;
constexpr int kTsXBox = kTsBM * 64 * 2;             // one 64-k activation box (32 KB)
constexpr int kTsXBytes = 2 * kTsXBox;              // 64 KB
constexpr int kTsCBytes = kTsBN * 64;               // 8 KB codes (INT4) / 6 KB indices (LUT3)
constexpr int kTsMBytes = 2048;                     // scales + zero points (INT4) / tables (LUT3)
constexpr int kTsOffC = kTsXBytes, kTsOffM = kTsOffC + kTsCBytes;
constexpr int kTsStageBytes = kTsOffM + kTsMBytes;  // 74 KB, a multiple of 1024
constexpr int kTsSmem = kTsStages * kTsStageBytes + 1024;
constexpr uint32_t kTsColA = 0, kTsColD = 256;
static_assert(kTsBM * kTsBN == kSkTileFloats, "a parked tile is one output tile");
static_assert(kTsStageBytes % 1024 == 0, "stages keep 1024-byte alignment");

struct GemmTsArgs {
  void* Y;                   // [M][N]
  const uint8_t* meta0;      // INT4: 128-channel-tiled scales; LUT3: I region (indices)
  const uint8_t* meta1;      // INT4: 128-channel-tiled zero points (ASYM); LUT3: T region (tables)
  int M, N, K, G, group;
  int n_tiles, m_tiles, k_blocks;  // channel tiles, token tiles, 64-k blocks
  int y_bf16;
  SkArgs sk;                 // the schedule (stream_k.cuh)
};

template <bool BF16, bool ASYM, bool LUT>
__global__ void __launch_bounds__(kTsThreads, 1) gemm_ts_kernel(const __grid_constant__ CUtensorMap tx,
                                                                const __grid_constant__ CUtensorMap tq,
                                                                const GemmTsArgs a) {
  extern __shared__ uint8_t dsmem[];
  __shared__ __align__(8) uint64_t full_bar[kTsStages], empty_bar[kTsStages];
  __shared__ __align__(8) uint64_t a_full[kTsABufs], a_empty[kTsABufs], d_full, d_empty;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int sk_ok_sh;  // the epilogue's wait for a parked part succeeded
  uint8_t* ring = dsmem + ((1024u - (smem_u32(dsmem) & 1023u)) & 1023u);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int i = 0; i < kTsStages; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], 1 + kTsConvWarps);
    }
    for (int i = 0; i < kTsABufs; ++i) {
      mbar_init(&a_full[i], kTsConvWarps);
      mbar_init(&a_empty[i], 1);
    }
    mbar_init(&d_full, 1);
    mbar_init(&d_empty, kTsEpWarps);
    fence_barrier_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 :: "r"(smem_u32(&tmem_base_sh)), "r"(512u) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tx);
      if (!LUT) tma_prefetch_desc(&tq);
      int it = 0;
      bool ok = true;
      SkSched sch(a.sk.dp_tiles, a.sk.sk_items, a.k_blocks, (int)blockIdx.x, (int)gridDim.x);
      SkItem w;
      while (ok && sch.next(w)) {
        int nt, mt;  // banded order: codes reused from L2 across a band's token tiles
        sk_tile_coords(w.tile, a.n_tiles, a.m_tiles, nt, mt);
        const int rows = min(kTsBN, a.N - nt * kTsBN);
        for (int kb = w.kb0; kb < w.kb1; ++kb, ++it) {
          const int s = it % kTsStages;
          if (it >= kTsStages && !mbar_wait_sleep(&empty_bar[s], ((it / kTsStages) & 1) ^ 1)) { ok = false; break; }
          uint8_t* st = ring + (size_t)s * kTsStageBytes;
          const int nxb = min(2, (a.K - kb * kTsBK + 63) / 64);  // 64-k activation boxes inside K
          if (LUT) {
            // the block's two 64-k LUT tiles: indices (24 B per channel) and tables (16 B per 8 channels)
            mbar_arrive_expect_tx(&full_bar[s], (uint32_t)(nxb * (kTsXBox + rows * 24 + (rows / 8) * 16)));
            for (int j = 0; j < nxb; ++j) {
              const int kt = kb * 2 + j;
              tma_load_2d(st + j * kTsXBox, &tx, kt * 64, mt * kTsBM, &full_bar[s]);
              bulk_load(st + kTsOffC + j * (kTsBN * 24), a.meta0 + ((size_t)kt * a.N + nt * kTsBN) * 24,
                        (uint32_t)(rows * 24), &full_bar[s]);
              bulk_load(st + kTsOffM + j * 256, a.meta1 + ((size_t)kt * (a.N / 8) + nt * (kTsBN / 8)) * 16,
                        (uint32_t)((rows / 8) * 16), &full_bar[s]);
            }
          } else {
            const int g0 = (kb * kTsBK) / a.group;
            const int ng = min(max(1, kTsBK / a.group), a.G - g0);  // K may end inside the block
            mbar_arrive_expect_tx(&full_bar[s], (uint32_t)(nxb * kTsXBox + kTsCBytes + ng * 128 * (ASYM ? 3 : 2)));
            for (int j = 0; j < nxb; ++j) tma_load_2d(st + j * kTsXBox, &tx, kb * kTsBK + 64 * j, mt * kTsBM, &full_bar[s]);
            tma_load_2d(st + kTsOffC, &tq, kb * (kTsBK / 2), nt * kTsBN, &full_bar[s]);
            const size_t m0 = ((size_t)nt * a.G + g0) * 128;
            bulk_load(st + kTsOffM, a.meta0 + m0 * 2, (uint32_t)(ng * 256), &full_bar[s]);
            if (ASYM) bulk_load(st + kTsOffM + 1024, a.meta1 + m0, (uint32_t)(ng * 128), &full_bar[s]);
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_m128(BF16, kTsBM);
      int it = 0, t_iter = 0;
      bool ok = true;
      SkSched sch(a.sk.dp_tiles, a.sk.sk_items, a.k_blocks, (int)blockIdx.x, (int)gridDim.x);
      SkItem w;
      for (; ok && sch.next(w); ++t_iter) {
        if (t_iter >= 1 && !mbar_wait_sleep(&d_empty, (t_iter - 1) & 1)) break;
        tc_fence_after();
        for (int kb = w.kb0; kb < w.kb1; ++kb, ++it) {
          const int s = it % kTsStages, b = it % kTsABufs;
          if (!mbar_wait_sleep(&full_bar[s], (it / kTsStages) & 1)) { ok = false; break; }
          if (!mbar_wait_sleep(&a_full[b], (it / kTsABufs) & 1)) { ok = false; break; }
          tc_fence_after();
          const uint32_t xb = smem_u32(ring + (size_t)s * kTsStageBytes);
          const int nkk = min(kTsBK, a.K - kb * kTsBK + 15) / 16;  // 16-k slices inside K (K % 32 == 0)
          for (int kk = 0; kk < nkk; ++kk) {
            const uint64_t db = umma_desc_sw128(xb + (uint32_t)(kk >> 2) * kTsXBox) + (uint64_t)((kk & 3) * 2);
            umma_ts(tmem + kTsColD, tmem + kTsColA + (uint32_t)b * 64 + (uint32_t)kk * 8, db, idesc,
                    (kb > w.kb0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&empty_bar[s]);
          umma_commit(&a_empty[b]);
        }
        if (ok) umma_commit(&d_full);
      }
    }
  } else if (warp < 2 + kTsConvWarps) {
    // ------------------------------------------------------------------ converters
    const int cw = warp - 2;
    const int q = warp & 3;          // TMEM lane quarter this warp may access
    const int part = cw >> 2;        // which chunks of the k-block this warp converts
    const int r = 32 * q + lane;     // channel within the tile
    const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16);
    int it = 0;
    bool ok = true;
    SkSched sch(a.sk.dp_tiles, a.sk.sk_items, a.k_blocks, (int)blockIdx.x, (int)gridDim.x);
    SkItem w;
    while (sch.next(w)) {
      int nt, mt_unused;
      sk_tile_coords(w.tile, a.n_tiles, a.m_tiles, nt, mt_unused);
      const bool row_ok = nt * kTsBN + r < a.N;
      for (int kb = w.kb0; kb < w.kb1; ++kb, ++it) {
        const int s = it % kTsStages, b = it % kTsABufs;
        if (ok && !mbar_wait_sleep(&full_bar[s], (it / kTsStages) & 1)) ok = false;
        if (ok && it >= kTsABufs && !mbar_wait_sleep(&a_empty[b], ((it / kTsABufs) & 1) ^ 1)) ok = false;
        tc_fence_after();
        const uint8_t* st = ring + (size_t)s * kTsStageBytes;
        // this thread's chunks of the block (32 k, 16 pairs each)
#pragma unroll
        for (int j = 0; j < kTsChunksPerConv; ++j) {
          const int ci = part * kTsChunksPerConv + j;  // chunk 0..3 of the block
          const int kc = ci * 32;                      // its first k within the block
          uint32_t o[16];
          if (ok && row_ok && kb * kTsBK + kc < a.K) {
            if (LUT) {
              const uint8_t* tile = st + kTsOffC + (ci >> 1) * (kTsBN * 24);  // LUT tile kb*2 + ci/2
              const uint32_t* wp = reinterpret_cast<const uint32_t*>(tile + r * 24 + (ci & 1) * 12);
              const uint32_t wa = wp[0], wb = wp[1], wc = wp[2];
              const uint4 tab = lds128(smem_u32(st + kTsOffM + (ci >> 1) * 256 + (r >> 3) * 16));
#pragma unroll
              for (int t = 0; t < 4; ++t) {
                uint32_t p[4];
                lut3_decode8(lut3_selector(t < 2 ? wa : wb, wc, t), tab, p);
                o[4 * t + 0] = p[0]; o[4 * t + 1] = p[1]; o[4 * t + 2] = p[2]; o[4 * t + 3] = p[3];
              }
            } else {
              const int gl = kc / a.group;  // group of the chunk among the block's groups
              const uint16_t sbits = *reinterpret_cast<const uint16_t*>(st + kTsOffM + (gl * 128 + r) * 2);
              const int z = ASYM ? (int)*reinterpret_cast<const int8_t*>(st + kTsOffM + 1024 + gl * 128 + r) : 8;
              uint32_t c1, c2;
              zero_consts<BF16>(z, c1, c2);
              const uint32_t s2 = scale_pair<BF16>(sbits);
              // the codes box is TMA-swizzled in 64-byte spans (16-byte chunk c of
              // row r at chunk c ^ ((r >> 1) & 3)): a quarter-warp's loads hit
              // eight different bank groups
              const uint4 wv = lds128(smem_u32(st + kTsOffC + r * 64 + ((ci ^ ((r >> 1) & 3)) << 4)));
              const uint32_t wd[4] = {wv.x, wv.y, wv.z, wv.w};
              constexpr uint32_t magic = BF16 ? 0x43004300u : 0x64006400u;
#pragma unroll
              for (int q4 = 0; q4 < 4; ++q4) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const uint32_t pq = and_or(wd[q4] >> (4 * e), 0x000F000Fu, magic);
                  o[4 * q4 + e] = BF16 ? bmul2_u32(bsub2_u32(pq, c1), s2) : hmul2_u32(hsub2_u32(pq, c1), s2);
                }
              }
            }
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) o[i] = 0u;
          }
          tmem_st16(lane_base + kTsColA + (uint32_t)b * 64 + (uint32_t)(kc / 2), o);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0 && ok) {
          mbar_arrive(&a_full[b]);
          mbar_arrive(&empty_bar[s]);
        }
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue
    // Every epilogue warp walks every item, also after a timed-out wait (then
    // it loads and stores nothing). The stores take no barrier: each warp
    // reads its own TMEM lanes and tokens and writes its own channels, and
    // releases its part of the accumulator as soon as it is in registers.
    const int q = warp & 3;
    const int r = 32 * q + lane;  // channel within the tile
    const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16);
    const int eg = (warp - 2 - kTsConvWarps) >> 2;  // epilogue group: tokens [64 kTsEpPairs eg, +64 kTsEpPairs)
    const bool lead = warp == 2 + kTsConvWarps && lane == 0;  // flags of cut tiles
    int t_iter = 0;
    bool ok = true;
    SkSched sch(a.sk.dp_tiles, a.sk.sk_items, a.k_blocks, (int)blockIdx.x, (int)gridDim.x);
    SkItem w;
    for (; sch.next(w); ++t_iter) {
      int nt, mt;
      sk_tile_coords(w.tile, a.n_tiles, a.m_tiles, nt, mt);
      if (ok && !mbar_wait_sleep(&d_full, t_iter & 1)) ok = false;
      tc_fence_after();
      // an earlier part: wait for the later part's sums in slot blockIdx.x + 1
      const float* park_in = a.sk.partials + (size_t)(blockIdx.x + 1) * kSkTileFloats + r;
      float* park_out = a.sk.partials + (size_t)blockIdx.x * kSkTileFloats + r;
      if (w.part == 2) {
        if (lead) sk_ok_sh = (ok && sk_wait_parked(a.sk)) ? 1 : 0;
        asm volatile("bar.sync 1, %0;" :: "r"(kTsEpWarps * 32) : "memory");
        ok = ok && sk_ok_sh != 0;
      }
      // two 32-token chunks per TMEM round trip (a load's wait costs about as
      // much as the chunk's stores)
#pragma unroll 1
      for (int jp = eg * kTsEpPairs; jp < (eg + 1) * kTsEpPairs; ++jp) {
        uint32_t vv[2][32];
        if (ok) {
          tmem_ld32_nowait(lane_base + kTsColD + (uint32_t)(jp * 64), vv[0]);
          tmem_ld32_nowait(lane_base + kTsColD + (uint32_t)(jp * 64 + 32), vv[1]);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) vv[0][i] = vv[1][i] = 0u;
        }
        if (jp == (eg + 1) * kTsEpPairs - 1) {  // this warp's part of the accumulator is in registers
          tc_fence_before();
          __syncwarp();
          if (lane == 0 && ok) mbar_arrive(&d_empty);
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int j = 2 * jp + h;
          uint32_t(&v)[32] = vv[h];
          if (w.part == 2 && ok) {  // own sums + parked sums, in that order
#pragma unroll
            for (int i = 0; i < 32; ++i)
              v[i] = __float_as_uint(__uint_as_float(v[i]) + __ldcg(park_in + (j * 32 + i) * kTsBN));
          }
          const int m0 = mt * kTsBM + j * 32;
          if (w.part == 1) {  // a later part: park the FP32 sums (all 256 tokens; rows past M hold zeros)
            if (ok) {
#pragma unroll
              for (int i = 0; i < 32; ++i) __stcg(park_out + (j * 32 + i) * kTsBN, __uint_as_float(v[i]));
            }
          } else {  // element stores: per warp, unordered
            const int n = nt * kTsBN + r;
            if (ok && n < a.N) {
#pragma unroll
              for (int i = 0; i < 32; ++i)
                if (m0 + i < a.M) store_out(a.Y, (size_t)(m0 + i) * a.N + n, __uint_as_float(v[i]), a.y_bf16);
            }
          }
        }
      }
      if (w.part == 1) {  // the parked sums are visible GPU-wide before the flag
        __threadfence();
        asm volatile("bar.sync 1, %0;" :: "r"(kTsEpWarps * 32) : "memory");
        if (lead && ok && !a.sk.debug_hold) st_release_u32(a.sk.flags + blockIdx.x, 1u);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem), "r"(512u) : "memory");
  }
}

}  // namespace lbq
