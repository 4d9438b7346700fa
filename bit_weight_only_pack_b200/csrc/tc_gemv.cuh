// Decode GEMV / skinny GEMM (batch 1..16) on INT4 weights with the 5th-generation
// tensor cores: Y^T[N, M] = dequant(W)^T[N, K] . X^T[K, M], the weight rows on
// the MMA M side (128 rows = the 128 lanes of tensor memory), the batch padded
// to the MMA's N = 16.
//
// Why tcgen05 here: at 4.1-4.75 bits per weight an SM must take in ~46 weights
// per clock to keep up with HBM, and the legacy warp-level MMA path runs out of
// tensor throughput well before that on this GPU. tcgen05.mma with the A operand
// in tensor memory takes 2048 weights per instruction from one issuing thread,
// so the per-weight cost is only the code -> operand conversion:
//
//  * 8 converter warps; thread (quarter q, lane l) owns weight row r = 32q + l,
//    which is TMEM lane r. Per 256-k stage each thread converts its row's 128
//    code bytes (read from the TMA-swizzled tile, conflict-free) into 128
//    FP16/BF16 pairs (q - z): a nibble OR-ed into the mantissa of 1024.0 /
//    128.0 is 1024 + q / 128 + q, and one packed subtract of 1024 + z / 128 + z
//    leaves q - z, all exact. They go to tensor memory with tcgen05.st (one
//    instruction per 32 weights). The two warps of a lane quarter split the
//    stage's k range.
//  * One MMA thread issues one MMA per 16-k slice into the group's accumulator
//    (16 TMEM columns, double-buffered by stage); per stage one commit frees the
//    A buffer, the shared-memory slot and publishes the accumulators.
//  * The converter threads then read their row's group accumulators
//    (tcgen05.ld) and add s * D to FP32 registers; the output (or a stream-K
//    partial) is written once per row tile.
//  * TMA producer warp: code tile (128 rows x 128 B, 128-byte swizzle), the
//    activation boxes (16 rows x 64 k, 128-byte swizzle: exactly the K-major
//    B-operand layout), and bulk copies of the tile's scales / zero points.
//    Weight copies for the first stages are issued before waiting on the
//    previous kernel (programmatic dependent launch); activations after.
//  * Stream-K over (128-row tile, 256-k stage) units, as in the warp-MMA kernel.
//
// Tensor memory (512 columns, one CTA per SM): A double buffer 2 x 128,
// accumulators 2 x (8 groups x 16).
#pragma once

#include "common.cuh"
#include "tma.cuh"
#include "skinny.cuh"
#include "gemm_tc.cuh"

namespace lbq {

constexpr int kTgStages = 6;
constexpr int kTgConvWarps = 8;
constexpr int kTgThreads = (2 + kTgConvWarps) * 32;
constexpr int kTgCodeBytes = 128 * 128;           // 128 rows x 256 k
constexpr int kTgXBox = 16 * 128;                 // 16 batch rows x 64 k (BF16/FP16)
constexpr int kTgOffX = kTgCodeBytes;
constexpr int kTgOffS = kTgOffX + 4 * kTgXBox;    // scales: up to 8 groups x 128 rows x 2 B
constexpr int kTgOffZ = kTgOffS + 8 * 128 * 2;    // zero points: up to 8 groups x 128 rows
constexpr int kTgSlot = kTgOffZ + 8 * 128;        // 27 KB, a multiple of 1024
constexpr int kTgSmem = kTgStages * kTgSlot + 1024;
constexpr uint32_t kTgColA = 0, kTgColD = 256;
static_assert(kTgSlot % 1024 == 0, "stage slots must keep 1024-byte alignment");

struct TcGemvArgs {
  void* Y;
  float* partials;          // [row_tiles][max_slots][M][128]
  unsigned int* counters;   // [row_tiles]
  const uint8_t* s_region;  // 128-channel-tiled scales
  const uint8_t* z_region;  // 128-channel-tiled zero points (ASYM)
  int K, N, M, G;
  int stages_per_tile, row_tiles, max_slots;
  long long units;
  int y_bf16;
};

__device__ __forceinline__ uint32_t umma_idesc_m128(bool bf16, int n) {
  return (1u << 4) | ((bf16 ? 1u : 0u) << 7) | ((bf16 ? 1u : 0u) << 10) | ((uint32_t)(n >> 3) << 17) |
         ((uint32_t)(128 >> 4) << 24);
}

// D[tmem] (+)= A[tmem] . B[smem descriptor]
__device__ __forceinline__ void umma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                        uint32_t acc) {
  asm volatile("{\n\t.reg .pred p;\n\t"
               "setp.ne.b32 p, %4, 0;\n\t"
               "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %5, %5, %5}, p;\n\t}"
               :: "r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(acc), "r"(0u)
               : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
               "%13, %14, %15, %16};"
               :: "r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]),
                  "r"(v[7]), "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
                  "r"(v[15])
               : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

template <int MC>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, float (&v)[MC]) {
  uint32_t r[MC];
  if constexpr (MC == 1) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(r[0]) : "r"(taddr));
  } else if constexpr (MC == 8) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
  } else {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
                 "%13, %14, %15}, [%16];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
                   "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
                   "=r"(r[15])
                 : "r"(taddr));
  }
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < MC; ++i) v[i] = __uint_as_float(r[i]);
}

// 8 codes of one word (nibble slots [k0 k2 k4 k6 k1 k3 k5 k7]) -> 4 operand
// pairs (q - z) in k order. zc holds (1024 + z) (FP16) or (128 + z) (BF16) twice.
template <bool BF16>
__device__ __forceinline__ void codes_to_pairs(uint32_t w, uint32_t zc, uint32_t* o) {
  constexpr uint32_t magic = BF16 ? 0x43004300u : 0x64006400u;
  const uint32_t p0 = and_or(w, 0x000F000Fu, magic), p1 = and_or(w >> 4, 0x000F000Fu, magic);
  const uint32_t p2 = and_or(w >> 8, 0x000F000Fu, magic), p3 = and_or(w >> 12, 0x000F000Fu, magic);
  if (BF16) {
    o[0] = bsub2_u32(p0, zc); o[1] = bsub2_u32(p1, zc); o[2] = bsub2_u32(p2, zc); o[3] = bsub2_u32(p3, zc);
  } else {
    o[0] = hsub2_u32(p0, zc); o[1] = hsub2_u32(p1, zc); o[2] = hsub2_u32(p2, zc); o[3] = hsub2_u32(p3, zc);
  }
}

// MC: accumulator columns read back (1, 8 or 16; >= M). GC: group / 32.
template <bool BF16, bool ASYM, int MC, int GC>
__global__ void __launch_bounds__(kTgThreads, 1) tc_gemv_kernel(const __grid_constant__ CUtensorMap tw,
                                                                const __grid_constant__ CUtensorMap tx,
                                                                const TcGemvArgs a) {
  extern __shared__ uint8_t dsmem[];
  __shared__ __align__(8) uint64_t full_bar[kTgStages], empty_bar[kTgStages];
  __shared__ __align__(8) uint64_t a_full[2], a_empty[2], d_full[2], d_empty[2];
  __shared__ uint32_t tmem_base_sh;
  __shared__ unsigned int s_last;
  __shared__ float red[16][128];  // the upper k half's row sums, added by the lower half at a flush
  uint8_t* ring = dsmem + ((1024u - (smem_u32(dsmem) & 1023u)) & 1023u);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int K = a.K, M = a.M;
  const int S_t = a.stages_per_tile;
  const long long u_begin = (long long)blockIdx.x * a.units / gridDim.x;
  const long long u_end = (long long)(blockIdx.x + 1) * a.units / gridDim.x;
  const int n_it = (int)(u_end - u_begin);
  constexpr int kGroupsPerStage = 8 / GC;

  if (tid == 0) {
    for (int i = 0; i < kTgStages; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], 1 + kTgConvWarps);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&a_full[i], kTgConvWarps);
      mbar_init(&a_empty[i], 1);
      mbar_init(&d_full[i], 1);
      mbar_init(&d_empty[i], kTgConvWarps);
    }
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
  asm volatile("griddepcontrol.launch_dependents;" :::);

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0 && n_it > 0) {
      tma_prefetch_desc(&tw);
      tma_prefetch_desc(&tx);
      const int nfirst = min(kTgStages, n_it);
      for (int it = 0; it < n_it; ++it) {
        const long long u = u_begin + it;
        const int rt = (int)(u / S_t);
        const int st = (int)(u - (long long)rt * S_t);
        const int slot = it % kTgStages;
        if (it >= kTgStages && !mbar_wait(&empty_bar[slot], ((it / kTgStages) & 1) ^ 1)) break;
        uint8_t* dst = ring + (size_t)slot * kTgSlot;
        const int gs0 = st * kGroupsPerStage;
        const int ng = min(kGroupsPerStage, a.G - gs0);
        const int nxb = min(4, (K - st * 256 + 63) / 64);
        mbar_arrive_expect_tx(&full_bar[slot],
                              (uint32_t)(kTgCodeBytes + nxb * kTgXBox + ng * 128 * (ASYM ? 3 : 2)));
        tma_load_2d(dst, &tw, st * 128, rt * 128, &full_bar[slot]);
        const size_t meta0 = ((size_t)rt * a.G + gs0) * 128;
        bulk_load(dst + kTgOffS, a.s_region + meta0 * 2, (uint32_t)(ng * 128 * 2), &full_bar[slot]);
        if (ASYM) bulk_load(dst + kTgOffZ, a.z_region + meta0, (uint32_t)(ng * 128), &full_bar[slot]);
        if (it + 1 == nfirst) {
          asm volatile("griddepcontrol.wait;" ::: "memory");  // X may come from the previous kernel
          for (int i = 0; i <= it; ++i) {
            const long long ui = u_begin + i;
            const int sti = (int)(ui - (ui / S_t) * S_t);
            const int nxi = min(4, (K - sti * 256 + 63) / 64);
            uint8_t* di = ring + (size_t)(i % kTgStages) * kTgSlot;
            for (int j = 0; j < nxi; ++j)
              tma_load_2d(di + kTgOffX + j * kTgXBox, &tx, sti * 256 + 64 * j, 0, &full_bar[i % kTgStages]);
          }
        } else if (it >= nfirst) {
          for (int j = 0; j < nxb; ++j) tma_load_2d(dst + kTgOffX + j * kTgXBox, &tx, st * 256 + 64 * j, 0, &full_bar[slot]);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_m128(BF16, 16);
      for (int it = 0; it < n_it; ++it) {
        const long long u = u_begin + it;
        const int st = (int)(u % S_t);
        const int slot = it % kTgStages, buf = it & 1;
        if (!mbar_wait(&full_bar[slot], (it / kTgStages) & 1)) break;
        if (!mbar_wait(&a_full[buf], (it >> 1) & 1)) break;
        if (it >= 2 && !mbar_wait(&d_empty[buf], ((it >> 1) & 1) ^ 1)) break;
        tc_fence_after();
        const int ng = min(kGroupsPerStage, a.G - st * kGroupsPerStage);
        const uint32_t xbase = smem_u32(ring + (size_t)slot * kTgSlot + kTgOffX);
        for (int gl = 0; gl < ng; ++gl) {
          const uint32_t d = tmem + kTgColD + (uint32_t)buf * 128 + (uint32_t)gl * 16;
#pragma unroll
          for (int j = 0; j < 2 * GC; ++j) {
            const int kk = gl * 2 * GC + j;  // 16-k slice of the stage
            const uint64_t b = umma_desc_sw128(xbase + (uint32_t)(kk >> 2) * kTgXBox) + (uint64_t)((kk & 3) * 2);
            umma_ts(d, tmem + kTgColA + (uint32_t)buf * 128 + (uint32_t)kk * 8, b, idesc, j > 0 ? 1u : 0u);
          }
        }
        umma_commit(&empty_bar[slot]);
        umma_commit(&a_empty[buf]);
        umma_commit(&d_full[buf]);
      }
    }
  } else {
    // ---------------------------------------------------------------- converters + epilogue
    const int cw = warp - 2;            // 0..7
    const int q = warp & 3;             // TMEM lane quarter this warp may access
    const int half = cw >> 2;           // k half of the stage: 0 -> k 0..127, 1 -> 128..255
    const int r = 32 * q + lane;        // weight row within the tile = TMEM lane
    const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16);
    constexpr int kMyGroups = kGroupsPerStage / 2;  // groups per k half (4, 2 or 1)
    float acc[MC];
#pragma unroll
    for (int m = 0; m < MC; ++m) acc[m] = 0.0f;
    float sc_prev[kMyGroups];
    int ng_prev = 0;
    bool ok = true;

    // Epilogue of iteration `e`: add s * D of this half's groups, then flush a
    // finished row tile. After a timed-out wait (ok == false) the work is
    // skipped but every converter thread still passes the same named barriers.
    auto epilogue = [&](int e) {
      const int eb = e & 1;
      if (ok && !mbar_wait(&d_full[eb], (e >> 1) & 1)) ok = false;
      if (ok) {
        tc_fence_after();
#pragma unroll
        for (int i = 0; i < kMyGroups; ++i) {
          const int gl = half * kMyGroups + i;
          if (gl < ng_prev) {
            float v[MC];
            tmem_ld_cols<MC>(lane_base + kTgColD + (uint32_t)eb * 128 + (uint32_t)gl * 16, v);
#pragma unroll
            for (int m = 0; m < MC; ++m) acc[m] = fmaf(sc_prev[i], v[m], acc[m]);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&d_empty[eb]);
      }
      const long long u = u_begin + e;
      const int rt = (int)(u / S_t);
      const int st = (int)(u - (long long)rt * S_t);
      if (!(st == S_t - 1 || u + 1 == u_end)) return;
      // ---- this CTA is done with row tile rt
      const long long tile_u0 = (long long)rt * S_t;
      const bool whole = (u_begin <= tile_u0) && (st == S_t - 1);
      if (half == 1) {
#pragma unroll
        for (int m = 0; m < MC; ++m) red[m][r] = acc[m];
      }
      asm volatile("bar.sync 1, %0;" :: "r"(kTgConvWarps * 32) : "memory");
      const int n = rt * 128 + r;
      if (half == 0 && ok) {
#pragma unroll
        for (int m = 0; m < MC; ++m) acc[m] += red[m][r];
        if (whole) {
          if (n < a.N)
#pragma unroll
            for (int m = 0; m < MC; ++m)
              if (m < M) store_out(a.Y, (size_t)m * a.N + n, acc[m], a.y_bf16);
        } else {
          const int first = sk_owner(tile_u0, a.units, gridDim.x);
          float* base = a.partials + (size_t)rt * a.max_slots * M * 128;
#pragma unroll
          for (int m = 0; m < MC; ++m)
            if (m < M) base[((size_t)(blockIdx.x - first) * M + m) * 128 + r] = acc[m];
        }
      }
      if (!whole) {
        __threadfence();
        asm volatile("bar.sync 1, %0;" :: "r"(kTgConvWarps * 32) : "memory");
        if (cw == 0 && lane == 0 && ok) {
          const long long lo = u_begin > tile_u0 ? u_begin : tile_u0;
          const unsigned int add = (unsigned int)(u + 1 - lo);
          const unsigned int prev = atomicAdd(&a.counters[rt], add);
          s_last = (prev + add == (unsigned int)S_t);
        }
        asm volatile("bar.sync 1, %0;" :: "r"(kTgConvWarps * 32) : "memory");
        if (s_last && half == 0 && ok) {
          __threadfence();
          const int first = sk_owner(tile_u0, a.units, gridDim.x);
          const int nslots = sk_owner(tile_u0 + S_t - 1, a.units, gridDim.x) - first + 1;
          const float* base = a.partials + (size_t)rt * a.max_slots * M * 128;
          if (n < a.N)
            for (int m = 0; m < M; ++m) {
              float sum = 0.0f;
              for (int sl = 0; sl < nslots; ++sl) sum += __ldcg(base + ((size_t)sl * M + m) * 128 + r);
              store_out(a.Y, (size_t)m * a.N + n, sum, a.y_bf16);
            }
          if (cw == 0 && lane == 0) a.counters[rt] = 0u;
        }
      }
      asm volatile("bar.sync 1, %0;" :: "r"(kTgConvWarps * 32) : "memory");
#pragma unroll
      for (int m = 0; m < MC; ++m) acc[m] = 0.0f;
    };

    for (int it = 0; it < n_it; ++it) {
      const long long u = u_begin + it;
      const int st = (int)(u % S_t);
      const int slot = it % kTgStages, buf = it & 1;
      if (ok && !mbar_wait(&full_bar[slot], (it / kTgStages) & 1)) ok = false;
      if (ok && it >= 2 && !mbar_wait(&a_empty[buf], ((it >> 1) & 1) ^ 1)) ok = false;
      tc_fence_after();
      const uint8_t* sp = ring + (size_t)slot * kTgSlot;
      const int ng = min(kGroupsPerStage, a.G - st * kGroupsPerStage);
      // scales (kept for the epilogue) and zero-point pairs of this half's groups
      float sc[kMyGroups];
      uint32_t zc[kMyGroups];
#pragma unroll
      for (int i = 0; i < kMyGroups; ++i) {
        const int gl = half * kMyGroups + i;
        sc[i] = 0.0f;
        zc[i] = 0u;
        if (ok && gl < ng) {
          sc[i] = h2f_bits(*reinterpret_cast<const uint16_t*>(sp + kTgOffS + (gl * 128 + r) * 2));
          const float z = ASYM ? (float)*reinterpret_cast<const int8_t*>(sp + kTgOffZ + gl * 128 + r) : 8.0f;
          zc[i] = BF16 ? pack_bf16x2(128.0f + z) : pack_f16x2(1024.0f + z);
        }
      }
      // codes of this half: 16-byte chunks p = 4*half .. 4*half+3 (32 k each)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int p = 4 * half + i;
        if (!ok || st * 256 + 32 * p >= K) break;
        const uint32_t z2 = zc[i / GC];
        const uint4 wv = lds128(smem_u32(sp) + sw128(r, p));
        uint32_t o[16];
        codes_to_pairs<BF16>(wv.x, z2, o);
        codes_to_pairs<BF16>(wv.y, z2, o + 4);
        codes_to_pairs<BF16>(wv.z, z2, o + 8);
        codes_to_pairs<BF16>(wv.w, z2, o + 12);
        tmem_st16(lane_base + kTgColA + (uint32_t)buf * 128 + (uint32_t)p * 16, o);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0 && ok) {
        mbar_arrive(&a_full[buf]);
        mbar_arrive(&empty_bar[slot]);
      }
      if (it > 0) epilogue(it - 1);
#pragma unroll
      for (int i = 0; i < kMyGroups; ++i) sc_prev[i] = sc[i];
      ng_prev = ng;
    }
    if (n_it > 0) epilogue(n_it - 1);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem), "r"(512u) : "memory");
  }
}

}  // namespace lbq
