// Decode GEMV at batch 1 on 3-bit LUT weights, fed by TMA and multiplied on
// the warp-level tensor cores:
//   y[n] = sum_k x[k] * e4m3(cb[tile][idx[k][n]]) * 2^(E[tile] - 127)
// (vLLM PR 62759 write-up, format section: a 3-bit index per weight into an
// 8-entry E4M3 codebook shared by 8 channels x 64 k, one UE8M0 exponent per
// such tile).
//
//  * Work unit: one codebook group (8 output rows) over all of K. One producer
//    lane streams a unit's indices (one 2-D TMA box: the group's 192 bytes of
//    every 64-k tile) and its BF16 decode tables (16 bytes per tile) into a
//    ring of shared-memory stages (mbarrier full / empty handshake, bounded
//    waits). A CTA's units are strided over the grid. The ring is kept short
//    on purpose: copies in flight together share the bandwidth and land
//    together, so a ring as long as the CTA's work would hold the decode back
//    until nearly all of it has arrived.
//  * Consumer warp w owns the 64-k tiles 4(KG w + i) + c (i < KG, c < 4) of
//    every unit; lane (g, c) decodes row g of tile 4(KG w + i) + c. The three
//    8-byte loads of a (row, tile) record give both 32-k chunks' index words.
//  * The batch is one column, so the m16n8k16 MMA's spare columns keep the two
//    32-k chunks of each tile apart: A rows 0..7 hold the 8 rows' weights of
//    the first chunks, rows 8..15 the same rows' weights of the second chunks,
//    each MMA taking 4 k of each of the quad's four tiles; B column 0 holds the
//    first chunks' activations, column 1 the second chunks', the other columns
//    zero. D[g][0] + D[g + 8][1] is then row g's dot product over the warp's
//    tiles, the quad sum done by the MMA.
//  * Decode per 8 indices: a byte-permute selector with one index per nibble
//    from the chunk's words, two lookups in the tile's low-byte and high-byte
//    tables and two byte interleaves per 4 weights: exact BF16 weights (the
//    tile exponent is folded into the tables), FP32 accumulation.
//  * Per unit each warp parks its 8 row sums in shared memory; after its last
//    unit the CTA adds the warps' sums in warp order, so results do not depend
//    on timing.
//  * With programmatic dependent launch the producer streams weights while the
//    previous kernel in the stream finishes; consumers read X only after
//    griddepcontrol.wait.
#pragma once

#include "common.cuh"
#include "tma.cuh"
#include "gemv_m1.cuh"
#include "gemv_tmma.cuh"
#include "lut3_gemv.cuh"

namespace lbq {

constexpr int kL3tMaxWarps = 16;   // consumer warps
constexpr int kL3tMaxStages = 16;

struct Lut3TmmaArgs {
  const uint16_t* X;  // [K] BF16 bits
  void* Y;            // [N]
  int K, N;
  int units;          // N / 8 codebook groups
  int nw;             // consumer warps
  int stages, stage_bytes, t_off;
  int max_units;      // units of the busiest CTA
  int y_bf16;
  int debug_drop;     // test hook: the producer issues nothing and the waits give up early
};

// Dynamic shared memory: [stages][stage_bytes] (1024-aligned; indices at 0,
// tables at t_off), then the row sums [max_units][nw][8] floats.
// KG: groups of four 64-k tiles per consumer warp (K <= 4096 KG, 16 warps).
template <int KG>
__global__ void __launch_bounds__((kL3tMaxWarps + 1) * 32, 1)
    lut3_tmma_kernel(const __grid_constant__ CUtensorMap mi, const __grid_constant__ CUtensorMap mt,
                     const Lut3TmmaArgs a) {
  extern __shared__ uint8_t l3t_dsmem[];
  __shared__ __align__(8) uint64_t full_bar[kL3tMaxStages];
  __shared__ __align__(8) uint64_t empty_bar[kL3tMaxStages];

  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(l3t_dsmem) + 1023) & ~uintptr_t(1023));
  const int S = a.stages, nw = a.nw;
  float* red = reinterpret_cast<float*>(ring + (size_t)S * a.stage_bytes);  // [max_units][nw][8]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int KT = a.K >> 6;

  if (tid == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], nw);
    }
    fence_barrier_init();
  }
  __syncthreads();
  griddep_launch_dependents();

  const uint32_t tx = (uint32_t)(KT * 192 + KT * 16);
  if (warp == nw) {
    // ---------------------------------------------------------------- producer
    if (lane != 0 || a.debug_drop) return;
    tma_prefetch_desc(&mi);
    tma_prefetch_desc(&mt);
    int u = 0, st = 0;
    uint32_t ph = 0;  // phase parity of stage st
    for (int rg = blockIdx.x; rg < a.units; rg += gridDim.x, ++u) {
      if (u >= S && !mbar_wait_sleep(&empty_bar[st], ph ^ 1)) break;
      uint8_t* dst = ring + (size_t)st * a.stage_bytes;
      mbar_arrive_expect_tx(&full_bar[st], tx);
      tma_load_2d(dst, &mi, rg * 24, 0, &full_bar[st]);
      tma_load_2d(dst + a.t_off, &mt, rg * 2, 0, &full_bar[st]);
      if (++st == S) {
        st = 0;
        ph ^= 1;
      }
    }
    // every copy this CTA issued lands before it may exit
    const int issued = u;
    for (int v = max(0, issued - S); v < issued; ++v)
      if (!mbar_wait_sleep(&full_bar[v % S], (v / S) & 1)) break;
    return;
  }

  // ------------------------------------------------------------------ consumers
  const int g = lane >> 2, c = lane & 3;
  const uint32_t ring_s = smem_u32(ring);
  int kt[KG];
  bool kok[KG];
#pragma unroll
  for (int i = 0; i < KG; ++i) {
    kt[i] = 4 * (KG * warp + i) + c;
    kok[i] = kt[i] < KT;
  }

  griddep_wait();  // X may be written by the previous kernel in the stream

  // activation operand: lane (0, c) carries the first 32-k chunk of its tiles
  // (B column 0), lane (1, c) the second (column 1); the other lanes zeros.
  // xb[i][t][j]: (b0, b1) of the MMA for k = 8t + 4j .. 8t + 4j + 3 of the chunk
  unsigned long long xb[KG][4][2];
#pragma unroll
  for (int i = 0; i < KG; ++i) {
    const bool on = g < 2 && kok[i];
    const uint4* xp = reinterpret_cast<const uint4*>(a.X + (size_t)(on ? kt[i] : 0) * 64 + 32 * (g & 1));
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (on) v = ld_nc_v4(xp + t);
      xb[i][t][0] = ((unsigned long long)v.y << 32) | v.x;
      xb[i][t][1] = ((unsigned long long)v.w << 32) | v.z;
    }
  }

  const uint32_t red_s = smem_u32(red) + (uint32_t)(warp * 8 + g) * 4u;
  const uint32_t red_step = (uint32_t)nw * 32u;
  const uint32_t dpoll = a.debug_drop ? 16u : kSleepPolls;
  int u = 0, st = 0;
  uint32_t ph = 0;  // phase parity of stage st
  for (int rg = blockIdx.x; rg < a.units; rg += gridDim.x, ++u) {
    // a timed-out wait raises the flag; the warp (as a whole) abandons its units
    if (!__all_sync(kFull, mbar_wait_sleep(&full_bar[st], ph, dpoll))) break;
    const uint32_t so = ring_s + (uint32_t)st * (uint32_t)a.stage_bytes;
    // this warp's words and tables to registers first, so the stage is
    // released before the arithmetic
    uint32_t w[KG][6];
    uint4 tab[KG];
#pragma unroll
    for (int i = 0; i < KG; ++i) {
      if (kok[i]) {
        const uint32_t ra = so + (uint32_t)(kt[i] * 192 + g * 24);
        const uint2 w01 = lds64(ra), w23 = lds64(ra + 8), w45 = lds64(ra + 16);
        w[i][0] = w01.x; w[i][1] = w01.y; w[i][2] = w23.x; w[i][3] = w23.y; w[i][4] = w45.x; w[i][5] = w45.y;
        tab[i] = lds128(so + (uint32_t)(a.t_off + kt[i] * 16));
      } else {
#pragma unroll
        for (int j = 0; j < 6; ++j) w[i][j] = 0u;
        tab[i] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty_bar[st]);  // this warp is done with the stage
    if (++st == S) {
      st = 0;
      ph ^= 1;
    }
    // two independent MMA chains (selector slices t even / odd)
    float d[2][4];
#pragma unroll
    for (int i = 0; i < KG; ++i)
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        // record words: A0 B0 C0 (chunk 0), A1 B1 C1 (chunk 1)
        const uint32_t s0 = lut3_selector(t < 2 ? w[i][0] : w[i][1], w[i][2], t);
        const uint32_t s1 = lut3_selector(t < 2 ? w[i][3] : w[i][4], w[i][5], t);
        uint32_t pa[4], pb[4];
        lut3_decode8(s0, tab[i], pa);
        lut3_decode8(s1, tab[i], pb);
        float(&dt)[4] = d[t & 1];
        if (i == 0 && t < 2) tm_mma<true, true>(dt, pa[0], pb[0], pa[1], pb[1], xb[i][t][0]);
        else tm_mma<true, false>(dt, pa[0], pb[0], pa[1], pb[1], xb[i][t][0]);
        tm_mma<true, false>(dt, pa[2], pb[2], pa[3], pb[3], xb[i][t][1]);
      }
    // accumulator: [0] = D[g][2c] (first chunks for c = 0), [3] = D[g+8][2c+1]
    // (second chunks for c = 0); lanes c > 0 hold the zero columns
    if (c == 0) {
      const float r = (d[0][0] + d[1][0]) + (d[0][3] + d[1][3]);
      asm volatile("st.shared.f32 [%0], %1;" :: "r"(red_s + (uint32_t)u * red_step), "f"(r) : "memory");
    }
  }

  // ------------------------------------------------- the CTA's rows, warp order
  const int units = u;  // of this warp (fewer only after a timed-out wait)
  int n_units = 0;
  for (int rg = blockIdx.x; rg < a.units; rg += gridDim.x) ++n_units;
  const bool complete = consumer_sync_and(units == n_units, nw * 32);
  if (!complete) return;
  for (int e = tid; e < n_units * 8; e += nw * 32) {
    const int uu = e >> 3, row = e & 7;
    const int n = (blockIdx.x + uu * gridDim.x) * 8 + row;
    const float* rp = red + (size_t)uu * nw * 8 + row;
    float sum = 0.f;
    for (int v = 0; v < nw; ++v) sum += rp[v * 8];
    store_out(a.Y, (size_t)n, sum, a.y_bf16);
  }
}

}  // namespace lbq
