// Decode GEMV at batches 2..16 on 3-bit LUT weights, fed by TMA and multiplied
// on the warp-level tensor cores:
//   Y[m][n] = sum_k X[m][k] * e4m3(cb[tile][idx[k][n]]) * 2^(E[tile] - 127)
// (vLLM PR 62759 write-up, format section). The batch-1 kernel's design
// (lut3_tmma.cuh) with the batch on the MMA's columns:
//  * Work unit: 16 output rows (two codebook groups) over all of K: one 2-D TMA
//    box of the two groups' 384 index bytes of every 64-k tile and one of their
//    two 16-byte BF16 decode tables per tile, into a short ring of stages.
//  * X (at most 16 rows) is staged in shared memory once per CTA.
//  * Consumer warp w takes tiles w, w + nw, ...; lane (g, t) decodes the
//    indices 8t .. 8t+7 of each 32-k chunk of row g of both groups (A rows
//    0..7 the first group, 8..15 the second): per chunk two m16n8k16 MMAs per
//    8 batch rows (NB blocks of 8), B column m of block b being X's row 8b + m,
//    all on the same decoded fragments. The tables fold the tile exponent in,
//    so one FP32 accumulator per block serves the unit.
//  * Per unit the warps' 16 x 8 NB sums meet in shared memory (warp order).
#pragma once

#include "common.cuh"
#include "tma.cuh"
#include "gemv_m1.cuh"
#include "gemv_tmma.cuh"
#include "lut3_gemv.cuh"
#include "lut3_tmma.cuh"

namespace lbq {

constexpr int kL3bMaxM = 16;
constexpr int kL3bRows = 16;

struct Lut3BatchArgs {
  const uint16_t* X;  // [M][K] BF16 bits
  void* Y;            // [M][N]
  int K, N, M;
  int tiles;          // 16-row units: ceil(N / 16)
  int nw;             // consumer warps
  int stages, stage_bytes, t_off;
  int xs_off, red_off;  // staged X [M][K], row sums [2][nw][16][8 NB]
  int y_bf16;
  int debug_drop;     // test hook: the producer issues nothing and the waits give up early
};

// KJ: tiles per consumer warp (at most); NB: blocks of 8 batch rows (1 or 2).
template <int KJ, int NB>
__global__ void __launch_bounds__((kL3tMaxWarps + 1) * 32, 1)
    lut3_tmma_batch_kernel(const __grid_constant__ CUtensorMap mi, const __grid_constant__ CUtensorMap mt,
                           const Lut3BatchArgs a) {
  extern __shared__ uint8_t l3b_dsmem[];
  __shared__ __align__(8) uint64_t full_bar[kL3tMaxStages];
  __shared__ __align__(8) uint64_t empty_bar[kL3tMaxStages];

  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(l3b_dsmem) + 1023) & ~uintptr_t(1023));
  const int S = a.stages, nw = a.nw;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int K = a.K, M = a.M, KT = K >> 6;

  if (tid == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], nw);
    }
    fence_barrier_init();
  }
  __syncthreads();
  griddep_launch_dependents();

  if (warp == nw) {
    // ---------------------------------------------------------------- producer
    if (lane != 0 || a.debug_drop) return;
    tma_prefetch_desc(&mi);
    tma_prefetch_desc(&mt);
    const uint32_t tx = (uint32_t)(KT * 384 + KT * 32);
    int u = 0, st = 0;
    uint32_t ph = 0;  // phase parity of stage st
    for (int rt = blockIdx.x; rt < a.tiles; rt += gridDim.x, ++u) {
      if (u >= S && !mbar_wait_sleep(&empty_bar[st], ph ^ 1)) break;
      uint8_t* dst = ring + (size_t)st * a.stage_bytes;
      mbar_arrive_expect_tx(&full_bar[st], tx);
      tma_load_2d(dst, &mi, rt * 48, 0, &full_bar[st]);  // a missing second group reads as zeros
      tma_load_2d(dst + a.t_off, &mt, rt * 4, 0, &full_bar[st]);
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
  const int nthreads = nw * 32;
  uint16_t* xs = reinterpret_cast<uint16_t*>(ring + a.xs_off);  // [M][K]
  float* red = reinterpret_cast<float*>(ring + a.red_off);       // [2][nw][16][8]
  griddep_wait();  // X may be written by the previous kernel in the stream
  for (int i = tid; i < M * K / 8; i += nthreads)
    reinterpret_cast<uint4*>(xs)[i] = ld_nc_v4(reinterpret_cast<const uint4*>(a.X) + i);
  consumer_sync(nthreads);

  const int g = lane >> 2, t = lane & 3;
  const uint32_t lo_shift = (uint32_t)(t & 1) * 2u;
  const uint32_t hi_rot = t == 0 ? 0u : t == 1 ? 31u : t == 2 ? 1u : 2u;
  const uint32_t ab_off = t < 2 ? 0u : 4u;
  bool col_ok[NB];  // B column g of block b = X row 8b + g
  uint32_t x_row[NB];
#pragma unroll
  for (int nb = 0; nb < NB; ++nb) {
    col_ok[nb] = 8 * nb + g < M;
    x_row[nb] = smem_u32(xs) + (uint32_t)(col_ok[nb] ? 8 * nb + g : 0) * (uint32_t)K * 2u + 16u * t;
  }
  const uint32_t dpoll = a.debug_drop ? 16u : kSleepPolls;
  int st = 0, buf = 0;
  uint32_t ph = 0;
  // a timed-out wait raises the flag; the warp then skips its work but keeps
  // the other warps' sequence of named barriers (every warp visits every unit)
  bool ok = true;
  for (int rt = blockIdx.x; rt < a.tiles; rt += gridDim.x) {
    if (ok && !__all_sync(kFull, mbar_wait_sleep(&full_bar[st], ph, dpoll))) ok = false;
    const uint32_t so = smem_u32(ring) + (uint32_t)st * (uint32_t)a.stage_bytes;
    float d[NB][2][4];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb)
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int e = 0; e < 4; ++e) d[nb][h][e] = 0.f;
#pragma unroll
    for (int jj = 0; jj < KJ; ++jj) {
      const int kt = warp + jj * nw;
      if (!ok || kt >= KT) continue;
      const uint32_t ra = so + (uint32_t)(kt * 384 + g * 24);  // row g of the first group; +192 the second
      const uint4 tabA = lds128(so + (uint32_t)(a.t_off + kt * 32));
      const uint4 tabB = lds128(so + (uint32_t)(a.t_off + kt * 32 + 16));
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t wA, cA, wB, cB;
        asm volatile("ld.shared.u32 %0, [%1];" : "=r"(wA) : "r"(ra + 12u * h + ab_off));
        asm volatile("ld.shared.u32 %0, [%1];" : "=r"(cA) : "r"(ra + 12u * h + 8u));
        asm volatile("ld.shared.u32 %0, [%1];" : "=r"(wB) : "r"(ra + 192u + 12u * h + ab_off));
        asm volatile("ld.shared.u32 %0, [%1];" : "=r"(cB) : "r"(ra + 192u + 12u * h + 8u));
        const uint32_t sA = ((wA >> lo_shift) & 0x33333333u) | (__funnelshift_l(cA, cA, hi_rot) & 0x44444444u);
        const uint32_t sB = ((wB >> lo_shift) & 0x33333333u) | (__funnelshift_l(cB, cB, hi_rot) & 0x44444444u);
        uint32_t pa[4], pb[4];
        lut3_decode8(sA, tabA, pa);
        lut3_decode8(sB, tabB, pb);
        // k = 64kt + 32h + 8t .. +7 of X row 8b + g: b0 / b1 of the block's two MMAs
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
          uint4 xv = make_uint4(0u, 0u, 0u, 0u);
          if (col_ok[nb]) xv = lds128(x_row[nb] + (uint32_t)(kt * 64 + 32 * h) * 2u);
          float(&dh)[4] = d[nb][h];
          tm_mma<true, false>(dh, pa[0], pb[0], pa[1], pb[1], ((unsigned long long)xv.y << 32) | xv.x);
          tm_mma<true, false>(dh, pa[2], pb[2], pa[3], pb[3], ((unsigned long long)xv.w << 32) | xv.z);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty_bar[st]);  // this warp is done with the stage
    if (++st == S) {
      st = 0;
      ph ^= 1;
    }
    // the warps' sums in warp order: red[buf][warp][row][column 8b + m]
    constexpr int kCols = 8 * NB, kTile = 16 * kCols;
    float* rb = red + ((size_t)buf * nw + warp) * kTile;
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
      rb[g * kCols + 8 * nb + 2 * t] = d[nb][0][0] + d[nb][1][0];
      rb[g * kCols + 8 * nb + 2 * t + 1] = d[nb][0][1] + d[nb][1][1];
      rb[(g + 8) * kCols + 8 * nb + 2 * t] = d[nb][0][2] + d[nb][1][2];
      rb[(g + 8) * kCols + 8 * nb + 2 * t + 1] = d[nb][0][3] + d[nb][1][3];
    }
    consumer_sync(nthreads);
    const int n0 = rt * kL3bRows;
    for (int i = tid; i < kL3bRows * M; i += nthreads) {
      const int r = i / M, m = i - r * M;
      if (n0 + r >= a.N) continue;
      const float* rp = red + (size_t)buf * nw * kTile + r * kCols + m;
      float sum = 0.f;
      for (int w = 0; w < nw; ++w) sum += rp[w * kTile];
      if (ok) store_out(a.Y, (size_t)m * a.N + n0 + r, sum, a.y_bf16);
    }
    buf ^= 1;
  }
}

}  // namespace lbq
