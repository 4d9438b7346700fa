// Decode GEMV at batch 1 on INT4 weights, fed by TMA and multiplied on the
// warp-level tensor cores: y[n] = sum_k x[k] * (q[k][n] - z) * s.
//
// "Low Bit ARM kernels" notes that decode at batch 1 is a GEMV and sets the
// latency; the weights stream once from HBM, so the kernel's job is to retire
// weights at HBM speed with as few instructions per weight as possible.
//
//  * Work unit: 16 output rows x one K-range of at most 4096 k (16 slices of
//    256 k). One producer lane streams each unit's codes (one 3-D TMA box:
//    128 bytes x 16 rows x the range's slices, 128-byte swizzle), scales and
//    zero points (one box each from the 128-channel-tiled regions) into a ring
//    of shared-memory stages (mbarrier full / empty handshake, bounded waits).
//  * Consumer warp w owns slice w of the CTA's K-range for every unit, so its
//    activation operand never changes: it is built once, in registers.
//  * The batch is one column, so 7 of the m16n8k16 MMA's 8 columns would be
//    idle; they keep 32-k chunks apart instead. Per MMA the A columns 0..7 hold
//    8 k of chunk X_j and columns 8..15 8 k of chunk Y_j, and the activation
//    operand puts chunk X_j's values in column 2j and Y_j's in column 2j+1 only.
//    16 MMAs (j = 0..3 chunk pairs x p = 0..3 code pairs per 32-bit word) cover
//    16 rows x 8 chunks, and column c of the accumulator is the dot product of
//    each row with chunk c alone, so the group scale (a group is a whole number
//    of chunks) is applied in FP32 afterwards.
//  * Codes become FP16 operands with one AND/OR per two codes: a nibble OR-ed
//    into the mantissa of 1024.0 (bits 0..3) or 64.0 (bits 4..7) gives 1024 + q
//    or 64 + q; one shift by 8 per word reaches the other four nibbles (BF16:
//    128 + q, one shift per pair). ldmatrix hands each thread one 32-bit word of
//    8 codes per matrix, in the MMA's A layout. The offsets and the zero point
//    are removed per chunk with the chunk's activation sums:
//      sum x (q - z) = acc - (1024 sA + 64 sB) - z (sA + sB).
//  * Per unit each warp reduces its two rows per thread over the quad and parks
//    16 row sums in shared memory; after its last unit the CTA adds the warps'
//    sums in warp order (one barrier per CTA, none per unit), so results do not
//    depend on timing. With K split into R ranges (R > 1) the ranges' FP32
//    sums meet in a workspace and the last CTA of a row tile (a device-scope
//    counter) adds them in range order and resets the counter.
//  * Up to 4 GEMVs with one K share a launch (q/k/v, gate/up): their row tiles
//    are numbered one after the other.
//  * With programmatic dependent launch the producer streams weights while the
//    previous kernel in the stream finishes; consumers read X only after
//    griddepcontrol.wait.
#pragma once

#include "common.cuh"
#include "tma.cuh"
#include "gemv_m1.cuh"

namespace lbq {

constexpr int kTmMaxItems = 4;
constexpr int kTmMaxSlices = 16;  // 256-k slices per K-range = consumer warps
constexpr int kTmMaxStages = 16;
constexpr int kTmDefaultStages = 3;  // the planner's ring depth (at most kTmMaxStages)
constexpr int kTmRows = 16;
constexpr int kTmSliceBytes = kTmRows * 128;  // one TMA box: 16 rows x 128 bytes of codes

struct GemvTmmaMaps {
  CUtensorMap q[kTmMaxItems];  // codes [K/256][N][128] bytes (3-D view), box 128 x 16 x nsl, 128-byte swizzle
  CUtensorMap s[kTmMaxItems];  // scales [tiles * G][128] u16, box 16 x krg
  CUtensorMap z[kTmMaxItems];  // zero points [tiles * G][128] u8, box 16 x krg
};

struct GemvTmmaArgs {
  const uint16_t* X[kTmMaxItems];  // [K] FP16 / BF16 bits
  void* Y[kTmMaxItems];            // [N]
  int N[kTmMaxItems];
  int rt_end[kTmMaxItems];         // cumulative 16-row tiles
  float* partials;                 // [R][N] FP32 (one item, R > 1)
  unsigned int* counters;          // [row tiles] (R > 1)
  int items, K, G, gshift;         // G groups over all of K; chunk c lies in group c >> gshift
  int R, nsl, krg;                 // K-ranges, slices per K-range, groups per K-range
  int row_tiles, stages, stage_bytes, s_off, z_off;
  int max_units;                   // units of the busiest CTA (row sums kept in shared memory)
  int y_bf16;
  int debug_drop;                  // test hook: the producer issues nothing and the waits give up early
};

// Codes of one 32-bit word (k = 8t .. 8t+7 of a chunk, nibble slots
// [k0 k2 k4 k6 k1 k3 k5 k7]) -> the FP16 / BF16 pair (k = 8t+2p, 8t+2p+1) in
// offset form. FP16: p even 1024 + q, p odd 64 + q. BF16: 128 + q.
template <bool BF16, int P>
__device__ __forceinline__ uint32_t tm_pair(uint32_t w, uint32_t w8) {
  if (BF16) return and_or(w >> (4 * P), 0x000F000Fu, 0x43004300u);
  if (P == 0) return and_or(w, 0x000F000Fu, 0x64006400u);
  if (P == 1) return and_or(w, 0x00F000F0u, 0x54005400u);
  if (P == 2) return and_or(w8, 0x000F000Fu, 0x64006400u);
  return and_or(w8, 0x00F000F0u, 0x54005400u);
}

// Barrier over the consumer warps (named barrier 1) that also ANDs a flag.
__device__ __forceinline__ bool consumer_sync_and(bool v, int nthreads) {
  int r;
  asm volatile("{\n\t.reg .pred p, q;\n\t"
               "setp.ne.s32 p, %1, 0;\n\t"
               "bar.red.and.pred q, 1, %2, p;\n\t"
               "selp.s32 %0, 1, 0, q;\n\t}"
               : "=r"(r) : "r"((int)v), "r"(nthreads) : "memory");
  return r != 0;
}

// d (+)= A . B on the warp-level tensor cores; plain (non-volatile) asm, so
// the compiler may interleave independent chains. The B fragment travels as
// one 64-bit value (an aligned register pair, no moves to assemble it). ZC:
// the chain's first MMA, accumulating onto zero.
template <bool BF16, bool ZC>
__device__ __forceinline__ void tm_mma(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                       unsigned long long b) {
#define LBQ_TM_MMA(TY, CIN, CONS)                                                                        \
  asm("{\n\t.reg .b32 b0, b1;\n\tmov.b64 {b0, b1}, %8;\n\t"                                           \
      "mma.sync.aligned.m16n8k16.row.col.f32." TY "." TY ".f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "    \
      "{b0, b1}, " CIN ";\n\t}"                                                                           \
      : CONS(d[0]), CONS(d[1]), CONS(d[2]), CONS(d[3])                                                  \
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "l"(b), "f"(0.0f))
#define LBQ_OUT(x) "=f"(x)
#define LBQ_INOUT(x) "+f"(x)
  if (ZC) {
    if (BF16) LBQ_TM_MMA("bf16", "{%9, %9, %9, %9}", LBQ_OUT);
    else LBQ_TM_MMA("f16", "{%9, %9, %9, %9}", LBQ_OUT);
  } else {
    if (BF16) LBQ_TM_MMA("bf16", "{%0, %1, %2, %3}", LBQ_INOUT);
    else LBQ_TM_MMA("f16", "{%0, %1, %2, %3}", LBQ_INOUT);
  }
#undef LBQ_TM_MMA
#undef LBQ_OUT
#undef LBQ_INOUT
}

__device__ __forceinline__ float lds_f16_as_f32(uint32_t addr) {
  uint16_t h;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(h) : "r"(addr));
  return h2f_bits(h);
}

__device__ __forceinline__ int lds_s8(uint32_t addr) {
  int v;
  asm volatile("ld.shared.s8 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ float lds_s8_as_f32(uint32_t addr) {
  int v;
  asm volatile("ld.shared.s8 %0, [%1];" : "=r"(v) : "r"(addr));
  // exact int8 -> float: 1.5 * 2^23 + v has unit spacing
  return __int_as_float(0x4B400000 + v) - 12582912.0f;
}

// Dynamic shared memory: [stages][stage_bytes] (1024-aligned), then the row
// sums [max_units][nsl][16] floats and one flag per unit.
// GS: log2(chunks per group) (0, 1, 2 for groups of 32, 64, 128), a template
// parameter so that every shared-memory offset below is an immediate.
template <bool BF16, bool ASYM, int GS>
__global__ void __launch_bounds__((kTmMaxSlices + 1) * 32, 1)
    gemv_tmma_kernel(const __grid_constant__ GemvTmmaMaps m, const GemvTmmaArgs a) {
  extern __shared__ uint8_t tm_dsmem[];
  __shared__ __align__(8) uint64_t full_bar[kTmMaxStages];
  __shared__ __align__(8) uint64_t empty_bar[kTmMaxStages];

  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(tm_dsmem) + 1023) & ~uintptr_t(1023));
  const int S = a.stages, nw = a.nsl;
  float* red = reinterpret_cast<float*>(ring + (size_t)S * a.stage_bytes);  // [max_units][nw][16]
  int* last_flag = reinterpret_cast<int*>(red + (size_t)a.max_units * nw * 16);  // [max_units]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int kr = blockIdx.x % a.R;
  const int cpk = gridDim.x / a.R;  // CTAs per K-range
  const int chunks = a.K >> 5;

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
    for (int i = 0; i < a.items; ++i) {
      tma_prefetch_desc(&m.q[i]);
      tma_prefetch_desc(&m.s[i]);
      if (ASYM) tma_prefetch_desc(&m.z[i]);
    }
    const int sl0 = kr * a.nsl;
    const uint32_t tx = (uint32_t)(a.nsl * kTmSliceBytes + a.krg * 32 + (ASYM ? a.krg * 16 : 0));
    int it = 0, u = 0, st = 0;
    uint32_t ph = 0;  // phase parity of stage st
    int item_end = a.rt_end[0];
    for (int rt = blockIdx.x / a.R; rt < a.row_tiles; rt += cpk, ++u) {
      if (u >= S && !mbar_wait_sleep(&empty_bar[st], ph ^ 1)) break;
      while (rt >= item_end) item_end = a.rt_end[++it];
      const int r0 = (rt - (it ? a.rt_end[it - 1] : 0)) * kTmRows;
      uint8_t* dst = ring + (size_t)st * a.stage_bytes;
      mbar_arrive_expect_tx(&full_bar[st], tx);
      tma_load_3d(dst, &m.q[it], 0, r0, sl0, &full_bar[st]);  // slices past K read as zeros
      const int my = (r0 >> 7) * a.G + kr * a.krg;
      tma_load_2d(dst + a.s_off, &m.s[it], r0 & 127, my, &full_bar[st]);
      if (ASYM) tma_load_2d(dst + a.z_off, &m.z[it], r0 & 127, my, &full_bar[st]);
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
  const int g = lane >> 2, t = lane & 3;
  const int cbase = (kr * a.nsl + warp) * 8;  // first chunk of this warp's slice
  // ldmatrix source of this lane: matrix mi = lane / 8 (rows 8*(mi & 1) ..,
  // chunk j + 4*(mi >> 1)), row lane % 8 of it; 128-byte swizzle
  const int mi = lane >> 3, mr = lane & 7;
  const uint32_t lrow = (uint32_t)(mr + 8 * (mi & 1));
  const uint32_t lcx = (uint32_t)(mr ^ (4 * (mi >> 1)));
  const uint32_t ring_s = smem_u32(ring);
  uint32_t lbase[4];  // this lane's ldmatrix address in stage 0, per chunk pair
#pragma unroll
  for (int j = 0; j < 4; ++j) lbase[j] = ring_s + (uint32_t)warp * kTmSliceBytes + lrow * 128u + ((j ^ lcx) << 4);
  // scales / zero points of this thread's chunks X_t = cbase + t and
  // Y_t = cbase + 4 + t for rows g and g + 8: one base per region, the rest
  // immediate offsets (group Y_t lies 4 >> GS groups after X_t)
  constexpr uint32_t kDY = 4u >> GS;
  const int gX = (warp * 8 + t) >> GS;
  const uint32_t sbase = ring_s + (uint32_t)(a.s_off + gX * 32 + g * 2);
  const uint32_t zbase = ring_s + (uint32_t)(a.z_off + gX * 16 + g);
  const uint32_t red_s = smem_u32(red) + (uint32_t)(warp * 16 + g) * 4u;
  const uint32_t red_step = (uint32_t)nw * 64u;

  griddep_wait();  // X may be written by the previous kernel in the stream

  // activation operand: thread (g, t) carries 8 values (k = 8t .. 8t+7) of
  // chunk X_{g/2} (g even, as b0 in the MMAs of pair g/2) or Y_{g/2} (g odd, b1)
  unsigned long long bf[4][4];  // (b0, b1) of MMA (j, p), low word b0
  float corrX = 0.f, corrY = 0.f, sxX = 0.f, sxY = 0.f;
  const uint16_t* x_loaded = nullptr;
  auto load_x = [&](const uint16_t* X) {
    x_loaded = X;
    const int cm = cbase + (g >> 1) + 4 * (g & 1);
    uint4 xv = make_uint4(0u, 0u, 0u, 0u);
    if (cm < chunks) xv = ld_nc_v4(X + (size_t)cm * 32 + 8 * t);
    const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        const unsigned long long v = xw[p];
        bf[j][p] = (g == 2 * j) ? v : (g == 2 * j + 1) ? (v << 32) : 0ull;
      }
    // chunk sums: class A (pairs 0, 2: 1024 + q) and class B (pairs 1, 3: 64 + q)
    float sA = 0.f, sB = 0.f;
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const float v = x2f<BF16>((uint16_t)(xw[p] & 0xFFFFu)) + x2f<BF16>((uint16_t)(xw[p] >> 16));
      if (p & 1) sB += v; else sA += v;
    }
    sA += __shfl_xor_sync(kFull, sA, 1);
    sB += __shfl_xor_sync(kFull, sB, 1);
    sA += __shfl_xor_sync(kFull, sA, 2);
    sB += __shfl_xor_sync(kFull, sB, 2);
    const float aX = __shfl_sync(kFull, sA, 8 * t), bX = __shfl_sync(kFull, sB, 8 * t);
    const float aY = __shfl_sync(kFull, sA, 8 * t + 4), bY = __shfl_sync(kFull, sB, 8 * t + 4);
    sxX = aX + bX;
    sxY = aY + bY;
    const float offX = BF16 ? 128.0f * sxX : fmaf(1024.0f, aX, 64.0f * bX);
    const float offY = BF16 ? 128.0f * sxY : fmaf(1024.0f, aY, 64.0f * bY);
    corrX = ASYM ? offX : fmaf(8.0f, sxX, offX);
    corrY = ASYM ? offY : fmaf(8.0f, sxY, offY);
  };

  int it = 0, u = 0, st = 0;
  uint32_t ph = 0;  // phase parity of stage st
  int item_end = a.rt_end[0];
  load_x(a.X[0]);
  const uint32_t dpoll = a.debug_drop ? 16u : kSleepPolls;
  for (int rt = blockIdx.x / a.R; rt < a.row_tiles; rt += cpk, ++u) {
    if (rt >= item_end) {  // the next GEMV of a grouped launch
      while (rt >= item_end) item_end = a.rt_end[++it];
      if (a.X[it] != x_loaded) load_x(a.X[it]);
    }
    // a timed-out wait raises the flag; the warp (as a whole) abandons its units
    if (!__all_sync(kFull, mbar_wait_sleep(&full_bar[st], ph, dpoll))) break;
    const uint32_t so = (uint32_t)st * (uint32_t)a.stage_bytes;
    // everything this warp needs from the stage goes to registers first, so
    // the stage is released before the arithmetic
    uint32_t r[4][4];
#pragma unroll
    for (int j = 0; j < 4; ++j) ldmatrix_x4(r[j], lbase[j] + so);
    const uint32_t sa = sbase + so;
    const float sXg = lds_f16_as_f32(sa), sXh = lds_f16_as_f32(sa + 16);
    const float sYg = lds_f16_as_f32(sa + kDY * 32), sYh = lds_f16_as_f32(sa + kDY * 32 + 16);
    int zXg = 0, zXh = 0, zYg = 0, zYh = 0;
    if (ASYM) {
      const uint32_t za = zbase + so;
      zXg = lds_s8(za);
      zXh = lds_s8(za + 8);
      zYg = lds_s8(za + kDY * 16);
      zYh = lds_s8(za + kDY * 16 + 8);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty_bar[st]);  // this warp is done with the stage
    if (++st == S) {
      st = 0;
      ph ^= 1;
    }
    // two independent MMA chains (chunk pairs 0, 2 and 1, 3)
    float d[2][4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t r8[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) r8[i] = BF16 ? 0u : r[j][i] >> 8;
      float(&dj)[4] = d[j & 1];
      if (j < 2)
        tm_mma<BF16, true>(dj, tm_pair<BF16, 0>(r[j][0], r8[0]), tm_pair<BF16, 0>(r[j][1], r8[1]),
                           tm_pair<BF16, 0>(r[j][2], r8[2]), tm_pair<BF16, 0>(r[j][3], r8[3]), bf[j][0]);
      else
        tm_mma<BF16, false>(dj, tm_pair<BF16, 0>(r[j][0], r8[0]), tm_pair<BF16, 0>(r[j][1], r8[1]),
                            tm_pair<BF16, 0>(r[j][2], r8[2]), tm_pair<BF16, 0>(r[j][3], r8[3]), bf[j][0]);
      tm_mma<BF16, false>(dj, tm_pair<BF16, 1>(r[j][0], r8[0]), tm_pair<BF16, 1>(r[j][1], r8[1]),
                          tm_pair<BF16, 1>(r[j][2], r8[2]), tm_pair<BF16, 1>(r[j][3], r8[3]), bf[j][1]);
      tm_mma<BF16, false>(dj, tm_pair<BF16, 2>(r[j][0], r8[0]), tm_pair<BF16, 2>(r[j][1], r8[1]),
                          tm_pair<BF16, 2>(r[j][2], r8[2]), tm_pair<BF16, 2>(r[j][3], r8[3]), bf[j][2]);
      tm_mma<BF16, false>(dj, tm_pair<BF16, 3>(r[j][0], r8[0]), tm_pair<BF16, 3>(r[j][1], r8[1]),
                          tm_pair<BF16, 3>(r[j][2], r8[2]), tm_pair<BF16, 3>(r[j][3], r8[3]), bf[j][3]);
    }
    // accumulator element i: [0] row g chunk X_t, [1] row g chunk Y_t, [2] row g+8 X_t, [3] row g+8 Y_t
    // (each chain writes only its own pairs' columns, the others stay zero)
    float cXg = corrX, cXh = corrX, cYg = corrY, cYh = corrY;
    if (ASYM) {
      cXg = fmaf(__int2float_rn(zXg), sxX, corrX);
      cXh = fmaf(__int2float_rn(zXh), sxX, corrX);
      cYg = fmaf(__int2float_rn(zYg), sxY, corrY);
      cYh = fmaf(__int2float_rn(zYh), sxY, corrY);
    }
    float pg = sXg * ((d[0][0] + d[1][0]) - cXg);
    pg = fmaf(sYg, (d[0][1] + d[1][1]) - cYg, pg);
    float ph_ = sXh * ((d[0][2] + d[1][2]) - cXh);
    ph_ = fmaf(sYh, (d[0][3] + d[1][3]) - cYh, ph_);
    pg += __shfl_xor_sync(kFull, pg, 1);
    ph_ += __shfl_xor_sync(kFull, ph_, 1);
    pg += __shfl_xor_sync(kFull, pg, 2);
    ph_ += __shfl_xor_sync(kFull, ph_, 2);
    if (t == 0) {
      const uint32_t rs = red_s + (uint32_t)u * red_step;
      asm volatile("st.shared.f32 [%0], %1;" :: "r"(rs), "f"(pg) : "memory");
      asm volatile("st.shared.f32 [%0], %1;" :: "r"(rs + 32u), "f"(ph_) : "memory");
    }
  }
  const int units = u;  // of this warp (fewer only after a timed-out wait)

  // ------------------------------------------------- the CTA's rows, warp order
  int n_units = 0;
  for (int rt = blockIdx.x / a.R; rt < a.row_tiles; rt += cpk) ++n_units;
  const bool complete = consumer_sync_and(units == n_units, nw * 32);
  for (int e = tid; e < n_units * 16; e += nw * 32) {
    const int uu = e >> 4, row = e & 15;
    const int rt = blockIdx.x / a.R + uu * cpk;
    int iu = 0;
    while (iu + 1 < a.items && rt >= a.rt_end[iu]) ++iu;
    const int n = (rt - (iu ? a.rt_end[iu - 1] : 0)) * kTmRows + row;
    float sum = 0.f;
    const float* rp = red + (size_t)uu * nw * 16 + row;
    for (int w = 0; w < nw; ++w) sum += rp[w * 16];
    if (!complete || n >= a.N[iu]) continue;
    if (a.R == 1) store_out(a.Y[iu], (size_t)n, sum, a.y_bf16);
    else a.partials[(size_t)kr * a.N[0] + n] = sum;
  }
  if (a.R == 1 || !complete) return;
  // K split over R CTAs: per row tile the last of them adds the ranges in order
  __threadfence();
  consumer_sync(nw * 32);
  for (int uu = tid; uu < n_units; uu += nw * 32) {
    const int rt = blockIdx.x / a.R + uu * cpk;
    last_flag[uu] = atomicAdd(&a.counters[rt], 1u) == (unsigned int)(a.R - 1);
  }
  consumer_sync(nw * 32);
  __threadfence();
  for (int e = tid; e < n_units * 16; e += nw * 32) {
    const int uu = e >> 4, row = e & 15;
    if (!last_flag[uu]) continue;
    const int rt = blockIdx.x / a.R + uu * cpk;
    const int n = rt * kTmRows + row;
    if (row == 0) a.counters[rt] = 0u;
    if (n >= a.N[0]) continue;
    float tot = 0.f;
    for (int k = 0; k < a.R; ++k) tot += __ldcg(a.partials + (size_t)k * a.N[0] + n);
    store_out(a.Y[0], (size_t)n, tot, a.y_bf16);
  }
}

}  // namespace lbq
