// Decode GEMV at batch 1 on INT4 weights: y[n] = sum_k x[k] * (q[k][n] - z) * s.
//
// "Low Bit ARM kernels" observes that decode at batch 1 is a GEMV and is where
// the latency goes; BaseRT's decode GEMV splits one weight row over many SIMD
// lanes and reduces. On B200 this kernel is HBM-bound, so it is built to keep
// enough bytes in flight and to touch every weight byte once:
//
//  * One producer thread streams tiles of the image (the codes of 8 rows for
//    this CTA's K-slice, plus their scales and zero points: 16-byte-wide boxes
//    of the 128-channel-tiled scale / zero-point regions) into a ring of
//    shared-memory slots with 2-D TMA copies, running up to `stages` slots
//    ahead of the consumers (mbarrier full/empty handshake, bounded waits).
//  * A consumer thread owns one 16-byte chunk (32 consecutive k, one scale)
//    of a row at a time; the 32 lanes of a warp read 512 contiguous bytes of
//    a row from shared memory. Its 32 activations stay in registers.
//  * Codes become FP16 (or BF16) values with one AND/OR per two codes: OR-ing
//    a nibble into the mantissa of 1024.0 (FP16) or 128.0 (BF16) gives 1024+q
//    (or 1024+16q for the upper nibble of a byte), with no conversion.
//  * Products x*(1024+q) are exact in FP32 and are accumulated in FP32 with
//    the mixed-precision FMA (fma.rn.f32.f16 / .bf16). The constant offsets
//    and the zero point are removed once per chunk using the per-chunk sums of
//    x:  sum x (q - z) = acc - (1024 xs_A + 64 xs_B + z xs),  then * s.
//  * Each thread accumulates 8 rows; a transposing butterfly reduces the 8
//    partial sums over the warp with 9 shuffles, and the warps of a row group
//    are summed in a fixed order through shared memory.
//  * Split-K: each K-slice writes FP32 partials; the last CTA of a row tile
//    (a device-scope counter) adds them in slice order and resets the counter,
//    so results are deterministic and the workspace is left zeroed.
//  * With programmatic dependent launch the producer starts streaming weights
//    while the previous kernel in the stream finishes; the consumers read X and
//    write Y only after griddepcontrol.wait.
#pragma once

#include "common.cuh"
#include "tma.cuh"

namespace lbq {

constexpr int kM1MaxStages = 8;
constexpr int kM1MaxConsumerThreads = 256;

constexpr int kM1SlotRows = 8;  // rows of the weight per ring slot

struct GemvM1Args {
  const uint16_t* X;        // [K] FP16/BF16 bits
  void* Y;                  // [N]
  float* partials;          // [splits][N] FP32 (splits > 1)
  unsigned int* counters;   // [row_tiles] (splits > 1)
  int K, N, G, gshift;      // chunk c lies in group c >> gshift
  int cps, splits;          // chunks per split (a multiple of 64 when splits > 1)
  int tpr, phases;          // consumer threads per row group (multiple of 32), row groups
  int stages;               // ring depth
  int nqbox;                // 256-byte code boxes per slot row
  int sbox_h, nsbox;        // groups per scale box and box count
  int zbox_h, nzbox;        // groups per zero-point box and box count
  int off_s, off_z, slot_bytes, tx_bytes;
  int row_tiles, total_tiles;  // tile = 8*phases rows of one K-slice
  int y_bf16;
};

constexpr unsigned kFull = 0xFFFFFFFFu;

// Reduce v[0..7] over the 32 lanes of a warp. Lane l ends with the total of
// row 4*bit4(l) + 2*bit3(l) + bit2(l).
__device__ __forceinline__ float butterfly8(const float (&v)[8], int lane) {
  const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4;
  float a[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float send = b4 ? v[i] : v[i + 4];
    const float keep = b4 ? v[i + 4] : v[i];
    a[i] = keep + __shfl_xor_sync(kFull, send, 16);
  }
  float b[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float send = b3 ? a[i] : a[i + 2];
    const float keep = b3 ? a[i + 2] : a[i];
    b[i] = keep + __shfl_xor_sync(kFull, send, 8);
  }
  float c = (b2 ? b[1] : b[0]) + __shfl_xor_sync(kFull, b2 ? b[0] : b[1], 4);
  c += __shfl_xor_sync(kFull, c, 2);
  c += __shfl_xor_sync(kFull, c, 1);
  return c;
}

__device__ __forceinline__ int butterfly8_row(int lane) {
  return ((lane >> 4) & 1) * 4 + ((lane >> 3) & 1) * 2 + ((lane >> 2) & 1);
}

// sum over the chunk of x * (offset-form weight). FP16: 1024+q in slots
// (0,4),(2,6) and 1024+16q in slots (1,5),(3,7); the result is scaled so both
// carry the 1024 offset. BF16: 128+q everywhere.
template <bool BF16>
__device__ __forceinline__ float chunk_acc(const uint4 w, const uint32_t (&x)[16]) {
  const uint32_t wd[4] = {w.x, w.y, w.z, w.w};
  if (!BF16) {
    float accA = 0.0f, accB = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t t = wd[i] >> 8;
      accA = fma2_f16_f32(x[4 * i + 0], and_or(wd[i], 0x000F000Fu, 0x64006400u), accA);
      accB = fma2_f16_f32(x[4 * i + 1], and_or(wd[i], 0x00F000F0u, 0x64006400u), accB);
      accA = fma2_f16_f32(x[4 * i + 2], and_or(t, 0x000F000Fu, 0x64006400u), accA);
      accB = fma2_f16_f32(x[4 * i + 3], and_or(t, 0x00F000F0u, 0x64006400u), accB);
    }
    return fmaf(accB, 0.0625f, accA);
  } else {
    float acc0 = 0.0f, acc1 = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc0 = fma2_bf16_f32(x[4 * i + 0], and_or(wd[i], 0x000F000Fu, 0x43004300u), acc0);
      acc1 = fma2_bf16_f32(x[4 * i + 1], and_or(wd[i] >> 4, 0x000F000Fu, 0x43004300u), acc1);
      acc0 = fma2_bf16_f32(x[4 * i + 2], and_or(wd[i] >> 8, 0x000F000Fu, 0x43004300u), acc0);
      acc1 = fma2_bf16_f32(x[4 * i + 3], and_or(wd[i] >> 12, 0x000F000Fu, 0x43004300u), acc1);
    }
    return acc0 + acc1;
  }
}

__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" :::); }
__device__ __forceinline__ void consumer_sync(int nthreads) {
  asm volatile("bar.sync 1, %0;" :: "r"(nthreads) : "memory");
}

template <bool BF16, bool ASYM, int RPT>
__global__ void __launch_bounds__(kM1MaxConsumerThreads + 32, 2) gemv_m1_kernel(
    const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap ts,
    const __grid_constant__ CUtensorMap tz, const GemvM1Args a) {
  extern __shared__ uint8_t dsmem[];
  __shared__ __align__(8) uint64_t full_bar[kM1MaxStages];
  __shared__ __align__(8) uint64_t empty_bar[kM1MaxStages];
  __shared__ float red[2][8][8];
  __shared__ unsigned int s_last;

  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
  const int nthreads_c = a.tpr * a.phases;
  const int ncw = nthreads_c >> 5;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr int R = kM1SlotRows;
  constexpr int CPT = 1;
  const int rows_per_tile = 8 * a.phases;

  if (tid == 0) {
    for (int i = 0; i < a.stages; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], ncw);
    }
    fence_barrier_init();
  }
  __syncthreads();
  griddep_launch_dependents();

  if (warp == ncw) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      tma_prefetch_desc(&tq);
      tma_prefetch_desc(&ts);
      if (ASYM) tma_prefetch_desc(&tz);
      int it = 0;
      for (int tile = blockIdx.x; tile < a.total_tiles; tile += gridDim.x) {
        const int split = tile / a.row_tiles;
        const int rt = tile - split * a.row_tiles;
        const int c0 = split * a.cps;
        const int g0 = c0 >> a.gshift;
        for (int sr = 0; sr < rows_per_tile; sr += R, ++it) {
          const int slot = it % a.stages;
          if (it >= a.stages && !mbar_wait(&empty_bar[slot], ((it / a.stages) & 1) ^ 1)) return;
          uint8_t* dst = ring + (size_t)slot * a.slot_bytes;
          const int r0 = rt * rows_per_tile + sr;
          if (r0 >= a.N) {
            mbar_arrive(&full_bar[slot]);
            continue;
          }
          mbar_arrive_expect_tx(&full_bar[slot], (uint32_t)a.tx_bytes);
          for (int b = 0; b < a.nqbox; ++b) tma_load_2d(dst + b * R * 256, &tq, c0 * 16 + b * 256, r0, &full_bar[slot]);
          // scales / zero points: rows r0..r0+7 of the 128-channel tile, groups g0..
          const int my = (r0 >> 7) * a.G + g0;
          for (int b = 0; b < a.nsbox; ++b)
            tma_load_2d(dst + a.off_s + b * a.sbox_h * 16, &ts, r0 & 127, my + b * a.sbox_h, &full_bar[slot]);
          if (ASYM)
            for (int b = 0; b < a.nzbox; ++b)
              tma_load_2d(dst + a.off_z + b * a.zbox_h * 16, &tz, (r0 & 127) & ~15, my + b * a.zbox_h, &full_bar[slot]);
        }
      }
    }
    return;
  }

  // ------------------------------------------------------------------ consumers
  const int phase = tid / a.tpr;
  const int lt = tid - phase * a.tpr;
  const int chunks = a.K >> 5;
  uint32_t xr[CPT][16];
  float xoff[CPT];  // offset-form correction: 1024 xs_A + 64 xs_B (FP16) or 128 xs (BF16), + 8 xs for SYM
  float xsum[CPT];
  // shared-memory offsets of this thread's chunk inside a ring slot (row 0 of
  // its phase); they depend only on the K-slice, so they are computed once
  uint32_t q_off[CPT], s_off[CPT], z_off[CPT];
  bool c_ok[CPT];
  const uint32_t q_rstride = (uint32_t)(a.phases * 256);
  const uint32_t s_rstride = (uint32_t)(a.phases * 2);
  const uint32_t z_rstride = (uint32_t)a.phases;
  int cur_split = -1;
  int it = 0;
  int buf = 0;
  bool timed_out = false;

  griddep_wait();  // X may be written by the previous kernel in the stream

  for (int tile = blockIdx.x; tile < a.total_tiles; tile += gridDim.x) {
    const int split = tile / a.row_tiles;
    const int rt = tile - split * a.row_tiles;

    if (split != cur_split) {
      cur_split = split;
      const int c0 = split * a.cps;
      const int nch = min(a.cps, chunks - c0);
#pragma unroll
      for (int j = 0; j < CPT; ++j) {
        const int c = lt + j * a.tpr;
        const int gi = c >> a.gshift;  // group within the K-slice
        c_ok[j] = c < nch;
        q_off[j] = (uint32_t)((c >> 4) * R * 256 + (c & 15) * 16 + phase * 256);
        s_off[j] = (uint32_t)(a.off_s + gi * 16 + phase * 2);
        z_off[j] = (uint32_t)(a.off_z + gi * 16 + phase);  // + the slot's row offset in its 16-row box
        float sA = 0.0f, sB = 0.0f;
        if (c_ok[j]) {
          const uint4* xp = reinterpret_cast<const uint4*>(a.X + (size_t)(c0 + c) * 32);
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const uint4 u = ld_nc_v4(xp + v);
            xr[j][4 * v + 0] = u.x; xr[j][4 * v + 1] = u.y; xr[j][4 * v + 2] = u.z; xr[j][4 * v + 3] = u.w;
          }
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float lo = x2f<BF16>((uint16_t)(xr[j][i] & 0xFFFFu));
            const float hi = x2f<BF16>((uint16_t)(xr[j][i] >> 16));
            if ((i & 1) == 0) sA += lo + hi; else sB += lo + hi;
          }
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) xr[j][i] = 0u;
        }
        const float xs = sA + sB;
        xsum[j] = xs;
        xoff[j] = (BF16 ? 128.0f * xs : 1024.0f * sA + 64.0f * sB) + (ASYM ? 0.0f : 8.0f * xs);
      }
    }

    float part[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) part[r] = 0.0f;

#pragma unroll
    for (int st = 0; st < 8 / RPT; ++st, ++it) {
      const int slot = it % a.stages;
      // after a timed-out wait the warp skips its work but keeps the same
      // sequence of consumer barriers as the other warps
      if (!timed_out && !mbar_wait(&full_bar[slot], (it / a.stages) & 1)) timed_out = true;
      if (timed_out) continue;
      const uint32_t sb = smem_u32(ring + (size_t)slot * a.slot_bytes);
      const uint32_t zrow = (uint32_t)((rt * rows_per_tile + st * R) & 8);  // 8-row half of the 16-row zp box
#pragma unroll
      for (int i = 0; i < RPT; ++i) {
#pragma unroll
        for (int j = 0; j < CPT; ++j) {
          if (c_ok[j]) {
            const uint4 w = lds128(sb + q_off[j] + i * q_rstride);
            uint16_t sbits;
            asm volatile("ld.shared.u16 %0, [%1];" : "=h"(sbits) : "r"(sb + s_off[j] + i * s_rstride));
            float corr = xoff[j];
            if (ASYM) {
              int zv;
              asm volatile("ld.shared.s8 %0, [%1];" : "=r"(zv) : "r"(sb + z_off[j] + zrow + i * z_rstride));
              corr = fmaf((float)zv, xsum[j], corr);
            }
            const float acc = chunk_acc<BF16>(w, xr[j]);
            part[st * RPT + i] = fmaf(h2f_bits(sbits), acc - corr, part[st * RPT + i]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty_bar[slot]);
    }

    const float total = butterfly8(part, lane);
    if ((lane & 3) == 0) red[buf][warp][butterfly8_row(lane)] = total;
    consumer_sync(nthreads_c);

    const int row0 = rt * rows_per_tile;
    if (tid < rows_per_tile) {
      const int p = tid % a.phases, idx = tid / a.phases;
      const int w0 = (p * a.tpr) >> 5, w1 = ((p + 1) * a.tpr) >> 5;
      float sum = 0.0f;
      for (int w = w0; w < w1; ++w) sum += red[buf][w][idx];
      const int n = row0 + tid;
      if (n < a.N && !timed_out) {
        if (a.splits == 1) store_out(a.Y, n, sum, a.y_bf16);
        else a.partials[(size_t)split * a.N + n] = sum;
      }
    }
    if (a.splits > 1) {
      __threadfence();
      consumer_sync(nthreads_c);
      if (tid == 0) {
        s_last = 0u;
        if (!timed_out) s_last = (atomicAdd(&a.counters[rt], 1u) == (unsigned int)(a.splits - 1));
      }
      consumer_sync(nthreads_c);
      if (s_last) {
        __threadfence();
        if (tid < rows_per_tile) {
          const int n = row0 + tid;
          if (n < a.N) {
            float sum = 0.0f;
            for (int sp = 0; sp < a.splits; ++sp) sum += __ldcg(a.partials + (size_t)sp * a.N + n);
            store_out(a.Y, n, sum, a.y_bf16);
          }
        }
        if (tid == 0) a.counters[rt] = 0u;
      }
    }
    buf ^= 1;
  }
}

}  // namespace lbq
