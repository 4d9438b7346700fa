// Decode GEMV at batch 1 on INT4 weights with plain vector loads:
// y[n] = sum_k x[k] * (q[k][n] - z) * s.
//
// At batch 1 every weight is used once, so the kernel is a stream: the code
// bytes go from HBM straight to registers (16-byte non-allocating loads, 512
// contiguous bytes per warp instruction), with no staging through shared
// memory and no producer/consumer handshakes.
//
//  * A CTA owns blocks of 8 output rows (grid-stride) and the whole K range;
//    lane l of warp w takes the 32-k chunk c = 32w + l (K <= 16384). Its
//    activations (32 values per chunk) and their offset sums stay in registers
//    while the CTA's row blocks use the same X.
//  * One launch may carry up to 4 GEMVs with the same K, group, mode and
//    dtypes (the projections that read one activation vector, e.g. q/k/v or
//    gate/up of a decoder layer): their row blocks are numbered one after the
//    other and spread over the same grid.
//  * Per row block and chunk a lane loads the 8 rows' 16-byte code chunks,
//    one 16-byte load of the 8 rows' scales and one 8-byte load of their zero
//    points (the image stores them 128 channels at a time, so 8 consecutive
//    rows are contiguous). The next row block's codes are loaded before the
//    current one is computed.
//  * Codes become FP16 (BF16) operands 1024 + q (128 + q) with one AND/OR per
//    pair, multiplied by x with FP32 accumulation (exact products); per chunk
//    the offset and the zero point are removed with the chunk's activation sum,
//    then the scale is applied.
//  * Each warp reduces its 8 row partials over its lanes (transposing
//    butterfly) and parks them in shared memory; after its last row block the
//    CTA adds the warps' sums in a fixed order (one barrier per CTA, none per
//    row block), so results do not depend on timing.
#pragma once

#include "common.cuh"
#include "gemv_m1.cuh"
#include "w4a8.cuh"

namespace lbq {

constexpr int kGdMaxWarps = 16;
constexpr int kGdMaxItems = 4;  // GEMVs of one launch (same K, group, mode and dtypes)

// One launch computes up to kGdMaxItems GEMVs; their 8-row blocks are numbered
// consecutively, item i owning blocks [rb_end[i-1], rb_end[i]).
struct GemvDirectArgs {
  const uint16_t* X[kGdMaxItems];  // [K] FP16/BF16 bits (the A8 kernel: [K] INT8 codes)
  const float* SX[kGdMaxItems];    // the A8 kernel: [K/32] activation scales
  void* Y[kGdMaxItems];            // [N]
  const uint8_t* q[kGdMaxItems];   // [N][K/2]
  const uint8_t* s[kGdMaxItems];   // 128-channel-tiled FP16 scales
  const uint8_t* z[kGdMaxItems];   // 128-channel-tiled int8 zero points (ASYM)
  int N[kGdMaxItems];
  int rb_end[kGdMaxItems];
  int items;
  int K, G;
  int row_blocks;                  // total over the items
  int y_bf16;
};

// sum over one 16-byte chunk (32 k) of x * (offset-form weight), FP32.
template <bool BF16>
__device__ __forceinline__ float gd_chunk(const uint4 w, const uint32_t (&x)[16]) { return chunk_acc<BF16>(w, x); }

// One chunk per lane: K <= 32 * 32 * kGdMaxWarps. Dynamic shared memory:
// float [row blocks of this CTA][warps][8] of per-warp row sums.
template <bool BF16, bool ASYM>
__global__ void __launch_bounds__(kGdMaxWarps * 32, 1) gemv_direct_kernel(const GemvDirectArgs a) {
  extern __shared__ float red[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nw = blockDim.x >> 5;
  const int chunks = a.K >> 5;
  const size_t rowb = (size_t)(a.K >> 1);  // code bytes per row
  const int gpc = (a.K / a.G) >> 5;        // chunks per group (1, 2 or 4)
  const int c = warp * 32 + lane;          // this lane's 32-k chunk
  const bool cok = c < chunks;

  auto item_of = [&](int rb) {
    int i = 0;
    while (i + 1 < a.items && rb >= a.rb_end[i]) ++i;
    return i;
  };
  // codes of the current and the next row block
  uint4 cur[8], nxt[8];
  auto load_block = [&](int rb, uint4 (&w)[8]) {
    const int it = item_of(rb);
    const int r0 = (rb - (it ? a.rb_end[it - 1] : 0)) * 8;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      w[i] = make_uint4(0u, 0u, 0u, 0u);
      if (cok && r0 + i < a.N[it]) w[i] = ld_stream_v4(a.q[it] + (size_t)(r0 + i) * rowb + (size_t)c * 16);
    }
  };

  // The weights are only read, so the first row block is requested before
  // waiting for the previous kernel in the stream (which may write X).
  int rb = blockIdx.x;
  if (rb < a.row_blocks) load_block(rb, cur);
  griddep_launch_dependents();
  griddep_wait();

  // this lane's activations and their offset sums, for the item being worked on
  uint32_t xr[16];
  float xoff = 0.0f, xsum = 0.0f;
  const uint16_t* x_loaded = nullptr;
  auto load_x = [&](const uint16_t* X) {
    x_loaded = X;
    float sA = 0.0f, sB = 0.0f;
    if (cok) {
      const uint4* xp = reinterpret_cast<const uint4*>(X + (size_t)c * 32);
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const uint4 u = ld_nc_v4(xp + v);
        xr[4 * v + 0] = u.x; xr[4 * v + 1] = u.y; xr[4 * v + 2] = u.z; xr[4 * v + 3] = u.w;
      }
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float lo = x2f<BF16>((uint16_t)(xr[i] & 0xFFFFu));
        const float hi = x2f<BF16>((uint16_t)(xr[i] >> 16));
        if ((i & 1) == 0) sA += lo + hi; else sB += lo + hi;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i) xr[i] = 0u;
    }
    xsum = sA + sB;
    // FP16: slots of class A carry 1024 + q, class B (1024 + 16 q)/16 after chunk_acc
    xoff = (BF16 ? 128.0f * xsum : 1024.0f * sA + 64.0f * sB) + (ASYM ? 0.0f : 8.0f * xsum);
  };

  int lb = 0;  // row block index within this CTA
  for (; rb < a.row_blocks; rb += gridDim.x, ++lb) {
    const int rbn = rb + gridDim.x;
    if (rbn < a.row_blocks) load_block(rbn, nxt);
    const int it = item_of(rb);
    if (a.X[it] != x_loaded) load_x(a.X[it]);
    const int r0 = (rb - (it ? a.rb_end[it - 1] : 0)) * 8;
    float part[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) part[i] = 0.0f;
    if (cok) {
      const int g = c / gpc;
      const size_t m0 = ((size_t)(r0 >> 7) * a.G + g) * 128 + (r0 & 127);  // 8 consecutive rows, 16-byte aligned
      const uint4 sv = ld_nc_v4(a.s[it] + m0 * 2);
      uint2 zv = make_uint2(0u, 0u);
      if (ASYM) zv = *reinterpret_cast<const uint2*>(a.z[it] + m0);
      const uint32_t sw[4] = {sv.x, sv.y, sv.z, sv.w};
#pragma unroll
      for (int i = 0; i < 8; i += 2) {
        const float2 sc = __half22float2(*reinterpret_cast<const __half2*>(&sw[i >> 1]));
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const float acc = gd_chunk<BF16>(cur[i + h], xr);
          float corr = xoff;
          if (ASYM) {
            const int zi = (int)(int8_t)(((i < 4 ? zv.x : zv.y) >> (8 * ((i + h) & 3))) & 0xFFu);
            corr = fmaf((float)zi, xsum, corr);
          }
          part[i + h] = fmaf(h ? sc.y : sc.x, acc - corr, part[i + h]);
        }
      }
    }
    const float total = butterfly8(part, lane);
    if ((lane & 3) == 0) red[(lb * nw + warp) * 8 + butterfly8_row(lane)] = total;
#pragma unroll
    for (int i = 0; i < 8; ++i) cur[i] = nxt[i];
  }
  // the warps' row sums of every row block of this CTA, added in warp order
  __syncthreads();
  for (int t = tid; t < lb * 8; t += blockDim.x) {
    const int l = t >> 3, row = t & 7;
    const int rbo = blockIdx.x + l * gridDim.x;
    const int it = item_of(rbo);
    const int r = (rbo - (it ? a.rb_end[it - 1] : 0)) * 8 + row;
    float sum = 0.0f;
    for (int w = 0; w < nw; ++w) sum += red[(l * nw + w) * 8 + row];
    if (r < a.N[it]) store_out(a.Y[it], (size_t)r, sum, a.y_bf16);
  }
}

// The same GEMV with the weights staged through shared memory by per-thread
// asynchronous copies: each lane keeps S row blocks of its chunk (8 rows of
// codes, their scales and zero points) in flight in its own shared-memory
// slots, so the bytes in flight per SM no longer depend on registers, and the
// scale and zero-point reads are prefetched with the codes. A lane reads back
// only what it copied itself, so a per-thread wait on its copy groups is the
// only synchronisation. Dynamic shared memory: uint4 codes [S][8][T], uint4
// scales [S][T], uint2 zero points [S][T] (T threads), then the row sums as in
// gemv_direct_kernel.
//
// A8 = true is the W4A8 form of the same kernel ("Low Bit ARM kernels": 4-bit
// weights with dynamic INT8 activations): X holds INT8 codes and SX one FP32
// scale per 32-k block (from lbq_quantize_int8); a chunk of a row is four
// pairs of byte dot products (dp4a) on the low nibbles and the in-place high
// nibbles (16 q), exact in int32; per chunk (s_w s_x) (sum xq q - z sum xq) is
// added in FP32.
template <bool BF16, bool ASYM, int S, bool A8 = false>
__global__ void __launch_bounds__(kGdMaxWarps * 32) gemv_direct_async_kernel(const GemvDirectArgs a) {
  extern __shared__ __align__(16) uint8_t gd_smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int T = blockDim.x, nw = T >> 5;
  // 32-bit shared addresses of this thread's slots: codes [S][8][T] x 16 B,
  // scales [S][T] x 16 B, zero points [S][T] x 8 B (lane-contiguous, so a
  // warp's copies of one row fill 512 contiguous bytes)
  const uint32_t T16 = (uint32_t)T * 16;
  const uint32_t sq_s = (uint32_t)__cvta_generic_to_shared(gd_smem) + (uint32_t)tid * 16;
  const uint32_t ss_s = sq_s + (uint32_t)S * 8 * T16;
  const uint32_t sz_s = (uint32_t)__cvta_generic_to_shared(gd_smem) + (uint32_t)S * 9 * T16 + (uint32_t)tid * 8;
  float* red = reinterpret_cast<float*>(gd_smem + (size_t)S * (9 * 16 + 8) * T);
  const int chunks = a.K >> 5;
  const size_t rowb = (size_t)(a.K >> 1);
  const int gpc = (a.K / a.G) >> 5;
  const int c = warp * 32 + lane;
  const bool cok = c < chunks;
  const int gidx = cok ? c / gpc : 0;  // this lane's group

  // the two row-block cursors (copies, compute) only move forward, so each
  // keeps its GEMV index
  int it_copy = 0, it_comp = 0;
  auto item_adv = [&](int& it, int rb) {
    while (it + 1 < a.items && rb >= a.rb_end[it]) ++it;
  };
  // copy row block rb's codes, scales and zero points for this lane into stage st
  auto issue = [&](int rb, int st) {
    if (cok && rb < a.row_blocks) {
      item_adv(it_copy, rb);
      const int it = it_copy;
      const int r0 = (rb - (it ? a.rb_end[it - 1] : 0)) * 8;
      const uint8_t* qc = a.q[it] + (size_t)r0 * rowb + (size_t)c * 16;
      const uint32_t dst = sq_s + (uint32_t)st * 8 * T16;
      const int nr = a.N[it] - r0;
      if (nr >= 8) {
#pragma unroll
        for (int i = 0; i < 8; ++i) cp_async16_s(dst + i * T16, qc + (size_t)i * rowb, 16);
      } else {  // rows past N read nothing and stage zeros
#pragma unroll
        for (int i = 0; i < 8; ++i) cp_async16_s(dst + i * T16, i < nr ? qc + (size_t)i * rowb : qc, i < nr ? 16 : 0);
      }
      const size_t m0 = ((size_t)(r0 >> 7) * a.G + gidx) * 128 + (r0 & 127);
      cp_async16_s(ss_s + (uint32_t)st * T16, a.s[it] + m0 * 2, 16);
      if (ASYM) cp_async8_s(sz_s + (uint32_t)st * 8 * T, a.z[it] + m0);
    }
    cp_async_commit();  // one group per stage, empty or not, keeps the wait count fixed
  };

  int rb = blockIdx.x;
  // the weights are only read: the first S row blocks are requested before
  // waiting for the previous kernel in the stream
#pragma unroll
  for (int st = 0; st < S; ++st) issue(rb + st * (int)gridDim.x, st);
  griddep_launch_dependents();
  griddep_wait();

  uint32_t xr[16];
  float xoff = 0.0f, xsum = 0.0f;
  float sx8 = 0.0f;  // A8: the block's activation scale and code sum
  int xs8 = 0;
  const uint16_t* x_loaded = nullptr;
  auto load_x = [&](const uint16_t* X) {
    x_loaded = X;
    if constexpr (A8) {
#pragma unroll
      for (int i = 0; i < 16; ++i) xr[i] = 0u;
      sx8 = 0.0f;
      xs8 = 0;
      if (cok) {
        uint32_t lo[4], hi[4];
        load_xq_block(reinterpret_cast<const int8_t*>(X) + (size_t)c * 32, lo, hi, xs8);
#pragma unroll
        for (int i = 0; i < 4; ++i) { xr[i] = lo[i]; xr[4 + i] = hi[i]; }
        sx8 = __ldg(a.SX[it_comp] + c);
      }
      return;
    }
    float sA = 0.0f, sB = 0.0f;
    if (cok) {
      const uint4* xp = reinterpret_cast<const uint4*>(X + (size_t)c * 32);
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const uint4 u = ld_nc_v4(xp + v);
        xr[4 * v + 0] = u.x; xr[4 * v + 1] = u.y; xr[4 * v + 2] = u.z; xr[4 * v + 3] = u.w;
      }
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float lo = x2f<BF16>((uint16_t)(xr[i] & 0xFFFFu));
        const float hi = x2f<BF16>((uint16_t)(xr[i] >> 16));
        if ((i & 1) == 0) sA += lo + hi; else sB += lo + hi;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i) xr[i] = 0u;
    }
    xsum = sA + sB;
    xoff = (BF16 ? 128.0f * xsum : 1024.0f * sA + 64.0f * sB) + (ASYM ? 0.0f : 8.0f * xsum);
  };

  int lb = 0, st = 0;
  for (; rb < a.row_blocks; rb += gridDim.x, ++lb) {
    cp_async_wait<S - 1>();  // this lane's copies of row block rb have landed
    item_adv(it_comp, rb);
    const int it = it_comp;
    if (a.X[it] != x_loaded) load_x(a.X[it]);
    float part[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) part[i] = 0.0f;
    if (cok) {
      const uint32_t src = sq_s + (uint32_t)st * 8 * T16;
      const uint4 sv = lds128(ss_s + (uint32_t)st * T16);
      const uint2 zv = ASYM ? lds64(sz_s + (uint32_t)st * 8 * T) : make_uint2(0u, 0u);
      const uint32_t sw[4] = {sv.x, sv.y, sv.z, sv.w};
#pragma unroll
      for (int i = 0; i < 8; i += 2) {
        const float2 sc = __half22float2(*reinterpret_cast<const __half2*>(&sw[i >> 1]));
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if constexpr (A8) {
            const uint4 wv = lds128(src + (uint32_t)(i + h) * T16);
            const uint32_t wd[4] = {wv.x, wv.y, wv.z, wv.w};
            int acc = 0, acc16 = 0;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              acc = dp4a_us(wd[j] & 0x0F0F0F0Fu, xr[j], acc);
              acc16 = dp4a_us(wd[j] & 0xF0F0F0F0u, xr[4 + j], acc16);
            }
            const int zi = ASYM ? (int)(int8_t)(((i < 4 ? zv.x : zv.y) >> (8 * ((i + h) & 3))) & 0xFFu) : 8;
            part[i + h] = (float)(acc + (acc16 >> 4) - zi * xs8) * ((h ? sc.y : sc.x) * sx8);
            continue;
          }
          const float acc = gd_chunk<BF16>(lds128(src + (uint32_t)(i + h) * T16), xr);
          float corr = xoff;
          if (ASYM) {
            const int zi = (int)(int8_t)(((i < 4 ? zv.x : zv.y) >> (8 * ((i + h) & 3))) & 0xFFu);
            corr = fmaf((float)zi, xsum, corr);
          }
          part[i + h] = fmaf(h ? sc.y : sc.x, acc - corr, part[i + h]);
        }
      }
    }
    const float total = butterfly8(part, lane);
    if ((lane & 3) == 0) red[(lb * nw + warp) * 8 + butterfly8_row(lane)] = total;
    issue(rb + S * (int)gridDim.x, st);  // refill the stage just read
    st = st + 1 == S ? 0 : st + 1;
  }
  cp_async_wait<0>();
  __syncthreads();
  int it = 0;
  for (int t = tid; t < lb * 8; t += blockDim.x) {
    const int l = t >> 3, row = t & 7;
    const int rbo = blockIdx.x + l * gridDim.x;
    item_adv(it, rbo);
    const int r = (rbo - (it ? a.rb_end[it - 1] : 0)) * 8 + row;
    float sum = 0.0f;
    for (int w = 0; w < nw; ++w) sum += red[(l * nw + w) * 8 + row];
    if (r < a.N[it]) store_out(a.Y[it], (size_t)r, sum, a.y_bf16);
  }
}

}  // namespace lbq
