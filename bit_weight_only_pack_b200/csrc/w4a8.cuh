// W4A8: INT4 weights (the lbq_pack image, SYM or ASYM) times dynamically
// quantised INT8 activations, with integer dot products.
//
// "Low Bit ARM kernels" runs its 4-bit-weight decode with dynamic INT8
// activations (group size 32): the weight codes are unpacked to int8 and
// multiplied with the int8 activations in an integer matrix-multiply
// instruction with int32 accumulation; the group scales are applied after the
// integer sum. On B200 the batch-1 shape is a GEMV, so the integer products
// run on the CUDA cores' 4-way byte dot product (dp4a: 4 multiply-adds per
// instruction, int32 accumulation):
//
//  * Activations: each row of X is quantised once per call, in blocks of 32
//    consecutive k, symmetric: s = amax / 127 in IEEE FP32 and xq = clamp(
//    rint(x / s), -127, 127) with the division in FP32 (s = 0 and xq = 0 for
//    an all-zero block) by lbq_quantize_int8; the GEMVs read xq and s (lane
//    l of warp w takes block 32 w + l: 32 bytes and one scale). Quantising in
//    every CTA of a GEMV instead would repeat the work a thousand times per
//    launch, and the projections that share an activation vector (q, k, v;
//    gate, up) share one quantisation.
//  * Weights: per 32-bit code word (8 k) the low nibbles AND 0x0F0F0F0F are
//    four unsigned bytes (k0, k4, k1, k5 in the INT4 image's slot order) and
//    the high nibbles AND 0xF0F0F0F0 four bytes 16 q (k2, k6, k3, k7), so two
//    logic operations and two dp4a retire eight weights; the activation bytes
//    are permuted once into the same orders, and the high-nibble sum is
//    divided by 16 (exactly) at the end of the block.
//  * Per block and row, exactly in int32:  I = sum xq q - z sum xq  (z = 8 for
//    SYM, the zero point for ASYM); the FP32 result adds (s_w s_x) I.
//  * The rest (row blocks of R = 8 / MB channels, 8 partial sums per lane,
//    transposing butterfly, warp totals met in shared memory in a fixed
//    order) follows the batch-1 GEMVs of this library.
#pragma once

#include "common.cuh"
#include "gemv_m1.cuh"

namespace lbq {

constexpr int kW8MaxWarps = 16;

// d = c + sum of the four products of unsigned bytes of a and signed bytes of b
__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

__device__ __forceinline__ void w8_griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void w8_griddep_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" :::); }

// One warp per 32-k block of X, one element per lane: the block maximum is a
// warp reduction and the warp writes its 32 codes as one 32-byte segment.
//
// xq = rint(RN(x / s)) needs the correctly rounded quotient only near a
// half-integer. The product t = RN(x RN(1/s)) is within 2^-15 of RN(x / s)
// (two roundings of relative size 2^-24 on a value below 128, plus half an
// ulp of RN(x / s)), so when t lies at least 2^-14 from every half-integer
// both round to the same integer; otherwise (and when 1/s is not finite) the
// code is taken from the IEEE quotient itself. Same codes as the division
// everywhere, one division per block on the common path.
// With programmatic dependent launch the GEMV that reads the codes may start
// (and stream its weights) while this kernel runs; X is read only after the
// previous kernel in the stream has finished.
template <bool BF16>
__global__ void __launch_bounds__(256) quantize_int8_kernel(const uint16_t* __restrict__ X, int M, int K,
                                                            int8_t* __restrict__ xq, float* __restrict__ sx) {
  w8_griddep_launch_dependents();
  w8_griddep_wait();
  const long long blk = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (blk >= (long long)M * (K / 32)) return;  // whole warps leave together
  const float x = x2f<BF16>(X[blk * 32 + lane]);
  float amax = fabsf(x);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
  const float s = __fdiv_rn(amax, 127.0f);
  const float inv = __fdiv_rn(1.0f, s);
  float r = 0.0f;
  if (s != 0.0f) {
    const float t = __fmul_rn(x, inv);
    r = rintf(t);
    if (!(inv <= 3.4028234663852886e38f) || 0.5f - fabsf(t - r) < 6.103515625e-05f) r = rintf(__fdiv_rn(x, s));
    r = fminf(fmaxf(r, -127.0f), 127.0f);
  }
  xq[blk * 32 + lane] = (int8_t)(int)r;
  if (lane == 0) sx[blk] = s;
}

// This lane's activation block: codes permuted into the weight words' byte
// orders (word i of a code chunk holds k = 8i .. 8i+7 as bytes (k0, k4, k1, k5)
// of its low nibbles and (k2, k6, k3, k7) of its high nibbles) and their sum.
__device__ __forceinline__ void load_xq_block(const int8_t* p, uint32_t (&xlo)[4], uint32_t (&xhi)[4], int& xsum) {
  const uint4 a = __ldg(reinterpret_cast<const uint4*>(p));
  const uint4 b = __ldg(reinterpret_cast<const uint4*>(p) + 1);
  const uint32_t nat[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  xsum = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    xlo[i] = __byte_perm(nat[2 * i], nat[2 * i + 1], 0x5140);
    xhi[i] = __byte_perm(nat[2 * i], nat[2 * i + 1], 0x7362);
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) xsum = __dp4a((int)nat[i], 0x01010101, xsum);
}

struct W4a8Args {
  const int8_t* XQ;   // [m_valid][K] INT8 activations
  const float* SX;    // [m_valid][K/32] their scales
  void* Y;            // [m_valid][N]
  const uint8_t* q;   // INT4 Q region [N][K/2]
  const uint8_t* s;   // 128-channel-tiled FP16 scales
  const uint8_t* z;   // 128-channel-tiled int8 zero points (ASYM)
  int K, N, G, gshift;  // block c lies in weight group c >> gshift
  int m_valid, row_blocks, y_bf16;
};

template <bool ASYM, int MB>
__global__ void __launch_bounds__(kW8MaxWarps * 32) w4a8_gemv_kernel(const W4a8Args a) {
  constexpr int R = 8 / MB;
  extern __shared__ float red[];  // [2][warps][8]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nw = blockDim.x >> 5;
  const int chunks = a.K >> 5;
  const int c = tid;
  const bool cok = c < chunks;
  const size_t rowb = (size_t)(a.K >> 1);
  const int gi = c >> a.gshift;

  // codes, scales and zero points of row block rb
  uint4 w[R];
  float s[R];
  int z[R];
  auto load_block = [&](int rb) {
    const int n0 = rb * R;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      w[r] = make_uint4(0u, 0u, 0u, 0u);
      if (cok && n0 + r < a.N) w[r] = ld_stream_v4(a.q + (size_t)(n0 + r) * rowb + (size_t)c * 16);
      s[r] = 0.0f;
      z[r] = 8;
    }
    if (cok) {
      // R consecutive channels of one 128-channel tile: contiguous, and padded
      // with zeros up to the tile's end, so the vector loads stay in the region.
      const size_t mi = meta_index(n0, gi, a.G);
      uint16_t sb[R];
      if constexpr (R == 8) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(a.s) + mi / 8);
        const uint32_t vs[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int r = 0; r < 8; ++r) sb[r] = (uint16_t)(vs[r >> 1] >> (16 * (r & 1)));
        if (ASYM) {
          const uint2 u = __ldg(reinterpret_cast<const uint2*>(a.z) + mi / 8);
          const uint32_t us[2] = {u.x, u.y};
#pragma unroll
          for (int r = 0; r < 8; ++r) z[r] = (int)(int8_t)(us[r >> 2] >> (8 * (r & 3)));
        }
      } else if constexpr (R == 4) {
        const uint2 v = __ldg(reinterpret_cast<const uint2*>(a.s) + mi / 4);
        const uint32_t vs[2] = {v.x, v.y};
#pragma unroll
        for (int r = 0; r < 4; ++r) sb[r] = (uint16_t)(vs[r >> 1] >> (16 * (r & 1)));
        if (ASYM) {
          const uint32_t u = __ldg(reinterpret_cast<const uint32_t*>(a.z) + mi / 4);
#pragma unroll
          for (int r = 0; r < 4; ++r) z[r] = (int)(int8_t)(u >> (8 * r));
        }
      } else {
        const uint32_t v = __ldg(reinterpret_cast<const uint32_t*>(a.s) + mi / 2);
#pragma unroll
        for (int r = 0; r < 2; ++r) sb[r] = (uint16_t)(v >> (16 * r));
        if (ASYM) {
          const uint16_t u = __ldg(reinterpret_cast<const uint16_t*>(a.z) + mi / 2);
#pragma unroll
          for (int r = 0; r < 2; ++r) z[r] = (int)(int8_t)(u >> (8 * r));
        }
      }
#pragma unroll
      for (int r = 0; r < R; ++r) s[r] = h2f_bits(sb[r]);
    }
  };
  // the first row block's loads are in flight while the activations are read;
  // the weights are only read, so they are requested before waiting for the
  // previous kernel in the stream (which may write the activations)
  if ((int)blockIdx.x < a.row_blocks) load_block(blockIdx.x);
  w8_griddep_launch_dependents();
  w8_griddep_wait();

  uint32_t xlo[MB][4], xhi[MB][4];
  float sx[MB];
  int xsum[MB];
#pragma unroll
  for (int m = 0; m < MB; ++m) {
    sx[m] = 0.0f;
    xsum[m] = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) { xlo[m][i] = 0u; xhi[m][i] = 0u; }
    if (cok && m < a.m_valid) {
      load_xq_block(a.XQ + (size_t)m * a.K + (size_t)c * 32, xlo[m], xhi[m], xsum[m]);
      sx[m] = __ldg(a.SX + (size_t)m * chunks + c);
    }
  }

  int buf = 0;
  for (int rb = blockIdx.x; rb < a.row_blocks; rb += gridDim.x) {
    const int n0 = rb * R;
    if (rb != (int)blockIdx.x) load_block(rb);

    float part[8];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      int acc[MB], acc16[MB];
#pragma unroll
      for (int m = 0; m < MB; ++m) { acc[m] = 0; acc16[m] = 0; }
      const uint32_t wd[4] = {w[r].x, w[r].y, w[r].z, w[r].w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t lo = wd[i] & 0x0F0F0F0Fu;
        const uint32_t hi = wd[i] & 0xF0F0F0F0u;  // bytes 16 q
#pragma unroll
        for (int m = 0; m < MB; ++m) {
          acc[m] = dp4a_us(lo, xlo[m][i], acc[m]);
          acc16[m] = dp4a_us(hi, xhi[m][i], acc16[m]);
        }
      }
#pragma unroll
      for (int m = 0; m < MB; ++m) {
        const int isum = acc[m] + (acc16[m] >> 4) - z[r] * xsum[m];
        part[m * R + r] = (s[r] * sx[m]) * (float)isum;
      }
    }

    const float total = butterfly8(part, lane);
    if ((lane & 3) == 0) red[(buf * nw + warp) * 8 + butterfly8_row(lane)] = total;
    __syncthreads();
    if (tid < 8) {
      const int m = tid / R, n = n0 + tid % R;
      if (m < a.m_valid && n < a.N) {
        float sum = 0.0f;
        for (int i = 0; i < nw; ++i) sum += red[(buf * nw + i) * 8 + tid];
        store_out(a.Y, (size_t)m * a.N + n, sum, a.y_bf16);
      }
    }
    buf ^= 1;
  }
}

}  // namespace lbq
