// Generic b-bit affine group-wise weights (b = 1..8): quantise + repack, the
// canonical unpack, and one decode GEMV per bit width and batch tile.
//
// "Low Bit ARM kernels" keeps one GEMV micro-kernel and one unpack routine per
// bit width 1..8 in a bit-width x tile table, and notes that 3-bit weights
// often keep 4-bit accuracy although they unpack less neatly. The affine form
// is that page's group-wise one: a code q in 0 .. 2^b - 1 per weight, value
// (q - zp) * s with one FP16 scale s and one int8 zero point zp per group of
// 32, 64 or 128 consecutive k of a column.
//
// Q region of the image: N rows of K b / 8 bytes; row n holds column n in
// chunks of 32 k, each b little-endian 32-bit words (4 b bytes). Inside a
// chunk the 16 even k (k = 2j) form one 16 b-bit stream kept in the LOW
// halves of the b words (stream bit t is bit t % 16 of the low half of word
// t / 16) and the 16 odd k (k = 2j + 1) a second stream in the HIGH halves at
// the same positions; code j of either stream takes stream bits [b j, b j + b).
// The pair (k, k + 1) therefore sits at one offset of the two halves of one
// word (two consecutive words when b j + b crosses a 16-bit boundary), and a
// shift plus an AND/OR turns both codes into a half2 / bf16x2 at once, the
// same pairing the INT4 image uses. Scales and zero points are tiled by 128
// channels exactly as for INT4 (8 consecutive channels are contiguous).
//
// Conversion without a convert instruction: a field of F bits shifted to bit
// position MANT - F of each half (MANT = 10 for FP16, 7 for BF16) and OR-ed
// with the bits of 2^F reads as the number 2^F + q, exactly (the mantissa's
// unit at that exponent is 1). The small offset 2^F keeps the FP32 sums of
// x * (2^F + q) close to the size of the wanted sums of x * q. BF16 has room
// for 7-bit fields, so 8-bit codes in BF16 go as two 4-bit fields,
// q = lo + 16 hi.
#pragma once

#include "common.cuh"
#include "gemv_m1.cuh"

namespace lbq {

// ----------------------------------------------------------------------------
// Quantise + repack, canonical unpack
// ----------------------------------------------------------------------------

// One thread per (group gi, column n); every step that decides a code is IEEE
// FP32 with round-to-nearest-even, as for INT4:
//   s = fp16((max w - min w) / (2^b - 1)); zp = clamp(rint(-min w / s), -128, 127);
//   q = clamp(rint(w / s) + zp, 0, 2^b - 1); a group whose stored s is 0 gets zp = 0, q = 0.
__global__ void __launch_bounds__(256) quantize_pack_affine_kernel(
    const float* __restrict__ W, int K, int N, int group, int bits,
    uint8_t* __restrict__ q_region, uint8_t* __restrict__ s_region, uint8_t* __restrict__ z_region) {
  const int G = K / group;
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= (long long)G * N) return;
  const int n = (int)(t % N);
  const int gi = (int)(t / N);
  const float* w = W + (size_t)gi * group * N + n;
  const float L = (float)((1 << bits) - 1);

  float lo = w[0], hi = w[0];
  for (int i = 1; i < group; ++i) {
    const float v = w[(size_t)i * N];
    lo = fminf(lo, v);
    hi = fmaxf(hi, v);
  }
  const __half s16 = __float2half_rn(__fdiv_rn(__fsub_rn(hi, lo), L));
  const float s = __half2float(s16);
  const float zp = (s == 0.0f) ? 0.0f : fminf(fmaxf(rintf(__fdiv_rn(-lo, s)), -128.0f), 127.0f);

  uint32_t* row = reinterpret_cast<uint32_t*>(q_region + (size_t)n * (size_t)(K / 32) * 4 * bits);
  const int c0 = gi * group / 32;
  for (int c = 0; c < group / 32; ++c) {
    uint32_t words[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
    for (int kk = 0; kk < 32; ++kk) {
      uint32_t q = 0u;
      if (s != 0.0f) {
        const float r = rintf(__fdiv_rn(w[(size_t)(c * 32 + kk) * N], s));
        q = (uint32_t)fminf(fmaxf(__fadd_rn(r, zp), 0.0f), L);
      }
      const int h = 16 * (kk & 1), p = bits * (kk >> 1), wi = p >> 4, o = p & 15;
      words[wi] |= ((q << o) & 0xFFFFu) << h;
      if (o + bits > 16) words[wi + 1] |= (q >> (16 - o)) << h;
    }
    for (int i = 0; i < bits; ++i) row[(size_t)(c0 + c) * bits + i] = words[i];
  }
  reinterpret_cast<uint16_t*>(s_region)[meta_index(n, gi, G)] = __half_as_ushort(s16);
  reinterpret_cast<int8_t*>(z_region)[meta_index(n, gi, G)] = (int8_t)(int)zp;
}

// Code of weight (k, n) read back from the image.
__device__ __forceinline__ uint32_t affine_code(const uint8_t* q_region, int K, int bits, int k, int n) {
  const uint32_t* cw = reinterpret_cast<const uint32_t*>(q_region + (size_t)n * (size_t)(K / 32) * 4 * bits) +
                       (size_t)(k >> 5) * bits;
  const int kk = k & 31, h = 16 * (kk & 1), p = bits * (kk >> 1), wi = p >> 4, o = p & 15;
  uint32_t v = (cw[wi] >> h) & 0xFFFFu;
  if (o + bits > 16) v |= ((cw[wi + 1] >> h) & 0xFFFFu) << 16;
  return (v >> o) & ((1u << bits) - 1u);
}

// Canonical arrays: per column n one little-endian bit stream, code k at bits
// [b k, b k + b); byte jb of column n's stream goes to q_stream[jb][n]
// (uint8 [K b / 8, N]). Scales and zero points transposed back to [K/group][N].
__global__ void __launch_bounds__(256) unpack_affine_kernel(
    const uint8_t* __restrict__ q_region, const uint8_t* __restrict__ s_region,
    const uint8_t* __restrict__ z_region, int K, int N, int group, int bits,
    uint8_t* __restrict__ q_stream, uint16_t* __restrict__ s_out, int8_t* __restrict__ z_out) {
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long nbytes = (long long)(K / 8) * bits * N;
  if (t < nbytes) {
    const int n = (int)(t % N);
    const long long jb = t / N;
    uint32_t byte = 0u;
    for (int i = 0; i < 8; ++i) {
      const long long P = 8 * jb + i;
      const int k = (int)(P / bits), b = (int)(P % bits);
      byte |= ((affine_code(q_region, K, bits, k, n) >> b) & 1u) << i;
    }
    q_stream[t] = (uint8_t)byte;
  }
  const int G = K / group;
  if (t < (long long)G * N) {
    const int n = (int)(t % N);
    const int gi = (int)(t / N);
    s_out[t] = reinterpret_cast<const uint16_t*>(s_region)[meta_index(n, gi, G)];
    z_out[t] = reinterpret_cast<const int8_t*>(z_region)[meta_index(n, gi, G)];
  }
}

// ----------------------------------------------------------------------------
// Decode GEMV: Y[m][n] = sum_k X[m][k] (q[k][n] - zp) s, 1 <= m < MB per launch
// ----------------------------------------------------------------------------
//
//  * Lane l of warp w owns the 32-k chunk c = 32 w + l (K <= 16384, one scale
//    per chunk); its MB x 32 activations and their per-row sums stay in
//    registers for all of the CTA's row blocks.
//  * A row block is R = 8 / MB output channels, so a lane carries R x MB = 8
//    partial sums: the 8-value transposing butterfly reduces them over the
//    warp, and the warps' totals meet in shared memory (double-buffered, one
//    barrier per row block, a fixed summation order).
//  * Per row block a lane issues R loads of its chunk (the widest vector that
//    4 b bytes allow), one vector load of the R scales and one of the R zero
//    points; consecutive lanes read consecutive chunks of a row, so a warp
//    instruction covers 128 b contiguous bytes. Latency is hidden by the
//    other warps resident on the SM (no staging, no handshakes); the first
//    row block is requested before the kernel waits for its predecessor in
//    the stream (programmatic dependent launch).
//  * Per pair of k one shift + one AND/OR (four operations when the pair's
//    field crosses a 16-bit boundary) give 2^F + q for both k, and two
//    mixed-precision FMAs accumulate x (2^F + q) in FP32 for each batch row.
//    Per chunk:  sum x (q - zp) = acc - (2^F + zp) sum x,  then times s.

constexpr int kAgMaxWarps = 16;

struct AffineGemvArgs {
  const uint16_t* X;  // [m_valid][K] FP16/BF16 bits
  void* Y;            // [m_valid][N]
  const uint8_t* q;   // Q region
  const uint8_t* s;   // S region
  const uint8_t* z;   // Z region
  int K, N, G, gshift;  // chunk c lies in group c >> gshift
  int m_valid, row_blocks, y_bf16;
};

__device__ __forceinline__ uint32_t ag_shift(uint32_t v, int s) { return s >= 0 ? (v >> s) : (v << -s); }

// (a & m) | (b & ~m)
__device__ __forceinline__ uint32_t bit_select(uint32_t a, uint32_t b, uint32_t m) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xE4;" : "=r"(d) : "r"(a), "r"(b), "r"(m));
  return d;
}

// The F-bit field at stream bit P of both halves, as 2^F + q in each half
// (FP16 bits for MANT = 10, BF16 for MANT = 7). P is a constant once the
// caller's loops are unrolled, so every branch and shift here folds away.
template <int B, int F, int MANT>
__device__ __forceinline__ uint32_t ag_field(const uint32_t (&w)[B], int P) {
  const int pos = MANT - F;
  const uint32_t fm = ((1u << F) - 1u) << pos;
  const uint32_t one = MANT == 10 ? (0x3C00u + ((uint32_t)F << 10)) : (0x3F80u + ((uint32_t)F << 7));
  const int wi = P >> 4, o = P & 15;
  if (o + F <= 16) return and_or(ag_shift(w[wi], o - pos), fm | (fm << 16), one | (one << 16));
  const int a = 16 - o;  // bits of the field in word wi; the rest open word wi + 1
  const uint32_t lm = ((1u << a) - 1u) << pos;
  const uint32_t t = bit_select(w[wi] >> (o - pos), w[wi + 1 < B ? wi + 1 : B - 1] << (pos + a), lm | (lm << 16));
  return and_or(t, fm | (fm << 16), one | (one << 16));
}

template <int B>
__device__ __forceinline__ void ag_load_chunk(const uint8_t* p, uint32_t (&w)[B]) {
  if constexpr (B % 4 == 0) {
#pragma unroll
    for (int i = 0; i < B / 4; ++i) {
      const uint4 v = ld_stream_v4(p + 16 * i);
      w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
    }
  } else if constexpr (B % 2 == 0) {
#pragma unroll
    for (int i = 0; i < B / 2; ++i) {
      uint32_t x, y;
      asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(x), "=r"(y) : "l"(p + 8 * i));
      w[2 * i] = x; w[2 * i + 1] = y;
    }
  } else {
#pragma unroll
    for (int i = 0; i < B; ++i) {
      uint32_t x;
      asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(x) : "l"(p + 4 * i));
      w[i] = x;
    }
  }
}

template <int B, bool BF16, int MB>
__global__ void __launch_bounds__(kAgMaxWarps * 32) affine_gemv_kernel(const AffineGemvArgs a) {
  constexpr int R = 8 / MB;                // rows per block
  constexpr bool kSplit = BF16 && B == 8;  // two 4-bit fields per code
  constexpr int F = kSplit ? 4 : B;
  constexpr int MANT = BF16 ? 7 : 10;
  constexpr float kOffset = kSplit ? 272.0f : (float)(1 << F);  // 16 + 16*16 for q = lo + 16 hi

  extern __shared__ float red[];  // [2][warps][8]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nw = blockDim.x >> 5;
  const int chunks = a.K >> 5;
  const int c = tid;
  const bool cok = c < chunks;
  const size_t rowb = (size_t)chunks * 4 * B;
  const int gi = c >> a.gshift;

  // codes, scales and zero points of row block rb
  uint32_t w[R][B];
  float s[R], zf[R];
  auto load_rows = [&](int rb) {
    const int n0 = rb * R;
#pragma unroll
    for (int r = 0; r < R; ++r) {
#pragma unroll
      for (int i = 0; i < B; ++i) w[r][i] = 0u;
      if (cok && n0 + r < a.N) ag_load_chunk<B>(a.q + (size_t)(n0 + r) * rowb + (size_t)c * 4 * B, w[r]);
      s[r] = 0.0f;
      zf[r] = 0.0f;
    }
    if (cok) {
      // R consecutive channels of one 128-channel tile: contiguous, and padded
      // with zeros up to the tile's end, so the vector loads stay in the region.
      const size_t mi = meta_index(n0, gi, a.G);
      uint16_t sb[R];
      int8_t zb[R];
      if constexpr (R == 8) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(a.s) + mi / 8);
        const uint2 u = __ldg(reinterpret_cast<const uint2*>(a.z) + mi / 8);
        const uint32_t vs[4] = {v.x, v.y, v.z, v.w}, us[2] = {u.x, u.y};
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          sb[r] = (uint16_t)(vs[r >> 1] >> (16 * (r & 1)));
          zb[r] = (int8_t)(us[r >> 2] >> (8 * (r & 3)));
        }
      } else if constexpr (R == 4) {
        const uint2 v = __ldg(reinterpret_cast<const uint2*>(a.s) + mi / 4);
        const uint32_t u = __ldg(reinterpret_cast<const uint32_t*>(a.z) + mi / 4);
        const uint32_t vs[2] = {v.x, v.y};
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          sb[r] = (uint16_t)(vs[r >> 1] >> (16 * (r & 1)));
          zb[r] = (int8_t)(u >> (8 * r));
        }
      } else {
        const uint32_t v = __ldg(reinterpret_cast<const uint32_t*>(a.s) + mi / 2);
        const uint16_t u = __ldg(reinterpret_cast<const uint16_t*>(a.z) + mi / 2);
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          sb[r] = (uint16_t)(v >> (16 * r));
          zb[r] = (int8_t)(u >> (8 * r));
        }
      }
#pragma unroll
      for (int r = 0; r < R; ++r) {
        s[r] = h2f_bits(sb[r]);
        zf[r] = (float)zb[r];
      }
    }
  };
  // the weights are only read: the first row block is requested before waiting
  // for the previous kernel in the stream (which may write X)
  if ((int)blockIdx.x < a.row_blocks) load_rows(blockIdx.x);
  griddep_launch_dependents();
  griddep_wait();

  uint32_t x[MB][16];
  float xs[MB];
#pragma unroll
  for (int m = 0; m < MB; ++m) {
    xs[m] = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) x[m][i] = 0u;
    if (cok && m < a.m_valid) {
      const uint4* xp = reinterpret_cast<const uint4*>(a.X + (size_t)m * a.K + (size_t)c * 32);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint4 v = __ldg(xp + i);
        x[m][4 * i] = v.x; x[m][4 * i + 1] = v.y; x[m][4 * i + 2] = v.z; x[m][4 * i + 3] = v.w;
      }
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        xs[m] += x2f<BF16>((uint16_t)(x[m][i] & 0xFFFFu));
        xs[m] += x2f<BF16>((uint16_t)(x[m][i] >> 16));
      }
    }
  }

  int buf = 0;
  for (int rb = blockIdx.x; rb < a.row_blocks; rb += gridDim.x) {
    const int n0 = rb * R;
    if (rb != (int)blockIdx.x) load_rows(rb);

    float part[8];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      float acc[MB], acc_hi[MB];
#pragma unroll
      for (int m = 0; m < MB; ++m) { acc[m] = 0.0f; acc_hi[m] = 0.0f; }
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        if constexpr (!kSplit) {
          const uint32_t wp = ag_field<B, F, MANT>(w[r], B * j);
#pragma unroll
          for (int m = 0; m < MB; ++m)
            acc[m] = BF16 ? fma2_bf16_f32(x[m][j], wp, acc[m]) : fma2_f16_f32(x[m][j], wp, acc[m]);
        } else {
          const uint32_t lo = ag_field<B, 4, MANT>(w[r], 8 * j);
          const uint32_t hi = ag_field<B, 4, MANT>(w[r], 8 * j + 4);
#pragma unroll
          for (int m = 0; m < MB; ++m) {
            acc[m] = fma2_bf16_f32(x[m][j], lo, acc[m]);
            acc_hi[m] = fma2_bf16_f32(x[m][j], hi, acc_hi[m]);
          }
        }
      }
#pragma unroll
      for (int m = 0; m < MB; ++m) {
        const float tot = kSplit ? fmaf(acc_hi[m], 16.0f, acc[m]) : acc[m];
        part[m * R + r] = s[r] * fmaf(-(kOffset + zf[r]), xs[m], tot);
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
