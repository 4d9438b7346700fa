// Decode GEMV at batch 1 on INT4 weights with the multiply-adds on the
// tensor cores: y[n] = sum_k x[k] * (q[k][n] - z) * s.
//
// A CUDA-core dot product spends about three instructions per weight here
// (nibble extraction, a conversion and an FMA per product) and tops out near
// 40 weights per clock per SM on B200, which is below what HBM delivers at
// batch 1. A legacy m16n8k16 MMA takes 256 weights per instruction, so the
// per-weight work left on the CUDA cores is the code-to-operand conversion.
//
// The batch is one column, so 7 of the MMA's 8 columns would be idle. They
// are used to keep 32-k chunks apart instead: in each MMA, thread t of a
// quad supplies the A columns {2t, 2t+1} from chunk c0+t and {2t+8, 2t+9}
// from chunk c0+4+t, and the activation fragment puts chunk c0+j's values in
// column j only. Column j of D is then the dot product of the 16 rows with
// chunk c0+j alone, so 16 MMAs over 8 chunks yield 8 per-chunk partial sums
// per row: a group (32, 64 or 128 k) is a whole number of chunks, and its
// scale is applied in FP32 to those sums.
//
//  * Operands are exact: a nibble OR-ed into the mantissa of 1024.0 (FP16)
//    or 128.0 (BF16) is 1024 + q, minus (1024 + z) gives q - z; the
//    upper-nibble class of FP16 (1024 + 16 q) goes through one FMA by 1/16.
//    The tensor cores accumulate x * (q - z) in FP32.
//  * A CTA owns 32-row tiles over the whole K and walks them grid-stride; its
//    warps split K into 8-chunk passes. A pass of a warp covers both 16-row
//    halves of the tile (two independent MMA chains). Each thread's 8 x 16
//    bytes of codes per pass (rows r, r+8, r+16, r+24; chunks c0+t, c0+4+t)
//    are copied into its own shared-memory slots S passes ahead (per-thread
//    asynchronous copies); the pass's scales and zero points travel in the
//    same copy group, copied by the warp's lanes (a warp-level sync makes
//    them visible to all lanes); the activations are staged once per CTA.
//  * Per row tile a warp's row sums are reduced over the quad with shuffles
//    and parked in shared memory; after its last tile the CTA adds the warps'
//    sums in warp order (one barrier per CTA), so results do not depend on
//    timing.
//  * Up to 4 GEMVs with the same K, group, mode and dtypes share one launch
//    (their 32-row tiles are numbered one after the other).
#pragma once

#include "common.cuh"
#include "gemv_m1.cuh"
#include "skinny.cuh"

namespace lbq {

constexpr int kDmMaxWarps = 16;
constexpr int kDmMaxItems = 4;
constexpr int kDmRows = 32;                                  // rows of a tile
constexpr int kDmMetaBytes = 8 * kDmRows * 2 + 8 * kDmRows;  // per warp and pass: 8 groups x 32 rows of scales, zero points

struct GemvDmmaArgs {
  const uint8_t* q[kDmMaxItems];  // [N][K/2]
  const uint8_t* s[kDmMaxItems];  // 128-channel-tiled FP16 scales
  const uint8_t* z[kDmMaxItems];  // 128-channel-tiled int8 zero points (ASYM)
  void* Y[kDmMaxItems];           // [N]
  int N[kDmMaxItems];
  int rt_end[kDmMaxItems];        // cumulative 32-row tiles
  int xi[kDmMaxItems];            // staged activation vector read by the item
  const uint16_t* X[kDmMaxItems]; // distinct activation vectors, [K] each
  int nx;
  int items;
  int K, G;
  int row_tiles;                  // total over the items
  int spw;                        // 8-chunk passes per warp
  int gshift;                     // log2(chunks per group)
  int y_bf16;
};

// Shared-memory bytes of one CTA: codes ring, scale / zero-point ring,
// staged activations, zero-point table; the row sums follow.
__host__ __device__ inline size_t dmma_smem_fixed(int stages, int threads, int nx, int K) {
  return (size_t)stages * 8 * threads * 16 + (size_t)stages * (threads / 32) * kDmMetaBytes + (size_t)nx * K * 2 +
         256 * 8 + (size_t)nx * (K / 32) * 8;
}

template <bool BF16, bool ASYM, int S, bool OFF>
__global__ void __launch_bounds__(kDmMaxWarps * 32, 1) gemv_dmma_kernel(const GemvDmmaArgs a) {
  extern __shared__ __align__(16) uint8_t dm_smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int T = blockDim.x, nw = T >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int K = a.K, chunks = K >> 5;
  const int gshift = a.gshift;
  const size_t rowb = (size_t)(K >> 1);
  const int spw = a.spw;
  uint4* ring = reinterpret_cast<uint4*>(dm_smem);                        // [S][8][T]
  uint8_t* mring = reinterpret_cast<uint8_t*>(ring + (size_t)S * 8 * T);  // [S][nw][kDmMetaBytes]
  uint16_t* xs = reinterpret_cast<uint16_t*>(mring + (size_t)S * nw * kDmMetaBytes);  // [nx][K]
  uint2* zlut = reinterpret_cast<uint2*>(xs + (size_t)a.nx * K);          // [256]
  float2* xsum = reinterpret_cast<float2*>(zlut + 256);                   // [nx][K/32]: per chunk (offset, sum)
  float* red = reinterpret_cast<float*>(xsum + (size_t)a.nx * chunks);    // [tiles][nw][32]

  // A pass is (local row tile lt, pass ss < spw of this warp's K range). Two
  // cursors walk them: the pass computed and the one copied S passes ahead.
  struct Cursor {
    int lt, ss, it;  // it: the GEMV of the tile (tiles only move forward)
  };
  auto advance = [&](Cursor& cu) {
    if (++cu.ss == spw) { cu.ss = 0; ++cu.lt; }
  };
  auto locate = [&](Cursor& cu, int& rt, int& n0, int& c0) {
    rt = blockIdx.x + cu.lt * (int)gridDim.x;
    while (cu.it + 1 < a.items && rt >= a.rt_end[cu.it]) ++cu.it;
    n0 = (rt - (cu.it ? a.rt_end[cu.it - 1] : 0)) * kDmRows;
    c0 = (warp * spw + cu.ss) * 8;
  };
  const size_t thr_off = (size_t)g * rowb + (size_t)t * 16;  // this thread's row / chunk within a pass
  const size_t rowb8 = rowb * 8;
  // 32-bit shared address of this thread's ring element (slot 0, j = 0); elements are T * 16 bytes apart
  const uint32_t T16 = (uint32_t)T * 16;
  const uint32_t ring_s = (uint32_t)__cvta_generic_to_shared(ring) + (uint32_t)tid * 16;
  // Copy a pass's codes (slot element j = 4h + 2f + e: row r + 16h + 8e,
  // chunk c0 + t + 4f) and, cooperatively, its scales and zero points.
  auto issue = [&](Cursor& cu, int slot) {
    int rt, n0, c0;
    locate(cu, rt, n0, c0);
    if (rt < a.row_tiles) {
      const int it = cu.it, N = a.N[it];
      const uint8_t* qb = a.q[it] + (size_t)n0 * rowb + (size_t)c0 * 16 + thr_off;
      const uint32_t dst = ring_s + (uint32_t)slot * 8 * T16;
      if (n0 + kDmRows <= N && c0 + 8 <= chunks) {
#pragma unroll
        for (int j = 0; j < 8; ++j)
          cp_async16_s(dst + j * T16, qb + (size_t)(2 * (j >> 2) + (j & 1)) * rowb8 + 64 * ((j >> 1) & 1), 16);
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int dr = 16 * (j >> 2) + 8 * (j & 1), dc = 4 * ((j >> 1) & 1);
          const bool ok = n0 + dr + g < N && c0 + dc + t < chunks;  // outside: nothing read, zeros staged
          cp_async16_s(dst + j * T16, ok ? qb + (size_t)dr * rowb + dc * 16 : a.q[it], ok ? 16 : 0);
        }
      }
      uint8_t* ms = mring + ((size_t)slot * nw + warp) * kDmMetaBytes;
      const int np = 8 >> gshift, gb = c0 >> gshift;
      const size_t tb = (size_t)(n0 >> 7) * a.G * 128 + (n0 & 127);  // (row n0, group 0); 32 rows stay in one 128-row tile
      {  // scales: lane = (group lane/4, rows 8 (lane%4) .. +7)
        const int lg = lane >> 2, rr = 8 * (lane & 3);
        const bool ok = lg < np && gb + lg < a.G;
        cp_async16(ms + lg * 64 + rr * 2, a.s[it] + (ok ? (tb + (size_t)(gb + lg) * 128 + rr) * 2 : 0), ok ? 16 : 0);
      }
      if (ASYM && lane < 16) {  // zero points: lane = (group lane/2, rows 16 (lane%2) .. +15)
        const int lg = lane >> 1, rr = 16 * (lane & 1);
        const bool ok = lg < np && gb + lg < a.G;
        cp_async16(ms + 512 + lg * 32 + rr, a.z[it] + (ok ? tb + (size_t)(gb + lg) * 128 + rr : 0), ok ? 16 : 0);
      }
    }
    cp_async_commit();  // one group per pass, empty or not, keeps the wait count fixed
    advance(cu);
  };

  // The weights are only read: the first passes' codes and scales are
  // requested before waiting for the previous kernel in the stream.
  Cursor cu_issue{0, 0, 0};
#pragma unroll
  for (int st = 0; st < S; ++st) issue(cu_issue, st);
  if (ASYM) {
    for (int i = tid; i < 256; i += T) {
      const float z = (float)(i - 128);
      zlut[i] = BF16 ? make_uint2(pack_bf16x2(128.0f + z), 0u)
                     : make_uint2(pack_f16x2(1024.0f + z), pack_f16x2(-(64.0f + z)));
    }
  }
  griddep_launch_dependents();
  griddep_wait();
  for (int v = 0; v < a.nx; ++v) {
    const uint4* src = reinterpret_cast<const uint4*>(a.X[v]);
    uint4* dst = reinterpret_cast<uint4*>(xs + (size_t)v * K);
    for (int i = tid; i < (K >> 3); i += T) dst[i] = ld_nc_v4(src + i);
  }
  __syncthreads();
  if (OFF) {
    // per chunk: the offset the operands carry, sum_k x * 1024 (FP16: pairs
    // 0, 2 of each 8-k word carry 1024 + q, pairs 1, 3 carry 1024 + 16 q and
    // are scaled by 1/16 afterwards, so they add 64 x) or 128 x (BF16), and
    // the plain sum used for the zero point
    for (int e = tid; e < a.nx * chunks; e += T) {
      const uint16_t* xc = xs + (size_t)e * 32;
      float sA = 0.0f, sB = 0.0f;
      for (int k = 0; k < 32; ++k) {
        const float v = x2f<BF16>(xc[k]);
        if (((k >> 1) & 1) == 0) sA += v; else sB += v;
      }
      xsum[e] = make_float2(BF16 ? 128.0f * (sA + sB) : 1024.0f * sA + 64.0f * sB, sA + sB);
    }
    __syncthreads();
  }

  // activation fragments (b0, b1): b0 feeds column t (lanes g == t), b1 column 4+t (lanes g == t+4)
  uint2 xb[16];
  int x_key = -1;
  const uint32_t za_sym = BF16 ? pack_bf16x2(136.0f) : pack_f16x2(1032.0f);
  const uint32_t zb_sym = BF16 ? 0u : pack_f16x2(-72.0f);
  float acc[2][2] = {{0.f, 0.f}, {0.f, 0.f}};  // [half][row r / r+8]
  Cursor cu{0, 0, 0};

  for (int slot = 0;; slot = slot + 1 == S ? 0 : slot + 1) {
    int rt, n0, c0;
    locate(cu, rt, n0, c0);
    if (rt >= a.row_tiles) break;
    const int lt = cu.lt;
    const bool tile_end = cu.ss == spw - 1;
    const int it = cu.it;
    cp_async_wait<S - 1>();  // this thread's copies of this pass have landed
    __syncwarp();            // ... and so have the scales the other lanes copied
    const uint8_t* ms = mring + ((size_t)slot * nw + warp) * kDmMetaBytes;
    const uint16_t* msc = reinterpret_cast<const uint16_t*>(ms);    // [group][32 rows]
    const int8_t* mzp = reinterpret_cast<const int8_t*>(ms + 512);  // [group][32 rows]
    const int key = a.xi[it] * 65536 + c0;
    if (key != x_key) {
      x_key = key;
      const uint16_t* xv = xs + (size_t)a.xi[it] * K;
      const int c = g == t ? c0 + t : c0 + 4 + t;
      const bool on = (g == t || g == t + 4) && c < chunks;
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const uint4 p = on ? *reinterpret_cast<const uint4*>(xv + (size_t)c * 32 + 8 * v) : make_uint4(0u, 0u, 0u, 0u);
        const uint32_t pw[4] = {p.x, p.y, p.z, p.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) xb[4 * v + e] = g < 4 ? make_uint2(pw[e], 0u) : make_uint2(0u, pw[e]);
      }
    }
    // codes and zero-point constants; element j = 4h + 2f + e
    uint32_t w[8][4], za[8], zb[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint4 v = lds128(ring_s + ((uint32_t)slot * 8 + j) * T16);
      w[j][0] = v.x; w[j][1] = v.y; w[j][2] = v.z; w[j][3] = v.w;
      if (ASYM && !OFF) {
        const int lg = (t + 4 * ((j >> 1) & 1)) >> gshift;
        const uint2 cz = zlut[mzp[lg * kDmRows + 16 * (j >> 2) + 8 * (j & 1) + g] + 128];
        za[j] = cz.x; zb[j] = cz.y;
      } else {
        za[j] = za_sym; zb[j] = zb_sym;
      }
    }
    // d[h][c]: half h, chain c (exact form: pairs alternate between two
    // chains; offset form: c = the pair's class, 1024 + q or 1024 + 16 q)
    float d[2][2][4];
#pragma unroll
    for (int i = 0; i < 16; ++i) {  // pair i of each chunk: k = 2i, 2i+1
      const int wi = i >> 2, p = i & 3;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t af[4];  // a0 row r / a1 row r+8 (chunk c0+t); a2 row r / a3 row r+8 (chunk c0+4+t)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int j = 4 * h + 2 * (q >> 1) + (q & 1);
          const uint32_t wd = w[j][wi];
          if (!BF16) {
            const uint32_t src = (p >= 2) ? (wd >> 8) : wd;
            const uint32_t o = and_or(src, (p & 1) ? 0x00F000F0u : 0x000F000Fu, 0x64006400u);
            if (OFF) af[q] = o;
            else if ((p & 1) == 0) af[q] = hsub2_u32(o, za[j]);
            else af[q] = hfma2_u32(o, 0x2C002C00u, zb[j]);
          } else {
            const uint32_t o = and_or(wd >> (4 * p), 0x000F000Fu, 0x43004300u);
            af[q] = OFF ? o : bsub2_u32(o, za[j]);
          }
        }
        const int c = p & 1;
        if (i < 2) mma_16816_zc(d[h][c], af, xb[i].x, xb[i].y, BF16);
        else mma_16816(d[h][c], af, xb[i].x, xb[i].y, BF16);
      }
    }
    // D columns 2t, 2t+1 are chunks c0+2t, c0+2t+1 of rows r (d0, d1) and r+8 (d2, d3)
    const int lg0 = (2 * t) >> gshift, lg1 = (2 * t + 1) >> gshift;
    float2 xo[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
    if (OFF) {
      const float2* xsv = xsum + (size_t)a.xi[it] * chunks;
      const int cc = c0 + 2 * t;
      xo[0] = cc < chunks ? xsv[cc] : make_float2(0.f, 0.f);
      xo[1] = cc + 1 < chunks ? xsv[cc + 1] : make_float2(0.f, 0.f);
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int r = 16 * h + 8 * e + g;
#pragma unroll
        for (int cl = 0; cl < 2; ++cl) {
          const int lg = cl ? lg1 : lg0;
          float v;
          if (OFF) {
            // sum x (q - z) = D(1024 + q) + D(1024 + 16 q) / 16 - offset - z * sum x
            v = BF16 ? d[h][0][2 * e + cl] + d[h][1][2 * e + cl] : fmaf(d[h][1][2 * e + cl], 0.0625f, d[h][0][2 * e + cl]);
            v -= xo[cl].x;
            const float zf = ASYM ? (float)mzp[lg * kDmRows + r] : 8.0f;
            v = fmaf(-zf, xo[cl].y, v);
          } else {
            v = d[h][0][2 * e + cl] + d[h][1][2 * e + cl];
          }
          acc[h][e] = fmaf(h2f_bits(msc[lg * kDmRows + r]), v, acc[h][e]);
        }
      }
    }
    __syncwarp();           // every lane has read the slot before any lane refills it
    issue(cu_issue, slot);  // refill the slot just read, S passes ahead
    if (tile_end) {
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          float v = acc[h][e];
          v += __shfl_xor_sync(0xffffffffu, v, 1);
          v += __shfl_xor_sync(0xffffffffu, v, 2);
          if (t == 0) red[((size_t)lt * nw + warp) * kDmRows + 16 * h + 8 * e + g] = v;
          acc[h][e] = 0.0f;
        }
    }
    advance(cu);
  }
  cp_async_wait<0>();
  __syncthreads();
  const int tiles = ((int)blockIdx.x < a.row_tiles) ? (a.row_tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  int it = 0;
  for (int e = tid; e < tiles * kDmRows; e += T) {
    const int l = e / kDmRows, r = e % kDmRows;
    const int rt = blockIdx.x + l * gridDim.x;
    while (it + 1 < a.items && rt >= a.rt_end[it]) ++it;
    const int n = (rt - (it ? a.rt_end[it - 1] : 0)) * kDmRows + r;
    float sum = 0.0f;
    for (int wv = 0; wv < nw; ++wv) sum += red[((size_t)l * nw + wv) * kDmRows + r];
    if (n < a.N[it]) store_out(a.Y[it], (size_t)n, sum, a.y_bf16);
  }
}

}  // namespace lbq
