// LUT3 weights x MXFP8 activations on the block-scaled FP8 tensor path:
// Y^T[N, M] = W^T[N, K] . X^T[K, M] with tcgen05.mma.kind::mxf8f6f4.block_scale.
//
// The vLLM PR 62759 write-up (format section, "LUT-B MoE with MXFP8
// activations") pairs the 3-bit LUT weights with MXFP8 activations: E4M3
// elements with one UE8M0 scale per 1 x 32 block. Its weights are indices into
// an E4M3 codebook, so the decoded weight is an E4M3 byte as it stands, and the
// tile's UE8M0 exponent is exactly a block scale of the weight operand: both
// 32-k halves of a 64-k tile carry it. The page's kernel gets the decode from
// Rubin's LUT decompressor; sm_100a has none, so here converter warps decode
// the indices in software (two byte permutes per eight weights) into a
// shared-memory operand tile, and the block-scaled MMA applies both scales.
// Every product of two E4M3 values and two powers of two is exact; only the
// FP32 accumulation order differs from the exact sum.
//
// Tile: 128 output channels (the MMA's M, the TMEM lanes) x 256 tokens (N),
// K in blocks of 128 (two LUT3 tiles, four MMAs of K = 32).
//
//   warp 0      TMA producer, per k-block: the tokens' E4M3 codes (256 rows x
//               128 bytes, 128-byte swizzle: the K-major B operand), the
//               channels' indices (bulk copies of the I region), the tiles'
//               codebook and exponent bytes (16 channel groups) and the
//               tokens' UE8M0 scale bytes.
//   warp 1      TMEM owner and MMA issuer: copies the block's scale atoms to
//               tensor memory (tcgen05.cp 32x128b.warpx4), then four
//               block-scaled MMAs with the scale byte of each 32-k step
//               selected by its ID, into one 256-column FP32 accumulator.
//   warps 2..9  converters: thread (warp w, lane l) owns channel 32 (w & 3) + l
//               and LUT3 tile (w - 2) / 4 of the block; it writes the channel's
//               64 E4M3 weights of that tile into the swizzled A tile and its
//               scale byte into the A scale atom; the first four warps also copy
//               the scale bytes of tokens r and 128 + r into the B scale atoms.
//               (Eight warps measured 3-5% faster than four, one per channel.)
//   warps 10..13 epilogue: tcgen05.ld the finished accumulator 64 tokens per
//               wait (thread = one channel), round 32 at a time into a [32 tokens][128
//               channels] shared-memory tile and write it with one TMA store
//               (two tiles alternate, so the rounding of one overlaps the store
//               of the other).
//
// Scale atoms (both operands): 128 rows x 4 k-steps of one byte, row r's four
// bytes at 16 (r % 32) + 4 (r / 32) + step; tcgen05.cp.32x128b.warpx4 places
// row r in TMEM lane r % 32 (and its copies in the other three lane quarters),
// column r / 32, byte = step, which is where the MMA reads it.
#pragma once

#include "common.cuh"
#include "tma.cuh"
#include "gemm_tc.cuh"
#include "lut3_gemv.cuh"
#include "stream_k.cuh"

namespace lbq {

constexpr int kMxBN = 128;            // channels per tile (TMEM lanes)
constexpr int kMxBM = 256;            // tokens per tile (MMA N)
constexpr int kMxBK = 128;            // k per block
constexpr int kMxStages = 3;          // TMA ring
constexpr int kMxABufs = 4;           // converted A tiles + scale atoms
constexpr int kMxConvWarps = 8, kMxEpWarps = 4;
constexpr int kMxThreads = (2 + kMxConvWarps + kMxEpWarps) * 32;
// stage layout for a tile of BM tokens
template <int BM>
struct MxStage {
  static constexpr int kOffX = 0;                          // BM x 128 B codes, 128-byte swizzle
  static constexpr int kOffI = kOffX + BM * kMxBK;         // 2 tiles x 128 channels x 24 B indices
  static constexpr int kOffC = kOffI + 2 * kMxBN * 24;     // codebooks: 16 groups x 16 B (2 tiles x 8 B)
  static constexpr int kOffE = kOffC + 16 * 16;            // exponents: 16 groups x 16 B (tiles in a 16-tile row)
  static constexpr int kOffS = kOffE + 16 * 16;            // token scales: BM x 16 B (4 blocks of a 512-k row)
  static constexpr int kBytes = (kOffS + BM * 16 + 1023) / 1024 * 1024;
};
constexpr int kMxOffX = MxStage<kMxBM>::kOffX;
constexpr int kMxOffI = MxStage<kMxBM>::kOffI;
constexpr int kMxOffC = MxStage<kMxBM>::kOffC;
constexpr int kMxOffE = MxStage<kMxBM>::kOffE;
constexpr int kMxOffS = MxStage<kMxBM>::kOffS;
constexpr int kMxStageBytes = MxStage<kMxBM>::kBytes;
// A buffer layout
constexpr int kMxOffA = 0;                            // 128 x 128 B weights, 128-byte swizzle
constexpr int kMxOffSA = kMxBN * kMxBK;               // A scale atom, 512 B
constexpr int kMxOffSB = kMxOffSA + 512;              // B scale atoms (one per 128 tokens), up to 1024 B
constexpr int kMxABufBytes = (kMxOffSB + 1024 + 1023) / 1024 * 1024;
constexpr int kMxOutBytes = 32 * kMxBN * 2;          // one [32 tokens][128 channels] output tile
constexpr int kMxSmem = kMxStages * kMxStageBytes + kMxABufs * kMxABufBytes + 2 * kMxOutBytes + 1024;
constexpr uint32_t kMxColD = 0, kMxColSF = 256;       // TMEM columns: accumulator, then 16 per A buffer
static_assert(kMxStageBytes % 1024 == 0 && kMxABufBytes % 1024 == 0, "1024-byte aligned tiles");

struct GemmMxArgs {
  void* Y;                   // [M][N]
  const uint8_t* i_region;   // LUT3 indices [K/64][N][24]
  int M, N, K;
  int n_tiles, m_tiles, k_blocks;
  int cb_rows;               // rows of the codebook / exponent boxes (min(16, N/8))
  int y_bf16;
  SkArgs sk;                 // the schedule: whole tiles, or stream-K over the last two waves (stream_k.cuh)
};

// Instruction descriptor of kind::mxf8f6f4.block_scale: A = B = E4M3, K-major,
// D = FP32, UE8M0 scales, N = 256, M = 128; the scale IDs pick the k-step's
// byte of each 32-bit scale column.
__host__ __device__ constexpr uint32_t umma_idesc_mx(uint32_t step, int n = kMxBM) {
  return ((uint32_t)(n >> 3) << 17) | (1u << 23) | ((uint32_t)(kMxBN >> 4) << 24) | (step << 29) | (step << 4);
}

// Shared-memory descriptor of a scale atom for tcgen05.cp: 32 rows of 16 bytes,
// no swizzle, 8-row core matrices 128 bytes apart.
__device__ __forceinline__ uint64_t sf_desc(uint32_t smem_addr) {
  return (uint64_t)((smem_addr >> 4) & 0x3FFFu) | ((uint64_t)(128 >> 4) << 16) | ((uint64_t)(128 >> 4) << 32) |
         ((uint64_t)1 << 46);
}

__device__ __forceinline__ void consumer_named_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" :: "r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ void tmem_cp_sf(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" :: "r"(taddr), "l"(sdesc) : "memory");
}

__device__ __forceinline__ void umma_mx(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                        uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t acc) {
  asm volatile("{\n\t.reg .pred p;\n\t"
               "setp.ne.b32 p, %6, 0;\n\t"
               "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%4], [%5], p;\n\t}"
               :: "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(sfa_tmem), "r"(sfb_tmem), "r"(acc)
               : "memory");
}

// Converter work of one k-block for channel r of the tile, LUT3 tiles
// h = hb .. he - 1 of the block (64 k each): the channel's E4M3 weights into
// the swizzled A tile and its tile exponents into the A scale atom (scale 1.0
// and zero weights when the channel does not exist, row_ok false); with
// copy_scales, also the k-block's scale bytes of tokens r + 128 hh into the B
// scale atoms. cbp points at the channel group's 16 codebook bytes of the
// block (tile h at cbp + 8 h), ep at its exponent byte of the block's first
// tile (tile h at ep[h]); st is the stage (layout MxStage<BM>), ab the A buffer.
template <int BM>
__device__ __forceinline__ void mx_convert_block(const uint8_t* st, uint8_t* ab, int r, int kb, bool row_ok,
                                                 const uint8_t* cbp, const uint8_t* ep, int hb, int he,
                                                 bool copy_scales) {
  using L = MxStage<BM>;
  const uint32_t arow = smem_u32(ab + kMxOffA) + (uint32_t)r * 128u;
  const uint32_t atom_off = (uint32_t)(16 * (r & 31) + 4 * (r >> 5));
  for (int h = hb; h < he; ++h) {
    uint32_t eh = 0x7F7Fu;  // scale 1.0 for channels past N
    if (row_ok) {
      // weights: 2 chunks x 4 groups of 8 k -> E4M3 bytes, 16 per swizzled chunk
      const uint32_t* w = reinterpret_cast<const uint32_t*>(st + L::kOffI + h * (kMxBN * 24) + r * 24);
      const uint2 cb = *reinterpret_cast<const uint2*>(cbp + h * 8);
      const uint32_t e = ep[h];
      eh = e | (e << 8);
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const uint32_t wa = w[3 * c], wb = w[3 * c + 1], wc = w[3 * c + 2];
#pragma unroll
        for (int tp = 0; tp < 2; ++tp) {
          uint32_t o[4];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int t = 2 * tp + u;
            const uint32_t sel = lut3_selector(t < 2 ? wa : wb, wc, t);
            o[2 * u] = prmt(cb.x, cb.y, sel);
            o[2 * u + 1] = prmt(cb.x, cb.y, sel >> 16);
          }
          const uint32_t chunk = (uint32_t)(4 * h + 2 * c + tp);  // 16-k chunk of the 128-k block
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};"
                       :: "r"(arow + ((chunk ^ (uint32_t)(r & 7)) << 4)), "r"(o[0]), "r"(o[1]), "r"(o[2]),
                          "r"(o[3]) : "memory");
        }
      }
    } else {
#pragma unroll
      for (uint32_t cc = 0; cc < 4; ++cc)
        asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" :: "r"(arow + ((4u * h + cc) << 4)), "r"(0u) : "memory");
    }
    // the two k-steps of tile h take bytes 2h, 2h + 1 of the channel's scale word
    *reinterpret_cast<uint16_t*>(ab + kMxOffSA + atom_off + 2 * h) = (uint16_t)eh;
  }
  if (copy_scales) {
    // token scales of this block: bytes 4 (kb % 4) .. +3 of each token's 16-byte row
#pragma unroll
    for (int hh = 0; hh < BM / 128; ++hh) {
      const uint32_t sw = *reinterpret_cast<const uint32_t*>(st + L::kOffS + (hh * 128 + r) * 16 + (kb & 3) * 4);
      *reinterpret_cast<uint32_t*>(ab + kMxOffSB + hh * 512 + atom_off) = sw;
    }
  }
}

__global__ void __launch_bounds__(kMxThreads, 1)
    gemm_mx_lut3_kernel(const __grid_constant__ CUtensorMap tx, const __grid_constant__ CUtensorMap ts,
                        const __grid_constant__ CUtensorMap tc, const __grid_constant__ CUtensorMap te,
                        const __grid_constant__ CUtensorMap ty, const GemmMxArgs a) {
  extern __shared__ uint8_t dsmem[];
  __shared__ __align__(8) uint64_t full_bar[kMxStages], empty_bar[kMxStages];
  __shared__ __align__(8) uint64_t a_full[kMxABufs], a_empty[kMxABufs], d_full, d_empty;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int sk_ok_sh;  // the epilogue's wait for a parked part succeeded
  uint8_t* ring = dsmem + ((1024u - (smem_u32(dsmem) & 1023u)) & 1023u);
  uint8_t* abuf = ring + (size_t)kMxStages * kMxStageBytes;
  uint8_t* obuf = abuf + (size_t)kMxABufs * kMxABufBytes;  // two output tiles

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int i = 0; i < kMxStages; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], 1 + kMxConvWarps);
    }
    for (int i = 0; i < kMxABufs; ++i) {
      mbar_init(&a_full[i], kMxConvWarps);
      mbar_init(&a_empty[i], 1);
    }
    mbar_init(&d_full, 1);
    mbar_init(&d_empty, kMxEpWarps);
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
      tma_prefetch_desc(&ts);
      tma_prefetch_desc(&tc);
      tma_prefetch_desc(&te);
      int it = 0;
      bool ok = true;
      SkSched sch(a.sk.dp_tiles, a.sk.sk_items, a.k_blocks, (int)blockIdx.x, (int)gridDim.x);
      SkItem w;
      while (ok && sch.next(w)) {
        const int nt = w.tile / a.m_tiles, mt = w.tile - nt * a.m_tiles;  // token tiles inner: indices reused from L2
        const int rows = min(kMxBN, a.N - nt * kMxBN);
        for (int kb = w.kb0; kb < w.kb1; ++kb, ++it) {
          const int s = it % kMxStages;
          if (it >= kMxStages && !mbar_wait_sleep(&empty_bar[s], ((it / kMxStages) & 1) ^ 1)) { ok = false; break; }
          uint8_t* st = ring + (size_t)s * kMxStageBytes;
          const uint32_t tx_bytes =
              (uint32_t)(kMxBM * kMxBK + 2 * rows * 24 + 2 * 16 * a.cb_rows + kMxBM * 16);
          mbar_arrive_expect_tx(&full_bar[s], tx_bytes);
          tma_load_2d(st + kMxOffX, &tx, kb * kMxBK, mt * kMxBM, &full_bar[s]);
          for (int h = 0; h < 2; ++h) {
            const int kt = kb * 2 + h;
            bulk_load(st + kMxOffI + h * (kMxBN * 24), a.i_region + ((size_t)kt * a.N + nt * kMxBN) * 24,
                      (uint32_t)(rows * 24), &full_bar[s]);
          }
          tma_load_2d(st + kMxOffC, &tc, kb * 16, nt * (kMxBN / 8), &full_bar[s]);
          tma_load_2d(st + kMxOffE, &te, (kb * 2 / 16) * 16, nt * (kMxBN / 8), &full_bar[s]);
          tma_load_2d(st + kMxOffS, &ts, (kb / 4) * 16, mt * kMxBM, &full_bar[s]);
        }
      }
      // every copy this CTA issued lands before it may exit
      for (int v = max(0, it - kMxStages); v < it; ++v)
        if (!mbar_wait_sleep(&full_bar[v % kMxStages], (v / kMxStages) & 1)) break;
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ scale copies + MMA issuer
    if (lane == 0) {
      int it = 0, t_iter = 0;
      bool ok = true;
      SkSched sch(a.sk.dp_tiles, a.sk.sk_items, a.k_blocks, (int)blockIdx.x, (int)gridDim.x);
      SkItem w;
      for (; ok && sch.next(w); ++t_iter) {
        if (t_iter >= 1 && !mbar_wait_sleep(&d_empty, (t_iter - 1) & 1)) break;
        tc_fence_after();
        for (int kb = w.kb0; kb < w.kb1; ++kb, ++it) {
          const int s = it % kMxStages, b = it % kMxABufs;
          if (!mbar_wait_sleep(&full_bar[s], (it / kMxStages) & 1)) { ok = false; break; }
          if (!mbar_wait_sleep(&a_full[b], (it / kMxABufs) & 1)) { ok = false; break; }
          tc_fence_after();
          const uint32_t ab = smem_u32(abuf + (size_t)b * kMxABufBytes);
          const uint32_t xb = smem_u32(ring + (size_t)s * kMxStageBytes + kMxOffX);
          const uint32_t sf = tmem + kMxColSF + (uint32_t)b * 16;
          tmem_cp_sf(sf, sf_desc(ab + kMxOffSA));
          tmem_cp_sf(sf + 4, sf_desc(ab + kMxOffSB));
          tmem_cp_sf(sf + 8, sf_desc(ab + kMxOffSB + 512));
#pragma unroll
          for (uint32_t kk = 0; kk < 4; ++kk) {
            const uint64_t da = umma_desc_sw128(ab + kMxOffA) + (uint64_t)(kk * 2);
            const uint64_t db = umma_desc_sw128(xb) + (uint64_t)(kk * 2);
            umma_mx(tmem + kMxColD, da, db, umma_idesc_mx(kk), sf | (kk << 30), (sf + 4) | (kk << 30),
                    (kb > w.kb0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&empty_bar[s]);
          umma_commit(&a_empty[b]);
        }
        if (ok) umma_commit(&d_full);
      }
    }
  } else if (warp < 2 + kMxConvWarps) {
    // ------------------------------------------------------------------ converters
    const int cw = warp - 2;
    const int r = (cw & 3) * 32 + lane;  // channel within the tile / token within each half
    const int h = cw >> 2;               // this warp's LUT3 tile of each k-block
    int it = 0;
    bool ok = true;
    SkSched sch(a.sk.dp_tiles, a.sk.sk_items, a.k_blocks, (int)blockIdx.x, (int)gridDim.x);
    SkItem w;
    while (sch.next(w)) {
      const int nt = w.tile / a.m_tiles;
      const bool row_ok = nt * kMxBN + r < a.N;
      for (int kb = w.kb0; kb < w.kb1; ++kb, ++it) {
        const int s = it % kMxStages, b = it % kMxABufs;
        if (ok && !mbar_wait_sleep(&full_bar[s], (it / kMxStages) & 1)) ok = false;
        if (ok && it >= kMxABufs && !mbar_wait_sleep(&a_empty[b], ((it / kMxABufs) & 1) ^ 1)) ok = false;
        tc_fence_after();
        const uint8_t* st = ring + (size_t)s * kMxStageBytes;
        uint8_t* ab = abuf + (size_t)b * kMxABufBytes;
        if (ok)
          mx_convert_block<kMxBM>(st, ab, r, kb, row_ok, st + kMxOffC + (r >> 3) * 16,
                                  st + kMxOffE + (r >> 3) * 16 + ((kb * 2) & 15), h, h + 1, h == 0);
        fence_proxy_async();  // the operand and scale writes, to the tensor core's proxy
        __syncwarp();
        if (lane == 0 && ok) {
          mbar_arrive(&a_full[b]);
          mbar_arrive(&empty_bar[s]);
        }
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int r = 32 * q + lane;  // channel within the tile
    const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16);
    const bool issuer = warp == 2 + kMxConvWarps && lane == 0;
    if (issuer) tma_prefetch_desc(&ty);
    // every epilogue warp runs every chunk and both named barriers of it, also
    // after a timed-out wait (then it loads and stores nothing), so the
    // barrier sequence stays the same in all four warps
    int t_iter = 0, ob = 0;
    bool ok = true;
    SkSched sch(a.sk.dp_tiles, a.sk.sk_items, a.k_blocks, (int)blockIdx.x, (int)gridDim.x);
    SkItem w;
    for (; sch.next(w); ++t_iter) {
      const int nt = w.tile / a.m_tiles, mt = w.tile - nt * a.m_tiles;
      if (ok && !mbar_wait_sleep(&d_full, t_iter & 1)) ok = false;
      tc_fence_after();
      // cut tiles: an earlier part adds the sums parked in slot blockIdx.x + 1;
      // a later part parks its own in slot blockIdx.x (stream_k.cuh)
      const float* park_in = a.sk.partials + (size_t)(blockIdx.x + 1) * kSkTileFloats + r;
      float* park_out = a.sk.partials + (size_t)blockIdx.x * kSkTileFloats + r;
      if (w.part == 2) {
        if (issuer) sk_ok_sh = (ok && sk_wait_parked(a.sk)) ? 1 : 0;
        consumer_named_sync(1, kMxEpWarps * 32);
        ok = ok && sk_ok_sh != 0;
      }
      // two 32-token chunks per TMEM round trip, each staged and stored as before
#pragma unroll 1
      for (int jp = 0; jp < kMxBM / 64; ++jp) {
        uint32_t vv[2][32];
        if (ok) {
          tmem_ld32_nowait(lane_base + kMxColD + (uint32_t)(jp * 64), vv[0]);
          tmem_ld32_nowait(lane_base + kMxColD + (uint32_t)(jp * 64 + 32), vv[1]);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) vv[0][i] = vv[1][i] = 0u;
        }
        if (jp == kMxBM / 64 - 1) {  // the accumulator is in registers: the MMAs may start the next tile
          tc_fence_before();
          __syncwarp();
          if (lane == 0 && ok) mbar_arrive(&d_empty);
        }
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int j = 2 * jp + hh;
          uint32_t(&v)[32] = vv[hh];
          if (w.part == 2 && ok) {  // own sums + parked sums, in that order
#pragma unroll
            for (int i = 0; i < 32; ++i)
              v[i] = __float_as_uint(__uint_as_float(v[i]) + __ldcg(park_in + (j * 32 + i) * kMxBN));
          }
          if (w.part == 1 && ok) {  // a later part: park the FP32 sums (all 256 tokens; rows past M hold zeros)
#pragma unroll
            for (int i = 0; i < 32; ++i) __stcg(park_out + (j * 32 + i) * kMxBN, __uint_as_float(v[i]));
          }
          // the tile written two chunks ago has been read by its TMA store
          if (issuer) bulk_wait_read<1>();
          consumer_named_sync(2, kMxEpWarps * 32);
          uint8_t* ot = obuf + (size_t)ob * kMxOutBytes;
          if (w.part != 1) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const float f = __uint_as_float(v[i]);
              const uint16_t h =
                  a.y_bf16 ? __bfloat16_as_ushort(__float2bfloat16_rn(f)) : __half_as_ushort(__float2half_rn(f));
              *reinterpret_cast<uint16_t*>(ot + (i * kMxBN + r) * 2) = h;
            }
          }
          fence_proxy_async();  // the tile, to the TMA unit
          consumer_named_sync(2, kMxEpWarps * 32);
          const int m0 = mt * kMxBM + j * 32;
          if (issuer && ok && w.part != 1 && m0 < a.M) {
            tma_store_2d(&ty, ot, nt * kMxBN, m0);
            bulk_commit();
          }
          ob ^= 1;
        }
      }
      if (w.part == 1) {  // the parked sums are visible GPU-wide before the flag
        __threadfence();
        consumer_named_sync(1, kMxEpWarps * 32);
        if (issuer && ok && !a.sk.debug_hold) st_release_u32(a.sk.flags + blockIdx.x, 1u);
      }
    }
    if (issuer) bulk_wait<0>();  // every output store has landed
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem), "r"(512u) : "memory");
  }
}

}  // namespace lbq
