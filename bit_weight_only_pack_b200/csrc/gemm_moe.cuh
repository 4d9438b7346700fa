// Grouped MoE GEMM: LUT3 expert weights x MXFP8 activations, token rows
// gathered through sorted_token_ids, plus the alignment that produces them.
//
// The vLLM PR 62759 write-up's native kernel is a grouped GEMM over the routed
// experts: moe_align_block_size lists each expert's (token, choice) pairs
// contiguously, padded to the M block, and the kernel takes one expert per M
// block, gathers the token rows of A through the list (a padding entry's row
// is filled with zeros through the copy's source size), and writes zeros for
// the valid rows of a block whose expert is not on this rank.
//
// Here the product is the LUT3 x MXFP8 kernel of gemm_mx.cuh with a 128-token
// tile (the write-up's M block) and three changes:
//  * warps 10..13 gather: thread g owns row g of the block; per k-block it
//    copies its token's 128 code bytes as eight 16-byte cp.async into the
//    128-byte-swizzled operand tile (the layout a TMA copy would write) and the
//    token's 4 scale bytes, source size 0 for a padding entry, then makes the
//    stage's mbarrier track those copies (cp.async.mbarrier.arrive.noinc);
//  * warp 0 copies the block's expert weights with bulk copies from that
//    expert's image (the images sit at a fixed stride, so no per-expert tensor
//    map is needed): per tile the 16 channel groups' codebook and exponent rows
//    for the whole K range (contiguous rows of the image: two copies, into a
//    double-buffered per-tile area), per k-block the two LUT3 tiles' indices.
//    Every bulk copy is a separate request to the copy unit, so the rows go
//    once per tile rather than 16 bytes per k-block. For a non-local expert it
//    copies nothing and the converters write zero weights;
//  * eight converter warps, one 64-k LUT3 tile of the k-block each (warps
//    2..5 the first, 6..9 the second);
//  * the epilogue writes each finished row to Y[pair id] with 16-byte stores
//    (rows of padding entries are not written).
#pragma once

#include "gemm_mx.cuh"

namespace lbq {

constexpr int kMoeBM = 128;  // tokens (sorted rows) per tile = the alignment block
// Ring depth and converted weight tiles in flight. Measured at the write-up's
// layer shape: 5 stages with 2 tiles, or 4 with 3 (or 2), change the time by 5%
// at most, at 1, 16 and 256 tokens alike.
constexpr int kMoeStages = 3;
constexpr int kMoeABufs = 4;
constexpr int kMoeConvWarps = 8, kMoeGatherWarps = 4;
constexpr int kMoeWarpEp = 2 + kMoeConvWarps;             // first epilogue warp
constexpr int kMoeWarpGather = kMoeWarpEp + kMxEpWarps;   // first gather warp
constexpr int kMoeThreads = (kMoeWarpGather + kMoeGatherWarps) * 32;
constexpr int kMoeMaxK = 8192;
using MoeStage = MxStage<kMoeBM>;
// fixed part of the dynamic shared memory; two per-tile codebook / exponent
// areas of moe_meta_bytes(K) follow
constexpr int kMoeSmemBase = kMoeStages * MoeStage::kBytes + kMoeABufs * kMxABufBytes + 2 * kMxOutBytes + 1024;
// TMEM columns: two accumulators (the MMAs fill one while the epilogue drains
// the other), then 16 per A buffer of scale atoms
constexpr uint32_t kMoeColD = 0, kMoeColSF = 256;
constexpr uint32_t kMoeTmemCols = 512;
__host__ __device__ constexpr int moe_meta_bytes(int s_stride, int z_stride) { return 16 * (s_stride + z_stride); }
static_assert(kMoeSmemBase + 2 * moe_meta_bytes(kMoeMaxK / 8, kMoeMaxK / 64) <= 227 * 1024, "MoE GEMM shared memory");

struct GemmMoeArgs {
  const uint8_t* codes;         // [T][K] E4M3 activations
  const uint8_t* scales;        // [T][K/32] UE8M0
  const int32_t* sorted_ids;    // [max_blocks * 128] pair ids, P = padding
  const int32_t* expert_ids;    // [max_blocks] local expert of each block (< 0: not on this rank)
  const int32_t* total;         // device scalar: entries of sorted_ids in use
  const uint8_t* images;        // local expert e's LUT3 image at images + e * image_stride
  size_t image_stride;
  size_t off_i, off_c, off_e;   // region offsets inside an image
  int s_stride, z_stride;       // codebook / exponent row strides (bytes)
  void* Y;                      // [P][N]
  int top_k, P, N, K;
  int n_tiles, max_blocks, k_blocks, num_experts;
  int y_bf16;
};

__device__ __forceinline__ void cp_async4_zfill(uint32_t smem, const void* gmem, int src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" :: "r"(smem), "l"(gmem), "r"(src_bytes) : "memory");
}
// The mbarrier completes one of its expected arrivals once every cp.async this
// thread issued before has landed.
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" :: "r"(smem_u32(bar)) : "memory");
}

__global__ void __launch_bounds__(kMoeThreads, 1) gemm_moe_lut3_mx_kernel(const GemmMoeArgs a) {
  extern __shared__ uint8_t dsmem[];
  __shared__ __align__(8) uint64_t full_bar[kMoeStages], empty_bar[kMoeStages];
  __shared__ __align__(8) uint64_t a_full[kMoeABufs], a_empty[kMoeABufs], d_full[2], d_empty[2];
  __shared__ __align__(8) uint64_t meta_full[2], meta_empty[2];
  __shared__ uint32_t tmem_base_sh;
  uint8_t* ring = dsmem + ((1024u - (smem_u32(dsmem) & 1023u)) & 1023u);
  uint8_t* abuf = ring + (size_t)kMoeStages * MoeStage::kBytes;
  uint8_t* obuf = abuf + (size_t)kMoeABufs * kMxABufBytes;  // two output tiles
  uint8_t* meta = obuf + 2 * kMxOutBytes;                   // two per-tile areas: codebook rows, exponent rows
  const int meta_bytes = moe_meta_bytes(a.s_stride, a.z_stride);
  const int meta_e = 16 * a.s_stride;                        // exponent rows inside an area

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // every role derives the same tile sequence from the same total
  const int nblk = min(max(__ldg(a.total), 0) / kMoeBM, a.max_blocks);
  const int total_tiles = a.n_tiles * nblk;
  const int nkb = a.k_blocks;
  auto expert_of = [&](int mb) {
    const int e = __ldg(a.expert_ids + mb);
    return e < a.num_experts ? e : -1;  // ids past the images count as not local
  };

  if (tid == 0) {
    for (int i = 0; i < kMoeStages; ++i) {
      mbar_init(&full_bar[i], 1 + kMoeGatherWarps * 32);
      mbar_init(&empty_bar[i], 1 + kMoeConvWarps);
    }
    for (int i = 0; i < kMoeABufs; ++i) {
      mbar_init(&a_full[i], kMoeConvWarps);
      mbar_init(&a_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&meta_full[i], 1);
      mbar_init(&meta_empty[i], kMoeConvWarps);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&d_full[i], 1);
      mbar_init(&d_empty[i], kMxEpWarps);
    }
    fence_barrier_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 :: "r"(smem_u32(&tmem_base_sh)), "r"(kMoeTmemCols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  if (warp == 0) {
    // ------------------------------------------------------------------ expert weights
    if (lane == 0) {
      int it = 0, t_iter = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x, ++t_iter) {
        const int nt = tile / nblk, mb = tile - nt * nblk;  // blocks inner: one expert's blocks are adjacent
        const int e = expert_of(mb);
        const int rows = min(kMxBN, a.N - nt * kMxBN);  // a multiple of 8
        const int groups = rows >> 3;
        const uint8_t* img = a.images + (size_t)(e < 0 ? 0 : e) * a.image_stride;
        // the tile's codebook and exponent rows (16 consecutive rows of each region)
        const int mi = t_iter & 1;
        if (t_iter >= 2 && !mbar_wait_sleep(&meta_empty[mi], ((t_iter >> 1) & 1) ^ 1)) { ok = false; break; }
        uint8_t* mt = meta + (size_t)mi * meta_bytes;
        const size_t g0 = (size_t)nt * (kMxBN / 8);
        mbar_arrive_expect_tx(&meta_full[mi], e < 0 ? 0u : (uint32_t)(groups * (a.s_stride + a.z_stride)));
        if (e >= 0) {
          bulk_load(mt, img + a.off_c + g0 * a.s_stride, (uint32_t)(groups * a.s_stride), &meta_full[mi]);
          bulk_load(mt + meta_e, img + a.off_e + g0 * a.z_stride, (uint32_t)(groups * a.z_stride), &meta_full[mi]);
        }
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = it % kMoeStages;
          if (it >= kMoeStages && !mbar_wait_sleep(&empty_bar[s], ((it / kMoeStages) & 1) ^ 1)) { ok = false; break; }
          uint8_t* st = ring + (size_t)s * MoeStage::kBytes;
          mbar_arrive_expect_tx(&full_bar[s], e < 0 ? 0u : (uint32_t)(2 * rows * 24));
          if (e >= 0)
            for (int h = 0; h < 2; ++h)
              bulk_load(st + MoeStage::kOffI + h * (kMxBN * 24),
                        img + a.off_i + ((size_t)(kb * 2 + h) * a.N + nt * kMxBN) * 24, (uint32_t)(rows * 24),
                        &full_bar[s]);
        }
      }
      // every copy this CTA issued lands before it may exit
      for (int v = max(0, it - kMoeStages); v < it; ++v)
        if (!mbar_wait_sleep(&full_bar[v % kMoeStages], (v / kMoeStages) & 1)) break;
      for (int v = max(0, t_iter - 2); v < t_iter; ++v)
        if (!mbar_wait_sleep(&meta_full[v & 1], (v >> 1) & 1)) break;
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ scale copies + MMA issuer
    if (lane == 0) {
      int it = 0, t_iter = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x, ++t_iter) {
        const int ai = t_iter & 1;  // accumulator of this tile
        if (t_iter >= 2 && !mbar_wait_sleep(&d_empty[ai], ((t_iter >> 1) & 1) ^ 1)) break;
        tc_fence_after();
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = it % kMoeStages, b = it % kMoeABufs;
          if (!mbar_wait_sleep(&full_bar[s], (it / kMoeStages) & 1)) { ok = false; break; }
          if (!mbar_wait_sleep(&a_full[b], (it / kMoeABufs) & 1)) { ok = false; break; }
          fence_proxy_async();  // the gathered rows (cp.async writes), to the tensor core's proxy
          tc_fence_after();
          const uint32_t ab = smem_u32(abuf + (size_t)b * kMxABufBytes);
          const uint32_t xb = smem_u32(ring + (size_t)s * MoeStage::kBytes + MoeStage::kOffX);
          const uint32_t sf = tmem + kMoeColSF + (uint32_t)b * 16;
          tmem_cp_sf(sf, sf_desc(ab + kMxOffSA));
          tmem_cp_sf(sf + 4, sf_desc(ab + kMxOffSB));
#pragma unroll
          for (uint32_t kk = 0; kk < 4; ++kk) {
            const uint64_t da = umma_desc_sw128(ab + kMxOffA) + (uint64_t)(kk * 2);
            const uint64_t db = umma_desc_sw128(xb) + (uint64_t)(kk * 2);
            umma_mx(tmem + kMoeColD + (uint32_t)ai * kMoeBM, da, db, umma_idesc_mx(kk, kMoeBM), sf | (kk << 30),
                    (sf + 4) | (kk << 30), (kb > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&empty_bar[s]);
          umma_commit(&a_empty[b]);
        }
        if (ok) umma_commit(&d_full[ai]);
      }
    }
  } else if (warp < kMoeWarpEp) {
    // ------------------------------------------------------------------ converters
    const int cw = warp - 2;
    const int r = (cw & 3) * 32 + lane;  // channel within the tile / token row of the block
    const int h = cw >> 2;               // this warp's LUT3 tile of each k-block
    int it = 0, t_iter = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x, ++t_iter) {
      const int nt = tile / nblk, mb = tile - nt * nblk;
      const bool row_ok = nt * kMxBN + r < a.N && expert_of(mb) >= 0;
      const int mi = t_iter & 1;
      if (ok && !mbar_wait_sleep(&meta_full[mi], (t_iter >> 1) & 1)) ok = false;
      const uint8_t* mt = meta + (size_t)mi * meta_bytes;
      for (int kb = 0; kb < nkb; ++kb, ++it) {
        const int s = it % kMoeStages, b = it % kMoeABufs;
        if (ok && !mbar_wait_sleep(&full_bar[s], (it / kMoeStages) & 1)) ok = false;
        if (ok && it >= kMoeABufs && !mbar_wait_sleep(&a_empty[b], ((it / kMoeABufs) & 1) ^ 1)) ok = false;
        tc_fence_after();
        const uint8_t* st = ring + (size_t)s * MoeStage::kBytes;
        uint8_t* ab = abuf + (size_t)b * kMxABufBytes;
        if (ok)
          mx_convert_block<kMoeBM>(st, ab, r, kb, row_ok, mt + (r >> 3) * a.s_stride + kb * 16,
                                   mt + meta_e + (r >> 3) * a.z_stride + kb * 2, h, h + 1, h == 0);
        fence_proxy_async();  // the operand and scale writes, to the tensor core's proxy
        __syncwarp();
        if (lane == 0 && ok) {
          mbar_arrive(&a_full[b]);
          mbar_arrive(&empty_bar[s]);
        }
      }
      __syncwarp();
      if (lane == 0 && ok) mbar_arrive(&meta_empty[mi]);
    }
  } else if (warp < kMoeWarpGather) {
    // ------------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int r = 32 * q + lane;  // channel within the tile
    const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16);
    const int ew = warp - kMoeWarpEp;  // 0..3: rows 8 ew .. 8 ew + 7 of each 32-row chunk
    // every epilogue warp runs every chunk and its named barrier, also after a
    // timed-out wait (then it loads and stores nothing)
    int t_iter = 0, ob = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x, ++t_iter) {
      const int nt = tile / nblk, mb = tile - nt * nblk;
      const int rows = min(kMxBN, a.N - nt * kMxBN);
      const int ai = t_iter & 1;
      if (ok && !mbar_wait_sleep(&d_full[ai], (t_iter >> 1) & 1)) ok = false;
      tc_fence_after();
#pragma unroll 1
      for (int j = 0; j < kMoeBM / 32; ++j) {
        // the pair ids of this warp's rows of the chunk, requested before the accumulator is read
        int sid[4];
#pragma unroll
        for (int pass = 0; pass < 4; ++pass)
          sid[pass] = __ldg(a.sorted_ids + (size_t)mb * kMoeBM + j * 32 + 8 * ew + 2 * pass + (lane >> 4));
        uint32_t v[32];
        if (ok) {
          tmem_ld32(lane_base + kMoeColD + (uint32_t)ai * kMoeBM + (uint32_t)(j * 32), v);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = 0u;
        }
        if (j == kMoeBM / 32 - 1) {  // the accumulator is in registers: the MMAs may start the next tile
          tc_fence_before();
          __syncwarp();
          if (lane == 0 && ok) mbar_arrive(&d_empty[ai]);
        }
        uint8_t* ot = obuf + (size_t)ob * kMxOutBytes;  // [32 rows][128 channels]
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float f = __uint_as_float(v[i]);
          const uint16_t h = a.y_bf16 ? __bfloat16_as_ushort(__float2bfloat16_rn(f)) : __half_as_ushort(__float2half_rn(f));
          *reinterpret_cast<uint16_t*>(ot + (i * kMxBN + r) * 2) = h;
        }
        consumer_named_sync(2, kMxEpWarps * 32);
        // rows 8 ew .. 8 ew + 7 of the chunk: two rows per pass, 16 lanes x 16 B each
#pragma unroll
        for (int pass = 0; pass < 4; ++pass) {
          const int i = 8 * ew + 2 * pass + (lane >> 4), cl = lane & 15;
          if (ok && sid[pass] >= 0 && sid[pass] < a.P && cl * 8 < rows) {
            const uint4 val = *reinterpret_cast<const uint4*>(ot + i * (kMxBN * 2) + cl * 16);
            *reinterpret_cast<uint4*>(static_cast<uint8_t*>(a.Y) + ((size_t)sid[pass] * a.N + nt * kMxBN) * 2 +
                                      cl * 16) = val;
          }
        }
        ob ^= 1;
      }
    }
  } else {
    // ------------------------------------------------------------------ token-row gather
    const int g = tid - kMoeWarpGather * 32;  // row of the block
    int it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
      const int nt = tile / nblk, mb = tile - nt * nblk;
      (void)nt;
      const int sid = __ldg(a.sorted_ids + (size_t)mb * kMoeBM + g);
      const bool valid = sid >= 0 && sid < a.P;
      const int token = valid ? sid / a.top_k : 0;
      const uint8_t* xsrc = a.codes + (size_t)token * a.K;
      const uint8_t* ssrc = a.scales + (size_t)token * (a.K / 32);
      const int nb = valid ? 16 : 0;
      for (int kb = 0; kb < nkb; ++kb, ++it) {
        const int s = it % kMoeStages;
        if (lane == 0 && it >= kMoeStages && !mbar_wait_sleep(&empty_bar[s], ((it / kMoeStages) & 1) ^ 1)) ok = false;
        ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
        if (!ok) break;
        const uint32_t st = smem_u32(ring + (size_t)s * MoeStage::kBytes);
        const uint32_t dst = st + MoeStage::kOffX + (uint32_t)g * 128u;
#pragma unroll
        for (int c = 0; c < 8; ++c)
          cp_async16_s(dst + (((uint32_t)c ^ (uint32_t)(g & 7)) << 4), xsrc + (size_t)kb * kMxBK + c * 16, nb);
        cp_async4_zfill(st + MoeStage::kOffS + (uint32_t)g * 16u + (uint32_t)(kb & 3) * 4u, ssrc + (size_t)kb * 4,
                        valid ? 4 : 0);
        cp_async_arrive_noinc(&full_bar[s]);
      }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");  // this thread's copies land before it may exit
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem), "r"(kMoeTmemCols) : "memory");
  }
}

// moe_align_block_size on one CTA: per-expert counts, runs padded to `block`
// in ascending expert order, the padding id P everywhere else, and each pair's
// id scattered into its expert's run (pairs of one expert in arrival order of
// the atomics: any order is as valid, each output row depends on its own pair).
// Shared memory: counts [E], run starts [E + 1], cursors [E].
__global__ void __launch_bounds__(1024) moe_align_kernel(const int32_t* __restrict__ topk_ids, int P, int E,
                                                         int block, const int32_t* __restrict__ expert_map,
                                                         int32_t* __restrict__ sorted_ids,
                                                         int32_t* __restrict__ expert_ids, int32_t* __restrict__ total,
                                                         int max_padded) {
  extern __shared__ int moe_sm[];
  int* cnt = moe_sm;
  int* start = cnt + E;
  int* cur = start + E + 1;
  const int tid = threadIdx.x, nt = blockDim.x;
  for (int e = tid; e < E; e += nt) { cnt[e] = 0; cur[e] = 0; }
  __syncthreads();
  for (int p = tid; p < P; p += nt) {
    const int e = topk_ids[p];
    if (e >= 0 && e < E) atomicAdd(&cnt[e], 1);
  }
  __syncthreads();
  {
    // start[e] = padded counts of the experts before e: each thread sums a
    // contiguous range of experts, then an exclusive scan over the threads
    // (warp shuffles, then one warp over the warp totals)
    __shared__ int warp_sum[32];
    const int per = (E + nt - 1) / nt, e0 = min(E, tid * per), e1 = min(E, e0 + per);
    int mine = 0;
    for (int e = e0; e < e1; ++e) mine += (cnt[e] + block - 1) / block * block;
    const int lane = tid & 31, warp = tid >> 5;
    int incl = mine;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int v = __shfl_up_sync(0xFFFFFFFFu, incl, d);
      if (lane >= d) incl += v;
    }
    if (lane == 31) warp_sum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const int nwarps = nt >> 5;
      int w = lane < nwarps ? warp_sum[lane] : 0;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int v = __shfl_up_sync(0xFFFFFFFFu, w, d);
        if (lane >= d) w += v;
      }
      if (lane < nwarps) warp_sum[lane] = w;  // inclusive totals of warps 0..lane
    }
    __syncthreads();
    int o = incl - mine + (warp > 0 ? warp_sum[warp - 1] : 0);
    for (int e = e0; e < e1; ++e) {
      start[e] = o;
      o += (cnt[e] + block - 1) / block * block;
    }
    if (tid == nt - 1) {
      start[E] = o;
      *total = o;
    }
  }
  for (int i = tid; i < max_padded; i += nt) sorted_ids[i] = P;
  for (int b = tid; b < max_padded / block; b += nt) expert_ids[b] = -1;
  __syncthreads();
  for (int e = tid; e < E; e += nt) {
    const int le = expert_map ? expert_map[e] : e;
    for (int b = start[e] / block; b < start[e + 1] / block; ++b) expert_ids[b] = le;
  }
  for (int p = tid; p < P; p += nt) {
    const int e = topk_ids[p];
    if (e >= 0 && e < E) sorted_ids[start[e] + atomicAdd(&cur[e], 1)] = p;
  }
}

}  // namespace lbq
