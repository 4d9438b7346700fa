// Stream-K schedule of the prefill GEMMs (128 channels x 256 tokens per tile,
// K in 128-k blocks), shared by the BF16-decode and the MXFP8 kernels.
//
// The CTAs (at most one per SM) take whole tiles strided over the grid; when
// the tiles leave a part-filled last wave, the last two waves' tiles are
// instead cut into (tile, k-block) items shared out evenly, so every SM ends
// at about the same time. Each CTA's share is at least one tile long, so a
// tile is cut at most once: its earlier part ends the share of CTA c - 1 and
// its later part starts the share of CTA c. The later part finishes first (it
// is its CTA's first item of the phase), parks its FP32 sums in workspace slot
// c and raises flag c; the earlier part waits for the flag (bounded), adds the
// parked sums to its own in a fixed order and writes the tile, so results do
// not depend on timing.
#pragma once

#include "common.cuh"
#include "tma.cuh"

namespace lbq {

// One work item: k-blocks [kb0, kb1) of a tile. part 0: the whole tile;
// 1: a later part (parks its sums in slot blockIdx.x); 2: an earlier part
// (adds the sums parked in slot blockIdx.x + 1, then writes the tile).
struct SkItem {
  int tile, kb0, kb1, part;
};

// The items of CTA `cta` of `grid` in order: the whole tiles cta, cta + grid,
// ... below dp_tiles, then its share [cta items / grid, (cta + 1) items / grid)
// of the sk_items (tile, k-block) items of the tiles after them. Every role of
// the CTA walks the same sequence (the host runs it too, for its checks).
struct SkSched {
  int tile, dp_tiles, step, nkb;
  long long pos, end;
  __host__ __device__ SkSched(int dp, long long sk_items, int k_blocks, int cta, int grid)
      : tile(cta), dp_tiles(dp), step(grid), nkb(k_blocks) {
    pos = sk_items * cta / grid;
    end = sk_items * (cta + 1) / grid;
  }
  __host__ __device__ bool next(SkItem& w) {
    if (tile < dp_tiles) {
      w.tile = tile;
      w.kb0 = 0;
      w.kb1 = nkb;
      w.part = 0;
      tile += step;
      return true;
    }
    if (pos >= end) return false;
    const long long t = pos / nkb;
    w.tile = dp_tiles + (int)t;
    w.kb0 = (int)(pos - t * nkb);
    w.kb1 = (int)(end - pos < (long long)(nkb - w.kb0) ? w.kb0 + (end - pos) : nkb);
    w.part = w.kb0 > 0 ? 1 : (w.kb1 < nkb ? 2 : 0);
    pos += w.kb1 - w.kb0;
    return true;
  }
};

// Kernel arguments of the schedule (all zero: whole tiles only, dp_tiles = tiles).
struct SkArgs {
  int dp_tiles;              // tiles taken whole, strided over the grid
  long long sk_items;        // (tile, k-block) items of the tiles after them (0: none)
  float* partials;           // [grid][256 tokens][128 channels] parked sums of cut tiles
  unsigned* flags;           // [grid] 1 while slot c holds a later part's sums; reset by the reader
  uint32_t flag_polls;       // bound on the wait for a parked part (about 1 us per poll)
  int debug_hold;            // test hook: later parts never raise their flag
};

constexpr int kSkTileFloats = 256 * 128;

// Banded tile order: bands of kSkBand token tiles; inside a band the channel
// tiles are outer and the band's token tiles inner. A wave of CTAs then shares
// one band's activations (8 x 256 tokens) instead of all of them, and each
// channel tile's codes are reused from L2 across the band. With at most
// kSkBand token tiles this is channel-tile-major order with token tiles inner.
// (Measured on B200, K=4096 N=14336 M=8192: INT4 +5%, LUT3 +9%; the LUT3 x
// MXFP8 GEMM, whose activations are half the bytes, did not gain and keeps the
// plain order.)
constexpr int kSkBand = 8;
__host__ __device__ __forceinline__ void sk_tile_coords(int tile, int n_tiles, int m_tiles, int& nt, int& mt) {
  const int band = tile / (kSkBand * n_tiles);
  const int mt0 = band * kSkBand;
  const int bw = m_tiles - mt0 < kSkBand ? m_tiles - mt0 : kSkBand;
  const int r = tile - band * kSkBand * n_tiles;
  nt = r / bw;
  mt = mt0 + (r - nt * bw);
}

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_u32(unsigned* p, unsigned v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" :: "l"(p), "r"(v) : "memory");
}

// One thread of an earlier part: wait (bounded) for the later part's flag in
// slot blockIdx.x + 1 and free the slot; false, with the device timeout flag
// raised, if it never came.
__device__ __forceinline__ bool sk_wait_parked(const SkArgs& s) {
  unsigned* f = s.flags + blockIdx.x + 1;
  for (uint32_t i = 0; i < s.flag_polls; ++i) {
    if (ld_acquire_u32(f) != 0u) {
      atomicExch(f, 0u);  // the slot is free for the next call
      return true;
    }
    __nanosleep(1000);
  }
  atomicOr(&g_device_error, kDevErrTimeout);
  return false;
}

}  // namespace lbq
