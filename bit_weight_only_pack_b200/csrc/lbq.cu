// The C ABI of the lbq library (declared in include/lbq.h): argument checks,
// shape-based kernel selection and launches. One translation unit includes
// every kernel header, so the library builds as a single object.
//
// Kernel selection by shape mirrors BaseRT's practice of choosing kernels
// from the layer shape ("BaseRT", kernel-selection section): M = 1 goes to
// the CUDA-core GEMV, 2 <= M <= 16 to the tensor-core skinny kernel, larger M
// to the tcgen05 prefill GEMM; split-K is chosen when the row tiles alone
// cannot fill the SMs.
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <algorithm>
#include <map>
#include <mutex>
#include <string>
#include <tuple>

#include "common.cuh"
#include "pack_int4.cuh"
#include "lut3.cuh"
#include "tma.cuh"
#include "gemv_m1.cuh"
#include "skinny.cuh"
#include "lut3_gemv.cuh"
#include "gemm_tc.cuh"
#include "tc_gemv.cuh"
#include "gemv_direct.cuh"
#include "gemv_tmma.cuh"
#include "mxfp8.cuh"
#include "gemm_ts.cuh"
#include "gemm_mx.cuh"
#include "lut3_direct.cuh"
#include "lut3_tmma.cuh"
#include "lut3_tmma_batch.cuh"
#include "affine.cuh"
#include "w4a8.cuh"
#include "gemm_moe.cuh"

namespace lbq {

static thread_local std::string g_last_error;
static std::atomic<uint64_t> g_launches{0};

static lbq_status fail(lbq_status st, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
static lbq_status fail(lbq_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

static lbq_status cuda_check(cudaError_t e, const char* what) {
  if (e != cudaSuccess) return fail(LBQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return LBQ_OK;
}

static lbq_status launch_check(const char* what) {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return cuda_check(cudaGetLastError(), what);
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static int num_sms() {
  static int sms = 0;
  static std::once_flag once;
  std::call_once(once, [] {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (sms <= 0) sms = 148;
  });
  return sms;
}

static int log2_exact(int v) {
  int l = 0;
  while ((1 << l) < v) ++l;
  return (1 << l) == v ? l : -1;
}

static lbq_status check_int4_shape(int K, int N, int group, int mode) {
  if (mode != LBQ_MODE_SYM && mode != LBQ_MODE_ASYM)
    return fail(LBQ_ERR_UNSUPPORTED, "mode %d is not an INT4 mode", mode);
  if (group != 32 && group != 64 && group != 128)
    return fail(LBQ_ERR_UNSUPPORTED, "group %d not in {32, 64, 128}", group);
  if (K <= 0 || N <= 0) return fail(LBQ_ERR_INVALID_ARG, "K=%d N=%d must be positive", K, N);
  if (K % group) return fail(LBQ_ERR_INVALID_ARG, "K=%d is not a multiple of group %d", K, group);
  return LBQ_OK;
}

static lbq_status check_lut3_shape(int K, int N) {
  if (K <= 0 || N <= 0) return fail(LBQ_ERR_INVALID_ARG, "K=%d N=%d must be positive", K, N);
  if (K % 64 || N % 8) return fail(LBQ_ERR_INVALID_ARG, "LUT3 needs K %% 64 == 0 and N %% 8 == 0 (K=%d N=%d)", K, N);
  return LBQ_OK;
}

__global__ void write_header_kernel(ImageHeader h, ImageHeader* dst) {
  if (threadIdx.x == 0) *dst = h;
}

// Reads the image header (a synchronous 64-byte copy; used by the debug calls only).
static lbq_status read_header(const void* image, ImageHeader* h) {
  return cuda_check(cudaMemcpy(h, image, sizeof(ImageHeader), cudaMemcpyDeviceToHost), "reading the image header");
}

static lbq_status check_header(const ImageHeader& h, int K, int N, int group, int mode) {
  const uint32_t magic = mode == LBQ_MODE_LUT3 ? kMagicLut3 : kMagicInt4;
  if (h.magic != magic || h.version != kImageVersion)
    return fail(LBQ_ERR_INVALID_ARG, "not an lbq image of this version (magic 0x%08x version %u)", h.magic, h.version);
  if (h.K != K || h.N != N || h.mode != mode || (mode != LBQ_MODE_LUT3 && h.group != group))
    return fail(LBQ_ERR_INVALID_ARG, "image holds K=%d N=%d group=%d mode=%d, call says K=%d N=%d group=%d mode=%d",
                h.K, h.N, h.group, h.mode, K, N, group, mode);
  return LBQ_OK;
}

// Resident blocks per SM for (kernel, block, dynamic smem). The first time a
// kernel is seen its dynamic shared-memory limit is raised to the device's
// opt-in maximum, once, so later calls with any smem size launch.
static int occupancy_for(const void* fn, int block, int smem) {
  static std::mutex mu;
  static std::map<const void*, bool> raised;
  static std::map<std::pair<const void*, long long>, int> cache;
  std::lock_guard<std::mutex> lk(mu);
  if (!raised[fn]) {
    int dev = 0, optin = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    cudaFuncAttributes fa{};
    cudaFuncGetAttributes(&fa, fn);
    cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, optin - (int)fa.sharedSizeBytes);
    raised[fn] = true;
  }
  auto key = std::make_pair(fn, (long long)smem * 4096 + block);
  auto itc = cache.find(key);
  if (itc != cache.end()) return itc->second;
  int occ = 0;
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, fn, block, smem);
  occ = std::max(occ, 1);
  cache[key] = occ;
  return occ;
}

// ----------------------------------------------------------------------------
// M = 1 GEMV planning
// ----------------------------------------------------------------------------

struct M1Plan {
  int splits, cps, rpt, tpr, phases;
  int nqbox, sbox_h, nsbox, zbox_h, nzbox, off_s, off_z, slot_bytes, tx_bytes, stages;
  int row_tiles, total_tiles, block, smem;
};

static int g_force_splits = 0;  // test hook: force a split count (0 = shape-based choice)
static int g_pdl = 0;           // launch GEMVs with programmatic dependent launch
static int g_force_skinny = 0;  // test hook: route M = 1 to the tensor-core skinny kernel
// test hook: GEMV kernel for M <= 16. 0 = the library's choice, 1 = the
// TMA-pipelined CUDA-core M = 1 kernel, 2 = the warp-MMA skinny kernel, 3 = the
// tcgen05 kernel, 4 = the direct-load CUDA-core M = 1 kernel.
static int g_gemv_path = 0;
enum { kPathAuto = 0, kPathM1 = 1, kPathMma = 2, kPathTc = 3, kPathDirect = 4, kPathTmma = 5 };

constexpr int kM1RingBudget = 100 * 1024;
constexpr int kM1MaxChunksPerSplit = 128;  // K-slices of at most 4096 k keep a ring slot near 20 KB

static void m1_slot_geometry(M1Plan& p, int group, bool asym) {
  const int gps = p.cps * 32 / group;  // groups per K-slice
  p.nqbox = (p.cps * 16 + 255) / 256;
  p.sbox_h = std::min(256, gps);
  p.nsbox = (gps + p.sbox_h - 1) / p.sbox_h;
  p.zbox_h = p.sbox_h;
  p.nzbox = asym ? p.nsbox : 0;
  const int qbytes = p.nqbox * kM1SlotRows * 256;
  p.off_s = (int)align_up(qbytes, 128);
  const int sbytes = p.nsbox * p.sbox_h * 16;
  p.off_z = (int)align_up(p.off_s + sbytes, 128);
  const int zbytes = p.nzbox * p.zbox_h * 16;
  p.slot_bytes = (int)align_up(p.off_z + zbytes, 1024);
  p.tx_bytes = qbytes + sbytes + zbytes;
}

// Shape-based plan: K-slices (split-K), threads per row, ring depth.
static M1Plan plan_m1(int K, int N, int group, bool asym, int force_splits) {
  const int chunks = K / 32;
  const int target = 2 * num_sms();
  M1Plan best{};
  const int max_splits = std::max(1, chunks / 64);
  for (int splits = 1; splits <= max_splits; ++splits) {
    if (force_splits > 0 && splits != std::min(force_splits, max_splits)) continue;
    int cps = chunks;
    if (splits > 1) cps = ((chunks + splits - 1) / splits + 63) / 64 * 64;  // slices start on 2048-k boundaries
    if ((chunks + cps - 1) / cps != splits) continue;
    if (cps > kM1MaxChunksPerSplit && splits < max_splits && force_splits == 0) continue;
    M1Plan p{};
    p.splits = splits;
    p.cps = cps;
    p.tpr = (cps + 31) / 32 * 32;
    if (p.tpr > kM1MaxConsumerThreads) continue;
    int phases = std::min(8, std::max(1, kM1MaxConsumerThreads / p.tpr));
    while (phases > 1 && (long long)((N + 8 * phases - 1) / (8 * phases)) * splits < target) phases /= 2;
    p.phases = phases;
    p.rpt = kM1SlotRows / phases;
    m1_slot_geometry(p, group, asym);
    p.stages = std::max(2, std::min(kM1MaxStages, kM1RingBudget / p.slot_bytes));
    p.row_tiles = (N + 8 * phases - 1) / (8 * phases);
    p.total_tiles = p.row_tiles * splits;
    p.block = p.tpr * phases + 32;
    p.smem = p.stages * p.slot_bytes + 1024;
    best = p;
    if (force_splits > 0 || (long long)p.total_tiles >= target) break;
  }
  return best;
}

static size_t m1_workspace_bytes(const M1Plan& p, int N) {
  if (p.splits <= 1) return 0;
  return align_up((size_t)p.splits * N * sizeof(float), 256) + align_up((size_t)p.row_tiles * sizeof(unsigned), 256);
}

typedef void (*M1Kernel)(CUtensorMap, CUtensorMap, CUtensorMap, GemvM1Args);

template <bool B, bool A>
static M1Kernel m1_kernel_for(int rpt) {
  if (rpt == 8) return gemv_m1_kernel<B, A, 8>;
  if (rpt == 4) return gemv_m1_kernel<B, A, 4>;
  if (rpt == 2) return gemv_m1_kernel<B, A, 2>;
  return gemv_m1_kernel<B, A, 1>;
}

static M1Kernel m1_kernel(bool bf16, bool asym, int rpt) {
  if (bf16) return asym ? m1_kernel_for<true, true>(rpt) : m1_kernel_for<true, false>(rpt);
  return asym ? m1_kernel_for<false, true>(rpt) : m1_kernel_for<false, false>(rpt);
}

static lbq_status launch_kernel_ex(const void* fn, dim3 grid, dim3 block, int smem, cudaStream_t st, bool pdl,
                                   void** args, const char* what) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  if (pdl) {
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  g_launches.fetch_add(1, std::memory_order_relaxed);
  const cudaError_t e = cudaLaunchKernelExC(&cfg, fn, args);
  if (e != cudaSuccess)
    return fail(LBQ_ERR_CUDA, "%s (grid %u, block %u, smem %d, pdl %d): %s", what, grid.x, block.x, smem, (int)pdl,
                cudaGetErrorString(e));
  return LBQ_OK;
}

static lbq_status run_m1(const uint16_t* X, bool xbf16, const void* image, const Layout& L, void* Y, bool ybf16,
                         void* ws, size_t ws_bytes, cudaStream_t st) {
  const bool asym = L.mode == LBQ_MODE_ASYM;
  const M1Plan p = plan_m1(L.K, L.N, L.group, asym, g_force_splits);
  if (p.block == 0) return fail(LBQ_ERR_UNSUPPORTED, "no GEMV plan for K=%d", L.K);
  const size_t need = m1_workspace_bytes(p, L.N);
  if (need > 0 && (ws == nullptr || ws_bytes < need))
    return fail(LBQ_ERR_INVALID_ARG, "workspace of %zu bytes is too small (need %zu)", ws_bytes, need);
  const uint8_t* img = static_cast<const uint8_t*>(image);
  const int G = L.K / L.group;
  const uint64_t meta_rows = (uint64_t)((L.N + 127) / 128) * G;  // (channel tile, group) rows of 128 entries
  CUtensorMap tq, ts, tz;
  if (!make_tmap_2d(&tq, img + L.off0, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)L.K / 2, (uint64_t)L.N,
                    (uint64_t)L.K / 2, 256, kM1SlotRows, CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_tmap_2d(&ts, img + L.off1, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, 128, meta_rows, 256, 8, (uint32_t)p.sbox_h,
                    CU_TENSOR_MAP_SWIZZLE_NONE))
    return fail(LBQ_ERR_CUDA, "cuTensorMapEncodeTiled failed for the GEMV tiles");
  tz = ts;
  if (asym && !make_tmap_2d(&tz, img + L.off2, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, 128, meta_rows, 128, 16,
                            (uint32_t)p.zbox_h, CU_TENSOR_MAP_SWIZZLE_NONE))
    return fail(LBQ_ERR_CUDA, "cuTensorMapEncodeTiled failed for the zero points");
  GemvM1Args a{};
  a.X = X;
  a.Y = Y;
  a.partials = need ? static_cast<float*>(ws) : nullptr;
  a.counters = need ? reinterpret_cast<unsigned*>(static_cast<uint8_t*>(ws) + align_up((size_t)p.splits * L.N * sizeof(float), 256)) : nullptr;
  a.K = L.K; a.N = L.N; a.G = G; a.gshift = log2_exact(L.group / 32);
  a.cps = p.cps; a.splits = p.splits; a.tpr = p.tpr; a.phases = p.phases;
  a.stages = p.stages; a.nqbox = p.nqbox; a.sbox_h = p.sbox_h; a.nsbox = p.nsbox; a.zbox_h = p.zbox_h;
  a.nzbox = p.nzbox; a.off_s = p.off_s; a.off_z = p.off_z; a.slot_bytes = p.slot_bytes; a.tx_bytes = p.tx_bytes;
  a.row_tiles = p.row_tiles; a.total_tiles = p.total_tiles; a.y_bf16 = ybf16 ? 1 : 0;
  const M1Kernel fn = m1_kernel(xbf16, asym, p.rpt);
  const int occ = occupancy_for((const void*)fn, p.block, p.smem);
  const int grid = std::min(p.total_tiles, num_sms() * occ);
  void* args[] = {&tq, &ts, &tz, &a};
  return launch_kernel_ex((const void*)fn, dim3(grid), dim3(p.block), p.smem, st, g_pdl != 0, args, "gemv_m1 launch");
}

// ----------------------------------------------------------------------------
// 2 <= M <= 16: tensor-core skinny kernel
// ----------------------------------------------------------------------------

struct SkPlan {
  int nt, gc, row_tiles, stages_per_tile, max_slots, grid, smem, slot;
  long long units;
};

typedef void (*SkKernel)(CUtensorMap, CUtensorMap, SkinnyArgs);

template <bool B, bool A, int NT, bool KF>
static SkKernel sk_for_gc(int gc) {
  if (gc == 1) return skinny_kernel<B, A, NT, 1, KF>;
  if (gc == 2) return skinny_kernel<B, A, NT, 2, KF>;
  return skinny_kernel<B, A, NT, 4, KF>;
}

template <bool B, bool A>
static SkKernel sk_for_nt(int nt, int gc, bool kfull) {
  if (nt == 1) return kfull ? sk_for_gc<B, A, 1, true>(gc) : sk_for_gc<B, A, 1, false>(gc);
  return kfull ? sk_for_gc<B, A, 2, true>(gc) : sk_for_gc<B, A, 2, false>(gc);
}

static SkKernel sk_kernel(bool bf16, bool asym, int nt, int gc, bool kfull) {
  if (bf16) return asym ? sk_for_nt<true, true>(nt, gc, kfull) : sk_for_nt<true, false>(nt, gc, kfull);
  return asym ? sk_for_nt<false, true>(nt, gc, kfull) : sk_for_nt<false, false>(nt, gc, kfull);
}

// Stream-K plan: units = row tiles x 256-k stages, split evenly over one wave
// of resident CTAs.
static SkPlan plan_skinny(int K, int N, int M, int group, bool asym, bool xbf16) {
  SkPlan p{};
  p.nt = M <= 8 ? 1 : 2;
  p.gc = group / 32;
  p.row_tiles = (N + kSkRows - 1) / kSkRows;
  p.stages_per_tile = (K + 255) / 256;
  p.units = (long long)p.row_tiles * p.stages_per_tile;
  p.slot = kSkWBytes + 4 * p.nt * 1024 + kSkSBytes + (asym ? kSkZBytes : 0);  // a multiple of 1024
  p.smem = kSkStages * p.slot + 1024;
  const SkKernel fn = sk_kernel(xbf16, asym, p.nt, p.gc, K % 256 == 0);
  const int occ = occupancy_for((const void*)fn, kSkThreads, p.smem);
  p.grid = (int)std::min<long long>(p.units, (long long)num_sms() * occ);
  const long long per = std::max<long long>(1, p.units / p.grid);
  p.max_slots = (int)((p.stages_per_tile + per - 1) / per + 1);
  return p;
}

static size_t skinny_workspace_bytes(const SkPlan& p, int M) {
  return align_up((size_t)p.row_tiles * p.max_slots * M * kSkRows * sizeof(float), 256) +
         align_up((size_t)p.row_tiles * sizeof(unsigned), 256);
}

static lbq_status run_skinny(const void* X, bool xbf16, int M, const void* image, const Layout& L, void* Y,
                             bool ybf16, void* ws, size_t ws_bytes, cudaStream_t st) {
  const bool asym = L.mode == LBQ_MODE_ASYM;
  const SkPlan p = plan_skinny(L.K, L.N, M, L.group, asym, xbf16);
  const size_t need = skinny_workspace_bytes(p, M);
  if (ws == nullptr || ws_bytes < need)
    return fail(LBQ_ERR_INVALID_ARG, "workspace of %zu bytes is too small (need %zu)", ws_bytes, need);
  const uint8_t* img = static_cast<const uint8_t*>(image);
  CUtensorMap tw, tx;
  const bool ok = make_tmap_2d(&tw, img + L.off0, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)L.K / 2, (uint64_t)L.N,
                               (uint64_t)L.K / 2, 128, kSkRows, CU_TENSOR_MAP_SWIZZLE_128B) &&
                  // X [M][K] as (32-k chunk, token, chunk index); box: 8 chunks of all M tokens
                  make_tmap_3d(&tx, X, CU_TENSOR_MAP_DATA_TYPE_UINT16, 32, (uint64_t)M, (uint64_t)L.K / 32,
                               (uint64_t)L.K * 2, 64, 32, (uint32_t)M, 8, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (!ok) return fail(LBQ_ERR_CUDA, "cuTensorMapEncodeTiled failed for the skinny kernel");
  SkinnyArgs a{};
  a.Y = Y;
  a.partials = static_cast<float*>(ws);
  a.counters = reinterpret_cast<unsigned*>(static_cast<uint8_t*>(ws) +
                                           align_up((size_t)p.row_tiles * p.max_slots * M * kSkRows * sizeof(float), 256));
  a.s_region = img + L.off1;
  a.z_region = asym ? img + L.off2 : nullptr;
  a.K = L.K; a.N = L.N; a.M = M; a.G = L.K / L.group;
  a.stages_per_tile = p.stages_per_tile; a.row_tiles = p.row_tiles; a.max_slots = p.max_slots; a.units = p.units;
  a.y_bf16 = ybf16 ? 1 : 0;
  const SkKernel fn = sk_kernel(xbf16, asym, p.nt, p.gc, L.K % 256 == 0);
  void* args[] = {&tw, &tx, &a};
  return launch_kernel_ex((const void*)fn, dim3(p.grid), dim3(kSkThreads), p.smem, st, g_pdl != 0, args,
                          "skinny launch");
}

// ----------------------------------------------------------------------------
// 1 <= M <= 16: tcgen05 GEMV (weights as the A operand in tensor memory)
// ----------------------------------------------------------------------------

typedef void (*TgKernel)(CUtensorMap, CUtensorMap, TcGemvArgs);

template <bool B, bool A, int MC>
static TgKernel tg_for_gc(int gc) {
  if (gc == 1) return tc_gemv_kernel<B, A, MC, 1>;
  if (gc == 2) return tc_gemv_kernel<B, A, MC, 2>;
  return tc_gemv_kernel<B, A, MC, 4>;
}

template <bool B, bool A>
static TgKernel tg_for_mc(int M, int gc) {
  if (M == 1) return tg_for_gc<B, A, 1>(gc);
  if (M <= 8) return tg_for_gc<B, A, 8>(gc);
  return tg_for_gc<B, A, 16>(gc);
}

static TgKernel tg_kernel(bool xbf16, bool asym, int M, int gc) {
  if (xbf16) return asym ? tg_for_mc<true, true>(M, gc) : tg_for_mc<true, false>(M, gc);
  return asym ? tg_for_mc<false, true>(M, gc) : tg_for_mc<false, false>(M, gc);
}

// One CTA per SM (the kernel holds all 512 tensor-memory columns).
static SkPlan plan_tcgemv(int K, int N) {
  SkPlan p{};
  p.row_tiles = (N + 127) / 128;
  p.stages_per_tile = (K + 255) / 256;
  p.units = (long long)p.row_tiles * p.stages_per_tile;
  p.smem = kTgSmem;
  p.grid = (int)std::min<long long>(p.units, (long long)num_sms());
  const long long per = std::max<long long>(1, p.units / p.grid);
  p.max_slots = (int)((p.stages_per_tile + per - 1) / per + 1);
  return p;
}

static lbq_status run_tcgemv(const void* X, bool xbf16, int M, const void* image, const Layout& L, void* Y,
                             bool ybf16, void* ws, size_t ws_bytes, cudaStream_t st) {
  const bool asym = L.mode == LBQ_MODE_ASYM;
  const SkPlan p = plan_tcgemv(L.K, L.N);
  const size_t need = skinny_workspace_bytes(p, M);
  if (ws == nullptr || ws_bytes < need)
    return fail(LBQ_ERR_INVALID_ARG, "workspace of %zu bytes is too small (need %zu)", ws_bytes, need);
  const uint8_t* img = static_cast<const uint8_t*>(image);
  CUtensorMap tw, tx;
  const bool ok = make_tmap_2d(&tw, img + L.off0, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)L.K / 2, (uint64_t)L.N,
                               (uint64_t)L.K / 2, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B) &&
                  make_tmap_2d(&tx, X, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, (uint64_t)L.K, (uint64_t)M,
                               (uint64_t)L.K * 2, 64, 16, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!ok) return fail(LBQ_ERR_CUDA, "cuTensorMapEncodeTiled failed for the tcgen05 GEMV");
  TcGemvArgs a{};
  a.Y = Y;
  a.partials = static_cast<float*>(ws);
  a.counters = reinterpret_cast<unsigned*>(static_cast<uint8_t*>(ws) +
                                           align_up((size_t)p.row_tiles * p.max_slots * M * kSkRows * sizeof(float), 256));
  a.s_region = img + L.off1;
  a.z_region = asym ? img + L.off2 : nullptr;
  a.K = L.K; a.N = L.N; a.M = M; a.G = L.K / L.group;
  a.stages_per_tile = p.stages_per_tile; a.row_tiles = p.row_tiles; a.max_slots = p.max_slots; a.units = p.units;
  a.y_bf16 = ybf16 ? 1 : 0;
  const TgKernel fn = tg_kernel(xbf16, asym, M, L.group / 32);
  occupancy_for((const void*)fn, kTgThreads, kTgSmem);
  void* args[] = {&tw, &tx, &a};
  return launch_kernel_ex((const void*)fn, dim3(p.grid), dim3(kTgThreads), kTgSmem, st, g_pdl != 0, args,
                          "tcgen05 GEMV launch");
}

// M = 1, direct loads (no workspace): `count` GEMVs of the same K / group /
// mode / dtypes in one launch.
// test hook: -1 = the library's choice, 0 = weights pipelined through
// registers, 2..4 = staged through shared memory with that many row blocks in
// flight
static int g_direct_stages = -1;
static int g_direct_ctas = 0;  // test hook: cap on resident CTAs per SM (0 = occupancy limit)

static const void* direct_async_kernel(bool bf16, bool asym, int stages, bool a8 = false) {
#define LBQ_GDA(S, A) (bf16 ? (asym ? (const void*)gemv_direct_async_kernel<true, true, S, A>              \
                                    : (const void*)gemv_direct_async_kernel<true, false, S, A>)             \
                            : (asym ? (const void*)gemv_direct_async_kernel<false, true, S, A>             \
                                    : (const void*)gemv_direct_async_kernel<false, false, S, A>))
#define LBQ_GDA8(S) (asym ? (const void*)gemv_direct_async_kernel<false, true, S, true> \
                         : (const void*)gemv_direct_async_kernel<false, false, S, true>)
  (void)bf16;
  if (a8) return stages >= 4 ? LBQ_GDA8(4) : stages == 3 ? LBQ_GDA8(3) : LBQ_GDA8(2);
#undef LBQ_GDA8
  return stages >= 4 ? LBQ_GDA(4, false) : stages == 3 ? LBQ_GDA(3, false) : LBQ_GDA(2, false);
#undef LBQ_GDA
}

// sx != nullptr selects the W4A8 form: items[i].X are INT8 codes and sx[i]
// their per-32-k scales.
static lbq_status run_direct(const lbq_gemv_item* items, int count, int K, int group, int mode, bool xbf16, bool ybf16,
                             cudaStream_t st, const float* const* sx = nullptr) {
  const bool a8 = sx != nullptr;
  const bool asym = mode == LBQ_MODE_ASYM;
  const int chunks = K / 32;
  const int nw = (chunks + 31) / 32;
  if (nw > kGdMaxWarps) return fail(LBQ_ERR_UNSUPPORTED, "direct GEMV needs K <= %d", 32 * 32 * kGdMaxWarps);
  if (count < 1 || count > kGdMaxItems) return fail(LBQ_ERR_INVALID_ARG, "count=%d not in 1..%d", count, kGdMaxItems);
  GemvDirectArgs a{};
  int rbs = 0;
  for (int i = 0; i < count; ++i) {
    const Layout L = make_layout(K, items[i].N, group, mode);
    const uint8_t* img = static_cast<const uint8_t*>(items[i].image);
    a.X[i] = static_cast<const uint16_t*>(items[i].X);
    a.SX[i] = a8 ? sx[i] : nullptr;
    a.Y[i] = items[i].Y;
    a.q[i] = img + L.off0;
    a.s[i] = img + L.off1;
    a.z[i] = asym ? img + L.off2 : nullptr;
    a.N[i] = items[i].N;
    rbs += (items[i].N + 7) / 8;
    a.rb_end[i] = rbs;
  }
  a.items = count;
  a.K = K; a.G = K / group;
  a.row_blocks = rbs;
  a.y_bf16 = ybf16 ? 1 : 0;
  const int T = nw * 32;
  const void* reg_fn =
      xbf16 ? (asym ? (const void*)gemv_direct_kernel<true, true> : (const void*)gemv_direct_kernel<true, false>)
            : (asym ? (const void*)gemv_direct_kernel<false, true> : (const void*)gemv_direct_kernel<false, false>);
  // Variant, measured on B200 over the decode-step shapes in one CUDA graph:
  // row blocks staged through shared memory, 3 in flight for large launches
  // with K <= 8192 and 2 for smaller launches (more CTAs per SM, one wave)
  // and for longer K (one CTA per SM either way, where the deeper ring
  // measured slower). The register-pipelined kernel is faster alone on small
  // launches but costs more than it saves when it runs between staged
  // launches in a step.
  int stages = g_direct_stages;
  if (stages < 0) stages = (K > 8192 || rbs < 4 * num_sms()) ? 2 : 3;
  // the most stages (<= the chosen count) whose slots fit a CTA
  while (stages >= 2 && (size_t)T * (size_t)(stages * (8 * 16 + 16 + 8)) > 220 * 1024) --stages;
  if (stages < 2) stages = 0;
  if (a8 && stages == 0) stages = 2;  // the INT8-activation form exists only staged (2 stages always fit)
  const int stage_bytes = stages ? T * stages * (8 * 16 + 16 + 8) : 0;
  const void* fn = stages == 0 ? reg_fn : direct_async_kernel(xbf16, asym, stages, a8);
  // one wave of CTAs; each keeps 8 floats per warp per row block in shared memory
  int occ = std::max(1, occupancy_for(fn, T, stage_bytes + 4096));
  if (g_direct_ctas > 0) occ = std::min(occ, g_direct_ctas);
  int grid = std::min(a.row_blocks, num_sms() * occ);
  int smem = ((a.row_blocks + grid - 1) / grid) * nw * 8 * (int)sizeof(float);
  while (smem > (stages ? 4096 : 96 * 1024) && grid < a.row_blocks) {  // very tall matrices: more CTAs, fewer blocks each
    grid = std::min(a.row_blocks, grid * 2);
    smem = ((a.row_blocks + grid - 1) / grid) * nw * 8 * (int)sizeof(float);
  }
  smem += stage_bytes;
  void* args[] = {&a};
  return launch_kernel_ex(fn, dim3(grid), dim3(T), smem, st, g_pdl != 0, args, "direct GEMV launch");
}

// ----------------------------------------------------------------------------
// M = 1: TMA-fed warp-MMA GEMV
// ----------------------------------------------------------------------------

// Tensor maps are encoded on the host; a decode step reuses the same images
// every step, so each (base, shape, box) is encoded once.
static bool cached_tmap_2d(CUtensorMap* out, const void* base, CUtensorMapDataType dt, int elem, uint64_t cols,
                           uint64_t rows, uint64_t row_stride, uint32_t box_cols, uint32_t box_rows,
                           CUtensorMapSwizzle swz) {
  struct Key {
    uintptr_t base;
    uint64_t cols, rows, stride;
    uint32_t bc, br;
    int dt, swz;
    bool operator<(const Key& o) const {
      return std::tie(base, cols, rows, stride, bc, br, dt, swz) <
             std::tie(o.base, o.cols, o.rows, o.stride, o.bc, o.br, o.dt, o.swz);
    }
  };
  struct Entry {
    alignas(64) CUtensorMap map;
  };
  static std::mutex mu;
  static std::map<Key, Entry> cache;
  const Key k{reinterpret_cast<uintptr_t>(base), cols, rows, row_stride, box_cols, box_rows, (int)dt, (int)swz};
  std::lock_guard<std::mutex> lk(mu);
  auto itc = cache.find(k);
  if (itc != cache.end()) {
    *out = itc->second.map;
    return true;
  }
  Entry e;
  if (!make_tmap_2d(&e.map, base, dt, elem, cols, rows, row_stride, box_cols, box_rows, swz)) return false;
  if (cache.size() >= 8192) cache.clear();
  cache.emplace(k, e);
  *out = e.map;
  return true;
}

// The codes [N][K/2] viewed as [K/256 slices][N rows][128 bytes] (row stride
// K/2, slice stride 128), box 128 x 16 rows x nsl slices, 128-byte swizzle.
static bool cached_tmap_3d(CUtensorMap* out, const void* base, uint64_t N, uint64_t K, uint32_t nsl) {
  struct Key {
    uintptr_t base;
    uint64_t N, K;
    uint32_t nsl;
    bool operator<(const Key& o) const { return std::tie(base, N, K, nsl) < std::tie(o.base, o.N, o.K, o.nsl); }
  };
  struct Entry {
    alignas(64) CUtensorMap map;
  };
  static std::mutex mu;
  static std::map<Key, Entry> cache;
  const Key k{reinterpret_cast<uintptr_t>(base), N, K, nsl};
  std::lock_guard<std::mutex> lk(mu);
  auto itc = cache.find(k);
  if (itc != cache.end()) {
    *out = itc->second.map;
    return true;
  }
  Entry e;
  if (!make_tmap_3d(&e.map, base, CU_TENSOR_MAP_DATA_TYPE_UINT8, 128, N, K / 256, K / 2, 128, 128, kTmRows, nsl,
                    CU_TENSOR_MAP_SWIZZLE_128B))
    return false;
  if (cache.size() >= 8192) cache.clear();
  cache.emplace(k, e);
  *out = e.map;
  return true;
}

struct TmPlan {
  int R, nsl, krg, row_tiles, grid, stages, stage_bytes, s_off, z_off, smem, block, max_units;
  size_t ws, cnt_off;
};

static int max_dynamic_smem() {
  static int optin = 0;
  static std::once_flag once;
  std::call_once(once, [] {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  });
  return optin;
}

// K is cut into R ranges of nsl 256-k slices (one consumer warp each, at most
// 16): the smallest R in {1, 2, 4} that fits (one CTA per SM, a fixed range per
// CTA). Several GEMVs in one launch keep R = 1 (no workspace).
static int g_tmma_split = 0;  // test hook: force the number of K-ranges (0 = the plan's choice)
static int g_debug_drop = 0;  // test hook: the TMA GEMV's producer issues nothing (its waits must give up)

static TmPlan plan_tmma(int K, const int* Ns, int count, int group, bool asym, bool allow_split = true) {
  TmPlan p{};
  const int chunks = K / 32;
  for (int i = 0; i < count; ++i) p.row_tiles += (Ns[i] + kTmRows - 1) / kTmRows;
  const int sms = num_sms();
  // the fewest ranges that fit: each range's CTA pays a fixed cost per unit
  // and the split adds a workspace pass, which balance rarely repays
  for (int R = 1; R <= 4; R *= 2) {
    if ((count > 1 || !allow_split) && R > 1) break;
    if (g_tmma_split > 0 && R != g_tmma_split && !((count > 1 || !allow_split) && R == 1)) continue;
    const int nsl = (chunks + 8 * R - 1) / (8 * R);
    if (nsl > kTmMaxSlices || (R - 1) * nsl * 8 >= chunks) continue;  // no range may be empty
    p.R = R;
    p.nsl = nsl;
    break;
  }
  if (p.nsl == 0) return p;
  p.krg = p.nsl * 256 / group;
  p.grid = p.R * std::max(1, std::min(p.row_tiles, sms / p.R));
  p.s_off = p.nsl * kTmSliceBytes;
  p.z_off = (int)align_up((size_t)p.s_off + (size_t)p.krg * 32, 128);
  p.stage_bytes = (int)align_up(asym ? (size_t)p.z_off + (size_t)p.krg * 16 : (size_t)p.z_off, 1024);
  const int cpk = p.grid / p.R;
  p.max_units = (p.row_tiles + cpk - 1) / cpk;
  const int avail = max_dynamic_smem() - 2 * kTmMaxStages * 8 - 1024;
  const int red_bytes = p.max_units * p.nsl * 16 * 4 + p.max_units * 4;
  // a short ring: the decode step (K=4096 launches, one CTA per SM) measured
  // 1071.5 us per step with at most three stages against 1077.3 with as many
  // as fit; copies in flight together land together and delay the decode
  int S = kTmDefaultStages;
  while (S >= 2 && S * p.stage_bytes + red_bytes > avail) --S;
  p.stages = S;
  p.smem = 1024 + S * p.stage_bytes + red_bytes;
  p.block = (p.nsl + 1) * 32;
  if (p.R > 1) {
    p.cnt_off = align_up((size_t)p.R * Ns[0] * sizeof(float), 256);
    p.ws = p.cnt_off + align_up((size_t)p.row_tiles * sizeof(unsigned), 256);
  }
  return p;
}

// Shapes the TMA-fed kernel takes: a 16-row box of codes and whole 256-k
// slices must fit the matrix; several GEMVs per launch need K <= 4096 (one
// range, no workspace).
static bool tmma_ok(int M, int K, const int* Ns, int count) {
  if (M != 1 || K < 256 || K > 16384 || K % 256) return false;
  if (count > 1 && K > 32 * 8 * kTmMaxSlices) return false;
  for (int i = 0; i < count; ++i)
    if (Ns[i] < kTmRows) return false;
  return true;
}

static const void* tmma_kernel(bool bf16, bool asym, int gshift) {
#define LBQ_TMK(GS)                                                                                        \
  (bf16 ? (asym ? (const void*)gemv_tmma_kernel<true, true, GS> : (const void*)gemv_tmma_kernel<true, false, GS>)   \
        : (asym ? (const void*)gemv_tmma_kernel<false, true, GS> : (const void*)gemv_tmma_kernel<false, false, GS>))
  return gshift == 0 ? LBQ_TMK(0) : gshift == 1 ? LBQ_TMK(1) : LBQ_TMK(2);
#undef LBQ_TMK
}

static lbq_status run_tmma(const lbq_gemv_item* items, int count, int K, int group, int mode, bool xbf16, bool ybf16,
                           void* ws, size_t ws_bytes, cudaStream_t st, bool allow_split = true) {
  const bool asym = mode == LBQ_MODE_ASYM;
  if (count < 1 || count > kTmMaxItems) return fail(LBQ_ERR_INVALID_ARG, "count=%d not in 1..%d", count, kTmMaxItems);
  int Ns[kTmMaxItems];
  for (int i = 0; i < count; ++i) Ns[i] = items[i].N;
  const TmPlan p = plan_tmma(K, Ns, count, group, asym, allow_split);
  if (p.nsl == 0 || p.stages < 2) return fail(LBQ_ERR_UNSUPPORTED, "no TMA GEMV plan for K=%d", K);
  GemvTmmaArgs a{};
  GemvTmmaMaps m;
  std::memset(&m, 0, sizeof(m));
  int tiles = 0;
  for (int i = 0; i < count; ++i) {
    const Layout L = make_layout(K, items[i].N, group, mode);
    const uint8_t* img = static_cast<const uint8_t*>(items[i].image);
    const uint64_t meta_rows = (uint64_t)((items[i].N + 127) / 128) * (uint64_t)(K / group);
    if (!cached_tmap_3d(&m.q[i], img + L.off0, (uint64_t)items[i].N, (uint64_t)K, (uint32_t)p.nsl) ||
        !cached_tmap_2d(&m.s[i], img + L.off1, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, 128, meta_rows, 256, 16,
                        (uint32_t)p.krg, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        (asym && !cached_tmap_2d(&m.z[i], img + L.off2, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, 128, meta_rows, 128, 16,
                                 (uint32_t)p.krg, CU_TENSOR_MAP_SWIZZLE_NONE)))
      return fail(LBQ_ERR_CUDA, "cuTensorMapEncodeTiled failed for the GEMV image %d", i);
    a.X[i] = static_cast<const uint16_t*>(items[i].X);
    a.Y[i] = items[i].Y;
    a.N[i] = items[i].N;
    tiles += (items[i].N + kTmRows - 1) / kTmRows;
    a.rt_end[i] = tiles;
  }
  if (p.R > 1) {
    if (!ws || ws_bytes < p.ws || !aligned16(ws))
      return fail(LBQ_ERR_INVALID_ARG, "workspace of %zu bytes (16-byte aligned) needed, got %zu", p.ws, ws_bytes);
    a.partials = static_cast<float*>(ws);
    a.counters = reinterpret_cast<unsigned int*>(static_cast<uint8_t*>(ws) + p.cnt_off);
  }
  a.items = count;
  a.K = K;
  a.G = K / group;
  a.gshift = group == 32 ? 0 : group == 64 ? 1 : 2;
  a.R = p.R;
  a.nsl = p.nsl;
  a.krg = p.krg;
  a.row_tiles = p.row_tiles;
  a.stages = p.stages;
  a.stage_bytes = p.stage_bytes;
  a.s_off = p.s_off;
  a.z_off = p.z_off;
  a.max_units = p.max_units;
  a.y_bf16 = ybf16 ? 1 : 0;
  a.debug_drop = g_debug_drop;
  const void* fn = tmma_kernel(xbf16, asym, a.gshift);
  occupancy_for(fn, p.block, p.smem);  // raises the kernel's dynamic shared-memory limit once
  void* args[] = {&m, &a};
  return launch_kernel_ex(fn, dim3(p.grid), dim3(p.block), p.smem, st, g_pdl != 0, args, "TMA GEMV launch");
}

// The kernel lbq_gemv runs for M <= 16. Measured on B200: at M = 1 the
// direct-load CUDA-core kernel is the fastest at every size it supports
// (K <= 16384; the warp-MMA kernel spends an MMA, 7/8 wasted, per 256 weights
// and legacy MMA throughput is its limit); from M = 2 the warp-MMA kernel wins.
// The tcgen05 kernel is slower at every batch size here (a 128 x 16 x N MMA
// costs the same ~185 cycles for N = 16 as for N = 256), so it is never the
// default.
// When the TMA-fed warp-MMA kernel is the M = 1 choice: 2 (the default) for
// launches of at least kTmmaMinTilesPerSm 16-row tiles per SM with K <= 4096,
// where it was measured faster than the staged CUDA-core kernel (the gate/up
// launch of the decode step: 4.74 against 4.32 TB/s; the step 1078 against
// 1127 us); smaller launches and longer K stay on the staged kernel, which
// starts streaming sooner. Test hook values: 0 never, 1 always.
static int g_tmma_default = 2;
constexpr int kTmmaMinTilesPerSm = 4;

static bool tmma_preferred(int K, const int* Ns, int count) {
  if (g_tmma_default == 1) return true;
  if (g_tmma_default != 2) return false;
  int tiles = 0;
  for (int i = 0; i < count; ++i) tiles += (Ns[i] + 15) / 16;
  return K <= 4096 && tiles >= kTmmaMinTilesPerSm * num_sms();
}

static int gemv_path(int M, int K, int N) {
  const long long weights = (long long)K * N;
  const bool direct_ok = M == 1 && K <= 32 * 32 * kGdMaxWarps;
  if (g_gemv_path == kPathTmma && tmma_ok(M, K, &N, 1)) return kPathTmma;
  if (g_gemv_path == kPathM1 && M == 1) return kPathM1;
  if (g_gemv_path == kPathDirect && direct_ok) return kPathDirect;
  if (g_gemv_path == kPathMma || g_gemv_path == kPathTc) return g_gemv_path;
  if (g_force_skinny) return kPathMma;
  if (M == 1 && g_force_splits) return kPathM1;
  if (M == 1 && g_gemv_path == kPathAuto && tmma_preferred(K, &N, 1) && tmma_ok(M, K, &N, 1)) return kPathTmma;
  if (M == 1) return direct_ok ? kPathDirect : (weights < (1LL << 27) ? kPathM1 : kPathMma);
  return kPathMma;
}

// Scratch of that kernel for one call: total bytes and where the tile counters
// sit (they must be zero when the kernel starts).
struct GemvScratch {
  size_t need, cnt_off, cnt_bytes;
};

static GemvScratch gemv_scratch(int M, int K, int N, int group, bool asym, bool xbf16) {
  GemvScratch g{0, 0, 0};
  const int path = gemv_path(M, K, N);
  if (path == kPathDirect) return g;
  if (path == kPathTmma) {
    const TmPlan p = plan_tmma(K, &N, 1, group, asym);
    g.need = p.ws;
    if (g.need) {
      g.cnt_off = p.cnt_off;
      g.cnt_bytes = (size_t)p.row_tiles * sizeof(unsigned);
    }
    return g;
  }
  if (path == kPathM1) {
    const M1Plan p = plan_m1(K, N, group, asym, g_force_splits);
    g.need = p.block == 0 ? 0 : m1_workspace_bytes(p, N);
    if (g.need) {
      g.cnt_off = align_up((size_t)p.splits * N * sizeof(float), 256);
      g.cnt_bytes = (size_t)p.row_tiles * sizeof(unsigned);
    }
    return g;
  }
  const SkPlan p = path == kPathMma ? plan_skinny(K, N, M, group, asym, xbf16) : plan_tcgemv(K, N);
  g.need = skinny_workspace_bytes(p, M);
  g.cnt_off = align_up((size_t)p.row_tiles * p.max_slots * M * kSkRows * sizeof(float), 256);
  g.cnt_bytes = (size_t)p.row_tiles * sizeof(unsigned);
  return g;
}

// ----------------------------------------------------------------------------
// M > 16: tcgen05 prefill GEMM
// ----------------------------------------------------------------------------

static int g_force_tc = 0;  // test hook: route every lbq_gemm call to the tcgen05 kernel
// test hook: prefill kernel. 0 = weights in tensor memory (A operand), 1 = the
// kernel with the weights dequantised into shared memory (B operand).
static int g_gemm_path = 0;

typedef void (*TsKernel)(CUtensorMap, CUtensorMap, GemmTsArgs);

// Prefill GEMM with the weights as the A operand in tensor memory (INT4 or LUT3).
// Prefill schedule: whole tiles strided over a grid of at most one CTA per
// SM; when that leaves a part-filled last wave whose idle share is worth more
// than the cut tiles' exchange (at least 5% of the whole schedule's SM time
// and 4 k-blocks per SM), the last two waves' tiles are shared out by k-block
// (stream-K) through a workspace of one flag and one FP32 tile per CTA.
// Measured on B200, K=4096 N=14336: M=512 +9%, M=2048 +10%, M=4096 +5%;
// at M=8192 (3% idle) whole tiles were 3% faster.
static int g_ts_stream_k = 1;       // test hook: 0 = whole tiles only
static int g_ts_hold = 0;           // test hook: later parts never raise their flag
static uint32_t g_ts_polls = 0;     // test hook: bound on the flag wait (0 = about 4 s)
struct TsPlan {
  int grid, dp_tiles;
  long long sk_items;
  size_t flags_bytes, ws_bytes;  // 0 without stream-K
};
static TsPlan plan_gemm_ts(int M, int K, int N) {
  const int T = ((N + kTsBN - 1) / kTsBN) * ((M + kTsBM - 1) / kTsBM);
  const int nkb = (K + kTsBK - 1) / kTsBK;
  TsPlan p{};
  p.grid = std::min(T, num_sms());
  p.dp_tiles = T;
  const int rem = T % p.grid;
  const long long waves = (T + p.grid - 1) / p.grid;
  if (T > p.grid && rem != 0 && (long long)nkb * (p.grid - rem) >= 4LL * p.grid &&
      20LL * (p.grid - rem) >= (long long)p.grid * waves) {
    p.dp_tiles = (T / p.grid - 1) * p.grid;
    p.sk_items = (long long)(T - p.dp_tiles) * nkb;
    p.flags_bytes = ((size_t)p.grid * 4 + 255) / 256 * 256;
    p.ws_bytes = p.flags_bytes + (size_t)p.grid * kSkTileFloats * 4;
  }
  return p;
}

// The schedule's kernel arguments: stream-K where the plan cuts tiles and the
// caller's workspace is large enough, else whole tiles.
static SkArgs sk_args(const TsPlan& p, int tiles, void* ws, size_t ws_bytes) {
  SkArgs k{};
  k.dp_tiles = tiles;
  k.flag_polls = g_ts_polls ? g_ts_polls : (1u << 22);
  k.debug_hold = g_ts_hold;
  if (p.ws_bytes && g_ts_stream_k && ws && ws_bytes >= p.ws_bytes) {
    k.dp_tiles = p.dp_tiles;
    k.sk_items = p.sk_items;
    k.flags = static_cast<unsigned*>(ws);
    k.partials = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + p.flags_bytes);
  }
  return k;
}

static lbq_status run_gemm_ts(const void* X, bool xbf16, int M, const void* image, const Layout& L, void* Y,
                              bool ybf16, void* ws, size_t ws_bytes, cudaStream_t st) {
  const bool lut = L.mode == LBQ_MODE_LUT3, asym = L.mode == LBQ_MODE_ASYM;
  const uint8_t* img = static_cast<const uint8_t*>(image);
  CUtensorMap tx, tq;
  if (!make_tmap_2d(&tx, X, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, (uint64_t)L.K, (uint64_t)M, (uint64_t)L.K * 2, 64,
                    kTsBM, CU_TENSOR_MAP_SWIZZLE_128B))
    return fail(LBQ_ERR_CUDA, "cuTensorMapEncodeTiled failed for the prefill activations");
  tq = tx;
  if (!lut && !make_tmap_2d(&tq, img + L.off0, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)L.K / 2, (uint64_t)L.N,
                            (uint64_t)L.K / 2, kTsBK / 2, kTsBN, CU_TENSOR_MAP_SWIZZLE_64B))
    return fail(LBQ_ERR_CUDA, "cuTensorMapEncodeTiled failed for the prefill codes");
  GemmTsArgs a{};
  a.Y = Y;
  a.meta0 = lut ? img + L.off0 : img + L.off1;
  a.meta1 = lut ? img + L.off3 : (asym ? img + L.off2 : nullptr);
  a.M = M; a.N = L.N; a.K = L.K;
  a.group = lut ? 64 : L.group;
  a.G = L.K / a.group;
  a.n_tiles = (L.N + kTsBN - 1) / kTsBN;
  a.m_tiles = (M + kTsBM - 1) / kTsBM;
  a.k_blocks = (L.K + kTsBK - 1) / kTsBK;
  a.y_bf16 = ybf16 ? 1 : 0;
  TsKernel fn;
  if (lut) fn = gemm_ts_kernel<true, false, true>;
  else if (xbf16) fn = asym ? gemm_ts_kernel<true, true, false> : gemm_ts_kernel<true, false, false>;
  else fn = asym ? gemm_ts_kernel<false, true, false> : gemm_ts_kernel<false, false, false>;
  const int smem = kTsSmem;
  occupancy_for((const void*)fn, kTsThreads, smem);
  const TsPlan p = plan_gemm_ts(M, L.K, L.N);
  const int grid = p.grid;
  a.sk = sk_args(p, a.n_tiles * a.m_tiles, ws, ws_bytes);
  void* args[] = {&tx, &tq, &a};
  return launch_kernel_ex((const void*)fn, dim3(grid), dim3(kTsThreads), smem, st, false, args,
                          "prefill GEMM launch");
}

static lbq_status run_gemm_tc(const void* X, bool xbf16, int M, const void* image, const Layout& L, void* Y,
                              bool ybf16, cudaStream_t st) {
  const bool asym = L.mode == LBQ_MODE_ASYM;
  const uint8_t* img = static_cast<const uint8_t*>(image);
  CUtensorMap tx, tq;
  const bool ok = make_tmap_2d(&tx, X, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, (uint64_t)L.K, (uint64_t)M,
                               (uint64_t)L.K * 2, kTcBK, kTcBM, CU_TENSOR_MAP_SWIZZLE_128B) &&
                  make_tmap_2d(&tq, img + L.off0, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)L.K / 2, (uint64_t)L.N,
                               (uint64_t)L.K / 2, kTcBK / 2, kTcBN, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (!ok) return fail(LBQ_ERR_CUDA, "cuTensorMapEncodeTiled failed for the prefill GEMM");
  GemmTcArgs a{};
  a.Y = Y;
  a.s_region = img + L.off1;
  a.z_region = asym ? img + L.off2 : nullptr;
  a.G = L.K / L.group;
  a.tiles128 = (L.N + 127) / 128;
  a.M = M; a.N = L.N; a.K = L.K; a.gshift64 = log2_exact(L.group / 32);
  a.m_tiles = (M + kTcBM - 1) / kTcBM;
  a.n_tiles = (L.N + kTcBN - 1) / kTcBN;
  a.k_blocks = (L.K + kTcBK - 1) / kTcBK;
  a.y_bf16 = ybf16 ? 1 : 0;
  const void* fn = xbf16 ? (asym ? (const void*)gemm_tc_kernel<true, true, false> : (const void*)gemm_tc_kernel<true, false, false>)
                         : (asym ? (const void*)gemm_tc_kernel<false, true, false> : (const void*)gemm_tc_kernel<false, false, false>);
  occupancy_for(fn, kTcThreads, kTcSmem);
  const int grid = std::min(a.m_tiles * a.n_tiles, num_sms());
  void* args[] = {&tx, &tq, &a};
  return launch_kernel_ex(fn, dim3(grid), dim3(kTcThreads), kTcSmem, st, false, args, "prefill GEMM launch");
}

// ----------------------------------------------------------------------------
// LUT3: skinny (M <= 16) and tcgen05 (M > 16)
// ----------------------------------------------------------------------------

static SkPlan plan_lut3(int K, int N, int M) {
  SkPlan p{};
  p.nt = M <= 8 ? 1 : 2;
  p.row_tiles = (N + kSkRows - 1) / kSkRows;
  p.stages_per_tile = (K + 255) / 256;
  p.units = (long long)p.row_tiles * p.stages_per_tile;
  p.slot = 13312 + 4 * p.nt * 1024;
  p.smem = kL3Stages * p.slot + 1024;
  const void* fn = p.nt == 1 ? (const void*)lut3_skinny_kernel<1> : (const void*)lut3_skinny_kernel<2>;
  const int occ = occupancy_for(fn, kSkThreads, p.smem);
  p.grid = (int)std::min<long long>(p.units, (long long)num_sms() * occ);
  const long long per = std::max<long long>(1, p.units / p.grid);
  p.max_slots = (int)((p.stages_per_tile + per - 1) / per + 1);
  return p;
}

static lbq_status run_lut3_skinny(const void* X, int M, const void* image, const Layout& L, void* Y, bool ybf16,
                                  void* ws, size_t ws_bytes, cudaStream_t st) {
  const SkPlan p = plan_lut3(L.K, L.N, M);
  const size_t need = skinny_workspace_bytes(p, M);
  if (ws == nullptr || ws_bytes < need)
    return fail(LBQ_ERR_INVALID_ARG, "workspace of %zu bytes is too small (need %zu)", ws_bytes, need);
  const uint8_t* img = static_cast<const uint8_t*>(image);
  CUtensorMap tx;
  if (!make_tmap_2d(&tx, X, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, (uint64_t)L.K, (uint64_t)M, (uint64_t)L.K * 2, 64,
                    (uint32_t)M, CU_TENSOR_MAP_SWIZZLE_128B))
    return fail(LBQ_ERR_CUDA, "cuTensorMapEncodeTiled failed for the LUT3 GEMV");
  Lut3SkinnyArgs a{};
  a.Y = Y;
  a.partials = static_cast<float*>(ws);
  a.counters = reinterpret_cast<unsigned*>(static_cast<uint8_t*>(ws) +
                                           align_up((size_t)p.row_tiles * p.max_slots * M * kSkRows * sizeof(float), 256));
  a.i_region = img + L.off0;
  a.t_region = img + L.off3;
  a.K = L.K; a.N = L.N; a.M = M;
  a.stages_per_tile = p.stages_per_tile; a.row_tiles = p.row_tiles; a.max_slots = p.max_slots; a.units = p.units;
  a.y_bf16 = ybf16 ? 1 : 0;
  const void* fn = p.nt == 1 ? (const void*)lut3_skinny_kernel<1> : (const void*)lut3_skinny_kernel<2>;
  void* args[] = {&tx, &a};
  return launch_kernel_ex(fn, dim3(p.grid), dim3(kSkThreads), p.smem, st, g_pdl != 0, args, "lut3 skinny launch");
}

// LUT3, M = 1, direct loads (no workspace).
static bool lut3_direct_ok(int M, int K) { return M == 1 && K / 64 <= 32 * kLdMaxWarps && g_gemv_path != kPathMma; }

// test hook: LUT3 batch-1 kernel (-1 = the library's choice, 0 = indices
// pipelined through registers, 2 / 3 = staged through shared memory)

static lbq_status run_lut3_direct(const void* X, const void* image, const Layout& L, void* Y, bool ybf16,
                                  cudaStream_t st) {
  const uint8_t* img = static_cast<const uint8_t*>(image);
  Lut3DirectArgs a{};
  a.X = static_cast<const uint16_t*>(X);
  a.Y = Y;
  a.i_region = img + L.off0;
  a.t_region = img + L.off3;
  a.K = L.K; a.N = L.N;
  a.row_blocks = L.N / 8;
  a.y_bf16 = ybf16 ? 1 : 0;
  const int nw = (L.K / 64 + 31) / 32;
  const int T = nw * 32;
  const void* fn = (const void*)lut3_direct_kernel;
  const int occ = std::max(1, occupancy_for(fn, T, 1024));
  int grid = std::min(a.row_blocks, num_sms() * occ);
  int smem = ((a.row_blocks + grid - 1) / grid) * nw * 8 * (int)sizeof(float);
  while (smem > 96 * 1024 && grid < a.row_blocks) {
    grid = std::min(a.row_blocks, grid * 2);
    smem = ((a.row_blocks + grid - 1) / grid) * nw * 8 * (int)sizeof(float);
  }
  void* args[] = {&a};
  return launch_kernel_ex(fn, dim3(grid), dim3(T), smem, st, g_pdl != 0, args, "LUT3 direct GEMV launch");
}

// LUT3, M = 1, TMA-fed warp-MMA kernel: one 8-row codebook group over all of
// K per unit, K <= 8192 (at most 16 consumer warps of 4 or 8 tiles each).
struct L3tPlan {
  int kg, nw, grid, max_units, stage_bytes, t_off, stages, smem;
};

static int g_l3t_stages = 0;  // test hook: ring stages of the LUT3 TMA GEMV (0 = the plan's choice)
// three stages (measured on B200, K=4096 N=14336 with programmatic dependent
// launch: 10.55 us against 10.67 with four, 10.95 with six, 12.4 with two)
static int g_l3t_default_stages = 3;

static L3tPlan plan_lut3_tmma(int K, int N) {
  L3tPlan p{};
  const int KT = K / 64;
  if (KT > 4 * 2 * kL3tMaxWarps) return p;
  p.kg = KT <= 4 * kL3tMaxWarps ? 1 : 2;
  p.nw = (KT + 4 * p.kg - 1) / (4 * p.kg);
  const int units = N / 8;
  p.grid = std::max(1, std::min(units, num_sms()));
  p.max_units = (units + p.grid - 1) / p.grid;
  p.t_off = (int)align_up((size_t)KT * 192, 128);
  p.stage_bytes = p.t_off + (int)align_up((size_t)KT * 16, 128);
  const int red_bytes = p.max_units * p.nw * 8 * 4;
  const int avail = max_dynamic_smem() - 2 * kL3tMaxStages * 8 - 1024 - red_bytes;
  // a short ring: copies in flight together land together (see the kernel)
  const int want = g_l3t_stages ? g_l3t_stages : g_l3t_default_stages;
  p.stages = std::min(std::min(std::min(p.max_units, want), kL3tMaxStages), avail / p.stage_bytes);
  p.smem = 1024 + p.stages * p.stage_bytes + red_bytes;
  return p;
}

static bool lut3_tmma_ok(int M, int K, int N, const void* X, const void* image) {
  if (M != 1 || g_gemv_path == kPathMma || g_gemv_path == kPathDirect) return false;
  if ((reinterpret_cast<uintptr_t>(X) & 15) || (reinterpret_cast<uintptr_t>(image) & 15)) return false;
  const L3tPlan p = plan_lut3_tmma(K, N);
  return p.nw > 0 && p.stages >= 1;
}

static lbq_status run_lut3_tmma(const void* X, const void* image, const Layout& L, void* Y, bool ybf16,
                                cudaStream_t st) {
  const L3tPlan p = plan_lut3_tmma(L.K, L.N);
  if (p.nw == 0 || p.stages < 1) return fail(LBQ_ERR_UNSUPPORTED, "no LUT3 TMA GEMV plan for K=%d N=%d", L.K, L.N);
  const uint8_t* img = static_cast<const uint8_t*>(image);
  const int KT = L.K / 64;
  CUtensorMap mi, mt;
  // indices [K/64][N * 24 bytes] as 8-byte elements, box: one group's 192 bytes x every tile
  if (!make_tmap_2d(&mi, img + L.off0, CU_TENSOR_MAP_DATA_TYPE_UINT64, 8, (uint64_t)L.N * 3, (uint64_t)KT,
                    (uint64_t)L.N * 24, 24, (uint32_t)KT, CU_TENSOR_MAP_SWIZZLE_NONE))
    return fail(LBQ_ERR_CUDA, "cuTensorMapEncodeTiled failed for the LUT3 indices");
  // tables [K/64][N/8 * 16 bytes], box: one group's 16 bytes x every tile
  if (!make_tmap_2d(&mt, img + L.off3, CU_TENSOR_MAP_DATA_TYPE_UINT64, 8, (uint64_t)L.N / 4, (uint64_t)KT,
                    (uint64_t)L.N * 2, 2, (uint32_t)KT, CU_TENSOR_MAP_SWIZZLE_NONE))
    return fail(LBQ_ERR_CUDA, "cuTensorMapEncodeTiled failed for the LUT3 tables");
  Lut3TmmaArgs a{};
  a.X = static_cast<const uint16_t*>(X);
  a.Y = Y;
  a.K = L.K; a.N = L.N;
  a.units = L.N / 8;
  a.nw = p.nw;
  a.stages = p.stages; a.stage_bytes = p.stage_bytes; a.t_off = p.t_off;
  a.max_units = p.max_units;
  a.y_bf16 = ybf16 ? 1 : 0;
  a.debug_drop = g_debug_drop;
  const void* fn = p.kg == 1 ? (const void*)lut3_tmma_kernel<1> : (const void*)lut3_tmma_kernel<2>;
  const int block = (p.nw + 1) * 32;
  occupancy_for(fn, block, p.smem);  // raises the kernel's dynamic shared-memory limit once
  void* args[] = {&mi, &mt, &a};
  return launch_kernel_ex(fn, dim3(p.grid), dim3(block), p.smem, st, g_pdl != 0, args, "LUT3 TMA GEMV launch");
}

// LUT3, M = 2..8, TMA-fed warp-MMA kernel with the batch on the MMA's columns.
static int g_l3b_off = 0;  // test hook: 1 = M = 2..8 on the skinny kernel instead

struct L3bPlan {
  int kj, nb, nw, grid, stage_bytes, t_off, stages, xs_off, red_off, smem;
};

static L3bPlan plan_lut3_batch(int M, int K, int N) {
  L3bPlan p{};
  const int KT = K / 64;
  // X staged whole: up to 64 KB for 8 rows, 128 KB for 16 (K <= 4096)
  p.nb = M > 8 ? 2 : 1;
  if (M < 2 || M > kL3bMaxM || KT > 8 * kL3tMaxWarps || (size_t)M * K * 2 > (size_t)p.nb * 64 * 1024) return L3bPlan{};
  p.nw = std::min(kL3tMaxWarps, KT);
  const int kj = (KT + p.nw - 1) / p.nw;
  p.kj = kj <= 2 ? 2 : kj <= 4 ? 4 : 8;
  const int tiles = (N + kL3bRows - 1) / kL3bRows;
  p.grid = std::max(1, std::min(tiles, num_sms()));
  const int max_units = (tiles + p.grid - 1) / p.grid;
  p.t_off = (int)align_up((size_t)KT * 384, 128);
  p.stage_bytes = p.t_off + (int)align_up((size_t)KT * 32, 128);
  const int x_bytes = (int)align_up((size_t)M * K * 2, 128);
  const int red_bytes = 2 * p.nw * 128 * p.nb * (int)sizeof(float);
  const int avail = max_dynamic_smem() - 2 * kL3tMaxStages * 8 - 1024 - x_bytes - red_bytes;
  // two stages: a deeper ring lands its copies together and delays the decode
  // (measured on B200, K=4096 N=14336 M=8: 16.95 us with two, 17.4 with three,
  // 17.9 with four, 21.3 with one)
  const int want = g_l3t_stages ? g_l3t_stages : 2;
  p.stages = std::min(std::min(std::min(max_units, want), kL3tMaxStages), avail / p.stage_bytes);
  p.xs_off = p.stages * p.stage_bytes;
  p.red_off = p.xs_off + x_bytes;
  p.smem = 1024 + p.red_off + red_bytes;
  return p;
}

static bool lut3_batch_ok(int M, int K, int N, const void* X, const void* image) {
  if (g_l3b_off || g_gemv_path == kPathMma) return false;
  if ((reinterpret_cast<uintptr_t>(X) & 15) || (reinterpret_cast<uintptr_t>(image) & 15)) return false;
  const L3bPlan p = plan_lut3_batch(M, K, N);
  return p.nw > 0 && p.stages >= 1;
}

static lbq_status run_lut3_batch(const void* X, int M, const void* image, const Layout& L, void* Y, bool ybf16,
                                 cudaStream_t st) {
  const L3bPlan p = plan_lut3_batch(M, L.K, L.N);
  if (p.nw == 0 || p.stages < 1) return fail(LBQ_ERR_UNSUPPORTED, "no LUT3 batch GEMV plan for M=%d K=%d", M, L.K);
  const uint8_t* img = static_cast<const uint8_t*>(image);
  const int KT = L.K / 64;
  CUtensorMap mi, mt;
  // indices [K/64][N * 24 bytes] as 8-byte words, box: two groups' 384 bytes x every tile
  if (!make_tmap_2d(&mi, img + L.off0, CU_TENSOR_MAP_DATA_TYPE_UINT64, 8, (uint64_t)L.N * 3, (uint64_t)KT,
                    (uint64_t)L.N * 24, 48, (uint32_t)KT, CU_TENSOR_MAP_SWIZZLE_NONE))
    return fail(LBQ_ERR_CUDA, "cuTensorMapEncodeTiled failed for the LUT3 indices");
  // tables [K/64][N/8 * 16 bytes], box: two groups' 32 bytes x every tile
  if (!make_tmap_2d(&mt, img + L.off3, CU_TENSOR_MAP_DATA_TYPE_UINT64, 8, (uint64_t)L.N / 4, (uint64_t)KT,
                    (uint64_t)L.N * 2, 4, (uint32_t)KT, CU_TENSOR_MAP_SWIZZLE_NONE))
    return fail(LBQ_ERR_CUDA, "cuTensorMapEncodeTiled failed for the LUT3 tables");
  Lut3BatchArgs a{};
  a.X = static_cast<const uint16_t*>(X);
  a.Y = Y;
  a.K = L.K; a.N = L.N; a.M = M;
  a.tiles = (L.N + kL3bRows - 1) / kL3bRows;
  a.nw = p.nw;
  a.stages = p.stages; a.stage_bytes = p.stage_bytes; a.t_off = p.t_off;
  a.xs_off = p.xs_off; a.red_off = p.red_off;
  a.y_bf16 = ybf16 ? 1 : 0;
  a.debug_drop = g_debug_drop;
  const void* fn;
  if (p.nb == 1)
    fn = p.kj == 2 ? (const void*)lut3_tmma_batch_kernel<2, 1>
       : p.kj == 4 ? (const void*)lut3_tmma_batch_kernel<4, 1> : (const void*)lut3_tmma_batch_kernel<8, 1>;
  else
    fn = p.kj == 2 ? (const void*)lut3_tmma_batch_kernel<2, 2>
       : p.kj == 4 ? (const void*)lut3_tmma_batch_kernel<4, 2> : (const void*)lut3_tmma_batch_kernel<8, 2>;
  const int block = (p.nw + 1) * 32;
  occupancy_for(fn, block, p.smem);  // raises the kernel's dynamic shared-memory limit once
  void* args[] = {&mi, &mt, &a};
  return launch_kernel_ex(fn, dim3(p.grid), dim3(block), p.smem, st, g_pdl != 0, args,
                          "LUT3 TMA batch GEMV launch");
}

static lbq_status run_lut3_gemm_tc(const void* X, int M, const void* image, const Layout& L, void* Y, bool ybf16,
                                   cudaStream_t st) {
  const uint8_t* img = static_cast<const uint8_t*>(image);
  CUtensorMap tx, tq;
  if (!make_tmap_2d(&tx, X, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, (uint64_t)L.K, (uint64_t)M, (uint64_t)L.K * 2, kTcBK,
                    kTcBM, CU_TENSOR_MAP_SWIZZLE_128B))
    return fail(LBQ_ERR_CUDA, "cuTensorMapEncodeTiled failed for the LUT3 GEMM");
  tq = tx;  // unused by the LUT3 producer
  GemmTcArgs a{};
  a.Y = Y;
  a.s_region = img + L.off0;  // indices
  a.z_region = img + L.off3;  // tables
  a.M = M; a.N = L.N; a.K = L.K; a.gshift64 = 1;
  a.m_tiles = (M + kTcBM - 1) / kTcBM;
  a.n_tiles = (L.N + kTcBN - 1) / kTcBN;
  a.k_blocks = L.K / kTcBK;
  a.y_bf16 = ybf16 ? 1 : 0;
  const void* fn = (const void*)gemm_tc_kernel<true, false, true>;
  occupancy_for(fn, kTcThreads, kTcSmem);
  const int grid = std::min(a.m_tiles * a.n_tiles, num_sms());
  void* args[] = {&tx, &tq, &a};
  return launch_kernel_ex(fn, dim3(grid), dim3(kTcThreads), kTcSmem, st, false, args, "LUT3 GEMM launch");
}

// ----------------------------------------------------------------------------
// LUT3 x MXFP8 on the block-scaled FP8 tensor path
// ----------------------------------------------------------------------------

static lbq_status run_lut3_mx(const uint8_t* codes, const uint8_t* scales, int M, const void* image, const Layout& L,
                              void* Y, bool ybf16, void* ws, size_t ws_bytes, cudaStream_t st) {
  const uint8_t* img = static_cast<const uint8_t*>(image);
  const int cb_rows = std::min(16, L.N / 8);
  CUtensorMap tx, ts, tc, te, ty;
  if (!make_tmap_2d(&ty, Y, ybf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, (uint64_t)L.N,
                    (uint64_t)M, (uint64_t)L.N * 2, kMxBN, 32, CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_tmap_2d(&tx, codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)L.K, (uint64_t)M, (uint64_t)L.K, kMxBK,
                    kMxBM, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_2d(&ts, scales, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)L.K / 32, (uint64_t)M,
                    (uint64_t)L.K / 32, 16, kMxBM, CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_tmap_2d(&tc, img + L.off1, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)L.s_stride, (uint64_t)L.N / 8,
                    (uint64_t)L.s_stride, 16, (uint32_t)cb_rows, CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_tmap_2d(&te, img + L.off2, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)L.z_stride, (uint64_t)L.N / 8,
                    (uint64_t)L.z_stride, 16, (uint32_t)cb_rows, CU_TENSOR_MAP_SWIZZLE_NONE))
    return fail(LBQ_ERR_CUDA, "cuTensorMapEncodeTiled failed for the LUT3 x MXFP8 operands");
  GemmMxArgs a{};
  a.Y = Y;
  a.i_region = img + L.off0;
  a.M = M;
  a.N = L.N;
  a.K = L.K;
  a.n_tiles = (L.N + kMxBN - 1) / kMxBN;
  a.m_tiles = (M + kMxBM - 1) / kMxBM;
  a.k_blocks = L.K / kMxBK;
  a.cb_rows = cb_rows;
  a.y_bf16 = ybf16 ? 1 : 0;
  const void* fn = (const void*)gemm_mx_lut3_kernel;
  occupancy_for(fn, kMxThreads, kMxSmem);
  // the tile and k-block of the BF16-decode prefill: the same schedule and workspace
  static_assert(kMxBN == kTsBN && kMxBM == kTsBM && kMxBK == kTsBK, "one stream-K plan for both prefill GEMMs");
  const TsPlan p = plan_gemm_ts(M, L.K, L.N);
  const int grid = p.grid;
  a.sk = sk_args(p, a.n_tiles * a.m_tiles, ws, ws_bytes);
  void* args[] = {&tx, &ts, &tc, &te, &ty, &a};
  return launch_kernel_ex(fn, dim3(grid), dim3(kMxThreads), kMxSmem, st, false, args, "LUT3 x MXFP8 GEMM launch");
}

// ----------------------------------------------------------------------------
// Grouped MoE: LUT3 experts x MXFP8 activations
// ----------------------------------------------------------------------------

static int moe_max_padded(long long P, int E, int block) {
  const long long runs = std::min<long long>(P, E);
  return (int)((P + runs * (block - 1)) / block * block);
}

// ----------------------------------------------------------------------------
// Generic b-bit affine weights
// ----------------------------------------------------------------------------

static lbq_status check_affine_shape(int K, int N, int group, int bits) {
  if (bits < 1 || bits > 8) return fail(LBQ_ERR_UNSUPPORTED, "bits %d not in 1..8", bits);
  if (group != 32 && group != 64 && group != 128)
    return fail(LBQ_ERR_UNSUPPORTED, "group %d not in {32, 64, 128}", group);
  if (K <= 0 || N <= 0) return fail(LBQ_ERR_INVALID_ARG, "K=%d N=%d must be positive", K, N);
  if (K % group) return fail(LBQ_ERR_INVALID_ARG, "K=%d is not a multiple of group %d", K, group);
  return LBQ_OK;
}

static lbq_status check_affine_header(const ImageHeader& h, int K, int N, int group, int bits) {
  if (h.magic != kMagicAffine || h.version != kImageVersion)
    return fail(LBQ_ERR_INVALID_ARG, "not an lbq affine image of this version (magic 0x%08x version %u)", h.magic,
                h.version);
  if (h.K != K || h.N != N || h.group != group || h.bits != bits || h.mode != LBQ_MODE_AFFINE)
    return fail(LBQ_ERR_INVALID_ARG, "image holds K=%d N=%d group=%d bits=%d, call says K=%d N=%d group=%d bits=%d",
                h.K, h.N, h.group, h.bits, K, N, group, bits);
  return LBQ_OK;
}

// The bit-width x batch-tile kernel table: [x dtype][bits - 1][tile], tiles
// of 1, 2 and 4 rows of X (8, 4 and 2 output channels per row block).
#define LBQ_AG_TILES(B, BF) \
  { (const void*)affine_gemv_kernel<B, BF, 1>, (const void*)affine_gemv_kernel<B, BF, 2>, \
    (const void*)affine_gemv_kernel<B, BF, 4> }
#define LBQ_AG_BITS(BF) \
  { LBQ_AG_TILES(1, BF), LBQ_AG_TILES(2, BF), LBQ_AG_TILES(3, BF), LBQ_AG_TILES(4, BF), \
    LBQ_AG_TILES(5, BF), LBQ_AG_TILES(6, BF), LBQ_AG_TILES(7, BF), LBQ_AG_TILES(8, BF) }
static const void* const kAffineGemv[2][8][3] = {LBQ_AG_BITS(false), LBQ_AG_BITS(true)};
#undef LBQ_AG_BITS
#undef LBQ_AG_TILES

static lbq_status run_affine_gemv(const uint16_t* X, bool xbf16, int M, const uint8_t* image, const Layout& L,
                                  void* Y, bool ybf16, cudaStream_t st) {
  const int chunks = L.K / 32;
  const int nw = (chunks + 31) / 32;
  if (nw > kAgMaxWarps) return fail(LBQ_ERR_UNSUPPORTED, "affine GEMV needs K <= %d", 32 * 32 * kAgMaxWarps);
  const int T = nw * 32;
  const int smem = 2 * nw * 8 * (int)sizeof(float);
  for (int m0 = 0; m0 < M; m0 += 4) {
    const int mv = std::min(4, M - m0);
    const int tile = mv == 1 ? 0 : mv == 2 ? 1 : 2;
    const int R = 8 >> tile;
    const void* fn = kAffineGemv[xbf16 ? 1 : 0][L.bits - 1][tile];
    AffineGemvArgs a{};
    a.X = X + (size_t)m0 * L.K;
    a.Y = static_cast<uint8_t*>(Y) + (size_t)m0 * L.N * 2;
    a.q = image + L.off0;
    a.s = image + L.off1;
    a.z = image + L.off2;
    a.K = L.K; a.N = L.N; a.G = L.K / L.group; a.gshift = log2_exact(L.group / 32);
    a.m_valid = mv;
    a.row_blocks = (L.N + R - 1) / R;
    a.y_bf16 = ybf16 ? 1 : 0;
    const int occ = std::max(1, occupancy_for(fn, T, smem));
    const int grid = std::min(a.row_blocks, num_sms() * occ);
    void* args[] = {&a};
    lbq_status s = launch_kernel_ex(fn, dim3(grid), dim3(T), smem, st, g_pdl != 0, args, "affine GEMV launch");
    if (s != LBQ_OK) return s;
  }
  return LBQ_OK;
}

// ----------------------------------------------------------------------------
// W4A8: INT4 weights x dynamic INT8 activations
// ----------------------------------------------------------------------------

static int g_w4a8_tiled = 0;  // test hook: batch-1 W4A8 on the tiled kernel instead of the staged one

// [asym][tile of 1, 2, 4 rows of X]
static const void* const kW4a8Gemv[2][3] = {
    {(const void*)w4a8_gemv_kernel<false, 1>, (const void*)w4a8_gemv_kernel<false, 2>,
     (const void*)w4a8_gemv_kernel<false, 4>},
    {(const void*)w4a8_gemv_kernel<true, 1>, (const void*)w4a8_gemv_kernel<true, 2>,
     (const void*)w4a8_gemv_kernel<true, 4>}};

static lbq_status run_w4a8_gemv(const int8_t* XQ, const float* SX, int M, const uint8_t* image, const Layout& L,
                                void* Y, bool ybf16, cudaStream_t st) {
  const int chunks = L.K / 32;
  const int nw = (chunks + 31) / 32;
  if (nw > kW8MaxWarps) return fail(LBQ_ERR_UNSUPPORTED, "W4A8 GEMV needs K <= %d", 32 * 32 * kW8MaxWarps);
  const int T = nw * 32;
  const int smem = 2 * nw * 8 * (int)sizeof(float);
  const bool asym = L.mode == LBQ_MODE_ASYM;
  for (int m0 = 0; m0 < M; m0 += 4) {
    const int mv = std::min(4, M - m0);
    const int tile = mv == 1 ? 0 : mv == 2 ? 1 : 2;
    const int R = 8 >> tile;
    const void* fn = kW4a8Gemv[asym ? 1 : 0][tile];
    W4a8Args a{};
    a.XQ = XQ + (size_t)m0 * L.K;
    a.SX = SX + (size_t)m0 * (L.K / 32);
    a.Y = static_cast<uint8_t*>(Y) + (size_t)m0 * L.N * 2;
    a.q = image + L.off0;
    a.s = image + L.off1;
    a.z = asym ? image + L.off2 : nullptr;
    a.K = L.K; a.N = L.N; a.G = L.K / L.group; a.gshift = log2_exact(L.group / 32);
    a.m_valid = mv;
    a.row_blocks = (L.N + R - 1) / R;
    a.y_bf16 = ybf16 ? 1 : 0;
    const int occ = std::max(1, occupancy_for(fn, T, smem));
    const int grid = std::min(a.row_blocks, num_sms() * occ);
    void* args[] = {&a};
    lbq_status s = launch_kernel_ex(fn, dim3(grid), dim3(T), smem, st, g_pdl != 0, args, "W4A8 GEMV launch");
    if (s != LBQ_OK) return s;
  }
  return LBQ_OK;
}

static lbq_status check_w4a8_args(const int8_t* xq, const float* sx, int M, const void* image, void* Y, int y_dtype) {
  if (!xq || !sx || !image || !Y) return fail(LBQ_ERR_INVALID_ARG, "xq, sx, image and Y must be non-null");
  if (!aligned16(xq) || !aligned16(image) || !aligned16(Y) || (reinterpret_cast<uintptr_t>(sx) & 3u))
    return fail(LBQ_ERR_INVALID_ARG, "xq, image and Y must be 16-byte aligned, sx 4-byte aligned");
  if (y_dtype != LBQ_DTYPE_F16 && y_dtype != LBQ_DTYPE_BF16) return fail(LBQ_ERR_UNSUPPORTED, "y_dtype %d", y_dtype);
  if (M <= 0) return fail(LBQ_ERR_INVALID_ARG, "M=%d must be positive", M);
  return LBQ_OK;
}

static lbq_status check_compute_args(const void* X, int x_dtype, int M, const void* image, void* Y, int y_dtype) {
  if (!X || !image || !Y) return fail(LBQ_ERR_INVALID_ARG, "X, image and Y must be non-null");
  if (!aligned16(X) || !aligned16(image) || !aligned16(Y))
    return fail(LBQ_ERR_INVALID_ARG, "X, image and Y must be 16-byte aligned");
  if (x_dtype != LBQ_DTYPE_F16 && x_dtype != LBQ_DTYPE_BF16) return fail(LBQ_ERR_UNSUPPORTED, "x_dtype %d", x_dtype);
  if (y_dtype != LBQ_DTYPE_F16 && y_dtype != LBQ_DTYPE_BF16) return fail(LBQ_ERR_UNSUPPORTED, "y_dtype %d", y_dtype);
  if (M <= 0) return fail(LBQ_ERR_INVALID_ARG, "M=%d must be positive", M);
  return LBQ_OK;
}

// ----------------------------------------------------------------------------
// Fixed scratch for lbq_gemv_noalloc
// ----------------------------------------------------------------------------
//
// Some callers cannot hand the library a workspace: a C program with no device
// allocator of its own, or a serving process whose device memory is carved up
// once at start-up and must not grow (or fragment) while requests are served.
// For them the split-K partial sums and tile counters of the GEMV live in this
// module-level array, which the CUDA runtime places when it loads the module;
// no call ever allocates or frees device memory.

constexpr size_t kNoAllocScratchBytes = (size_t)8 << 20;  // 8 MiB per device
constexpr int kNoAllocMaxDevices = 64;

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch on the current device. Outside stream
// capture it is looked up on every call (cheap once the module is loaded), so
// a module reloaded after cudaDeviceReset is found at its new address; while
// `stream` is being captured the address of the last uncaptured call on this
// device is used, because the first lookup may load the module, which capture
// does not allow.
static uint8_t* noalloc_scratch(cudaStream_t stream, lbq_status* st) {
  static std::mutex mu;
  static uint8_t* ptr[kNoAllocMaxDevices] = {};
  int dev = 0;
  if ((*st = cuda_check(cudaGetDevice(&dev), "cudaGetDevice")) != LBQ_OK) return nullptr;
  if (dev < 0 || dev >= kNoAllocMaxDevices) {
    *st = fail(LBQ_ERR_UNSUPPORTED, "device %d is beyond the %d devices the fixed scratch supports", dev,
               kNoAllocMaxDevices);
    return nullptr;
  }
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if ((*st = cuda_check(cudaStreamIsCapturing(stream, &cap), "cudaStreamIsCapturing")) != LBQ_OK) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (cap == cudaStreamCaptureStatusNone) {
    void* p = nullptr;
    if ((*st = cuda_check(cudaGetSymbolAddress(&p, g_noalloc_scratch), "cudaGetSymbolAddress of the fixed scratch")) !=
        LBQ_OK)
      return nullptr;
    ptr[dev] = static_cast<uint8_t*>(p);
  } else if (ptr[dev] == nullptr) {
    *st = fail(LBQ_ERR_INVALID_ARG,
               "lbq_gemv_noalloc: the first call on a device must come before any stream capture (it looks up the "
               "fixed scratch's address)");
    return nullptr;
  }
  *st = LBQ_OK;
  return ptr[dev];
}

}  // namespace lbq

using namespace lbq;

extern "C" {

const char* lbq_last_error(void) { return g_last_error.c_str(); }

int lbq_version(void) { return 100; }

uint64_t lbq_launch_count(void) { return g_launches.load(); }

// Test hook (not in the public header): force the split-K count of the M = 1
// GEMV; 0 restores the shape-based choice.
void lbq_debug_force_splits(int splits) { g_force_splits = splits < 0 ? 0 : splits; }

// Test hook (not in the public header): route every lbq_gemm call, any M, to
// the tcgen05 prefill kernel.
void lbq_debug_force_tc(int on) { g_force_tc = on ? 1 : 0; }

// Test hook (not in the public header): route M = 1 through the skinny kernel.
void lbq_debug_force_skinny(int on) { g_force_skinny = on ? 1 : 0; }

// Test hook (not in the public header): pick the prefill kernel (0 = weights in
// tensor memory, 1 = weights dequantised into shared memory).
void lbq_debug_gemm_path(int path) { g_gemm_path = path == 1 ? 1 : 0; }

// Test hook (not in the public header): pick the GEMV kernel for M <= 16
// (0 = the library's choice, 1 = TMA-pipelined CUDA-core M = 1, 2 = warp MMA,
// 3 = tcgen05, 4 = direct-load CUDA-core M = 1, 5 = TMA-fed warp-MMA M = 1).
void lbq_debug_gemv_path(int path) { g_gemv_path = (path >= 0 && path <= 5) ? path : 0; }

// Test hook (not in the public header): when the TMA-fed warp-MMA kernel is
// the batch-1 choice: 0 never, 1 always, 2 (and any other value: the library's
// default) for launches of at least 4 16-row tiles per SM with K <= 4096.
void lbq_debug_tmma_default(int mode) { g_tmma_default = (mode >= 0 && mode <= 2) ? mode : 2; }

// Test hook (not in the public header): force the TMA-fed kernel's K split
// (1, 2 or 4 ranges; 0 = the plan's choice). A forced split that the shape
// cannot take leaves the kernel without a plan (the call then fails).
void lbq_debug_tmma_split(int r) { g_tmma_split = (r == 1 || r == 2 || r == 4) ? r : 0; }

// Test hook (not in the public header): the next TMA-fed GEMV launches issue
// no copies, so every consumer wait runs out (after a short spin limit); the
// kernel returns without writing Y and raises the device flag that
// lbq_device_status() reports. No copy is in flight when the CTA exits.
void lbq_debug_drop_copies(int on) { g_debug_drop = on ? 1 : 0; }

// Test hook (not in the public header): direct batch-1 kernel variant
// (-1 = the library's choice, 0 = weights pipelined through registers, 2..4 =
// staged through shared memory with that many row blocks in flight) and a cap
// on resident CTAs per SM.
void lbq_debug_direct_variant(int variant, int ctas_per_sm) {
  g_direct_stages = (variant == 0 || (variant >= 2 && variant <= 4)) ? variant : -1;
  g_direct_ctas = ctas_per_sm > 0 ? ctas_per_sm : 0;
}

// Test hook (not in the public header): batch-1 lbq_w4a8_gemv on the tiled
// W4A8 kernel (the one for M > 1) instead of the staged direct kernel.
void lbq_debug_w4a8_tiled(int on) { g_w4a8_tiled = on ? 1 : 0; }

// Test hook (not in the public header): ring stages of the TMA-fed LUT3
// batch-1 kernel (1..16, capped by the CTA's units and shared memory; 0 = the
// plan's choice).
void lbq_debug_lut3_stages(int stages) { g_l3t_stages = (stages >= 1 && stages <= kL3tMaxStages) ? stages : 0; }

// Test hook (not in the public header): 1 = LUT3 at M = 2..8 on the skinny
// kernel instead of the TMA-fed batch kernel (0 = the library's choice).
void lbq_debug_lut3_batch_off(int on) { g_l3b_off = on ? 1 : 0; }

// Test hook (not in the public header): prefill stream-K on (1, the library's
// choice) or off (0: whole tiles, as without a workspace).
void lbq_debug_gemm_stream_k(int on) { g_ts_stream_k = on ? 1 : 0; }

// Test hook (not in the public header): with polls > 0 the prefill's later
// parts never raise their flag and each earlier part gives up after `polls`
// waits of about 1 us: it writes nothing and raises the device flag that
// lbq_device_status() reports. polls = 0 restores the library's behaviour.
void lbq_debug_gemm_hold(int polls) {
  g_ts_hold = polls > 0 ? 1 : 0;
  g_ts_polls = polls > 0 ? (uint32_t)polls : 0u;
}

// Test hook (not in the public header): the prefill schedule of CTA `cta` for
// this shape, as the kernel walks it. Writes up to `max_items` items as
// (tile, kb0, kb1, part) int quadruples to `items` (host) and returns the
// item count; *grid receives the grid size, *k_blocks the 128-k blocks per tile.
int lbq_debug_gemm_schedule(int M, int K, int N, int stream_k, int cta, int* grid, int* k_blocks, int* items,
                            int max_items) {
  const TsPlan p = plan_gemm_ts(M, K, N);
  const int nkb = (K + kTsBK - 1) / kTsBK;
  *grid = p.grid;
  *k_blocks = nkb;
  const bool sk = stream_k && p.ws_bytes;
  SkSched sch(sk ? p.dp_tiles : ((N + kTsBN - 1) / kTsBN) * ((M + kTsBM - 1) / kTsBM), sk ? p.sk_items : 0, nkb,
              cta, p.grid);
  SkItem w;
  int n = 0;
  while (sch.next(w)) {
    if (n < max_items) {
      items[4 * n] = w.tile;
      items[4 * n + 1] = w.kb0;
      items[4 * n + 2] = w.kb1;
      items[4 * n + 3] = w.part;
    }
    ++n;
  }
  return n;
}

// Test hook (not in the public header): the (channel tile, token tile) of a
// prefill tile index in the banded order the kernel uses.
void lbq_debug_tile_coords(int tile, int n_tiles, int m_tiles, int* nt, int* mt) {
  sk_tile_coords(tile, n_tiles, m_tiles, *nt, *mt);
}

lbq_status lbq_set_option(int option, int value) {
  if (option == LBQ_OPT_PDL) {
    g_pdl = value ? 1 : 0;
    return LBQ_OK;
  }
  return fail(LBQ_ERR_INVALID_ARG, "unknown option %d", option);
}

lbq_status lbq_packed_size(int K, int N, int group, int mode, size_t* bytes) {
  if (!bytes) return fail(LBQ_ERR_INVALID_ARG, "bytes must be non-null");
  lbq_status st = mode == LBQ_MODE_LUT3 ? check_lut3_shape(K, N) : check_int4_shape(K, N, group, mode);
  if (st != LBQ_OK) return st;
  *bytes = make_layout(K, N, mode == LBQ_MODE_LUT3 ? 0 : group, mode).total;
  return LBQ_OK;
}

lbq_status lbq_pack(const float* W, int K, int N, int group, int mode, void* image, size_t image_bytes, void* stream) {
  lbq_status st = check_int4_shape(K, N, group, mode);
  if (st != LBQ_OK) return st;
  if (!W || !image) return fail(LBQ_ERR_INVALID_ARG, "W and image must be non-null");
  if (!aligned16(W) || !aligned16(image)) return fail(LBQ_ERR_INVALID_ARG, "W and image must be 16-byte aligned");
  const Layout L = make_layout(K, N, group, mode);
  if (image_bytes < L.total) return fail(LBQ_ERR_INVALID_ARG, "image buffer %zu bytes < %zu needed", image_bytes, L.total);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* img = static_cast<uint8_t*>(image);
  write_header_kernel<<<1, 32, 0, s>>>(make_header(L), reinterpret_cast<ImageHeader*>(img));
  if ((st = launch_check("header launch")) != LBQ_OK) return st;
  // zero the scale / zero-point regions so their row padding is deterministic
  if ((st = cuda_check(cudaMemsetAsync(img + L.off1, 0, L.total - L.off1, s), "clearing the scale regions")) != LBQ_OK)
    return st;
  const long long work = (long long)(K / group) * N;
  const int block = 256;
  const unsigned grid = (unsigned)((work + block - 1) / block);
  if (mode == LBQ_MODE_SYM)
    quantize_pack_int4_kernel<false><<<grid, block, 0, s>>>(W, K, N, group, img + L.off0, img + L.off1, nullptr);
  else
    quantize_pack_int4_kernel<true><<<grid, block, 0, s>>>(W, K, N, group, img + L.off0, img + L.off1, img + L.off2);
  return launch_check("quantize_pack launch");
}

lbq_status lbq_pack_lut3(const uint8_t* idx, const uint8_t* codebooks, const uint8_t* exponents, int K, int N,
                         void* image, size_t image_bytes, void* stream) {
  lbq_status st = check_lut3_shape(K, N);
  if (st != LBQ_OK) return st;
  if (!idx || !codebooks || !exponents || !image)
    return fail(LBQ_ERR_INVALID_ARG, "idx, codebooks, exponents and image must be non-null");
  if (!aligned16(image)) return fail(LBQ_ERR_INVALID_ARG, "image must be 16-byte aligned");
  const Layout L = make_layout(K, N, 0, LBQ_MODE_LUT3);
  if (image_bytes < L.total) return fail(LBQ_ERR_INVALID_ARG, "image buffer %zu bytes < %zu needed", image_bytes, L.total);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* img = static_cast<uint8_t*>(image);
  write_header_kernel<<<1, 32, 0, s>>>(make_header(L), reinterpret_cast<ImageHeader*>(img));
  if ((st = launch_check("header launch")) != LBQ_OK) return st;
  if ((st = cuda_check(cudaMemsetAsync(img + L.off1, 0, L.total - L.off1, s), "clearing the table regions")) != LBQ_OK)
    return st;
  const long long work = (long long)(K / 64) * N;
  pack_lut3_kernel<<<(unsigned)((work + 255) / 256), 256, 0, s>>>(idx, codebooks, exponents, K, N, img + L.off0,
                                                                  img + L.off1, img + L.off2, img + L.off3);
  return launch_check("pack_lut3 launch");
}

lbq_status lbq_workspace_size(int op, int M, int K, int N, int group, int mode, size_t* bytes) {
  if (!bytes) return fail(LBQ_ERR_INVALID_ARG, "bytes must be non-null");
  *bytes = 0;
  if (op == 0 || op == 1) {
    lbq_status st = check_int4_shape(K, N, group, mode);
    if (st != LBQ_OK) return st;
    if (M <= 0) return fail(LBQ_ERR_INVALID_ARG, "M must be positive");
    if (op == 1 && g_force_tc) return LBQ_OK;  // the alternative tensor-core GEMM needs no workspace
    if (op == 1 && M > 16) {  // the prefill GEMM: stream-K's flags and parked tiles, where it cuts tiles
      *bytes = plan_gemm_ts(M, K, N).ws_bytes;
      return LBQ_OK;
    }
    if (M <= 16) {
      // the plan may depend on the activation dtype through a kernel's
      // occupancy; take the larger of the two
      const bool asym = mode == LBQ_MODE_ASYM;
      *bytes = std::max(gemv_scratch(M, K, N, group, asym, false).need, gemv_scratch(M, K, N, group, asym, true).need);
    }
    return LBQ_OK;
  }
  if (op == 2) {
    lbq_status st = check_lut3_shape(K, N);
    if (st != LBQ_OK) return st;
    if (M <= 0) return fail(LBQ_ERR_INVALID_ARG, "M must be positive");
    if (M <= 16 && !g_force_tc && !lut3_direct_ok(M, K)) *bytes = skinny_workspace_bytes(plan_lut3(K, N, M), M);
    if (M > 16 && !g_force_tc) *bytes = plan_gemm_ts(M, K, N).ws_bytes;
    return LBQ_OK;
  }
  return fail(LBQ_ERR_INVALID_ARG, "op %d not in {0, 1, 2}", op);
}

lbq_status lbq_gemv(const void* X, int x_dtype, int M, int K, int N, int group, int mode, const void* image, void* Y,
                    int y_dtype, void* ws, size_t ws_bytes, void* stream) {
  lbq_status st = check_int4_shape(K, N, group, mode);
  if (st != LBQ_OK) return st;
  if ((st = check_compute_args(X, x_dtype, M, image, Y, y_dtype)) != LBQ_OK) return st;
  if (M > 16) return fail(LBQ_ERR_UNSUPPORTED, "lbq_gemv takes M <= 16 (M=%d); use lbq_gemm", M);
  const Layout L = make_layout(K, N, group, mode);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int path = gemv_path(M, K, N);
  if (path == kPathDirect || path == kPathTmma) {
    const lbq_gemv_item item{X, image, Y, N};
    if (path == kPathTmma)
      return run_tmma(&item, 1, K, group, mode, x_dtype == LBQ_DTYPE_BF16, y_dtype == LBQ_DTYPE_BF16, ws, ws_bytes,
                      s);
    return run_direct(&item, 1, K, group, mode, x_dtype == LBQ_DTYPE_BF16, y_dtype == LBQ_DTYPE_BF16, s);
  }
  if (path == kPathM1)
    return run_m1(static_cast<const uint16_t*>(X), x_dtype == LBQ_DTYPE_BF16, image, L, Y, y_dtype == LBQ_DTYPE_BF16,
                  ws, ws_bytes, s);
  if (path == kPathMma)
    return run_skinny(X, x_dtype == LBQ_DTYPE_BF16, M, image, L, Y, y_dtype == LBQ_DTYPE_BF16, ws, ws_bytes, s);
  return run_tcgemv(X, x_dtype == LBQ_DTYPE_BF16, M, image, L, Y, y_dtype == LBQ_DTYPE_BF16, ws, ws_bytes, s);
}

lbq_status lbq_gemm(const void* X, int x_dtype, int M, int K, int N, int group, int mode, const void* image, void* Y,
                    int y_dtype, void* ws, size_t ws_bytes, void* stream) {
  if (M <= 16 && !g_force_tc) return lbq_gemv(X, x_dtype, M, K, N, group, mode, image, Y, y_dtype, ws, ws_bytes, stream);
  lbq_status st = check_int4_shape(K, N, group, mode);
  if (st != LBQ_OK) return st;
  if ((st = check_compute_args(X, x_dtype, M, image, Y, y_dtype)) != LBQ_OK) return st;
  if (g_gemm_path == 0)
    return run_gemm_ts(X, x_dtype == LBQ_DTYPE_BF16, M, image, make_layout(K, N, group, mode), Y,
                       y_dtype == LBQ_DTYPE_BF16, ws, ws_bytes, static_cast<cudaStream_t>(stream));
  return run_gemm_tc(X, x_dtype == LBQ_DTYPE_BF16, M, image, make_layout(K, N, group, mode), Y,
                     y_dtype == LBQ_DTYPE_BF16, static_cast<cudaStream_t>(stream));
}

lbq_status lbq_lut3_gemm(const void* X, int x_dtype, int M, int K, int N, const void* image, void* Y, int y_dtype,
                         void* ws, size_t ws_bytes, void* stream) {
  lbq_status st = check_lut3_shape(K, N);
  if (st != LBQ_OK) return st;
  if ((st = check_compute_args(X, x_dtype, M, image, Y, y_dtype)) != LBQ_OK) return st;
  if (x_dtype != LBQ_DTYPE_BF16) return fail(LBQ_ERR_UNSUPPORTED, "LUT3 kernels take BF16 activations");
  const Layout L = make_layout(K, N, 0, LBQ_MODE_LUT3);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (lut3_tmma_ok(M, K, N, X, image) && !g_force_tc) return run_lut3_tmma(X, image, L, Y, y_dtype == LBQ_DTYPE_BF16, s);
  if (lut3_direct_ok(M, K) && !g_force_tc) return run_lut3_direct(X, image, L, Y, y_dtype == LBQ_DTYPE_BF16, s);
  if (lut3_batch_ok(M, K, N, X, image) && !g_force_tc)
    return run_lut3_batch(X, M, image, L, Y, y_dtype == LBQ_DTYPE_BF16, s);
  if (M <= 16 && !g_force_tc) return run_lut3_skinny(X, M, image, L, Y, y_dtype == LBQ_DTYPE_BF16, ws, ws_bytes, s);
  if (g_gemm_path == 0) return run_gemm_ts(X, true, M, image, L, Y, y_dtype == LBQ_DTYPE_BF16, ws, ws_bytes, s);
  return run_lut3_gemm_tc(X, M, image, L, Y, y_dtype == LBQ_DTYPE_BF16, s);
}

lbq_status lbq_unpack_canonical(const void* image, int K, int N, int group, int mode, uint8_t* q_packed,
                                uint16_t* scales, int8_t* zp, void* stream) {
  lbq_status st = check_int4_shape(K, N, group, mode);
  if (st != LBQ_OK) return st;
  if (!image || !q_packed || !scales) return fail(LBQ_ERR_INVALID_ARG, "image, q_packed and scales must be non-null");
  if (mode == LBQ_MODE_ASYM && !zp) return fail(LBQ_ERR_INVALID_ARG, "zp must be non-null for ASYM");
  ImageHeader h;
  if ((st = read_header(image, &h)) != LBQ_OK) return st;
  if ((st = check_header(h, K, N, group, mode)) != LBQ_OK) return st;
  const Layout L = make_layout(K, N, group, mode);
  const uint8_t* img = static_cast<const uint8_t*>(image);
  const long long work = (long long)(K / 2) * N;
  unpack_int4_kernel<<<(unsigned)((work + 255) / 256), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      img + L.off0, img + L.off1, mode == LBQ_MODE_ASYM ? img + L.off2 : nullptr, K, N, group, q_packed, scales,
      mode == LBQ_MODE_ASYM ? zp : nullptr);
  return launch_check("unpack launch");
}

lbq_status lbq_unpack_lut3_canonical(const void* image, int K, int N, uint8_t* idx_stream, uint8_t* codebooks,
                                     uint8_t* exponents, void* stream) {
  lbq_status st = check_lut3_shape(K, N);
  if (st != LBQ_OK) return st;
  if (!image || !idx_stream || !codebooks || !exponents)
    return fail(LBQ_ERR_INVALID_ARG, "image, idx_stream, codebooks and exponents must be non-null");
  ImageHeader h;
  if ((st = read_header(image, &h)) != LBQ_OK) return st;
  if ((st = check_header(h, K, N, 0, LBQ_MODE_LUT3)) != LBQ_OK) return st;
  const Layout L = make_layout(K, N, 0, LBQ_MODE_LUT3);
  const uint8_t* img = static_cast<const uint8_t*>(image);
  const long long work = (long long)(K / 64) * N;
  unpack_lut3_kernel<<<(unsigned)((work + 255) / 256), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      img + L.off0, img + L.off1, img + L.off2, K, N, idx_stream, codebooks, exponents);
  return launch_check("unpack_lut3 launch");
}

lbq_status lbq_dequant(const void* image, int K, int N, int group, int mode, float* W_out, void* stream) {
  lbq_status st = mode == LBQ_MODE_LUT3 ? check_lut3_shape(K, N) : check_int4_shape(K, N, group, mode);
  if (st != LBQ_OK) return st;
  if (!image || !W_out) return fail(LBQ_ERR_INVALID_ARG, "image and W_out must be non-null");
  ImageHeader h;
  if ((st = read_header(image, &h)) != LBQ_OK) return st;
  if ((st = check_header(h, K, N, group, mode)) != LBQ_OK) return st;
  if (mode == LBQ_MODE_LUT3) {
    const Layout L = make_layout(K, N, 0, LBQ_MODE_LUT3);
    const uint8_t* img = static_cast<const uint8_t*>(image);
    const long long work = (long long)K * N;
    dequant_lut3_kernel<<<(unsigned)((work + 255) / 256), 256, 0, static_cast<cudaStream_t>(stream)>>>(
        img + L.off0, img + L.off1, img + L.off2, K, N, W_out);
    return launch_check("dequant_lut3 launch");
  }
  const Layout L = make_layout(K, N, group, mode);
  const uint8_t* img = static_cast<const uint8_t*>(image);
  const long long work = (long long)K * N;
  dequant_int4_kernel<<<(unsigned)((work + 255) / 256), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      img + L.off0, img + L.off1, mode == LBQ_MODE_ASYM ? img + L.off2 : nullptr, K, N, group, W_out);
  return launch_check("dequant launch");
}

lbq_status lbq_affine_packed_size(int K, int N, int group, int bits, size_t* bytes) {
  if (!bytes) return fail(LBQ_ERR_INVALID_ARG, "bytes must be non-null");
  lbq_status st = check_affine_shape(K, N, group, bits);
  if (st != LBQ_OK) return st;
  *bytes = make_layout(K, N, group, LBQ_MODE_AFFINE, bits).total;
  return LBQ_OK;
}

lbq_status lbq_pack_affine(const float* W, int K, int N, int group, int bits, void* image, size_t image_bytes,
                           void* stream) {
  lbq_status st = check_affine_shape(K, N, group, bits);
  if (st != LBQ_OK) return st;
  if (!W || !image) return fail(LBQ_ERR_INVALID_ARG, "W and image must be non-null");
  if (!aligned16(W) || !aligned16(image)) return fail(LBQ_ERR_INVALID_ARG, "W and image must be 16-byte aligned");
  const Layout L = make_layout(K, N, group, LBQ_MODE_AFFINE, bits);
  if (image_bytes < L.total) return fail(LBQ_ERR_INVALID_ARG, "image buffer %zu bytes < %zu needed", image_bytes, L.total);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* img = static_cast<uint8_t*>(image);
  write_header_kernel<<<1, 32, 0, s>>>(make_header(L), reinterpret_cast<ImageHeader*>(img));
  if ((st = launch_check("header launch")) != LBQ_OK) return st;
  if ((st = cuda_check(cudaMemsetAsync(img + L.off1, 0, L.total - L.off1, s), "clearing the scale regions")) != LBQ_OK)
    return st;
  const long long work = (long long)(K / group) * N;
  quantize_pack_affine_kernel<<<(unsigned)((work + 255) / 256), 256, 0, s>>>(W, K, N, group, bits, img + L.off0,
                                                                           img + L.off1, img + L.off2);
  return launch_check("quantize_pack_affine launch");
}

lbq_status lbq_affine_gemv(const void* X, int x_dtype, int M, int K, int N, int group, int bits, const void* image,
                           void* Y, int y_dtype, void* stream) {
  lbq_status st = check_affine_shape(K, N, group, bits);
  if (st != LBQ_OK) return st;
  if ((st = check_compute_args(X, x_dtype, M, image, Y, y_dtype)) != LBQ_OK) return st;
  if (M > 16) return fail(LBQ_ERR_UNSUPPORTED, "lbq_affine_gemv takes 1 <= M <= 16 (M=%d)", M);
  const Layout L = make_layout(K, N, group, LBQ_MODE_AFFINE, bits);
  // 4-bit codes: the image's chunks, scales and zero points are byte for byte
  // the asymmetric INT4 image (pair-split nibbles = the INT4 slot order, same
  // region offsets), so batch 1 runs on the INT4 GEMVs (none of them needs a
  // workspace at batch 1 when the TMA-fed kernel takes the whole K range)
  if (bits == 4 && M == 1 && K <= 32 * 32 * kGdMaxWarps) {
    const lbq_gemv_item item{X, image, Y, N};
    const bool xbf16 = x_dtype == LBQ_DTYPE_BF16, ybf16 = y_dtype == LBQ_DTYPE_BF16;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (tmma_ok(1, K, &N, 1) && tmma_preferred(K, &N, 1) && plan_tmma(K, &N, 1, group, true, false).nsl > 0)
      return run_tmma(&item, 1, K, group, LBQ_MODE_ASYM, xbf16, ybf16, nullptr, 0, s, false);
    return run_direct(&item, 1, K, group, LBQ_MODE_ASYM, xbf16, ybf16, s);
  }
  return run_affine_gemv(static_cast<const uint16_t*>(X), x_dtype == LBQ_DTYPE_BF16, M,
                         static_cast<const uint8_t*>(image), L, Y, y_dtype == LBQ_DTYPE_BF16,
                         static_cast<cudaStream_t>(stream));
}

lbq_status lbq_unpack_affine_canonical(const void* image, int K, int N, int group, int bits, uint8_t* q_stream,
                                       uint16_t* scales, int8_t* zp, void* stream) {
  lbq_status st = check_affine_shape(K, N, group, bits);
  if (st != LBQ_OK) return st;
  if (!image || !q_stream || !scales || !zp)
    return fail(LBQ_ERR_INVALID_ARG, "image, q_stream, scales and zp must be non-null");
  ImageHeader h;
  if ((st = read_header(image, &h)) != LBQ_OK) return st;
  if ((st = check_affine_header(h, K, N, group, bits)) != LBQ_OK) return st;
  const Layout L = make_layout(K, N, group, LBQ_MODE_AFFINE, bits);
  const uint8_t* img = static_cast<const uint8_t*>(image);
  const long long work = (long long)(K / 8) * bits * N;
  unpack_affine_kernel<<<(unsigned)((work + 255) / 256), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      img + L.off0, img + L.off1, img + L.off2, K, N, group, bits, q_stream, scales, zp);
  return launch_check("unpack_affine launch");
}

lbq_status lbq_quantize_int8(const void* X, int x_dtype, int M, int K, int8_t* xq, float* sx, void* stream) {
  if (!X || !xq || !sx) return fail(LBQ_ERR_INVALID_ARG, "X, xq and sx must be non-null");
  if (!aligned16(X) || !aligned16(xq)) return fail(LBQ_ERR_INVALID_ARG, "X and xq must be 16-byte aligned");
  if (x_dtype != LBQ_DTYPE_F16 && x_dtype != LBQ_DTYPE_BF16) return fail(LBQ_ERR_UNSUPPORTED, "x_dtype %d", x_dtype);
  if (M <= 0 || K <= 0 || K % 32) return fail(LBQ_ERR_INVALID_ARG, "M=%d K=%d: need M > 0 and K a positive multiple of 32", M, K);
  const long long warps = (long long)M * (K / 32);  // one warp per 32-k block
  const unsigned grid = (unsigned)((warps * 32 + 255) / 256);
  const void* fn = x_dtype == LBQ_DTYPE_BF16 ? (const void*)quantize_int8_kernel<true>
                                             : (const void*)quantize_int8_kernel<false>;
  const uint16_t* Xp = static_cast<const uint16_t*>(X);
  void* args[] = {(void*)&Xp, (void*)&M, (void*)&K, (void*)&xq, (void*)&sx};
  return launch_kernel_ex(fn, dim3(grid), dim3(256), 0, static_cast<cudaStream_t>(stream), g_pdl != 0, args,
                          "quantize_int8 launch");
}

lbq_status lbq_w4a8_gemv_grouped(const lbq_w4a8_item* items, int count, int K, int group, int mode, int y_dtype,
                                 void* stream) {
  if (!items || count < 1 || count > kGdMaxItems) return fail(LBQ_ERR_INVALID_ARG, "count=%d not in 1..%d", count, kGdMaxItems);
  lbq_status st;
  lbq_gemv_item gi[kGdMaxItems];
  const float* sx[kGdMaxItems];
  for (int i = 0; i < count; ++i) {
    if ((st = check_int4_shape(K, items[i].N, group, mode)) != LBQ_OK) return st;
    if ((st = check_w4a8_args(items[i].xq, items[i].sx, 1, items[i].image, items[i].Y, y_dtype)) != LBQ_OK) return st;
    gi[i] = lbq_gemv_item{items[i].xq, items[i].image, items[i].Y, items[i].N};
    sx[i] = items[i].sx;
  }
  return run_direct(gi, count, K, group, mode, false, y_dtype == LBQ_DTYPE_BF16, static_cast<cudaStream_t>(stream), sx);
}

lbq_status lbq_w4a8_gemv(const int8_t* xq, const float* sx, int M, int K, int N, int group, int mode,
                         const void* image, void* Y, int y_dtype, void* stream) {
  lbq_status st = check_int4_shape(K, N, group, mode);
  if (st != LBQ_OK) return st;
  if ((st = check_w4a8_args(xq, sx, M, image, Y, y_dtype)) != LBQ_OK) return st;
  if (M > 16) return fail(LBQ_ERR_UNSUPPORTED, "lbq_w4a8_gemv takes 1 <= M <= 16 (M=%d)", M);
  if (M == 1 && !g_w4a8_tiled) {
    const lbq_gemv_item item{xq, image, Y, N};
    return run_direct(&item, 1, K, group, mode, false, y_dtype == LBQ_DTYPE_BF16, static_cast<cudaStream_t>(stream),
                      &sx);
  }
  const Layout L = make_layout(K, N, group, mode);
  return run_w4a8_gemv(xq, sx, M, static_cast<const uint8_t*>(image), L, Y, y_dtype == LBQ_DTYPE_BF16,
                       static_cast<cudaStream_t>(stream));
}

lbq_status lbq_device_status(void* stream) {
  lbq_status st = cuda_check(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)), "stream synchronize");
  if (st != LBQ_OK) return st;
  unsigned int v = 0;
  const unsigned int zero = 0;
  if ((st = cuda_check(cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v)), "reading the device flag")) != LBQ_OK) return st;
  if (v == 0) return LBQ_OK;
  if ((st = cuda_check(cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero)), "clearing the device flag")) != LBQ_OK) return st;
  return fail(LBQ_ERR_DEVICE, "a kernel reported device error flags 0x%x", v);
}

lbq_status lbq_gemv_grouped(const lbq_gemv_item* items, int count, int K, int group, int mode, int x_dtype,
                            int y_dtype, void* stream) {
  if (!items) return fail(LBQ_ERR_INVALID_ARG, "items must be non-null");
  if (count < 1 || count > kGdMaxItems) return fail(LBQ_ERR_INVALID_ARG, "count=%d not in 1..%d", count, kGdMaxItems);
  if (K > 32 * 32 * kGdMaxWarps) return fail(LBQ_ERR_UNSUPPORTED, "lbq_gemv_grouped needs K <= %d", 32 * 32 * kGdMaxWarps);
  for (int i = 0; i < count; ++i) {
    lbq_status st = check_int4_shape(K, items[i].N, group, mode);
    if (st != LBQ_OK) return st;
    if ((st = check_compute_args(items[i].X, x_dtype, 1, items[i].image, items[i].Y, y_dtype)) != LBQ_OK) return st;
  }
  int Ns[kGdMaxItems];
  for (int i = 0; i < count; ++i) Ns[i] = items[i].N;
  const bool tmma = (g_gemv_path == kPathTmma || (g_gemv_path == kPathAuto && tmma_preferred(K, Ns, count))) &&
                    tmma_ok(1, K, Ns, count) && count <= kTmMaxItems &&
                    plan_tmma(K, Ns, count, group, mode == LBQ_MODE_ASYM, false).nsl > 0;
  if (tmma)
    return run_tmma(items, count, K, group, mode, x_dtype == LBQ_DTYPE_BF16, y_dtype == LBQ_DTYPE_BF16, nullptr, 0,
                    static_cast<cudaStream_t>(stream), false);
  return run_direct(items, count, K, group, mode, x_dtype == LBQ_DTYPE_BF16, y_dtype == LBQ_DTYPE_BF16,
                    static_cast<cudaStream_t>(stream));
}

lbq_status lbq_quantize_mxfp8(const void* X, int x_dtype, int M, int K, uint8_t* codes, uint8_t* scales,
                              void* stream) {
  if (!X || !codes || !scales) return fail(LBQ_ERR_INVALID_ARG, "X, codes and scales must be non-null");
  if (M <= 0 || K <= 0 || K % 32) return fail(LBQ_ERR_INVALID_ARG, "M=%d K=%d: need M >= 1 and K a multiple of 32", M, K);
  if (!aligned16(X) || !aligned16(codes))
    return fail(LBQ_ERR_INVALID_ARG, "X and codes must be 16-byte aligned");
  if (x_dtype != LBQ_DTYPE_F16 && x_dtype != LBQ_DTYPE_BF16) return fail(LBQ_ERR_UNSUPPORTED, "x_dtype %d", x_dtype);
  const long long blocks = (long long)M * (K / 32);
  const unsigned grid = (unsigned)((blocks + 255) / 256);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (x_dtype == LBQ_DTYPE_BF16)
    quantize_mxfp8_kernel<true><<<grid, 256, 0, s>>>(static_cast<const uint16_t*>(X), codes, scales, blocks);
  else
    quantize_mxfp8_kernel<false><<<grid, 256, 0, s>>>(static_cast<const uint16_t*>(X), codes, scales, blocks);
  return launch_check("MXFP8 quantisation launch");
}

lbq_status lbq_gemv_noalloc(const void* X, int x_dtype, int M, int K, int N, int group, int mode, const void* image,
                            void* Y, int y_dtype, void* stream) {
  lbq_status st = check_int4_shape(K, N, group, mode);
  if (st != LBQ_OK) return st;
  if ((st = check_compute_args(X, x_dtype, M, image, Y, y_dtype)) != LBQ_OK) return st;
  if (M > 16) return fail(LBQ_ERR_UNSUPPORTED, "lbq_gemv_noalloc takes M <= 16 (M=%d)", M);
  // The scratch the dispatch of lbq_gemv needs for this call, and where in it
  // the tile counters sit (the same plans lbq_gemv makes).
  const GemvScratch g = gemv_scratch(M, K, N, group, mode == LBQ_MODE_ASYM, x_dtype == LBQ_DTYPE_BF16);
  const size_t need = g.need, cnt_off = g.cnt_off, cnt_bytes = g.cnt_bytes;
  if (need > kNoAllocScratchBytes)
    return fail(LBQ_ERR_UNSUPPORTED,
                "lbq_gemv_noalloc: M=%d K=%d N=%d needs %zu bytes of scratch, more than its fixed %zu; use lbq_gemv "
                "with a workspace",
                M, K, N, need, kNoAllocScratchBytes);
  uint8_t* scratch = nullptr;
  if (need) {
    scratch = noalloc_scratch(static_cast<cudaStream_t>(stream), &st);
    if (!scratch) return st;
    // The counters must be zero when the kernel starts; the previous call may
    // have left partial sums where this shape keeps its counters.
    if ((st = cuda_check(cudaMemsetAsync(scratch + cnt_off, 0, cnt_bytes, static_cast<cudaStream_t>(stream)),
                         "clearing the fixed scratch's tile counters")) != LBQ_OK)
      return st;
  }
  return lbq_gemv(X, x_dtype, M, K, N, group, mode, image, Y, y_dtype, scratch, need ? kNoAllocScratchBytes : 0,
                  stream);
}

lbq_status lbq_lut3_mx_gemm(const uint8_t* codes, const uint8_t* scales, int M, int K, int N, const void* image,
                            void* Y, int y_dtype, void* ws, size_t ws_bytes, void* stream) {
  lbq_status st = check_lut3_shape(K, N);
  if (st != LBQ_OK) return st;
  if (K % 512) return fail(LBQ_ERR_UNSUPPORTED, "lbq_lut3_mx_gemm needs K %% 512 == 0 (K=%d)", K);
  if (M <= 0) return fail(LBQ_ERR_INVALID_ARG, "M=%d must be positive", M);
  if (!codes || !scales || !image || !Y) return fail(LBQ_ERR_INVALID_ARG, "codes, scales, image and Y must be non-null");
  if (!aligned16(codes) || !aligned16(scales) || !aligned16(image) || !aligned16(Y))
    return fail(LBQ_ERR_INVALID_ARG, "codes, scales, image and Y must be 16-byte aligned");
  if (y_dtype != LBQ_DTYPE_F16 && y_dtype != LBQ_DTYPE_BF16) return fail(LBQ_ERR_UNSUPPORTED, "y_dtype %d", y_dtype);
  return run_lut3_mx(codes, scales, M, image, make_layout(K, N, 0, LBQ_MODE_LUT3), Y, y_dtype == LBQ_DTYPE_BF16,
                     ws, ws_bytes, static_cast<cudaStream_t>(stream));
}

lbq_status lbq_moe_max_padded(int num_pairs, int num_experts, int block, int* max_padded) {
  if (!max_padded) return fail(LBQ_ERR_INVALID_ARG, "max_padded must be non-null");
  if (num_pairs <= 0 || num_experts <= 0 || block <= 0)
    return fail(LBQ_ERR_INVALID_ARG, "num_pairs=%d num_experts=%d block=%d must be positive", num_pairs, num_experts, block);
  const long long bound = (long long)num_pairs + (long long)std::min(num_pairs, num_experts) * (block - 1);
  if (bound > (1LL << 30)) return fail(LBQ_ERR_INVALID_ARG, "the padded pair list would exceed 2^30 entries");
  *max_padded = moe_max_padded(num_pairs, num_experts, block);
  return LBQ_OK;
}

lbq_status lbq_moe_align(const int32_t* topk_ids, int num_pairs, int num_experts, int block, const int32_t* expert_map,
                         int32_t* sorted_ids, int32_t* expert_ids, int32_t* total, int max_padded, void* stream) {
  if (!topk_ids || !sorted_ids || !expert_ids || !total)
    return fail(LBQ_ERR_INVALID_ARG, "topk_ids, sorted_ids, expert_ids and total must be non-null");
  if (num_pairs <= 0 || num_experts <= 0 || num_experts > 2048 || block <= 0)
    return fail(LBQ_ERR_INVALID_ARG, "num_pairs=%d num_experts=%d (1..2048) block=%d", num_pairs, num_experts, block);
  int need = 0;
  lbq_status st = lbq_moe_max_padded(num_pairs, num_experts, block, &need);
  if (st != LBQ_OK) return st;
  if (max_padded < need) return fail(LBQ_ERR_INVALID_ARG, "max_padded=%d < %d (lbq_moe_max_padded)", max_padded, need);
  const int smem = (3 * num_experts + 1) * (int)sizeof(int);
  void* args[] = {(void*)&topk_ids, (void*)&num_pairs, (void*)&num_experts, (void*)&block, (void*)&expert_map,
                  (void*)&sorted_ids, (void*)&expert_ids, (void*)&total, (void*)&max_padded};
  return launch_kernel_ex((const void*)moe_align_kernel, dim3(1), dim3(1024), smem, static_cast<cudaStream_t>(stream),
                          false, args, "MoE align launch");
}

lbq_status lbq_moe_lut3_mx_gemm(const uint8_t* codes, const uint8_t* scales, int T, int top_k, int K, int N,
                                const int32_t* sorted_ids, const int32_t* expert_ids, const int32_t* total,
                                int max_padded, const void* images, size_t image_stride, int num_local_experts,
                                void* Y, int y_dtype, void* stream) {
  lbq_status st = check_lut3_shape(K, N);
  if (st != LBQ_OK) return st;
  if (K % 128 || K > kMoeMaxK)
    return fail(LBQ_ERR_UNSUPPORTED, "lbq_moe_lut3_mx_gemm needs K %% 128 == 0 and K <= %d (K=%d)", kMoeMaxK, K);
  if (T <= 0 || top_k <= 0 || num_local_experts <= 0)
    return fail(LBQ_ERR_INVALID_ARG, "T=%d top_k=%d num_local_experts=%d must be positive", T, top_k, num_local_experts);
  if ((long long)T * top_k >= (1LL << 30)) return fail(LBQ_ERR_INVALID_ARG, "T * top_k too large");
  if (max_padded <= 0 || max_padded % kMoeBM)
    return fail(LBQ_ERR_INVALID_ARG, "max_padded=%d must be a positive multiple of %d", max_padded, kMoeBM);
  if (!codes || !scales || !sorted_ids || !expert_ids || !total || !images || !Y)
    return fail(LBQ_ERR_INVALID_ARG, "codes, scales, sorted_ids, expert_ids, total, images and Y must be non-null");
  if (!aligned16(codes) || !aligned16(scales) || !aligned16(images) || !aligned16(Y) || image_stride % 16)
    return fail(LBQ_ERR_INVALID_ARG, "codes, scales, images, Y and image_stride must be 16-byte aligned");
  if (y_dtype != LBQ_DTYPE_F16 && y_dtype != LBQ_DTYPE_BF16) return fail(LBQ_ERR_UNSUPPORTED, "y_dtype %d", y_dtype);
  const Layout L = make_layout(K, N, 0, LBQ_MODE_LUT3);
  if (image_stride < L.total) return fail(LBQ_ERR_INVALID_ARG, "image_stride %zu < image size %zu", image_stride, L.total);
  GemmMoeArgs a{};
  a.codes = codes;
  a.scales = scales;
  a.sorted_ids = sorted_ids;
  a.expert_ids = expert_ids;
  a.total = total;
  a.images = static_cast<const uint8_t*>(images);
  a.image_stride = image_stride;
  a.off_i = L.off0; a.off_c = L.off1; a.off_e = L.off2;
  a.s_stride = (int)L.s_stride; a.z_stride = (int)L.z_stride;
  a.Y = Y;
  a.top_k = top_k; a.P = T * top_k; a.N = N; a.K = K;
  a.n_tiles = (N + kMxBN - 1) / kMxBN;
  a.max_blocks = max_padded / kMoeBM;
  a.k_blocks = K / kMxBK;
  a.num_experts = num_local_experts;
  a.y_bf16 = y_dtype == LBQ_DTYPE_BF16 ? 1 : 0;
  const int smem = kMoeSmemBase + 2 * moe_meta_bytes(a.s_stride, a.z_stride);
  const void* fn = (const void*)gemm_moe_lut3_mx_kernel;
  occupancy_for(fn, kMoeThreads, smem);
  const int grid = (int)std::min<long long>((long long)a.n_tiles * a.max_blocks, num_sms());
  void* args[] = {&a};
  return launch_kernel_ex(fn, dim3(grid), dim3(kMoeThreads), smem, static_cast<cudaStream_t>(stream), false, args,
                          "MoE LUT3 x MXFP8 GEMM launch");
}

}  // extern "C"
