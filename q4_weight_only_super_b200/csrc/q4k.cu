// C ABI of the Q4_K library (declared in include/q4k.h): argument checks,
// launch configuration and kernel launches. All kernels live in the
// included headers; this is the only translation unit of libq4k.so.
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <type_traits>

#include "common.cuh"
#include "dequant.cuh"
#include "gemm_tc.cuh"
#include "gemv.cuh"
#include "gemv_sk.cuh"
#include "gemv_sk6.cuh"
#include "gemv_skg.cuh"
#include "moe.cuh"

using namespace q4k;

namespace {

constexpr int kMaxDevices = 64;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int current_device() {
  int d = 0;
  cudaGetDevice(&d);
  return d;
}

// Raise a kernel's dynamic shared-memory limit once per device. `set_to` must be
// distinct for every kernel (the caller owns one per kernel instantiation).
template <typename F>
cudaError_t ensure_smem(F* func, size_t bytes, std::atomic<size_t> (&set_to)[kMaxDevices]) {
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  if (bytes <= 48 * 1024 || set_to[dev].load() >= bytes) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(func),
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess)  // prefer the largest shared-memory carveout (two CTAs per SM)
    e = cudaFuncSetAttribute(reinterpret_cast<const void*>(func),
                             cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  if (e == cudaSuccess) set_to[dev].store(bytes);
  return e;
}

q4k_status launch_status(cudaError_t e) {
  if (e == cudaSuccess) return Q4K_OK;
  cudaGetLastError();  // clear the sticky launch error of this thread
  return Q4K_ERR_LAUNCH;
}

// Launch `k` as a programmatic dependent of the previous kernel in `s`: it may
// start while that kernel finishes; every such kernel here executes
// griddepcontrol.wait before it reads anything the previous kernel writes.
template <typename... KArgs, typename... Args>
q4k_status launch_pdl(void (*k)(KArgs...), dim3 grid, dim3 block, cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return launch_status(cudaLaunchKernelEx(&cfg, k, static_cast<KArgs>(args)...));
}

// ---------------------------------------------------------------- GEMV ----

struct GemvCfg {
  int mt, warps, tiles, ksplit, wstages, xstages;
};

// Ring depths per token class (weight stages, activation stages). Every class
// must fit two CTAs per SM: 228 KiB of shared memory per SM, 1 KiB of it
// reserved per CTA. Then one cluster-fit table serves every class, so the K
// split -- and with it the summation order -- does not depend on the class.
constexpr size_t kGemvTwoPerSm = 233472 / 2 - 1024;
constexpr int kGemvStages[3][2] = {{4, 6}, {4, 2}, {3, 2}};  // mt = 1, 2, 4
static_assert(GemvSmem<1, 4, 2>::total(kGemvStages[0][0], kGemvStages[0][1]) <= kGemvTwoPerSm, "mt 1");
static_assert(GemvSmem<2, 4, 2>::total(kGemvStages[1][0], kGemvStages[1][1]) <= kGemvTwoPerSm, "mt 2");
static_assert(GemvSmem<4, 4, 2>::total(kGemvStages[2][0], kGemvStages[2][1]) <= kGemvTwoPerSm, "mt 4");
// Q5_K: 176-byte rows take a shallower weight ring at the same two CTAs per SM
constexpr int kGemvStagesQ5[3][2] = {{3, 6}, {3, 2}, {2, 2}};
static_assert(GemvSmem<1, 4, 2, false, kQtQ5K>::total(kGemvStagesQ5[0][0], kGemvStagesQ5[0][1]) <= kGemvTwoPerSm, "q5 mt 1");
static_assert(GemvSmem<2, 4, 2, false, kQtQ5K>::total(kGemvStagesQ5[1][0], kGemvStagesQ5[1][1]) <= kGemvTwoPerSm, "q5 mt 2");
static_assert(GemvSmem<4, 4, 2, false, kQtQ5K>::total(kGemvStagesQ5[2][0], kGemvStagesQ5[2][1]) <= kGemvTwoPerSm, "q5 mt 4");
// Q8_0: 272-byte rows, two weight stages (the reduction buffer shares the ring)
constexpr int kGemvStagesQ80[3][2] = {{2, 6}, {2, 2}, {2, 2}};
static_assert(GemvSmem<1, 4, 2, false, kQtQ80>::total(kGemvStagesQ80[0][0], kGemvStagesQ80[0][1]) <= kGemvTwoPerSm, "q8 mt 1");
static_assert(GemvSmem<2, 4, 2, false, kQtQ80>::total(kGemvStagesQ80[1][0], kGemvStagesQ80[1][1]) <= kGemvTwoPerSm, "q8 mt 2");
static_assert(GemvSmem<4, 4, 2, false, kQtQ80>::total(kGemvStagesQ80[2][0], kGemvStagesQ80[2][1]) <= kGemvTwoPerSm, "q8 mt 4");
static_assert(GemvSmem<4, 4, 2, false, kQtQ80>::red_bytes <= 2 * GemvSmem<4, 4, 2, false, kQtQ80>::wstage,
              "q8: reduction buffer inside the weight ring");
// Q6_K: 224-byte row copies, two or three weight stages
constexpr int kGemvStagesQ6[3][2] = {{3, 5}, {3, 2}, {2, 2}};
static_assert(GemvSmem<1, 4, 2, false, kQtQ6K>::total(kGemvStagesQ6[0][0], kGemvStagesQ6[0][1]) <= kGemvTwoPerSm, "q6 mt 1");
static_assert(GemvSmem<2, 4, 2, false, kQtQ6K>::total(kGemvStagesQ6[1][0], kGemvStagesQ6[1][1]) <= kGemvTwoPerSm, "q6 mt 2");
static_assert(GemvSmem<4, 4, 2, false, kQtQ6K>::total(kGemvStagesQ6[2][0], kGemvStagesQ6[2][1]) <= kGemvTwoPerSm, "q6 mt 4");

// fit[d][ks]: clusters of ks GEMV CTAs that can be resident at once on device d
// (a cluster must sit inside one GPC, so this is below 2 * SMs / ks).
std::atomic<int> g_gemv_fit[kMaxDevices][9];
std::atomic<size_t> g_gemv_fit_smem_set[kMaxDevices];

q4k_status gemv_cluster_fit(int ks, int* fit) {
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices || ks < 1 || ks > 8) return Q4K_ERR_CUDA;
  int v = g_gemv_fit[dev][ks].load();
  if (v <= 0) {
    auto* k = gemv_kernel<1, 4, 2, false, false>;
    const size_t smem = GemvSmem<1, 4, 2>::total(kGemvStages[0][0], kGemvStages[0][1]);
    if (ensure_smem(k, smem, g_gemv_fit_smem_set) != cudaSuccess) return launch_status(cudaErrorUnknown);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(ks * 64), 1, 1);
    cfg.blockDim = dim3(32 * (4 + 2), 1, 1);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)ks;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&v, k, &cfg) != cudaSuccess || v <= 0) {
      cudaGetLastError();
      return Q4K_ERR_CUDA;
    }
    g_gemv_fit[dev][ks].store(v);
  }
  *fit = v;
  return Q4K_OK;
}

// Launch shape for `tokens` (<= 32) tokens against `rows_out` weight rows per
// matrix and `nkb` super-blocks per row, with `groups` matrices (experts)
// processed side by side. Depends only on (rows, nkb, groups) and the device,
// so the summation order of a token's result never depends on the batch. The
// K split (cluster size, at most 8) is the largest that keeps every cluster
// resident at once: a cluster that does not fit waits for a whole second wave.
q4k_status pick_gemv(int tokens, int rows_out, int nkb, int groups, GemvCfg* out) {
  GemvCfg c;
  c.mt = tokens <= 8 ? 1 : (tokens <= 16 ? 2 : 4);
  const int cls = c.mt == 1 ? 0 : (c.mt == 2 ? 1 : 2);
  // 128 weight rows per CTA: 4 consumer warps x two 16-row tiles, so each
  // activation fragment, barrier wait and min-term operand serves 32 rows
  // (measured 2-6% faster than 8 warps x one tile at 1..16 tokens)
  c.tiles = 2;
  c.warps = 4;
  c.wstages = kGemvStages[cls][0];
  c.xstages = kGemvStages[cls][1];
  const long clusters = (long)((rows_out + 128 - 1) / 128) * groups;
  int ks = std::max(1, std::min(8, nkb));
  for (; ks > 1; --ks) {
    int fit = 0;
    const q4k_status st = gemv_cluster_fit(ks, &fit);
    if (st != Q4K_OK) return st;
    if ((long)fit >= clusters) break;
  }
  c.ksplit = ks;
  *out = c;
  return Q4K_OK;
}

template <int MT, int WARPS, int TILES, bool GROUPED, bool SWIGLU, bool REPACK = false, int QT = kQtQ4K>
q4k_status launch_gemv_t(const GemvParams& p, int rows_total, int tiles, int groups, cudaStream_t s) {
  auto* k = gemv_kernel<MT, WARPS, TILES, GROUPED, SWIGLU, REPACK, QT>;
  static std::atomic<size_t> smem_set[kMaxDevices];  // one per instantiation
  CUtensorMap tmap = {};  // repacked and Q6_K weights stream by plain bulk copies: no tensor map
  using LS = GemvSmem<MT, WARPS, TILES, REPACK, QT>;
  const int bb = QT == kQtQ80 ? kQ80GroupBytes : (QT == kQtQ5K ? kQ5BlockBytes : BLOCK_BYTES);
  if (!REPACK && QT != kQtQ6K && !make_tmap_w_rowgroup(&tmap, p.W, rows_total, (int64_t)p.nkb * bb, 16 * TILES, LS::pitch,
                                       QT == kQtQ80 ? 2 : 1))
    return Q4K_ERR_CUDA;
  const size_t smem = GemvSmem<MT, WARPS, TILES, REPACK, QT>::total(p.wstages, p.xstages);
  if (ensure_smem(k, smem, smem_set) != cudaSuccess) return Q4K_ERR_LAUNCH;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(tiles * p.ksplit), (unsigned)groups, 1);
  cfg.blockDim = dim3(32 * (WARPS + 2), 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)p.ksplit;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  // programmatic dependent launch: the weight stream starts while the activation
  // pre-pass still runs; the kernel waits for it before reading its records
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return launch_status(cudaLaunchKernelEx(&cfg, k, tmap, p));
}

// Activation pre-pass (rows of X, gathered when `gather` is set) then the GEMV.
template <bool GROUPED, bool SWIGLU, bool REPACK = false, int QT = kQtQ4K>
q4k_status launch_gemv(const GemvCfg& c, GemvParams p, const uint16_t* X, const int32_t* gather,
                       int rows, int K, void* ws, int rows_out, int groups, cudaStream_t s) {
  p.ksplit = c.ksplit;
  p.wstages = c.wstages;
  p.xstages = c.xstages;
  p.rows_pad = rows + kXPadRows;
  p.xprep = static_cast<const uint8_t*>(ws);
  const int total_rows = (int)(GROUPED ? (int64_t)p.E * p.N : p.N);
  const int64_t recs = (int64_t)p.rows_pad * p.nkb;
  const q4k_status st = launch_pdl(QT == kQtQ4KxQ8 ? gemv_prep_q8_kernel : gemv_prep_kernel,
                                   dim3((unsigned)((recs + 7) / 8)), dim3(256), s, X, gather, rows, p.rows_pad, K,
                                   p.nkb, static_cast<uint8_t*>(ws));
  if (st != Q4K_OK) return st;
  const int tiles = (rows_out + 128 - 1) / 128;
  if (c.mt == 1) return launch_gemv_t<1, 4, 2, GROUPED, SWIGLU, REPACK, QT>(p, total_rows, tiles, groups, s);
  if (c.mt == 2) return launch_gemv_t<2, 4, 2, GROUPED, SWIGLU, REPACK, QT>(p, total_rows, tiles, groups, s);
  return launch_gemv_t<4, 4, 2, GROUPED, SWIGLU, REPACK, QT>(p, total_rows, tiles, groups, s);
}

// ------------------------------------------------ stationary GEMV (1..8 tokens) ----

// sk_fit[d][kpw-1][P]: clusters of P stationary-GEMV CTAs (one per SM) resident at
// once on device d.
// Q6: the Q6_K form of the kernel (gemv_sk6_kernel), with its own tables.
std::atomic<int> g_sk_fit[2][kMaxDevices][2][9];
std::atomic<size_t> g_sk_smem_set[2][2][kMaxDevices];

template <int KPW, bool Q6 = false>
q4k_status sk_cluster_fit_t(int P, int* fit) {
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices || P < 1 || P > 8) return Q4K_ERR_CUDA;
  int v = g_sk_fit[Q6][dev][KPW - 1][P].load();
  if (v <= 0) {
    auto* k = Q6 ? gemv_sk6_kernel<KPW> : gemv_sk_kernel<KPW>;
    if (ensure_smem(k, kSkSmemBudget, g_sk_smem_set[Q6][KPW - 1]) != cudaSuccess) return Q4K_ERR_LAUNCH;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(P * 64), 1, 1);
    cfg.blockDim = dim3(SkMax<KPW>::threads, 1, 1);
    cfg.dynamicSmemBytes = kSkSmemBudget;  // one CTA per SM
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)P;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&v, k, &cfg) != cudaSuccess || v <= 0) {
      cudaGetLastError();
      return Q4K_ERR_CUDA;
    }
    g_sk_fit[Q6][dev][KPW - 1][P].store(v);
  }
  *fit = v;
  return Q4K_OK;
}

// The stationary GEMV's launch shape for an N x K matrix; *ok = false when the shape
// is outside what it covers (more than 8 K parts). q6: the Q6_K form.
q4k_status pick_sk(int N, int nkb, SkCfg* c, bool* ok, bool q6 = false) {
  *ok = false;
  if (!(q6 ? sk6_shape(N, nkb, c) : sk_shape(N, nkb, c))) return Q4K_OK;
  int fit = 0;
  const q4k_status st = q6 ? (c->kpw == 2 ? sk_cluster_fit_t<2, true>(c->P, &fit) : sk_cluster_fit_t<1, true>(c->P, &fit))
                           : (c->kpw == 2 ? sk_cluster_fit_t<2>(c->P, &fit) : sk_cluster_fit_t<1>(c->P, &fit));
  if (st != Q4K_OK) return Q4K_OK;  // not resident on this device: the ring kernel takes the shape
  *ok = sk_finish(fit, c);
  return Q4K_OK;
}

template <int KPW, bool Q6 = false>
q4k_status launch_sk_t(const SkCfg& c, const void* W, const uint16_t* X, float* Y, int M, int N, int K,
                       cudaStream_t s) {
  auto* k = Q6 ? gemv_sk6_kernel<KPW> : gemv_sk_kernel<KPW>;
  if (ensure_smem(k, kSkSmemBudget, g_sk_smem_set[Q6][KPW - 1]) != cudaSuccess) return Q4K_ERR_LAUNCH;
  SkParams p = {};
  p.W = static_cast<const uint8_t*>(W);
  p.X = X;
  p.Y = Y;
  p.M = M;
  p.N = N;
  p.K = K;
  p.nkb = K / QK;
  p.P = c.P;
  p.KU = c.KU;
  p.CW = c.CW;
  p.units = c.units;
  p.pitch = c.pitch;
  p.stages = c.stages;
  p.uslots = c.uslots;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)c.grid, 1, 1);
  cfg.blockDim = dim3((unsigned)(32 * (c.CW + 2)), 1, 1);
  cfg.dynamicSmemBytes = c.smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = (unsigned)c.P;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = c.P > 1 ? 2 : 1;
  return launch_status(cudaLaunchKernelEx(&cfg, k, p));
}

q4k_status launch_sk(const SkCfg& c, const void* W, const uint16_t* X, float* Y, int M, int N, int K,
                     cudaStream_t s, bool q6 = false) {
  if (q6)
    return c.kpw == 2 ? launch_sk_t<2, true>(c, W, X, Y, M, N, K, s) : launch_sk_t<1, true>(c, W, X, Y, M, N, K, s);
  return c.kpw == 2 ? launch_sk_t<2>(c, W, X, Y, M, N, K, s) : launch_sk_t<1>(c, W, X, Y, M, N, K, s);
}

// ------------------------------------ grouped stationary GEMV (MoE decode) ----

std::atomic<int> g_sm_count[kMaxDevices];

int sm_count() {
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return 0;
  int v = g_sm_count[dev].load();
  if (v <= 0) {
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) v = 0;
    g_sm_count[dev].store(v);
  }
  return v;
}

// Shared memory one grouped-GEMV CTA may take: one CTA per SM with two super-blocks a
// warp; with one, two CTAs per SM, or four when K has at most four super-blocks (at
// most six warps a CTA: four fit the registers too).
size_t skg_budget(int nkb) {
  return nkb > 10 ? kSkSmemBudget : (nkb <= 4 ? 233472 / 4 - 1024 : kGemvTwoPerSm);
}

// Every CTA resident at once: the kernel deals the units over the whole grid.
template <int KPW, bool SWIGLU, int PL = 0>
q4k_status launch_skg_t(const SkgCfg& c, const SkgParams& p, cudaStream_t s) {
  auto* k = gemv_skg_kernel<KPW, SWIGLU, PL>;
  static std::atomic<size_t> smem_set[kMaxDevices];
  // resident CTAs per SM for the last (threads, smem) asked on each device, packed
  // as (threads << 40) | (smem << 8) | count
  static std::atomic<uint64_t> occ[kMaxDevices];
  if (ensure_smem(k, c.smem, smem_set) != cudaSuccess) return Q4K_ERR_LAUNCH;
  const int dev = current_device();
  const int threads = 32 * (c.CW + 2);
  const uint64_t key = ((uint64_t)threads << 40) | ((uint64_t)c.smem << 8);
  uint64_t o = occ[dev].load();
  if ((o & ~(uint64_t)0xFF) != key) {
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, threads, c.smem) != cudaSuccess || per_sm <= 0)
      return launch_status(cudaErrorUnknown);
    o = key | (uint64_t)std::min(per_sm, 255);
    occ[dev].store(o);
  }
  const int grid = (int)(o & 0xFF) * sm_count();
  if (grid <= 0) return Q4K_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid, 1, 1);
  cfg.blockDim = dim3((unsigned)threads, 1, 1);
  cfg.dynamicSmemBytes = c.smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return launch_status(cudaLaunchKernelEx(&cfg, k, p));
}

q4k_status launch_skg(const SkgCfg& c, const SkgParams& p, bool swiglu, cudaStream_t s) {
  if (c.kpw == 2)
    return swiglu ? launch_skg_t<2, true>(c, p, s) : launch_skg_t<2, false>(c, p, s);
  return swiglu ? launch_skg_t<1, true>(c, p, s) : launch_skg_t<1, false>(c, p, s);
}

// The grouped gate_up + SwiGLU GEMV with the routing prologue; PL = logits per lane.
template <int PL>
q4k_status launch_skg_route_t(const SkgCfg& c, const SkgParams& p, cudaStream_t s) {
  return c.kpw == 2 ? launch_skg_t<2, true, PL>(c, p, s) : launch_skg_t<1, true, PL>(c, p, s);
}

// Routing kernels keep each lane's share of a logit row in registers: pick the
// instantiation whose per-lane slot count PL covers E (E <= 32 * PL).
template <typename F>
q4k_status route_pl_dispatch(int E, F&& f) {
  if (E <= 32) return f(std::integral_constant<int, 1>());
  if (E <= 64) return f(std::integral_constant<int, 2>());
  if (E <= 128) return f(std::integral_constant<int, 4>());
  if (E <= 256) return f(std::integral_constant<int, 8>());
  if (E <= 512) return f(std::integral_constant<int, 16>());
  return f(std::integral_constant<int, 32>());
}

// Fixed scratch of moe_route_permute_noalloc: one array per device that loads
// this library, alive until process exit. Host code must not pass the symbol
// itself to a kernel (on the host it names a host-side stand-in, not device
// memory): its device address is looked up once per device, with that device
// current, and cached.
constexpr size_t kNoAllocRouteInts = 65536;  // 256 KiB
static __device__ __align__(256) int32_t g_noalloc_route_scratch[kNoAllocRouteInts];
std::atomic<int32_t*> g_noalloc_route_ptr[kMaxDevices];

q4k_status noalloc_route_scratch(int32_t** out) {
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return Q4K_ERR_CUDA;
  int32_t* p = g_noalloc_route_ptr[dev].load();
  if (!p) {
    void* addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_noalloc_route_scratch) != cudaSuccess || !addr) {
      cudaGetLastError();
      return Q4K_ERR_CUDA;
    }
    p = static_cast<int32_t*>(addr);
    g_noalloc_route_ptr[dev].store(p);
  }
  *out = p;
  return Q4K_OK;
}

}  // namespace

extern "C" {

const char* q4k_status_string(int s) {
  switch (s) {
    case Q4K_OK: return "ok";
    case Q4K_ERR_NULL: return "null pointer";
    case Q4K_ERR_ALIGN: return "pointer not 16-byte aligned";
    case Q4K_ERR_SHAPE: return "invalid shape";
    case Q4K_ERR_UNSUPPORTED: return "unsupported shape";
    case Q4K_ERR_WORKSPACE: return "workspace missing or too small";
    case Q4K_ERR_LAUNCH: return "kernel launch failed";
    case Q4K_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    case Q4K_ERR_DEVICE_BOUNDS: return "device-side index out of range";
    case Q4K_ERR_CUDA: return "CUDA runtime error";
    case Q4K_ERR_DEVICE_RANGE: return "value outside the fp16 range of the tensor-core grouped path";
    case Q4K_ERR_TOO_LARGE: return "problem exceeds the fixed scratch of the no-allocation entry point";
    default: return "unknown status";
  }
}

q4k_status q4k_dequant(const void* W, int64_t nblocks, int out_bf16, void* out, void* stream) {
  if (nblocks < 0) return Q4K_ERR_SHAPE;
  if (nblocks == 0) return Q4K_OK;
  if (!W || !out) return Q4K_ERR_NULL;
  if (!aligned16(W) || !aligned16(out)) return Q4K_ERR_ALIGN;
  const int64_t threads = nblocks * 32;
  const int64_t grid = (threads + 255) / 256;
  if (grid > 0x7fffffffLL) return Q4K_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (out_bf16)
    dequant_kernel<true><<<(unsigned)grid, 256, 0, s>>>(static_cast<const uint8_t*>(W), nblocks, out);
  else
    dequant_kernel<false><<<(unsigned)grid, 256, 0, s>>>(static_cast<const uint8_t*>(W), nblocks, out);
  return launch_status(cudaGetLastError());
}

q4k_status q4k_gemv(const void* W, const uint16_t* X, float* Y, int M, int N, int K, void* ws,
                    size_t ws_bytes, void* stream) {
  if (M < 0 || N < 0 || K <= 0 || K % QK) return Q4K_ERR_SHAPE;
  if (M == 0 || N == 0) return Q4K_OK;
  if (!W || !X || !Y || !ws) return Q4K_ERR_NULL;
  if (!aligned16(W) || !aligned16(X) || !aligned16(Y) || !aligned16(ws)) return Q4K_ERR_ALIGN;
  if (M > 32 || N % 16) return Q4K_ERR_UNSUPPORTED;
  if (ws_bytes < gemv_ws_bytes(M, K)) return Q4K_ERR_WORKSPACE;
  if (M <= 8) {  // super-block-stationary kernel: no pre-pass, no workspace traffic
    SkCfg sc;
    bool ok = false;
    const q4k_status st = pick_sk(N, K / QK, &sc, &ok);
    if (st != Q4K_OK) return st;
    if (ok) return launch_sk(sc, W, X, Y, M, N, K, static_cast<cudaStream_t>(stream));
  }
  GemvParams p = {};
  p.W = static_cast<const uint8_t*>(W);
  p.out = Y;
  p.M = M;
  p.N = N;
  p.nkb = K / QK;
  GemvCfg c;
  const q4k_status st = pick_gemv(M, N, p.nkb, 1, &c);
  if (st != Q4K_OK) return st;
  return launch_gemv<false, false>(c, p, X, nullptr, M, K, ws, N, 1, static_cast<cudaStream_t>(stream));
}


int64_t q4k_repacked_bytes(int N, int K) {
  if (N <= 0 || K <= 0 || K % QK) return 0;
  return repacked_bytes(N, K);
}

q4k_status q4k_gemv_q8(const void* W, const uint16_t* X, float* Y, int M, int N, int K, void* ws,
                       size_t ws_bytes, void* stream) {
  if (M < 0 || N < 0 || K <= 0 || K % QK) return Q4K_ERR_SHAPE;
  if (M == 0 || N == 0) return Q4K_OK;
  if (!W || !X || !Y || !ws) return Q4K_ERR_NULL;
  if (!aligned16(W) || !aligned16(X) || !aligned16(Y) || !aligned16(ws)) return Q4K_ERR_ALIGN;
  if (M > 32 || N % 16) return Q4K_ERR_UNSUPPORTED;
  if (ws_bytes < gemv_ws_bytes(M, K)) return Q4K_ERR_WORKSPACE;
  GemvParams p = {};
  p.W = static_cast<const uint8_t*>(W);
  p.out = Y;
  p.M = M;
  p.N = N;
  p.nkb = K / QK;
  GemvCfg c;
  const q4k_status st = pick_gemv(M, N, p.nkb, 1, &c);  // Q4_K rows: the Q4_K ring depths and K split
  if (st != Q4K_OK) return st;
  return launch_gemv<false, false, false, kQtQ4KxQ8>(c, p, X, nullptr, M, K, ws, N, 1,
                                                      static_cast<cudaStream_t>(stream));
}

q4k_status q80_gemv(const void* W, const uint16_t* X, float* Y, int M, int N, int K, void* ws, size_t ws_bytes,
                    void* stream) {
  if (M < 0 || N < 0 || K <= 0 || K % QK) return Q4K_ERR_SHAPE;
  if (M == 0 || N == 0) return Q4K_OK;
  if (!W || !X || !Y || !ws) return Q4K_ERR_NULL;
  if (!aligned16(W) || !aligned16(X) || !aligned16(Y) || !aligned16(ws)) return Q4K_ERR_ALIGN;
  if (M > 32 || N % 16) return Q4K_ERR_UNSUPPORTED;
  if (ws_bytes < gemv_ws_bytes(M, K)) return Q4K_ERR_WORKSPACE;
  GemvParams p = {};
  p.W = static_cast<const uint8_t*>(W);
  p.out = Y;
  p.M = M;
  p.N = N;
  p.nkb = K / QK;
  GemvCfg c;
  const q4k_status st = pick_gemv(M, N, p.nkb, 1, &c);  // the Q4_K K split: same cluster fit
  if (st != Q4K_OK) return st;
  const int cls = c.mt == 1 ? 0 : (c.mt == 2 ? 1 : 2);
  c.wstages = kGemvStagesQ80[cls][0];
  c.xstages = kGemvStagesQ80[cls][1];
  return launch_gemv<false, false, false, kQtQ80>(c, p, X, nullptr, M, K, ws, N, 1, static_cast<cudaStream_t>(stream));
}

q4k_status q5k_gemv(const void* W, const uint16_t* X, float* Y, int M, int N, int K, void* ws, size_t ws_bytes,
                    void* stream) {
  if (M < 0 || N < 0 || K <= 0 || K % QK) return Q4K_ERR_SHAPE;
  if (M == 0 || N == 0) return Q4K_OK;
  if (!W || !X || !Y || !ws) return Q4K_ERR_NULL;
  if (!aligned16(W) || !aligned16(X) || !aligned16(Y) || !aligned16(ws)) return Q4K_ERR_ALIGN;
  if (M > 32 || N % 16) return Q4K_ERR_UNSUPPORTED;
  if (ws_bytes < gemv_ws_bytes(M, K)) return Q4K_ERR_WORKSPACE;
  GemvParams p = {};
  p.W = static_cast<const uint8_t*>(W);
  p.out = Y;
  p.M = M;
  p.N = N;
  p.nkb = K / QK;
  GemvCfg c;
  const q4k_status st = pick_gemv(M, N, p.nkb, 1, &c);  // the Q4_K K split: same cluster fit
  if (st != Q4K_OK) return st;
  const int cls = c.mt == 1 ? 0 : (c.mt == 2 ? 1 : 2);
  c.wstages = kGemvStagesQ5[cls][0];
  c.xstages = kGemvStagesQ5[cls][1];
  return launch_gemv<false, false, false, kQtQ5K>(c, p, X, nullptr, M, K, ws, N, 1, static_cast<cudaStream_t>(stream));
}

q4k_status q6k_gemv(const void* W, const uint16_t* X, float* Y, int M, int N, int K, void* ws, size_t ws_bytes,
                    void* stream) {
  if (M < 0 || N < 0 || K <= 0 || K % QK) return Q4K_ERR_SHAPE;
  if (M == 0 || N == 0) return Q4K_OK;
  if (!W || !X || !Y || !ws) return Q4K_ERR_NULL;
  if (!aligned16(W) || !aligned16(X) || !aligned16(Y) || !aligned16(ws)) return Q4K_ERR_ALIGN;
  if (M > 32 || N % 16) return Q4K_ERR_UNSUPPORTED;
  if (ws_bytes < gemv_ws_bytes(M, K)) return Q4K_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int nkb = K / QK;
  if (M <= 8) {  // 1..8 tokens: the stationary form, one launch, no pre-pass
    SkCfg sc;
    bool ok = false;
    const q4k_status st = pick_sk(N, nkb, &sc, &ok, true);
    if (st != Q4K_OK) return st;
    if (ok) return launch_sk(sc, W, X, Y, M, N, K, s, true);
  }
  // 9..32 tokens (and shapes the stationary form does not cover): the ring GEMV, the
  // weights streamed by per-row bulk copies
  GemvParams p = {};
  p.W = static_cast<const uint8_t*>(W);
  p.out = Y;
  p.M = M;
  p.N = N;
  p.nkb = nkb;
  GemvCfg c;
  const q4k_status st = pick_gemv(M, N, nkb, 1, &c);  // the Q4_K K split: same cluster fit
  if (st != Q4K_OK) return st;
  const int cls = c.mt == 1 ? 0 : (c.mt == 2 ? 1 : 2);
  c.wstages = kGemvStagesQ6[cls][0];
  c.xstages = kGemvStagesQ6[cls][1];
  return launch_gemv<false, false, false, kQtQ6K>(c, p, X, nullptr, M, K, ws, N, 1, s);
}

q4k_status q4k_repack(const void* W, int N, int K, void* Wr, void* stream) {
  if (N < 0 || K <= 0 || K % QK) return Q4K_ERR_SHAPE;
  if (N == 0) return Q4K_OK;
  if (!W || !Wr) return Q4K_ERR_NULL;
  if (!aligned16(W) || !aligned16(Wr)) return Q4K_ERR_ALIGN;
  const int64_t units = repacked_bytes(N, K) / 8;
  const int64_t grid = std::min<int64_t>((units + 255) / 256, 148 * 32);
  repack_kernel<<<(unsigned)grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint8_t*>(W), N, K / QK, static_cast<uint8_t*>(Wr), units);
  return launch_status(cudaGetLastError());
}

q4k_status q4k_gemv_repacked(const void* Wr, const uint16_t* X, float* Y, int M, int N, int K, void* ws,
                             size_t ws_bytes, void* stream) {
  if (M < 0 || N < 0 || K <= 0 || K % QK) return Q4K_ERR_SHAPE;
  if (M == 0 || N == 0) return Q4K_OK;
  if (!Wr || !X || !Y || !ws) return Q4K_ERR_NULL;
  if (!aligned16(Wr) || !aligned16(X) || !aligned16(Y) || !aligned16(ws)) return Q4K_ERR_ALIGN;
  if (M > 32 || N % 16) return Q4K_ERR_UNSUPPORTED;
  if (ws_bytes < gemv_ws_bytes(M, K)) return Q4K_ERR_WORKSPACE;
  GemvParams p = {};
  p.W = static_cast<const uint8_t*>(Wr);
  p.out = Y;
  p.M = M;
  p.N = N;
  p.nkb = K / QK;
  GemvCfg c;
  const q4k_status st = pick_gemv(M, N, p.nkb, 1, &c);  // the raw-layout choice: same sums, same order
  if (st != Q4K_OK) return st;
  return launch_gemv<false, false, true>(c, p, X, nullptr, M, K, ws, N, 1, static_cast<cudaStream_t>(stream));
}

q4k_status q4k_gemm(const void* W, const uint16_t* X, float* Y, int M, int N, int K, void* ws,
                    size_t ws_bytes, void* stream) {
  (void)ws;
  (void)ws_bytes;
  if (M < 0 || N < 0 || K <= 0 || K % QK) return Q4K_ERR_SHAPE;
  if (M == 0 || N == 0) return Q4K_OK;
  if (!W || !X || !Y) return Q4K_ERR_NULL;
  if (!aligned16(W) || !aligned16(X) || !aligned16(Y)) return Q4K_ERR_ALIGN;
  if (N % kGemmBN) return Q4K_ERR_UNSUPPORTED;
  GemmParams p = {};
  p.W = static_cast<const uint8_t*>(W);
  p.X = X;
  p.Y = Y;
  p.M = M;
  p.N = N;
  p.K = K;
  return launch_gemm_tc(p, static_cast<cudaStream_t>(stream));
}

q4k_status bf16w_gemm(const uint16_t* Wb, const uint16_t* X, float* Y, int M, int N, int K, void* stream) {
  if (M < 0 || N < 0 || K <= 0 || K % QK) return Q4K_ERR_SHAPE;
  if (M == 0 || N == 0) return Q4K_OK;
  if (!Wb || !X || !Y) return Q4K_ERR_NULL;
  if (!aligned16(Wb) || !aligned16(X) || !aligned16(Y)) return Q4K_ERR_ALIGN;
  if (N % kGemmBN) return Q4K_ERR_UNSUPPORTED;
  GemmParams p = {};
  p.W = reinterpret_cast<const uint8_t*>(Wb);
  p.X = X;
  p.Y = Y;
  p.M = M;
  p.N = N;
  p.K = K;
  return launch_gemm_tc_bf16w(p, static_cast<cudaStream_t>(stream));
}

size_t q4k_workspace_bytes(int op, int M, int N, int K, int E, int topk) {
  (void)N;
  (void)topk;
  if (op == Q4K_OP_ROUTE) {
    if (M <= 0 || E <= 0) return 0;
    const size_t tiles = (size_t)(M + kRouteTokPerCta - 1) / kRouteTokPerCta;
    return tiles * (size_t)E * sizeof(int32_t);
  }
  if (op == Q4K_OP_GEMV || op == Q4K_OP_GROUPED) {
    if (M <= 0 || K <= 0 || K % QK) return 0;
    return gemv_ws_bytes(M, K);
  }
  return 0;
}

q4k_status moe_route_permute(const float* logits, int M, int E, int topk, int32_t* topk_ids,
                             float* topk_w, int32_t* expert_offsets, int32_t* perm,
                             int32_t* inv_perm, int32_t* row_token, void* ws, size_t ws_bytes,
                             void* stream) {
  if (M < 0 || E <= 0 || topk <= 0) return Q4K_ERR_SHAPE;
  if (E > kMaxE || topk > kMaxTopk || topk > E) return Q4K_ERR_UNSUPPORTED;
  if ((int64_t)M * topk > 0x7fffffffLL) return Q4K_ERR_UNSUPPORTED;
  if (!expert_offsets) return Q4K_ERR_NULL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (M == 0) {
    return cudaMemsetAsync(expert_offsets, 0, sizeof(int32_t) * (E + 1), s) == cudaSuccess
               ? Q4K_OK : Q4K_ERR_CUDA;
  }
  if (!logits || !topk_ids || !topk_w || !perm || !inv_perm || !row_token || !ws)
    return Q4K_ERR_NULL;
  if (!aligned16(logits) || !aligned16(topk_ids) || !aligned16(topk_w) ||
      !aligned16(expert_offsets) || !aligned16(perm) || !aligned16(inv_perm) ||
      !aligned16(row_token) || !aligned16(ws))
    return Q4K_ERR_ALIGN;
  if (ws_bytes < q4k_workspace_bytes(Q4K_OP_ROUTE, M, 0, 0, E, topk)) return Q4K_ERR_WORKSPACE;
  const int tiles = (M + kRouteTokPerCta - 1) / kRouteTokPerCta;
  if (tiles == 1)  // one CTA routes and places everything: one launch, no histogram in ws
    return route_pl_dispatch(E, [&](auto pl) {
      return launch_pdl(route_permute_one_kernel<decltype(pl)::value>, dim3(1), dim3(32 * kRouteOneWarps), s, logits,
                        M, E, topk, topk_ids, topk_w, expert_offsets, perm, inv_perm, row_token);
    });
  int32_t* counts = static_cast<int32_t*>(ws);
  const q4k_status st = route_pl_dispatch(E, [&](auto pl) {
    return launch_pdl(route_kernel<decltype(pl)::value>, dim3(tiles), dim3(32 * kRouteWarps), s, logits, M, E,
                      topk, topk_ids, topk_w, counts);
  });
  if (st != Q4K_OK) return st;
  return launch_pdl(permute_kernel, dim3(tiles), dim3(256), s, topk_ids, counts, M, E, topk, tiles,
                    expert_offsets, perm, inv_perm, row_token);
}

// The no-allocation variant: same checks and kernels as moe_route_permute, with
// the per-tile histograms in the library's fixed device array.
q4k_status moe_route_permute_noalloc(const float* logits, int M, int E, int topk, int32_t* topk_ids,
                                     float* topk_w, int32_t* expert_offsets, int32_t* perm,
                                     int32_t* inv_perm, int32_t* row_token, void* stream) {
  if (M < 0 || E <= 0 || topk <= 0) return Q4K_ERR_SHAPE;
  if (E > kMaxE || topk > kMaxTopk || topk > E) return Q4K_ERR_UNSUPPORTED;
  if ((int64_t)M * topk > 0x7fffffffLL) return Q4K_ERR_UNSUPPORTED;
  if (!expert_offsets) return Q4K_ERR_NULL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (M == 0) {
    return cudaMemsetAsync(expert_offsets, 0, sizeof(int32_t) * (E + 1), s) == cudaSuccess
               ? Q4K_OK : Q4K_ERR_CUDA;
  }
  if (!logits || !topk_ids || !topk_w || !perm || !inv_perm || !row_token) return Q4K_ERR_NULL;
  if (!aligned16(logits) || !aligned16(topk_ids) || !aligned16(topk_w) ||
      !aligned16(expert_offsets) || !aligned16(perm) || !aligned16(inv_perm) ||
      !aligned16(row_token))
    return Q4K_ERR_ALIGN;
  const int tiles = (M + kRouteTokPerCta - 1) / kRouteTokPerCta;
  if ((size_t)tiles * (size_t)E > kNoAllocRouteInts) return Q4K_ERR_TOO_LARGE;
  int32_t* counts = nullptr;
  const q4k_status sst = noalloc_route_scratch(&counts);
  if (sst != Q4K_OK) return sst;
  // route_kernel writes every histogram entry permute_kernel reads, so the
  // array's previous contents never matter and nothing is cleared.
  q4k_status st = route_pl_dispatch(E, [&](auto pl) {
    route_kernel<decltype(pl)::value><<<tiles, 32 * kRouteWarps, 0, s>>>(logits, M, E, topk, topk_ids, topk_w,
                                                                          counts);
    return launch_status(cudaGetLastError());
  });
  if (st != Q4K_OK) return st;
  permute_kernel<<<tiles, 256, 0, s>>>(topk_ids, counts, M, E, topk, tiles, expert_offsets, perm,
                                       inv_perm, row_token);
  return launch_status(cudaGetLastError());
}

q4k_status moe_q4k_grouped(const void* W_experts, int E, int N, int K, const uint16_t* A,
                           const int32_t* row_gather, const int32_t* expert_offsets, int rows,
                           int max_rows_hint, int act, void* out, void* ws, size_t ws_bytes,
                           void* stream) {
  if (E <= 0 || N <= 0 || K <= 0 || K % QK || rows < 0 || max_rows_hint < 0) return Q4K_ERR_SHAPE;
  if (act != Q4K_ACT_NONE && act != Q4K_ACT_SWIGLU) return Q4K_ERR_UNSUPPORTED;
  if (rows == 0) return Q4K_OK;
  if (!W_experts || !A || !expert_offsets || !out) return Q4K_ERR_NULL;
  if (!aligned16(W_experts) || !aligned16(A) || !aligned16(out) || !aligned16(expert_offsets) ||
      (row_gather && !aligned16(row_gather)))
    return Q4K_ERR_ALIGN;
  if (N % 32 || E > kMaxE) return Q4K_ERR_UNSUPPORTED;
  const int nkb = K / QK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int hint = std::min(max_rows_hint == 0 ? rows : max_rows_hint, rows);
  if (hint <= 32) {
    if (!ws) return Q4K_ERR_NULL;
    if (!aligned16(ws)) return Q4K_ERR_ALIGN;
    if (ws_bytes < gemv_ws_bytes(rows, K)) return Q4K_ERR_WORKSPACE;
    // K within one CTA's warps: the grouped stationary GEMV (no activation pre-pass,
    // any number of rows per expert); else the ring kernel below
    SkgCfg sc;
    if (skg_shape(nkb, E, skg_budget(nkb), &sc) && ((int64_t)(rows + 7) / 8 + E) * (N / kSkRows) < 0x7fffffffLL) {
      SkgParams sp = {};
      sp.W = static_cast<const uint8_t*>(W_experts);
      sp.A = A;
      sp.gather = row_gather;
      sp.offsets = expert_offsets;
      sp.out = out;
      sp.E = E;
      sp.N = N;
      sp.K = K;
      sp.nkb = nkb;
      sp.rows = rows;
      sp.CW = sc.CW;
      sp.pitch = sc.pitch;
      sp.stages = sc.stages;
      return launch_skg(sc, sp, act == Q4K_ACT_SWIGLU, s);
    }
    GemvParams p = {};
    p.W = static_cast<const uint8_t*>(W_experts);
    p.out = out;
    p.offsets = expert_offsets;
    p.N = N;
    p.nkb = nkb;
    p.E = E;
    const int groups = std::min(E, rows);
    // The same launch shape (hence the same K partition and summation order) for
    // the fp32 and the SwiGLU outputs: a SwiGLU CTA covers as many weight rows.
    GemvCfg c;
    const q4k_status st = pick_gemv(hint, N, nkb, groups, &c);
    if (st != Q4K_OK) return st;
    if (act == Q4K_ACT_SWIGLU)
      return launch_gemv<true, true>(c, p, A, row_gather, rows, K, ws, N, groups, s);
    return launch_gemv<true, false>(c, p, A, row_gather, rows, K, ws, N, groups, s);
  }
  if (N % kGemmBN) return Q4K_ERR_UNSUPPORTED;
  GemmParams p = {};
  p.W = static_cast<const uint8_t*>(W_experts);
  p.X = A;
  p.Y = out;
  p.N = N;
  p.K = K;
  p.E = E;
  p.offsets = expert_offsets;
  p.gather = row_gather;
  p.rows = rows;
  p.act = act;
  p.expert_stride = (int64_t)N * nkb * BLOCK_BYTES;
  return launch_gemm_tc_grouped(p, s);
}

q4k_status moe_route_gate_up(const float* logits, int M, int E, int topk, int32_t* topk_ids, float* topk_w,
                             int32_t* expert_offsets, int32_t* perm, int32_t* inv_perm, int32_t* row_token,
                             const void* W_gate_up, int N, int K, const uint16_t* X, void* h, void* stream) {
  if (M < 0 || E <= 0 || topk <= 0 || N <= 0 || K <= 0 || K % QK) return Q4K_ERR_SHAPE;
  if (M > kRouteTokPerCta || E > 256 || topk > kMaxTopk || topk > E) return Q4K_ERR_UNSUPPORTED;
  if (N % 32) return Q4K_ERR_UNSUPPORTED;
  if (!expert_offsets) return Q4K_ERR_NULL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (M == 0) {
    return cudaMemsetAsync(expert_offsets, 0, sizeof(int32_t) * (E + 1), s) == cudaSuccess ? Q4K_OK
                                                                                          : Q4K_ERR_CUDA;
  }
  if (!logits || !topk_ids || !topk_w || !perm || !inv_perm || !row_token || !W_gate_up || !X || !h)
    return Q4K_ERR_NULL;
  if (!aligned16(logits) || !aligned16(topk_ids) || !aligned16(topk_w) || !aligned16(expert_offsets) ||
      !aligned16(perm) || !aligned16(inv_perm) || !aligned16(row_token) || !aligned16(W_gate_up) ||
      !aligned16(X) || !aligned16(h))
    return Q4K_ERR_ALIGN;
  const int nkb = K / QK;
  const int rows = M * topk;
  SkgCfg sc;
  // the routing warps of the prologue must exist: CW + 2 >= kSkgRouteWarps
  if (!skg_shape(nkb, E, skg_budget(nkb), &sc, true) || sc.CW + 2 < kSkgRouteWarps ||
      ((int64_t)(rows + 7) / 8 + E) * (N / kSkRows) >= 0x7fffffffLL)
    return Q4K_ERR_UNSUPPORTED;  // use moe_route_permute and moe_q4k_grouped
  SkgParams sp = {};
  sp.W = static_cast<const uint8_t*>(W_gate_up);
  sp.A = X;
  sp.out = h;
  sp.E = E;
  sp.N = N;
  sp.K = K;
  sp.nkb = nkb;
  sp.rows = rows;
  sp.CW = sc.CW;
  sp.pitch = sc.pitch;
  sp.stages = sc.stages;
  sp.logits = logits;
  sp.M = M;
  sp.topk = topk;
  sp.topk_ids = topk_ids;
  sp.topk_w = topk_w;
  sp.offsets_out = expert_offsets;
  sp.perm = perm;
  sp.inv_perm = inv_perm;
  sp.row_token = row_token;
  if (E <= 32) return launch_skg_route_t<1>(sc, sp, s);
  if (E <= 64) return launch_skg_route_t<2>(sc, sp, s);
  if (E <= 128) return launch_skg_route_t<4>(sc, sp, s);
  return launch_skg_route_t<8>(sc, sp, s);
}

q4k_status moe_combine(const float* O, const int32_t* inv_perm, const float* topk_w, int M,
                       int topk, int H, float* Y, void* stream) {
  if (M < 0 || topk <= 0 || H <= 0) return Q4K_ERR_SHAPE;
  if (M == 0) return Q4K_OK;
  if (!O || !inv_perm || !topk_w || !Y) return Q4K_ERR_NULL;
  if (!aligned16(O) || !aligned16(inv_perm) || !aligned16(topk_w) || !aligned16(Y))
    return Q4K_ERR_ALIGN;
  if (H % 4 || M > 65535 || topk > kMaxTopk) return Q4K_ERR_UNSUPPORTED;
  const int n4 = H / 4;
  dim3 grid((n4 + 255) / 256, M);
  return launch_pdl(combine_kernel<false>, grid, dim3(256), static_cast<cudaStream_t>(stream), O, inv_perm, topk_w,
                    M, topk, H, static_cast<const float*>(nullptr), Y);
}

q4k_status moe_combine_residual(const float* O, const int32_t* inv_perm, const float* topk_w,
                                const float* residual, int M, int topk, int H, float* Y, void* stream) {
  if (M < 0 || topk <= 0 || H <= 0) return Q4K_ERR_SHAPE;
  if (M == 0) return Q4K_OK;
  if (!O || !inv_perm || !topk_w || !residual || !Y) return Q4K_ERR_NULL;
  if (!aligned16(O) || !aligned16(inv_perm) || !aligned16(topk_w) || !aligned16(residual) || !aligned16(Y))
    return Q4K_ERR_ALIGN;
  if (H % 4 || M > 65535 || topk > kMaxTopk) return Q4K_ERR_UNSUPPORTED;
  const int n4 = H / 4;
  dim3 grid((n4 + 255) / 256, M);
  return launch_pdl(combine_kernel<true>, grid, dim3(256), static_cast<cudaStream_t>(stream), O, inv_perm, topk_w,
                    M, topk, H, residual, Y);
}

q4k_status moe_route_permute_hidden(const uint16_t* X, const uint16_t* W_router, int M, int E, int H, int topk,
                                    float* logits, int32_t* topk_ids, float* topk_w, int32_t* expert_offsets,
                                    int32_t* perm, int32_t* inv_perm, int32_t* row_token, void* ws, size_t ws_bytes,
                                    void* stream) {
  if (M < 0 || E <= 0 || topk <= 0 || H <= 0 || H % 8) return Q4K_ERR_SHAPE;
  if (E > kMaxE || topk > kMaxTopk || topk > E || M > 65535) return Q4K_ERR_UNSUPPORTED;
  if (M > 0) {
    if (!X || !W_router || !logits) return Q4K_ERR_NULL;
    if (!aligned16(X) || !aligned16(W_router) || !aligned16(logits)) return Q4K_ERR_ALIGN;
    // the routing call's own checks run before anything is launched
    if (!topk_ids || !topk_w || !expert_offsets || !perm || !inv_perm || !row_token || !ws) return Q4K_ERR_NULL;
    if (!aligned16(topk_ids) || !aligned16(topk_w) || !aligned16(expert_offsets) || !aligned16(perm) ||
        !aligned16(inv_perm) || !aligned16(row_token) || !aligned16(ws))
      return Q4K_ERR_ALIGN;
    if (ws_bytes < q4k_workspace_bytes(Q4K_OP_ROUTE, M, 0, 0, E, topk)) return Q4K_ERR_WORKSPACE;
    const q4k_status st = launch_pdl(router_logits_kernel, dim3((unsigned)M, (unsigned)((E + 31) / 32)), dim3(256),
                                     static_cast<cudaStream_t>(stream), X, W_router, M, E, H, logits);
    if (st != Q4K_OK) return st;
  }
  return moe_route_permute(logits, M, E, topk, topk_ids, topk_w, expert_offsets, perm, inv_perm, row_token, ws,
                           ws_bytes, stream);
}

q4k_status q4k_test_wait_fault(int drop_stage, uint64_t wait_limit_ns) {
  const int drop = drop_stage < 0 ? -1 : drop_stage;
  const unsigned long long lim = wait_limit_ns ? (unsigned long long)wait_limit_ns : 2000000000ull;
  if (cudaMemcpyToSymbol(g_test_drop_stage, &drop, sizeof(int)) != cudaSuccess ||
      cudaMemcpyToSymbol(g_wait_limit_ns, &lim, sizeof(lim)) != cudaSuccess) {
    cudaGetLastError();
    return Q4K_ERR_CUDA;
  }
  return Q4K_OK;
}

q4k_status q4k_last_device_status(void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return Q4K_ERR_CUDA;
  int v = 0;
  const int zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(int)) != cudaSuccess) return Q4K_ERR_CUDA;
  if (cudaMemcpyToSymbol(g_status, &zero, sizeof(int)) != cudaSuccess) return Q4K_ERR_CUDA;
  return static_cast<q4k_status>(v);
}

}  // extern "C"
