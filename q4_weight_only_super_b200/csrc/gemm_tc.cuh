// Q4_K prefill GEMM and grouped expert GEMM on 5th-generation tensor cores
// (tcgen05 + TMEM), with the weights dequantised tile by tile into shared
// memory (hipEngine 0.3.0 README, "GGUF Support": the bulk-prefill path;
// hipster README claims table: "MoE grouped GEMM").
//
//   D[m][n] = sum_k X[m][k] * w[n][k],  w = RN_bf16(RN_fp32(d*sc*q - dmin*m))
//
// CTA tile 256 (tokens) x 256 (weight rows), K step 64, one tile per CTA:
//   warp 0      TMA producer: activation tile (bf16, 128-byte swizzle) and the
//               raw Q4_K bytes of the weight tile (block headers + 32 quant
//               bytes per row per K step), into a 3-deep ring.
//   warp 1      allocates 512 TMEM columns; lane 0 issues tcgen05.mma
//               (M=128, N=256, K=16, bf16 x bf16 -> fp32) for both 128-row
//               halves of the token tile; frees TMEM at the end.
//   warps 2-9   dequantise one weight row each per K step into the canonical
//               K-major 128-byte-swizzled bf16 layout the MMA reads (2-deep
//               ring); afterwards they drain TMEM (tcgen05.ld) to global.
//   warps 10-13 (grouped variant) load activation rows by index (gathered or
//               contiguous), convert bf16 -> fp16 in registers and store them
//               in the same swizzled layout.
// Dense GEMM above 256 tokens (PAIR): a cluster of two CTAs on two SMs computes a
// 512-token x 256-weight-row tile with tcgen05.mma.cta_group::2 (M=256, N=256,
// issued by the even CTA): each CTA holds 256 token rows of A (128 per MMA, one
// MMA per 256-token half) and dequantises 128 of the 256 weight rows -- half the
// per-SM dequantisation -- into 4-deep rings; its TMEM receives its own token rows
// x all 256 weight rows. The odd CTA's MMA lane relays "stage ready" to the even
// CTA by one remote mbarrier arrive per K step; the MMA completions are committed
// to the barriers of both CTAs (multicast commit).
// The dense GEMM multiplies bf16 x bf16. The grouped (mixture-of-experts) GEMM
// multiplies fp16 x fp16: its activations can be heavy-tailed (SwiGLU outputs),
// where bf16-rounded weights (unit roundoff 2^-8) would not keep the
// 2e-3 * sum|w*x| error bound; fp16 weights (2^-11) do. Values outside the fp16
// range latch Q4K_ERR_DEVICE_RANGE.
// Every wait is bounded; on expiry the kernel latches Q4K_ERR_DEVICE_TIMEOUT,
// stops all roles, drains its own copies (bounded), frees TMEM and returns.
#pragma once
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>

#include "common.cuh"

namespace q4k {

constexpr int kGemmBM = 256;
constexpr int kGemmBN = 256;
constexpr int kGemmBK = 64;
constexpr int kStagesAW = 3;
constexpr int kStagesB = 2;
constexpr int kDqWarps = 8;
constexpr int kGatherWarps = 8;  // grouped: activation-row gather (4 were the bound, 8 measured 10% faster)
constexpr uint32_t kATileBytes = kGemmBM * 128;       // 32 KB per K step
constexpr uint32_t kBTileBytes = kGemmBN * 128;       // 32 KB per K step
constexpr uint32_t kWRawPart = kGemmBN * 16;          // 4 KB: one 16-byte column per row
constexpr uint32_t kWRawBytes = 3 * kWRawPart;        // header, quants 0-15, quants 16-31
constexpr uint32_t kSmemA = 0;
// epilogue staging: per epilogue warp 32 rows x kEpiPitch words, inside the
// activation stages (free once the last MMA has completed)
constexpr int kEpiPitch = 36;
constexpr uint32_t kSmemB = kSmemA + kStagesAW * kATileBytes;
static_assert(kDqWarps * 32 * kEpiPitch * 4 <= kStagesAW * kATileBytes, "epilogue staging fits the A stages");
constexpr uint32_t kSmemW = kSmemB + kStagesB * kBTileBytes;
constexpr uint32_t kSmemBar = kSmemW + kStagesAW * kWRawBytes;

// Shared-memory layout of one CTA. PAIR: a CTA pair (a cluster of two) computes a
// 512-token x 256-weight-row tile with tcgen05.mma.cta_group::2 (M = 256, N = 256):
// each CTA holds 256 token rows of A (two 128-row halves, one per MMA) and half the
// weight tile -- 128 rows, which it alone dequantises -- and its TMEM receives its
// own token rows x all 256 weight rows. Half the dequantisation per SM leaves room
// for 4-deep rings.
template <bool PAIR>
struct GemmLayout {
  static constexpr int SA = PAIR ? 4 : kStagesAW;                 // A (and raw weight) stages
  static constexpr int SB = PAIR ? 4 : kStagesB;                  // B stages
  static constexpr int BROWS = PAIR ? kGemmBN / 2 : kGemmBN;      // weight rows per CTA
  static constexpr uint32_t BTile = (uint32_t)BROWS * 128;        // bytes per B stage
  static constexpr uint32_t WPart = (uint32_t)BROWS * 16;         // one 16-byte column of the rows
  static constexpr uint32_t WRaw = 3 * WPart;                     // header, quants 0-15, quants 16-31
  static constexpr uint32_t SmemB = kSmemA + SA * kATileBytes;
  static constexpr uint32_t SmemW = SmemB + SB * BTile;
  static constexpr uint32_t SmemBar = SmemW + SA * WRaw;
  static constexpr size_t Launch = SmemBar + 256 + 1024;          // + barriers, + alignment slack
};
static_assert(GemmLayout<false>::SmemBar == kSmemBar, "one-CTA layout unchanged");
static_assert(GemmLayout<true>::Launch <= 232448, "pair layout fits one SM's shared memory");

struct GemmParams {
  const uint8_t* W;        // dense [N][nkb][144]; grouped [E][N][nkb][144]; bf16-weight form: bf16 [N][K]
  const uint16_t* X;       // activations bf16 (dense [M][K]; grouped: rows of A)
  void* Y;                 // dense fp32 [M][N]; grouped fp32 [rows][N] or bf16 [rows][N/2]
  int M, N, K;
  int E;
  const int32_t* offsets;  // grouped: [E+1]
  const int32_t* gather;   // grouped: optional sorted row -> A row
  int rows;                // grouped: total rows
  int act;
  int64_t expert_stride;
  int n_tiles;             // N / 256
  int m_tiles;             // dense: ceil(M/256); grouped: upper bound of (expert, m-tile) tasks
};

// ---- PTX wrappers -----------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(bar),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// As mbar_try_wait, but the thread may sleep in hardware (up to ~1 ms) until the
// phase completes instead of returning at once: waiting warps do not spin and
// take no issue slots from the warps that work.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3;\n"
      " selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(1000000u)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Bounded wait; returns false (after latching a timeout) if the phase never
// completes within g_wait_limit_ns or another role has already aborted.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  const uint64_t limit = *const_cast<volatile unsigned long long*>(&g_wait_limit_ns);
  for (;;) {
    if (mbar_try_wait_sleep(bar, parity)) return true;
    if (*abort_flag) return false;
    if (global_timer_ns() - t0 > limit) {
      latch_status(Q4K_ERR_DEVICE_TIMEOUT);
      *abort_flag = 1;
      return false;
    }
  }
}

// As mbar_wait, with the limit passed in (read once per thread by the caller).
__device__ __forceinline__ bool mbar_wait_l(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                            uint64_t limit) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (;;) {
    if (mbar_try_wait_sleep(bar, parity)) return true;
    if (*abort_flag) return false;
    if (global_timer_ns() - t0 > limit) {
      latch_status(Q4K_ERR_DEVICE_TIMEOUT);
      *abort_flag = 1;
      return false;
    }
  }
}

// Wait for copies this CTA issued itself to land before it exits, whatever the
// abort flag says (shared memory must not be released under an asynchronous
// write); bounded by the same limit, after which it latches a timeout.
__device__ __forceinline__ bool mbar_wait_drain(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  const uint64_t limit = *const_cast<volatile unsigned long long*>(&g_wait_limit_ns);
  for (;;) {
    if (mbar_try_wait_sleep(bar, parity)) return true;
    if (global_timer_ns() - t0 > limit) {
      latch_status(Q4K_ERR_DEVICE_TIMEOUT);
      return false;
    }
  }
}

// As mbar_wait, with cluster-scope acquire: for a barrier that a thread of the
// other CTA of the cluster arrives on (release, cluster scope).
__device__ __forceinline__ bool mbar_wait_cluster(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
  auto try_once = [&]() {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
  };
  if (try_once()) return true;
  const uint64_t t0 = global_timer_ns();
  const uint64_t limit = *const_cast<volatile unsigned long long*>(&g_wait_limit_ns);
  for (;;) {
    if (try_once()) return true;
    if (*abort_flag) return false;
    if (global_timer_ns() - t0 > limit) {
      latch_status(Q4K_ERR_DEVICE_TIMEOUT);
      *abort_flag = 1;
      return false;
    }
  }
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], "
      "[%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// K-major, 128-byte swizzle shared-memory matrix descriptor: 8-row atoms of
// 128-byte rows, atoms 1024 bytes apart (stride byte offset), descriptor
// version 1, swizzle mode 2 (128B).
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor: fp32 accumulate, A and B both bf16 (format 1) or both
// fp16 (format 0), both K-major, M=128, N=256.
constexpr uint32_t kIdescBf16 = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(256 >> 3) << 17) |
                                ((uint32_t)(128 >> 4) << 24);
constexpr uint32_t kIdescF16 = (1u << 4) | ((uint32_t)(256 >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
// bf16 x bf16 -> fp32, K-major, M=256 (a CTA pair, 128 rows each), N=256
constexpr uint32_t kIdescBf16Pair = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(256 >> 3) << 17) |
                                    ((uint32_t)(256 >> 4) << 24);

__device__ __forceinline__ void umma_f16kind(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
      : "memory");
}

// The CTA-pair MMA (issued by the even CTA of the cluster): A rows 0..127 from
// this CTA's shared memory and 128..255 from the peer's, at the same offsets; B
// rows (weight rows) 0..127 from this CTA, 128..255 from the peer; D rows 0..127
// into this CTA's TMEM and 128..255 into the peer's, at the same address.
__device__ __forceinline__ void umma2_f16kind(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                              uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Completion of the pair's MMAs issued so far, signalled on the barrier at this
// offset in both CTAs of the pair.
__device__ __forceinline__ void umma2_commit_both(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
      "h"((uint16_t)3)
      : "memory");
}

// Arrive (release, cluster scope) on the barrier at this offset in CTA `rank` of the cluster.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t bar, uint32_t rank) {
  asm volatile(
      "{\n .reg .b32 ra;\n mapa.shared::cluster.u32 ra, %0, %1;\n"
      " mbarrier.arrive.release.cluster.shared::cluster.b64 _, [ra];\n}" ::"r"(bar),
      "r"(rank)
      : "memory");
}

// All threads of both CTAs of the cluster (release / acquire).
__device__ __forceinline__ void cluster_barrier() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
        "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]),
        "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]),
        "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}


// Byte offset of 16-byte chunk `c` (0..7) of row `r` in a K-major 128-byte
// swizzled tile (rows of 128 bytes, 8-row atoms of 1024 bytes).
__device__ __forceinline__ uint32_t sw128_offset(int r, int c) {
  return (uint32_t)((r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4));
}

// ---- dequantisation of one row's 64-weight K step ---------------------------

// Four consecutive weights (l = 4p .. 4p+3 of one sub-block) from the nibbles
// of one quant word, as exact fp32 q*ds - dm. Each nibble is placed in the
// mantissa of a float whose exponent makes the nibble's lowest bit worth 1
// (2^E + q), so q*ds = fma(2^E + q, ds, -2^E*ds) exactly.
__device__ __forceinline__ void dq4(uint32_t word, int h, float ds, float dm, float cA, float cB,
                                    float (&w)[4]) {
  // bytes 0,1 of the word in bits 0..15; bytes 2,3 after a 16-bit shift
  const uint32_t lo = word, hi = word >> 16;
  // nibble h of byte b (b in {0,1} of a 16-bit half) sits at bit 8b + 4h
  const uint32_t mA = 0x0Fu << (4 * h), mB = 0x0F00u << (4 * h);
  // exponents: bit 4h -> 2^(23-4h) unit; bit 8+4h -> 2^(15-4h) unit
  const uint32_t eA = (uint32_t)(127 + 23 - 4 * h) << 23, eB = (uint32_t)(127 + 15 - 4 * h) << 23;
  w[0] = fmaf(__uint_as_float((lo & mA) | eA), ds, cA) - dm;
  w[1] = fmaf(__uint_as_float((lo & mB) | eB), ds, cB) - dm;
  w[2] = fmaf(__uint_as_float((hi & mA) | eA), ds, cA) - dm;
  w[3] = fmaf(__uint_as_float((hi & mB) | eB), ds, cB) - dm;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  const __nv_bfloat162 p = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&p);
}
__device__ __forceinline__ uint32_t pack_f16x2(float a, float b) {
  const __half2 p = __floats2half2_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&p);
}
template <bool F16>
__device__ __forceinline__ uint32_t pack2(float a, float b) {
  return F16 ? pack_f16x2(a, b) : pack_bf16x2(a, b);
}

// Dequantise half H of weight row `r`'s K step (super-block ks/4, chunk ks%4: the
// 32 weights of sub-block 2*chunk + H) from its raw header (16 B) and 32 quant
// bytes into the swizzled B tile.
template <bool F16, int H>
__device__ __forceinline__ void dequant_row_half(uint8_t* btile, int r, int chunk, uint4 hdr, uint4 qa, uint4 qb) {
  const float d = half_bits_to_float(hdr.x), dmin = half_bits_to_float(hdr.x >> 16);
  const uint32_t qw[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};  // bytes l = 4i..4i+3
  uint32_t sc, m;
  scale_min(hdr.y, hdr.z, hdr.w, 2 * chunk + H, sc, m);
  const float ds = d * (float)sc;   // exact
  const float dm = dmin * (float)m; // exact
  const float cA = -ds * __uint_as_float((uint32_t)(127 + 23 - 4 * H) << 23);
  const float cB = -ds * __uint_as_float((uint32_t)(127 + 15 - 4 * H) << 23);
  if (F16 && fmaf(15.f, fabsf(ds), fabsf(dm)) > 65504.f) latch_status(Q4K_ERR_DEVICE_RANGE);
#pragma unroll
  for (int c8 = 0; c8 < 4; ++c8) {  // 8 weights: l = 8*c8 .. 8*c8+7 of the sub-block
    float w0[4], w1[4];
    dq4(qw[2 * c8], H, ds, dm, cA, cB, w0);
    dq4(qw[2 * c8 + 1], H, ds, dm, cA, cB, w1);
    // dq4 returns weights in byte order (b0, b1, b2, b3)
    uint4 o;
    o.x = pack2<F16>(w0[0], w0[1]);
    o.y = pack2<F16>(w0[2], w0[3]);
    o.z = pack2<F16>(w1[0], w1[1]);
    o.w = pack2<F16>(w1[2], w1[3]);
    *reinterpret_cast<uint4*>(btile + sw128_offset(r, 4 * H + c8)) = o;
  }
}

// Both halves of weight row `r`'s K step.
template <bool F16>
__device__ __forceinline__ void dequant_row_step(uint8_t* btile, int r, int chunk, uint4 hdr, uint4 qa,
                                                 uint4 qb) {
  dequant_row_half<F16, 0>(btile, r, chunk, hdr, qa, qb);
  dequant_row_half<F16, 1>(btile, r, chunk, hdr, qa, qb);
}

// ---- the kernel -----------------------------------------------------------------

// BF16W: the weights arrive already dequantised, as bf16 [N][K] (the unfused chain:
// q4k_dequant to bf16, then this GEMM); the producer loads each K step's weight tile
// by TMA with the 128-byte swizzle -- the very layout the dequantising warps write --
// and everything else (tiles, MMAs and their order, epilogue) is the fused GEMM's,
// so the two give bit-identical results for the same bf16 weights.
template <bool GROUPED, bool SWIGLU, bool BF16W = false, bool PAIR = false>
__global__ void __launch_bounds__(32 * (2 + kDqWarps + (GROUPED ? kGatherWarps : 0)), 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
               GemmParams p) {
  static_assert(!BF16W || !GROUPED, "bf16-weight form: dense only");
  static_assert(!PAIR || !GROUPED, "CTA pairs: dense only");
  using LY = GemmLayout<PAIR>;
  constexpr int SA = LY::SA, SB = LY::SB;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base, formed by pointer arithmetic on the shared array so the
  // compiler keeps the shared address space (plain LDS/STS, not generic accesses)
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // barriers (8 bytes each) at SmemBar: [0..3] full_aw, [4..7] empty_aw, [8..11] full_b,
  // [12..15] empty_b, [16] tmem_full, [17..20] pair_full (PAIR, bf16 weights: the odd
  // CTA's stage is ready, arrived on in the even CTA)
  auto bar_full_aw = [&](int s) { return sbase + LY::SmemBar + 8u * s; };
  auto bar_empty_aw = [&](int s) { return sbase + LY::SmemBar + 8u * (4 + s); };
  auto bar_full_b = [&](int s) { return sbase + LY::SmemBar + 8u * (8 + s); };
  auto bar_empty_b = [&](int s) { return sbase + LY::SmemBar + 8u * (12 + s); };
  const uint32_t bar_tmem_full = sbase + LY::SmemBar + 8u * 16;
  auto bar_pair_full = [&](int s) { return sbase + LY::SmemBar + 8u * (17 + s); };
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + LY::SmemBar + 192);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + LY::SmemBar + 196);
  int* task_info = reinterpret_cast<int*>(smem + LY::SmemBar + 200);  // expert, row_base, count, m0

  // ---- tile coordinates ----
  // PAIR: CTAs 2i and 2i+1 form cluster i (rank = blockIdx.x % 2) and share its tile
  const int rank = PAIR ? (int)(blockIdx.x & 1u) : 0;
  const unsigned tile_id = PAIR ? blockIdx.x >> 1 : blockIdx.x;
  const int n_tile = (int)(tile_id % (unsigned)p.n_tiles);
  const int task = (int)(tile_id / (unsigned)p.n_tiles);
  if (threadIdx.x == 0) {
    for (int s = 0; s < SA; ++s) {
      mbar_init(bar_full_aw(s), GROUPED ? 1 + kGatherWarps : 1);
      mbar_init(bar_empty_aw(s), BF16W ? 1 : 1 + kDqWarps);
    }
    // PAIR: the even CTA's full_b also takes the odd CTA's dequantising warps (remote
    // arrivals, made after they have seen their own stage's copies land)
    for (int s = 0; s < SB; ++s) {
      mbar_init(bar_full_b(s), BF16W ? 1 : kDqWarps);
      mbar_init(bar_empty_b(s), 1);
    }
    if (PAIR)
      for (int s = 0; s < SA; ++s) mbar_init(bar_pair_full(s), 1);
    mbar_init(bar_tmem_full, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    // Resolve the task: dense -> m tile (PAIR: 512 tokens); grouped -> (expert, m tile within expert).
    int expert = 0, row_base = 0, count = p.M, m0 = task * (PAIR ? 2 * kGemmBM : kGemmBM);
    if (GROUPED) {
      int seen = 0;
      expert = -1;
      for (int e0 = 0; e0 < p.E && expert < 0; e0 += 32) {
        const int e = e0 + lane;
        int c = 0;
        if (e < p.E) c = p.offsets[e + 1] - p.offsets[e];
        const int t = (c + kGemmBM - 1) / kGemmBM;
        int incl = t;
        for (int off = 1; off < 32; off <<= 1) {
          const int o = __shfl_up_sync(0xffffffffu, incl, off);
          if (lane >= off) incl += o;
        }
        const unsigned hit = __ballot_sync(0xffffffffu, task < seen + incl && t > 0);
        if (hit) {
          const int L = __ffs(hit) - 1;
          expert = e0 + L;
          const int incl_l = __shfl_sync(0xffffffffu, incl, L);
          const int t_l = __shfl_sync(0xffffffffu, t, L);
          m0 = (task - (seen + incl_l - t_l)) * kGemmBM;
        }
        seen += __shfl_sync(0xffffffffu, incl, 31);
      }
      if (expert >= 0) {
        row_base = p.offsets[expert];
        count = p.offsets[expert + 1] - row_base;
      }
    }
    if (lane == 0) {
      task_info[0] = expert;
      task_info[1] = row_base;
      task_info[2] = count;
      task_info[3] = m0;
    }
  }
  if (warp == 1) {
    if (PAIR) {  // warp 1 of both CTAs, the same slot offset: the same TMEM address in each
      asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(
                       smem_u32(const_cast<uint32_t*>(tmem_slot)))
                   : "memory");
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    } else {
      asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(
                       smem_u32(const_cast<uint32_t*>(tmem_slot)))
                   : "memory");
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
  }
  tc_fence_before();
  if (PAIR)
    cluster_barrier();  // both CTAs' barriers initialised and TMEM allocated
  else
    __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int expert = task_info[0], row_base = task_info[1], count = task_info[2], m0 = task_info[3];
  const bool active = GROUPED ? (expert >= 0) : (m0 < p.M);
  const int nks = p.K / kGemmBK;

  if (active) {
    if (warp == 0) {
      // ---------------- TMA producer ----------------
      if (lane == 0) {
        const int drop = g_test_drop_stage;  // test hook; -1 in normal use
        int issued = 0;
        // weight rows of this tile in the [rows][row_bytes] view of W
        int wy0, wy1;
        if (SWIGLU) {
          const int half = p.N / 2;
          const int g0 = n_tile * (kGemmBN / 2);
          wy0 = (GROUPED ? expert * p.N : 0) + g0;
          wy1 = wy0 + half;
        } else {
          // PAIR: this CTA's 128 of the tile's 256 weight rows
          wy0 = (GROUPED ? expert * p.N : 0) + n_tile * kGemmBN + (PAIR ? 128 * rank : 0);
          wy1 = wy0 + kGemmBN / 2;
        }
        // token rows of the two A halves (PAIR: MMA h takes tokens m0 + 256h + 128 rank ..)
        const int ay = GROUPED ? row_base + m0 : m0 + (PAIR ? 128 * rank : 0);
        const int ay1 = ay + (PAIR ? 256 : 128);
        for (int ks = 0; ks < nks; ++ks) {
          const int s = ks % SA, u = ks / SA;
          if (u >= 1 && !mbar_wait(bar_empty_aw(s), (u - 1) & 1, abort_flag)) break;
          if (BF16W) {  // the weight tile's B stage must be free too
            const int sb = ks % SB, ub = ks / SB;
            if (ub >= 1 && !mbar_wait(bar_empty_b(sb), (ub - 1) & 1, abort_flag)) break;
          }
          ++issued;
          if (ks == drop) continue;  // test hook: this stage never arrives
          const uint32_t bytes = (GROUPED ? 0u : kATileBytes) + (BF16W ? 0u : LY::WRaw);
          mbar_arrive_expect_tx(bar_full_aw(s), bytes);
          const uint32_t a_dst = sbase + kSmemA + s * kATileBytes;
          if (!GROUPED) {
            tma_load_2d(a_dst, &tmap_x, ks * kGemmBK, ay, bar_full_aw(s));
            tma_load_2d(a_dst + kATileBytes / 2, &tmap_x, ks * kGemmBK, ay1, bar_full_aw(s));
          }
          if (BF16W) {  // the CTA's weight rows x 64 bf16, 128-byte swizzled, into the B stage
            const int sb = ks % SB;
            mbar_arrive_expect_tx(bar_full_b(sb), LY::BTile);
            tma_load_2d(sbase + LY::SmemB + sb * LY::BTile, &tmap_w, ks * kGemmBK,
                        n_tile * kGemmBN + (PAIR ? 128 * rank : 0), bar_full_b(sb));
            continue;
          }
          const int kb = ks >> 2, c = ks & 3;
          const int xh = kb * BLOCK_BYTES, xq = xh + 16 + 32 * c;
          const uint32_t w_dst = sbase + LY::SmemW + s * LY::WRaw;
          if (PAIR) {  // 128 rows: one box per 16-byte column
            tma_load_2d(w_dst, &tmap_w, xh, wy0, bar_full_aw(s));
            tma_load_2d(w_dst + LY::WPart, &tmap_w, xq, wy0, bar_full_aw(s));
            tma_load_2d(w_dst + 2 * LY::WPart, &tmap_w, xq + 16, wy0, bar_full_aw(s));
            continue;
          }
          tma_load_2d(w_dst, &tmap_w, xh, wy0, bar_full_aw(s));
          tma_load_2d(w_dst + 2048, &tmap_w, xh, wy1, bar_full_aw(s));
          tma_load_2d(w_dst + kWRawPart, &tmap_w, xq, wy0, bar_full_aw(s));
          tma_load_2d(w_dst + kWRawPart + 2048, &tmap_w, xq, wy1, bar_full_aw(s));
          tma_load_2d(w_dst + 2 * kWRawPart, &tmap_w, xq + 16, wy0, bar_full_aw(s));
          tma_load_2d(w_dst + 2 * kWRawPart + 2048, &tmap_w, xq + 16, wy1, bar_full_aw(s));
        }
        // Drain: every issued stage must have landed before this CTA may exit. On the
        // normal path the consumers have waited for all of them already.
        if (*abort_flag) {
          for (int ks = (issued > SA ? issued - SA : 0); ks < issued; ++ks)
            if (ks != drop) mbar_wait_drain(bar_full_aw(ks % SA), (ks / SA) & 1);
          if (BF16W)
            for (int ks = (issued > SB ? issued - SB : 0); ks < issued; ++ks)
              if (ks != drop) mbar_wait_drain(bar_full_b(ks % SB), (ks / SB) & 1);
        }
      }
    } else if (warp == 1) {
      // ---------------- MMA issuer ----------------
      // PAIR: the even CTA issues the pair's MMAs. Its full_b also counts the odd CTA's
      // dequantising warps, which arrive once their own stage's copies (A included) have
      // landed and their B half is written. With bf16 weights (no dequantising warps) the
      // odd CTA's lane relays "my stage is ready" instead (a remote arrive on pair_full).
      if (lane == 0) {
        bool ok = true;
        for (int ks = 0; ks < nks && ok; ++ks) {
          const int s = ks % SA, sb = ks % SB;
          ok = mbar_wait(bar_full_aw(s), (ks / SA) & 1, abort_flag) &&
               mbar_wait(bar_full_b(sb), (ks / SB) & 1, abort_flag);
          if (!ok) break;
          if (PAIR && rank == 1) {
            mbar_arrive_remote(bar_pair_full(s), 0);
            continue;
          }
          if (PAIR && !(ok = mbar_wait_cluster(bar_pair_full(s), (ks / SA) & 1, abort_flag))) break;
          tc_fence_after();
          const uint32_t a0 = sbase + kSmemA + s * kATileBytes;
          const uint32_t b0 = sbase + LY::SmemB + sb * LY::BTile;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
#pragma unroll
            for (int kk = 0; kk < kGemmBK / 16; ++kk) {
              if (PAIR)
                umma2_f16kind(tmem + h * 256, umma_desc_sw128(a0 + h * (kATileBytes / 2) + kk * 32),
                              umma_desc_sw128(b0 + kk * 32), kIdescBf16Pair, (ks | kk) != 0);
              else
                umma_f16kind(tmem + h * 256, umma_desc_sw128(a0 + h * (kATileBytes / 2) + kk * 32),
                             umma_desc_sw128(b0 + kk * 32), GROUPED ? kIdescF16 : kIdescBf16,
                             (ks | kk) != 0);
            }
          }
          if (PAIR) {
            umma2_commit_both(bar_empty_aw(s));
            umma2_commit_both(bar_empty_b(sb));
          } else {
            umma_commit(bar_empty_aw(s));
            umma_commit(bar_empty_b(sb));
          }
        }
        if (ok && PAIR && rank == 0) umma2_commit_both(bar_tmem_full);
        if (ok && !PAIR) umma_commit(bar_tmem_full);
      }
    } else if (warp < 2 + kDqWarps) {
      // ---------------- dequantisation, then epilogue ----------------
      // weight row of the B tile (0..255); PAIR: row 0..127 of the CTA's half, and the
      // 32-weight half of the K step (warps 2-5: the first, 6-9: the second)
      const int r = PAIR ? ((warp - 2) & 3) * 32 + lane : (warp - 2) * 32 + lane;
      const int hh = (warp - 2) >> 2;
      bool ok = true;
      for (int ks = 0; ks < (BF16W ? 0 : nks); ++ks) {  // (bf16 weights: loaded by TMA)
        const int s = ks % SA, sb = ks % SB, ub = ks / SB;
        if (!__all_sync(0xffffffffu, mbar_wait(bar_full_aw(s), (ks / SA) & 1, abort_flag))) {
          ok = false;
          break;
        }
        if (ub >= 1 &&
            !__all_sync(0xffffffffu, mbar_wait(bar_empty_b(sb), (ub - 1) & 1, abort_flag))) {
          ok = false;
          break;
        }
        {
          const uint8_t* wr = smem + LY::SmemW + s * LY::WRaw;
          const uint4 hdr = *reinterpret_cast<const uint4*>(wr + r * 16);
          const uint4 qa = *reinterpret_cast<const uint4*>(wr + LY::WPart + r * 16);
          const uint4 qb = *reinterpret_cast<const uint4*>(wr + 2 * LY::WPart + r * 16);
          __syncwarp();
          if (lane == 0) mbar_arrive(bar_empty_aw(s));
          uint8_t* bt = smem + LY::SmemB + sb * LY::BTile;
          if (!PAIR)
            dequant_row_step<GROUPED>(bt, r, ks & 3, hdr, qa, qb);
          else if (hh == 0)
            dequant_row_half<GROUPED, 0>(bt, r, ks & 3, hdr, qa, qb);
          else
            dequant_row_half<GROUPED, 1>(bt, r, ks & 3, hdr, qa, qb);
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_full_b(sb));
      }
      // epilogue: warp w reads TMEM lanes 32*(w%4).. of accumulator half (w-2)/4
      if (ok && __all_sync(0xffffffffu, mbar_wait(bar_tmem_full, 0, abort_flag))) {
        tc_fence_after();
        const int q = warp & 3, hm = (warp - 2) >> 2;
        // first of this warp's 32 token rows (PAIR: MMA hm's rows of this CTA)
        const int mbase = PAIR ? m0 + hm * 256 + rank * 128 + q * 32 : m0 + hm * 128 + q * 32;
        const int limit = GROUPED ? count : p.M;
        const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(hm * 256);
        // Coalesced stores through a per-warp staging tile (the activation stages are
        // free once the last MMA has completed): tcgen05.ld gives each lane 32 columns of
        // its own row; the tile is written back so that every store instruction covers
        // whole 64- or 128-byte segments of four or eight rows.
        uint32_t* stg = reinterpret_cast<uint32_t*>(smem + kSmemA) + (warp - 2) * (32 * kEpiPitch);
        if (SWIGLU) {
          const int half = p.N / 2;
          uint16_t* out = static_cast<uint16_t*>(p.Y) + (int64_t)row_base * half + n_tile * (kGemmBN / 2);
#pragma unroll 1
          for (int cb = 0; cb < 4; ++cb) {
            uint32_t g[32], u[32];
            tmem_ld32(tbase + cb * 32, g);
            tmem_ld32(tbase + 128 + cb * 32, u);
#pragma unroll
            for (int i = 0; i < 32; i += 8) {
              uint4 o;
              uint32_t* op = &o.x;
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float g0 = __uint_as_float(g[i + 2 * e]), g1 = __uint_as_float(g[i + 2 * e + 1]);
                const float u0 = __uint_as_float(u[i + 2 * e]), u1 = __uint_as_float(u[i + 2 * e + 1]);
                op[e] = pack_bf16x2(silu_mul(g0, u0), silu_mul(g1, u1));
              }
              *reinterpret_cast<uint4*>(stg + lane * kEpiPitch + i / 2) = o;
            }
            __syncwarp();
            // 32 rows x 64 bytes: each instruction stores eight rows (four lanes per row)
#pragma unroll
            for (int it = 0; it < 4; ++it) {
              const int r = it * 8 + (lane >> 2), c = lane & 3;
              if (mbase + r < limit)
                *reinterpret_cast<uint4*>(out + (int64_t)(mbase + r) * half + cb * 32 + c * 8) =
                    *reinterpret_cast<const uint4*>(stg + r * kEpiPitch + c * 4);
            }
            __syncwarp();
          }
        } else {
          float* out = static_cast<float*>(p.Y) + (int64_t)(GROUPED ? row_base : 0) * p.N + n_tile * kGemmBN;
#pragma unroll 1
          for (int cb = 0; cb < 8; ++cb) {
            uint32_t v[32];
            tmem_ld32(tbase + cb * 32, v);
#pragma unroll
            for (int i = 0; i < 32; i += 4)
              *reinterpret_cast<uint4*>(stg + lane * kEpiPitch + i) = make_uint4(v[i], v[i + 1], v[i + 2], v[i + 3]);
            __syncwarp();
            // 32 rows x 128 bytes: each instruction stores four rows (eight lanes per row)
#pragma unroll
            for (int it = 0; it < 8; ++it) {
              const int r = it * 4 + (lane >> 3), c = lane & 7;
              if (mbase + r < limit)
                *reinterpret_cast<float4*>(out + (int64_t)(mbase + r) * p.N + cb * 32 + c * 4) =
                    *reinterpret_cast<const float4*>(stg + r * kEpiPitch + c * 4);
            }
            __syncwarp();
          }
        }
      }
    } else if (GROUPED) {
      // ---------------- activation rows: load, bf16 -> fp16, store swizzled ----------------
      constexpr int RS = kGatherWarps * 4;                // row stride: 8 lanes cover a 128-byte row
      const int gt = (warp - 2 - kDqWarps) * 32 + lane;  // 0..32*kGatherWarps-1
      const int ch = gt & 7;                              // 16-byte chunk within the 128-byte row
      const int r0 = gt >> 3;                             // rows r0, r0+RS, ...
      const uint16_t* src_row[kGemmBM / RS];
#pragma unroll
      for (int j = 0; j < kGemmBM / RS; ++j) {
        const int mrow = m0 + r0 + RS * j;
        src_row[j] = nullptr;
        if (mrow < count) {
          const int64_t sr = p.gather ? p.gather[row_base + mrow] : (row_base + mrow);
          src_row[j] = p.X + sr * p.K + ch * 8;
        }
      }
      uint4 buf[kGemmBM / RS];
      auto load = [&](int ks) {
#pragma unroll
        for (int j = 0; j < kGemmBM / RS; ++j)
          buf[j] = src_row[j] ? ldg_u4(src_row[j] + ks * kGemmBK) : make_uint4(0u, 0u, 0u, 0u);
      };
      uint32_t amax = 0;  // largest |bf16| bit pattern seen, per 16-bit half
      if (nks > 0) load(0);
      for (int ks = 0; ks < nks; ++ks) {
        const int s = ks % SA, u = ks / SA;
        if (u >= 1 &&
            !__all_sync(0xffffffffu, mbar_wait(bar_empty_aw(s), (u - 1) & 1, abort_flag)))
          break;
        uint8_t* a_dst = smem + kSmemA + s * kATileBytes;
#pragma unroll
        for (int j = 0; j < kGemmBM / RS; ++j) {
          const uint32_t w[4] = {buf[j].x, buf[j].y, buf[j].z, buf[j].w};
          uint4 o;
          uint32_t* op = &o.x;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            amax = __vmaxu2(amax, w[e] & 0x7FFF7FFFu);
            op[e] = pack_f16x2(__uint_as_float(w[e] << 16), __uint_as_float(w[e] & 0xFFFF0000u));
          }
          *reinterpret_cast<uint4*>(a_dst + sw128_offset(r0 + RS * j, ch)) = o;
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_full_aw(s));
        if (ks + 1 < nks) load(ks + 1);  // next stage's rows in flight during the next wait
      }
      // |x| >= 65536 (bf16 0x4780) does not fit fp16
      if ((amax & 0xFFFFu) >= 0x4780u || (amax >> 16) >= 0x4780u) latch_status(Q4K_ERR_DEVICE_RANGE);
    }
  }

  // ---- teardown ----
  tc_fence_before();
  if (PAIR)
    cluster_barrier();  // neither CTA leaves while the pair's MMAs or arrivals may touch it
  else
    __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    if (PAIR)
      asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
    else
      asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
  }
}

// ---- host side ----------------------------------------------------------------------

inline PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult qres;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &qres) ==
            cudaSuccess &&
        qres == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// bf16 [rows][K] activations, box 64 x 128, 128-byte swizzle.
inline bool make_tmap_x(CUtensorMap* m, const void* base, int64_t rows, int K) {
  auto enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)K * 2};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Raw Q4_K rows viewed as bytes [rows][row_bytes], box 16 bytes x 128 rows.
inline bool make_tmap_w(CUtensorMap* m, const void* base, int64_t rows, int64_t row_bytes) {
  auto enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)row_bytes, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
  cuuint32_t box[2] = {16, 128};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// PAIR: clusters of two CTAs, m_tiles counting 512-token tiles.
template <bool GROUPED, bool SWIGLU, bool BF16W = false, bool PAIR = false>
inline q4k_status launch_gemm_t(const CUtensorMap& tx, const CUtensorMap& tw, const GemmParams& p,
                                cudaStream_t s) {
  auto* k = gemm_tc_kernel<GROUPED, SWIGLU, BF16W, PAIR>;
  constexpr size_t smem = GemmLayout<PAIR>::Launch;
  static std::atomic<int> attr_set[64];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return Q4K_ERR_CUDA;
  if (!attr_set[dev].load()) {
    if (cudaFuncSetAttribute(reinterpret_cast<const void*>(k), cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
      return Q4K_ERR_LAUNCH;
    attr_set[dev].store(1);
  }
  const dim3 block(32 * (2 + kDqWarps + (GROUPED ? kGatherWarps : 0)));
  if (!PAIR) {
    const dim3 grid((unsigned)(p.n_tiles * p.m_tiles));
    k<<<grid, block, smem, s>>>(tx, tw, p);
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? Q4K_OK : Q4K_ERR_LAUNCH;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(2 * p.n_tiles * p.m_tiles), 1, 1);
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, k, tx, tw, p);
  if (e != cudaSuccess) cudaGetLastError();
  return e == cudaSuccess ? Q4K_OK : Q4K_ERR_LAUNCH;
}

// More than 256 tokens: CTA pairs on 512-token tiles (tcgen05.mma.cta_group::2);
// up to 256: one CTA per 256-token tile.
constexpr int kGemmPairMinM = 257;

inline q4k_status launch_gemm_tc(GemmParams p, cudaStream_t s) {
  CUtensorMap tx, tw;
  const int64_t row_bytes = (int64_t)(p.K / QK) * BLOCK_BYTES;
  if (!make_tmap_x(&tx, p.X, p.M, p.K) || !make_tmap_w(&tw, p.W, p.N, row_bytes))
    return Q4K_ERR_CUDA;
  p.n_tiles = p.N / kGemmBN;
  if (p.M >= kGemmPairMinM) {
    p.m_tiles = (p.M + 2 * kGemmBM - 1) / (2 * kGemmBM);
    return launch_gemm_t<false, false, false, true>(tx, tw, p, s);
  }
  p.m_tiles = (p.M + kGemmBM - 1) / kGemmBM;
  return launch_gemm_t<false, false>(tx, tw, p, s);
}

// bf16 weights [N][K], box 64 x box_rows (one B stage), 128-byte swizzle.
inline bool make_tmap_wb(CUtensorMap* m, const void* base, int64_t rows, int K, int box_rows) {
  auto enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)K * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The GEMM of the unfused chain: bf16 weights [N][K] (e.g. from q4k_dequant), the
// fused kernel's tiles and MMA order.
inline q4k_status launch_gemm_tc_bf16w(GemmParams p, cudaStream_t s) {
  CUtensorMap tx, tw;
  const bool pair = p.M >= kGemmPairMinM;
  if (!make_tmap_x(&tx, p.X, p.M, p.K) || !make_tmap_wb(&tw, p.W, p.N, p.K, pair ? kGemmBN / 2 : kGemmBN))
    return Q4K_ERR_CUDA;
  p.n_tiles = p.N / kGemmBN;
  if (pair) {
    p.m_tiles = (p.M + 2 * kGemmBM - 1) / (2 * kGemmBM);
    return launch_gemm_t<false, false, true, true>(tx, tw, p, s);
  }
  p.m_tiles = (p.M + kGemmBM - 1) / kGemmBM;
  return launch_gemm_t<false, false, true>(tx, tw, p, s);
}

// Grouped: tasks are (expert, 256-row tile of that expert's rows); their number
// is at most ceil(rows/256) + min(E, rows). CTAs past the real count exit.
// Activation rows are fetched by the loader warps (by index when `gather` is
// set), so the activation tensor map is unused.
inline q4k_status launch_gemm_tc_grouped(GemmParams p, cudaStream_t s) {
  CUtensorMap tx, tw;
  const int64_t row_bytes = (int64_t)(p.K / QK) * BLOCK_BYTES;
  if (!make_tmap_x(&tx, p.X, 1, p.K) || !make_tmap_w(&tw, p.W, (int64_t)p.E * p.N, row_bytes))
    return Q4K_ERR_CUDA;
  const bool swiglu = p.act == Q4K_ACT_SWIGLU;
  if (swiglu && (p.N / 2) % (kGemmBN / 2)) return Q4K_ERR_UNSUPPORTED;
  p.n_tiles = swiglu ? (p.N / 2) / (kGemmBN / 2) : p.N / kGemmBN;
  p.m_tiles = (p.rows + kGemmBM - 1) / kGemmBM + std::min(p.E, p.rows);
  return swiglu ? launch_gemm_t<true, true>(tx, tw, p, s) : launch_gemm_t<true, false>(tx, tw, p, s);
}

}  // namespace q4k
