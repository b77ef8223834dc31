// Q4_K decode GEMV (1..32 tokens) and its grouped mixture-of-experts form.
//
// Operation: Y[m][n] = sum_k w[n][k] * X[m][k] over Q4_K weights (hipEngine
// 0.3.0 README, "Quickstart": the GEMV-decode profile; hipster README claims
// table: "GEMV ... GB/s"). The weight stream from HBM is the roofline.
//
// Design (sm_100a):
//  * A pre-pass (gemv_prep_kernel) turns each activation row, one 256-wide
//    super-block column at a time, into a 576-byte record: the 256 values
//    scaled by a power of two 2^k (chosen so the column's largest magnitude
//    lands in [2^14, 2^15): exact, and fp16 can neither overflow nor lose the
//    small values), rounded to fp16, stored in the order the MMA fragments
//    read them; the eight 32-wide sub-block sums of the scaled values (times
//    2^-6) as fp16 hi + lo pairs; and 2^-k. It runs once per call, so every
//    CTA only copies prepared records.
//  * In the GEMV a producer warp streams the CTA's weight rows (one
//    super-block column per stage) into a shared-memory ring with TMA, a
//    second producer warp copies the matching activation records with 1-D
//    bulk copies; mbarriers track both. The GEMV is launched as a programmatic
//    dependent of the pre-pass, so its weight stream starts while the pre-pass
//    runs and only the activation copies wait for it.
//  * Consumer warps own 16 or 32 weight rows each (one or two 16-row MMA
//    tiles; with two, every activation fragment feeds two MMAs). The A operand
//    takes one of two exact forms:
//    - 1..16 tokens: the nibble field itself read as fp16 bits -- q * 2^-24 for
//      a low nibble, 16q * 2^-24 for a high one, fp16 subnormals that the
//      tensor core multiplies exactly -- one AND per two weights. A sub-block's
//      two k-steps accumulate on their own (C_j, fp32) and the block sum is
//      C = sum_j s_j * C_j with s_j = sc_j (sc_j/16 for high nibbles) as an
//      exact fp32; 2^24 is folded into d.
//    - 17..32 tokens: fp16 q*sc (<= 945, exact): a nibble ORed into 0x6400 is
//      1024+q (low) or 1024+16q (high), and one fp16x2 FMA with (sc or sc/16)
//      and -1024*that removes the bias, so the mma.sync m16n8k16 accumulator
//      runs over the whole super-block (scaling per result would grow with the
//      four token groups).
//  * The min term, dmin * sum_j m_j * X_j over the eight sub-blocks, is one
//    more MMA per tile: A = m_j (fp16, exact), B = the sub-block sums
//    (hi + lo, two MMAs), k = sub-block index.
//  * Per super-block the result is y += d*2^-k*C - 64*dmin*2^-k*Cm.
//  * The k order inside a sub-block is free for a dot product, so each
//    thread takes the nibbles in the order the masks produce them, and the
//    pre-pass stores the activations in that same order.
//  * A CTA owns 16*TILES*WARPS weight rows and a contiguous range of super-blocks;
//    a thread-block cluster of KSPLIT CTAs covers the whole K range and its
//    partial sums are reduced in rank order through distributed shared memory
//    (deterministic, no atomics). The decomposition depends only on (N, K), and
//    the pre-pass record of a row depends only on that row, so within a token
//    class (1..16, 17..32) a token's result never depends on the other tokens
//    in the batch.
#pragma once
#include <cooperative_groups.h>

#include "common.cuh"
#include "gemm_tc.cuh"  // mbarrier / TMA wrappers

namespace q4k {

namespace cg = cooperative_groups;

// Prepared activation record of one (row, super-block): bytes [0,512) fp16 values
// in fragment order [sub-block 8][quarter 4][8], [512,528) fp16 sub-block sums
// (hi), [528,544) (lo), [544,548) fp32 2^-k, rest padding. 576 = 64 mod 128
// keeps the per-thread 16-byte fragment reads bank-conflict-free.
constexpr int kXRec = 576;
constexpr int kXPadRows = 32;  // zero records appended after the real rows

// The MMA wrappers are plain (not volatile) asm: they have no side effects, so the
// compiler may schedule independent MMAs (and their operand set-up) around one
// another instead of keeping every MMA in program order; an MMA whose accumulator
// comes from the previous one otherwise stalls the warp for its full latency.
__device__ __forceinline__ void mma_f16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                              uint32_t a3, uint32_t b0, uint32_t b1, bool zero_c) {
  if (zero_c) {
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%10,%10,%10,%10};"
        : "=f"(c[0]), "=f"(c[1]), "=f"(c[2]), "=f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.0f));
  } else {
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  }
}

// (a & b) | c in one logic instruction.
__device__ __forceinline__ uint32_t and_or(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

__device__ __forceinline__ uint32_t h2_bits(__half2 v) { return *reinterpret_cast<uint32_t*>(&v); }
__device__ __forceinline__ __half2 bits_h2(uint32_t v) { return *reinterpret_cast<__half2*>(&v); }

// fp16x2 (1024 + b_lo, 1024 + b_hi) from bytes `lo` and `hi` (0..3) of `word`
// (each <= 63, so it fits the 10-bit mantissa of 1024).
// Q5_K: bit b of bytes 0 and 2 of `w`, moved to bit `to` of each 16-bit half
// (b and to are compile-time constants after unrolling).
__device__ __forceinline__ uint32_t fifth_bits(uint32_t w, int b, int to) {
  const uint32_t s = to >= b ? (w << (to - b)) : (w >> (b - to));
  return s & (0x00010001u << to);
}

__device__ __forceinline__ uint32_t bytes_1024(uint32_t word, uint32_t lo, uint32_t hi) {
  return __byte_perm(word, 0x64u, (4u << 12) | (hi << 8) | (4u << 4) | lo);
}

// ------------------------------------------------------------------ pre-pass ---

// One warp per (row, super-block) record; rows >= `rows` (padding) become zeros.
__global__ void __launch_bounds__(256) gemv_prep_kernel(const uint16_t* __restrict__ X,
                                                        const int32_t* __restrict__ gather, int rows,
                                                        int rows_pad, int K, int nkb,
                                                        uint8_t* __restrict__ ws) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // X and the gather indices may come from the previous kernel. (The GEMV, the
  // only reader of this workspace, never signals its dependents early, so this
  // pre-pass cannot start while an earlier GEMV still reads the workspace.)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int lane = threadIdx.x & 31;
  const int64_t w = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (w >= (int64_t)rows_pad * nkb) return;  // uniform per warp
  const int kb = (int)(w / rows_pad), r = (int)(w % rows_pad);
  uint8_t* rec = ws + w * kXRec;  // record index kb * rows_pad + r
  const int sb = lane >> 2, tq = lane & 3;
  uint4 v = make_uint4(0u, 0u, 0u, 0u);
  if (r < rows) {
    const int64_t src = gather ? gather[r] : r;
    v = ldg_u4(X + src * K + (int64_t)kb * QK + sb * 32 + tq * 8);
  }
  const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
  float x[8];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    x[2 * e] = bf16_bits_to_float(wv[e] & 0xFFFFu);
    x[2 * e + 1] = bf16_bits_to_float(wv[e] >> 16);
  }
  uint32_t amax = 0;
#pragma unroll
  for (int e = 0; e < 8; ++e) amax = max(amax, __float_as_uint(x[e]) & 0x7FFFFFFFu);
  amax = __reduce_max_sync(0xffffffffu, amax);  // bit order = magnitude order for |x|
  int k = 0;
  if (amax != 0) {
    const int E = max(1, (int)(amax >> 23));  // biased exponent of the largest |x|
    k = min(126, max(-126, 141 - E));          // largest |x| * 2^k in [2^14, 2^15)
  }
  const float f = __uint_as_float((uint32_t)(127 + k) << 23);  // 2^k
  float xs[8];
  float sum = 0.f;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    xs[e] = x[e] * f;  // exact
    sum += xs[e];
  }
  uint4 o;  // fragment order (e0,e2),(e1,e3),(e4,e6),(e5,e7)
  o.x = h2_bits(__floats2half2_rn(xs[0], xs[2]));
  o.y = h2_bits(__floats2half2_rn(xs[1], xs[3]));
  o.z = h2_bits(__floats2half2_rn(xs[4], xs[6]));
  o.w = h2_bits(__floats2half2_rn(xs[5], xs[7]));
  *reinterpret_cast<uint4*>(rec + (sb * 4 + tq) * 16) = o;
  sum += __shfl_xor_sync(0xffffffffu, sum, 1);
  sum += __shfl_xor_sync(0xffffffffu, sum, 2);
  const float s2 = sum * 0.015625f;  // 2^-6: |s2| < 2^14
  const __half hi = __float2half_rn(s2);
  const __half lo = __float2half_rn(s2 - __half2float(hi));
  if (tq == 0) {
    reinterpret_cast<__half*>(rec + 512)[sb] = hi;
    reinterpret_cast<__half*>(rec + 528)[sb] = lo;
  }
  if (lane == 0) *reinterpret_cast<float*>(rec + 544) = __uint_as_float((uint32_t)(127 - k) << 23);
}

// Q8 activation lane: the same records (one warp each, rows >= `rows` zero), holding
// the 256 values of the column as int8 codes in natural order (bytes 0..255), the
// eight sub-block sums of the codes times 2^-6 as fp16 hi + lo (exact: |sum| <=
// 4064), and the column scale d_x at byte 544. amax = max |x|, d_x = amax / 127,
// inv = 127 / amax, q = rint(x * inv) clamped to +-127, each step one IEEE fp32
// operation in round-to-nearest-even.
__global__ void __launch_bounds__(256) gemv_prep_q8_kernel(const uint16_t* __restrict__ X,
                                                           const int32_t* __restrict__ gather, int rows,
                                                           int rows_pad, int K, int nkb,
                                                           uint8_t* __restrict__ ws) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");  // as gemv_prep_kernel
  const int lane = threadIdx.x & 31;
  const int64_t w = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (w >= (int64_t)rows_pad * nkb) return;  // uniform per warp
  const int kb = (int)(w / rows_pad), r = (int)(w % rows_pad);
  uint8_t* rec = ws + w * kXRec;
  uint4 v = make_uint4(0u, 0u, 0u, 0u);
  if (r < rows) {
    const int64_t src = gather ? gather[r] : r;
    v = ldg_u4(X + src * K + (int64_t)kb * QK + lane * 8);  // values 8*lane .. 8*lane+7
  }
  const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
  float x[8];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    x[2 * e] = bf16_bits_to_float(wv[e] & 0xFFFFu);
    x[2 * e + 1] = bf16_bits_to_float(wv[e] >> 16);
  }
  uint32_t amax = 0;
#pragma unroll
  for (int e = 0; e < 8; ++e) amax = max(amax, __float_as_uint(x[e]) & 0x7FFFFFFFu);
  amax = __reduce_max_sync(0xffffffffu, amax);
  float dx = 0.f, inv = 0.f;
  if (amax != 0) {
    dx = __fdiv_rn(__uint_as_float(amax), 127.f);
    inv = __fdiv_rn(127.f, __uint_as_float(amax));
  }
  uint32_t packed[2] = {0u, 0u};
  int isum = 0;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const int qv = max(-127, min(127, __float2int_rn(__fmul_rn(x[e], inv))));
    isum += qv;
    packed[e >> 2] |= ((uint32_t)qv & 0xFFu) << (8 * (e & 3));
  }
  *reinterpret_cast<uint2*>(rec + 8 * lane) = make_uint2(packed[0], packed[1]);
  isum += __shfl_xor_sync(0xffffffffu, isum, 1);  // the four lanes of sub-block lane / 4
  isum += __shfl_xor_sync(0xffffffffu, isum, 2);
  const float s2 = (float)isum * 0.015625f;
  const __half hi = __float2half_rn(s2);
  const __half lo = __float2half_rn(s2 - __half2float(hi));
  if ((lane & 3) == 0) {
    reinterpret_cast<__half*>(rec + 512)[lane >> 2] = hi;
    reinterpret_cast<__half*>(rec + 528)[lane >> 2] = lo;
  }
  if (lane == 0) *reinterpret_cast<float*>(rec + 544) = dx;
}

// m16n8k32 integer MMA, u8 A x s8 B -> s32, zero accumulator in.
__device__ __forceinline__ void imma_16832(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                           uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%10,%10,%10};"
      : "=r"(c[0]), "=r"(c[1]), "=r"(c[2]), "=r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "r"(0));
}

// ---------------------------------------------------------------------- GEMV ---

struct GemvParams {
  const uint8_t* W;          // dense: [N][nkb][144]; grouped: [E][N][nkb][144]
  const uint8_t* xprep;      // prepared records [nkb][rows_pad][576]
  void* out;                 // fp32 [rows][N] or bf16 [rows][N/2] (SWIGLU)
  const int32_t* offsets;    // grouped: [E+1] rows per expert (device); dense: nullptr
  int M;                     // dense: tokens; grouped: unused
  int N;                     // weight rows per matrix
  int nkb;                   // K / 256
  int E;                     // grouped: experts
  int rows_pad;              // records per super-block column
  int ksplit;                // cluster size along K
  int wstages;               // weight ring depth
  int xstages;               // activation ring depth
};

// Each consumer warp owns 16*TILES weight rows (TILES 16-row MMA tiles). A stage
// of the weight ring holds, per warp, those rows x 160 bytes: one 144-byte
// super-block plus the first 16 bytes of the next (read and ignored) -- the
// 160-byte pitch makes the per-thread 8-byte quant reads bank-conflict-free.
constexpr int kGemvPitch = 160;
// Q5_K super-block (Q4_K's fields plus 32 bytes of fifth bits): 176 bytes, read
// in 176-byte boxes
constexpr int kQ5BlockBytes = 176;
constexpr int kQ5QhOff = 16;   // qh[32]: bit 2c+h of qh[l] is the fifth bit of weight 64c+32h+l
constexpr int kQ5QsOff = 48;   // the 128 nibble bytes, ordered as in Q4_K
// Q8_0: blocks of 32 weights in 34 bytes (fp16 d, then 32 signed bytes); the
// GEMV reads them eight at a time (one 256-wide column of the matrix, 272 bytes
// per row), and block j of a group plays the part of Q4_K's sub-block j
constexpr int kQ80GroupBytes = 272;
// Q6_K: 210-byte super-blocks (ql[128], qh[64], sixteen signed byte scales at 192, fp16
// d at 208). Rows are then only 2-byte aligned, out of reach of a TMA box, so each row's
// block of a stage is one 224-byte bulk copy of its 16-byte-aligned superset (the block
// starts 0..14 bytes in; 224 = 14 * 16 also ends each copy at or before the next block's
// end, and the last copy of the matrix exactly at its end, the matrix being a multiple of
// 16 bytes long)
constexpr int kQ6BB = 210;
constexpr int kQ6Copy = 224;
// weight formats of the GEMV kernel
constexpr int kQtQ4K = 0, kQtQ5K = 1, kQtQ80 = 2;
constexpr int kQtQ4KxQ8 = 3;  // Q4_K weights, int8 activations (the Q8 lane)
constexpr int kQtQ6K = 4;

// Shared memory layout (dynamic):
//   wring [wstages][WARPS][16*TILES rows][160 B]   weight tiles (TMA destination)
//   xring [xstages][8*MT tokens][576 B]            activation records (bulk-copy destination)
//   red   [16*TILES*WARPS rows][8*MT] fp32         per-CTA partial result
//   bars  wfull, wempty [wstages], xfull, xempty [xstages]; abort flag
// Repacked weights (q4k_repack): 128-row tiles whose super-block columns are
// contiguous and whose row-blocks keep each thread's 32 quant bytes together;
// the stage is one bulk copy and the smem pitch the block size itself.
constexpr int kRepackRows = 128;

template <int MT, int WARPS, int TILES, bool REPACK = false, int QT = kQtQ4K>
struct GemvSmem {
  static constexpr int TOK = 8 * MT;
  static constexpr int pitch =
      QT == kQtQ6K ? kQ6Copy
                   : (QT == kQtQ80 ? kQ80GroupBytes
                                   : (QT == kQtQ5K ? kQ5BlockBytes : (REPACK ? BLOCK_BYTES : kGemvPitch)));
  // Q8_0 (272-byte rows): the reduction buffer lies in the weight ring, which is
  // free once every stage has been consumed, so 32 tokens still fit two CTAs per SM
  static constexpr bool red_in_ring = QT == kQtQ80;
  static constexpr size_t red_bytes = (size_t)16 * TILES * WARPS * TOK * 4;
  static constexpr int warp_tile = 16 * TILES * pitch;
  static constexpr size_t wstage = (size_t)WARPS * warp_tile;
  static constexpr size_t xstage = (size_t)TOK * kXRec;
  static constexpr __host__ __device__ size_t xring_off(int ws) { return (size_t)ws * wstage; }
  static constexpr __host__ __device__ size_t red_off(int ws, int xsn) {
    return red_in_ring ? 0 : xring_off(ws) + (size_t)xsn * xstage;
  }
  static constexpr __host__ __device__ size_t bar_off(int ws, int xsn) {
    return xring_off(ws) + (size_t)xsn * xstage + (red_in_ring ? 0 : red_bytes);
  }
  static constexpr __host__ __device__ size_t total(int ws, int xsn) { return bar_off(ws, xsn) + 16 * (ws + xsn) + 16; }
};

// The eight six-bit scales and mins of a block, four per word as bytes:
// sc[0] = sc0..3, sc[1] = sc4..7, mn[0] = m0..3, mn[1] = m4..7.
__device__ __forceinline__ void unpack_scales(uint32_t s0, uint32_t s1, uint32_t s2, uint32_t (&sc)[2],
                                              uint32_t (&mn)[2]) {
  sc[0] = s0 & 0x3F3F3F3Fu;
  mn[0] = s1 & 0x3F3F3F3Fu;
  sc[1] = (s2 & 0x0F0F0F0Fu) | ((s0 >> 2) & 0x30303030u);
  mn[1] = ((s2 >> 4) & 0x0F0F0F0Fu) | ((s1 >> 2) & 0x30303030u);
}

__device__ __forceinline__ void bulk_copy_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// The 4 bytes at a 2-byte-aligned shared-memory address (its row has slack after it).
__device__ __forceinline__ uint32_t lds_word_a2(const uint8_t* p) {
  const uintptr_t a = reinterpret_cast<uintptr_t>(p);
  const uint32_t* q = reinterpret_cast<const uint32_t*>(a & ~static_cast<uintptr_t>(3));
  return __funnelshift_r(q[0], q[1], (uint32_t)(a & 3) * 8u);
}

// Signed scale byte j (0..3) of a word, as an exact fp32: (2^23 + 128 + s) - (2^23 + 128).
__device__ __forceinline__ float s8_to_f32(uint32_t w, int j) {
  return __uint_as_float(__byte_perm(w ^ 0x80808080u, 0x4B000000u, 0x7650u | (uint32_t)j)) - 8388736.f;
}

// One Q6_K stage of a consumer warp: its rows g + 8r (r < 2*TILES) of the warp tile wt,
// row r's block starting off[r] bytes into its copy, times the stage's activation
// records xb for MT token groups; acc += d * 2^-k * sum_i scale_i * (q . x)_i.
// One mma.sync m16n8k16 per 16-weight sub-block (n, u, lh), tile and token group: thread
// t takes weights 16lh + 4t + {0..3}, so its ql and qh data are one word each per row;
// the six bits go into the low byte of 0x6400 = 1024 + (q + 32) and one fp16 add of
// -1056 leaves q itself, exact. The signed scale multiplies the fp32 MMA result. The
// record holds the matching activations in the 8-byte half t%2 of chunk
// 4(4n + u) + 2lh + t/2 (the order the pre-pass gives every 32-wide column).
template <int MT, int TILES>
__device__ __forceinline__ void q6_stage(float (&acc)[TILES][MT][4], const uint8_t* wt, const int (&off)[2 * TILES],
                                         const uint8_t* xb, int g, int t) {
  constexpr int R = 2 * TILES;
  const uint8_t* rb[R];
  uint32_t sc[R][4];
  float d[R];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    rb[r] = wt + (g + 8 * r) * kQ6Copy + off[r];
#pragma unroll
    for (int i = 0; i < 4; ++i) sc[r][i] = lds_word_a2(rb[r] + 192 + 4 * i);
    d[r] = __half2float(*reinterpret_cast<const __half*>(rb[r] + 208));
  }
  const __half2 m1056 = __float2half2_rn(-1056.f);
  float C[TILES][MT][4];
#pragma unroll
  for (int n = 0; n < 2; ++n) {
#pragma unroll
    for (int lh = 0; lh < 2; ++lh) {
      const int o = 64 * n + 16 * lh + 4 * t;
      uint32_t la[R], lb[R], hq[R];  // ql words for u = 0, 2 and u = 1, 3; qh for all four
#pragma unroll
      for (int r = 0; r < R; ++r) {
        la[r] = lds_word_a2(rb[r] + o);
        lb[r] = lds_word_a2(rb[r] + o + 32);
        hq[r] = lds_word_a2(rb[r] + 128 + 32 * n + 16 * lh + 4 * t);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int si = 8 * n + 2 * u + lh;  // scale index (weight / 16)
        uint32_t lo[R], hi[R];
        float s[R];
#pragma unroll
        for (int r = 0; r < R; ++r) {
          // six-bit values q + 32 of the four weights, one per byte
          const uint32_t v = ((((u & 1) ? lb[r] : la[r]) >> (4 * (u >> 1))) & 0x0F0F0F0Fu) |
                             (((hq[r] >> (2 * u)) & 0x03030303u) << 4);
          lo[r] = h2_bits(__hadd2(bits_h2(__byte_perm(v, 0x64646464u, 0x4240u)), m1056));  // weights 4t, 4t+2
          hi[r] = h2_bits(__hadd2(bits_h2(__byte_perm(v, 0x64646464u, 0x4341u)), m1056));  // 4t+1, 4t+3
          s[r] = s8_to_f32(sc[r][si >> 2], si & 3);
        }
        const int boff = (4 * (4 * n + u) + 2 * lh + (t >> 1)) * 16 + 8 * (t & 1);
#pragma unroll
        for (int f = 0; f < MT; ++f) {
          const uint2 bx = *reinterpret_cast<const uint2*>(xb + (8 * f + g) * kXRec + boff);
#pragma unroll
          for (int tt = 0; tt < TILES; ++tt) {
            // A: rows g (regs 0, 2) and g+8 (regs 1, 3) of tile tt
            float Cj[4];
            mma_f16_16816(Cj, lo[2 * tt], lo[2 * tt + 1], hi[2 * tt], hi[2 * tt + 1], bx.x, bx.y, true);
            const float sa = s[2 * tt], sb = s[2 * tt + 1];
            if (si == 0) {
              C[tt][f][0] = sa * Cj[0];
              C[tt][f][1] = sa * Cj[1];
              C[tt][f][2] = sb * Cj[2];
              C[tt][f][3] = sb * Cj[3];
            } else {
              C[tt][f][0] = fmaf(sa, Cj[0], C[tt][f][0]);
              C[tt][f][1] = fmaf(sa, Cj[1], C[tt][f][1]);
              C[tt][f][2] = fmaf(sb, Cj[2], C[tt][f][2]);
              C[tt][f][3] = fmaf(sb, Cj[3], C[tt][f][3]);
            }
          }
        }
      }
    }
  }
  // y += d * 2^-k * C (2^-k of tokens 2t and 2t+1 of each group, from the records)
#pragma unroll
  for (int f = 0; f < MT; ++f) {
    const float k0 = *reinterpret_cast<const float*>(xb + (8 * f + 2 * t) * kXRec + 544);
    const float k1 = *reinterpret_cast<const float*>(xb + (8 * f + 2 * t + 1) * kXRec + 544);
#pragma unroll
    for (int tt = 0; tt < TILES; ++tt) {
      const float da = d[2 * tt], db = d[2 * tt + 1];
      acc[tt][f][0] = fmaf(da * k0, C[tt][f][0], acc[tt][f][0]);
      acc[tt][f][1] = fmaf(da * k1, C[tt][f][1], acc[tt][f][1]);
      acc[tt][f][2] = fmaf(db * k0, C[tt][f][2], acc[tt][f][2]);
      acc[tt][f][3] = fmaf(db * k1, C[tt][f][3], acc[tt][f][3]);
    }
  }
}

// Roles: warps 0..WARPS-1 consume (16*TILES weight rows each); warp WARPS issues
// the weight TMA; warp WARPS+1 copies the activation records.
// GROUPED: blockIdx.y enumerates non-empty experts (the y-th expert with a
// non-zero row count); SWIGLU: the first WARPS/2 consumer warps hold gate rows
// and the last WARPS/2 the matching up rows (at +N/2).
// QT: the weight format.
//  * Q5_K (176-byte super-blocks): the fifth bit of each quant is ORed into the
//    nibble field before either A form is built, so q runs to 31 and the
//    arithmetic stays exact (q*sc <= 1953 and 1024+16q <= 1520 in fp16).
//  * Q8_0 (eight 34-byte blocks per 256-wide column): the per-sub-block scaling
//    of the subnormal form at every token count, with A = the signed q itself as
//    an fp16 integer (-128..127, exact) and the block's d as the sub-block scale;
//    no min term.
//  * Q6_K (210-byte super-blocks): the weight producer warp issues one 224-byte
//    bulk copy per row (the block's 16-byte-aligned superset) instead of a TMA
//    box, and the consumers run q6_stage on each row from its own offset; no min
//    term.
template <int MT, int WARPS, int TILES, bool GROUPED, bool SWIGLU, bool REPACK = false, int QT = kQtQ4K>
__global__ void __launch_bounds__(32 * (WARPS + 2), 2) gemv_kernel(const __grid_constant__ CUtensorMap tmap_w,
                                                                   GemvParams p) {
  using L = GemvSmem<MT, WARPS, TILES, REPACK, QT>;
  static_assert(!REPACK || (!GROUPED && 16 * TILES * WARPS == kRepackRows), "repacked: dense, 128-row tiles");
  static_assert(QT == kQtQ4K || (!GROUPED && !REPACK), "Q5_K, Q8_0, Q6_K: dense raw layout");
  static_assert(QT != kQtQ6K || !SWIGLU, "Q6_K: plain output");
  constexpr bool Q5 = QT == kQtQ5K, Q80 = QT == kQtQ80, Q8X = QT == kQtQ4KxQ8, Q6 = QT == kQtQ6K;
  constexpr int BB = Q80 ? kQ80GroupBytes : (Q5 ? kQ5BlockBytes : BLOCK_BYTES);  // bytes per 256-wide column
  constexpr int QO = Q5 ? kQ5QsOff : 16;                                         // offset of the nibble bytes
  constexpr int TOK = 8 * MT;
  // 1..16 tokens: the subnormal-nibble A operand with per-sub-block scaling after the
  // MMA (fewer instructions per weight); 17..32: fp16 sc*q built before the MMA
  // (the per-result scaling would grow with the token groups).
  constexpr bool SUBN = !Q8X && (Q80 || MT <= 2);
  constexpr int WROWS = 16 * TILES;    // weight rows per consumer warp
  constexpr int ROWS = WROWS * WARPS;  // weight rows per CTA
  extern __shared__ __align__(128) uint8_t smem[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int SW = p.wstages, SX = p.xstages;
  if (!REPACK && !Q6 && threadIdx.x == 32 * WARPS)  // the weight-TMA thread: fetch the descriptor meanwhile
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_w)) : "memory");

  const int rank = (int)(blockIdx.x % (unsigned)p.ksplit);
  const int tile = (int)(blockIdx.x / (unsigned)p.ksplit);
  const int kb0 = (int)((int64_t)rank * p.nkb / p.ksplit);
  const int kb1 = (int)((int64_t)(rank + 1) * p.nkb / p.ksplit);
  const int nk = kb1 - kb0;

  // ---- which tokens / matrix ----
  int expert = 0, row_base = 0, count = p.M;
  if (GROUPED) {
    // the expert offsets come from the routing kernels: wait for the pre-pass
    // (which itself waited for them) before reading
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // Find the blockIdx.y-th expert with a non-empty row range (every warp does
    // the same scan, so the result is uniform). The offsets of 128 experts are
    // loaded at once: one memory latency instead of one per 32 experts.
    const int want = (int)blockIdx.y;
    int found = -1, seen = 0;
    for (int e0 = 0; e0 < p.E && found < 0; e0 += 128) {
      bool ne[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int e = e0 + 32 * i + lane;
        ne[i] = e < p.E && __ldg(p.offsets + e + 1) > __ldg(p.offsets + e);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const unsigned bal = __ballot_sync(0xffffffffu, ne[i]);
        const int n = __popc(bal);
        if (found < 0 && want < seen + n) {
          unsigned b = bal;
          for (int j = 0; j < want - seen; ++j) b &= b - 1;
          found = e0 + 32 * i + __ffs(b) - 1;
        }
        seen += n;
      }
    }
    if (found < 0) return;  // uniform over the cluster (depends on blockIdx.y only)
    expert = found;
    row_base = p.offsets[found];
    count = p.offsets[found + 1] - row_base;
    if (count > TOK) {
      if (threadIdx.x == 0 && rank == 0) latch_status(Q4K_ERR_DEVICE_BOUNDS);
      count = TOK;
    }
  }

  uint8_t* xring = smem + L::xring_off(SW);
  float* red = reinterpret_cast<float*>(smem + L::red_off(SW, SX));
  const uint32_t bar0 = smem_u32(smem + L::bar_off(SW, SX));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::bar_off(SW, SX) + 16 * (SW + SX));
  auto wfull = [&](int s) { return bar0 + 8u * s; };
  auto wempty = [&](int s) { return bar0 + 8u * (SW + s); };
  auto xfull = [&](int s) { return bar0 + 8u * (2 * SW + s); };
  auto xempty = [&](int s) { return bar0 + 8u * (2 * SW + SX + s); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < SW; ++s) {
      mbar_init(wfull(s), 1);
      mbar_init(wempty(s), WARPS);
    }
    for (int s = 0; s < SX; ++s) {
      mbar_init(xfull(s), 1);
      mbar_init(xempty(s), WARPS);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  if (warp == WARPS) {
    if (Q6) {
      // ---------------- weight producer, Q6_K: one 224-byte bulk copy per row ----------------
      // lane l copies row l of every warp tile; rows past N are not copied (no MMA tile
      // mixes them with real rows, and their results are never written)
      static_assert(!Q6 || 16 * TILES == 32, "Q6_K: one row per lane and warp tile");
      const int drop = g_test_drop_stage;  // test hook; -1 in normal use
      const int64_t row_bytes = (int64_t)p.nkb * kQ6BB;
      const int rbase = tile * ROWS + lane;
      uint32_t nrows = 0;
#pragma unroll
      for (int w = 0; w < WARPS; ++w) nrows += rbase + WROWS * w < p.N ? 1u : 0u;
      const uint32_t tx = __reduce_add_sync(0xffffffffu, nrows) * (uint32_t)kQ6Copy;
      int issued = 0, s = 0;
      uint32_t ph = 0;
      for (int ks = 0; ks < nk; ++ks) {
        int ok = 1;
        if (lane == 0) {
          if (ks >= SW) mbar_wait(wempty(s), ph ^ 1u, abort_flag);
          ok = !*abort_flag;
        }
        if (!__shfl_sync(0xffffffffu, ok, 0)) break;
        if (ks != drop) {
          if (lane == 0) mbar_arrive_expect_tx(wfull(s), tx);
          __syncwarp();
          const int64_t kofs = (int64_t)(kb0 + ks) * kQ6BB;
          const uint32_t dst = smem_u32(smem) + (uint32_t)(s * L::wstage) + (uint32_t)(lane * kQ6Copy);
#pragma unroll
          for (int w = 0; w < WARPS; ++w) {
            const int r = rbase + WROWS * w;
            if (r < p.N)
              bulk_copy_g2s(dst + (uint32_t)(w * L::warp_tile), p.W + (((int64_t)r * row_bytes + kofs) & ~(int64_t)15),
                            (uint32_t)kQ6Copy, wfull(s));
          }
        }
        ++issued;
        if (++s == SW) {
          s = 0;
          ph ^= 1u;
        }
      }
      if (lane == 0)
        for (int ks = (issued > SW ? issued - SW : 0); ks < issued; ++ks)
          if (ks != drop) mbar_wait_drain(wfull(ks % SW), (ks / SW) & 1);
    } else if (lane == 0) {
      // ---------------- weight producer: TMA ----------------
      const int lim = SWIGLU ? p.N / 2 : p.N;
      const int drop = g_test_drop_stage;  // test hook; -1 in normal use
      int issued = 0;
      int s = 0;
      uint32_t ph = 0;  // stage index and the parity of its current use (no divisions)
      for (int ks = 0; ks < nk; ++ks) {
        if (ks >= SW) mbar_wait(wempty(s), ph ^ 1u, abort_flag);
        if (*abort_flag) break;
        if (ks == drop) {  // test hook: this stage never arrives
          ++issued;
          if (++s == SW) {
            s = 0;
            ph ^= 1u;
          }
          continue;
        }
        mbar_arrive_expect_tx(wfull(s), (uint32_t)(WARPS * L::warp_tile));
        const uint32_t dst = smem_u32(smem) + (uint32_t)(s * L::wstage);
        const int x = (kb0 + ks) * BB / (Q80 ? 2 : 1);  // Q8_0: 16-bit elements (272 bytes = 136)
        if (REPACK) {  // the tile's super-block column is one contiguous 18 KB run
          const uint8_t* src = p.W + ((size_t)tile * p.nkb + (kb0 + ks)) * (size_t)L::wstage;
          bulk_copy_g2s(dst, src, (uint32_t)L::wstage, wfull(s));
        }
#pragma unroll
        for (int w = 0; w < (REPACK ? 0 : WARPS); ++w) {
          int r0 = SWIGLU ? tile * (ROWS / 2) + WROWS * (w % (WARPS / 2)) : tile * ROWS + WROWS * w;
          r0 = min(r0, lim);  // rows past the end read zeros (or are ignored)
          const int row = expert * p.N + (SWIGLU && w >= WARPS / 2 ? p.N / 2 : 0) + r0;
          tma_load_2d(dst + w * L::warp_tile, &tmap_w, x, row, wfull(s));
        }
        ++issued;
        if (++s == SW) {
          s = 0;
          ph ^= 1u;
        }
      }
      // Every issued stage must land before the CTA exits, abort or not (normally
      // the consumers have already waited for all of them).
      for (int ks = (issued > SW ? issued - SW : 0); ks < issued; ++ks)
        if (ks != drop) mbar_wait_drain(wfull(ks % SW), (ks / SW) & 1);
    }
  } else if (warp == WARPS + 1) {
    // ---------------- activation producer: bulk copies of prepared records ----------------
    if (lane == 0) {
      asm volatile("griddepcontrol.wait;" ::: "memory");  // the pre-pass has finished
      // only the token groups that hold rows of this call (or expert) are copied
      const uint32_t xbytes = (uint32_t)(((count + 7) / 8) * 8 * kXRec);
      int issued = 0;
      int s = 0;
      uint32_t ph = 0;
      for (int ks = 0; ks < nk; ++ks) {
        if (ks >= SX) mbar_wait(xempty(s), ph ^ 1u, abort_flag);
        if (*abort_flag) break;
        mbar_arrive_expect_tx(xfull(s), xbytes);
        const uint8_t* src = p.xprep + ((int64_t)(kb0 + ks) * p.rows_pad + row_base) * kXRec;
        bulk_copy_g2s(smem_u32(xring) + (uint32_t)(s * L::xstage), src, xbytes, xfull(s));
        ++issued;
        if (++s == SX) {
          s = 0;
          ph ^= 1u;
        }
      }
      for (int ks = (issued > SX ? issued - SX : 0); ks < issued; ++ks)
        mbar_wait_drain(xfull(ks % SX), (ks / SX) & 1);
    }
  } else {
    // ---------------- consumers ----------------
    const int r0 = SWIGLU ? tile * (ROWS / 2) + WROWS * (warp % (WARPS / 2)) : tile * ROWS + WROWS * warp;
    const bool valid = r0 < (SWIGLU ? p.N / 2 : p.N);
    float acc[TILES][MT][4];
#pragma unroll
    for (int r = 0; r < TILES; ++r)
#pragma unroll
      for (int f = 0; f < MT; ++f)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[r][f][e] = 0.f;
    const __half2 neg1024 = __float2half2_rn(-1024.f);
    const __half2 sixteenth = __float2half2_rn(0.0625f);
    const __half2 neg64 = __float2half2_rn(-64.f);

    // Q6_K: row g + 8r of this warp starts (its offset + 210 kb) mod 16 bytes into its copy
    int q6off[Q6 ? 2 * TILES : 1];
#pragma unroll
    for (int r = 0; r < (Q6 ? 2 * TILES : 0); ++r)
      q6off[r] = (int)(((int64_t)(r0 + g + 8 * r) * ((int64_t)p.nkb * kQ6BB)) & 15);
    int sw = 0, sx = 0;
    uint32_t pw = 0, px = 0;  // ring stage indices and phase parities (no divisions)
    for (int ks = 0; ks < nk; ++ks) {
      mbar_wait(wfull(sw), pw, abort_flag);
      const int sw_cur = sw;
      const uint8_t* wt = smem + sw * L::wstage + warp * L::warp_tile;
      if (Q6) {
        // the stage's weights are read from shared memory until the end: both rings are
        // released together
        mbar_wait(xfull(sx), px, abort_flag);
        if (valid) {
          int off[2 * TILES];
#pragma unroll
          for (int r = 0; r < 2 * TILES; ++r) off[r] = (q6off[r] + (kb0 + ks) * kQ6BB) & 15;
          q6_stage<MT, TILES>(acc, wt, off, xring + (size_t)sx * L::xstage, g, t);
        }
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(wempty(sw));
          mbar_arrive(xempty(sx));
        }
        if (++sw == SW) {
          sw = 0;
          pw ^= 1u;
        }
        if (++sx == SX) {
          sx = 0;
          px ^= 1u;
        }
        continue;
      }
      // rows g, g+8 (tile 0), g+16, g+24 (tile 1), ... of this warp's rows
      constexpr int R = 2 * TILES;
      uint32_t hdx[R];
      uint32_t scw[R][2], mnw[R][2];
      uint2 qv[R][4];  // [row][chunk]
      uint2 qhv[R];    // Q5: this thread's fifth-bit bytes qh[8t .. 8t+7] of each row
#pragma unroll
      for (int r = 0; r < (Q80 ? 0 : R); ++r) {  // Q8_0 reads its blocks sub-block by sub-block below
        const uint8_t* rp = wt + (g + 8 * r) * L::pitch;
        const uint4 hd = *reinterpret_cast<const uint4*>(rp);
        hdx[r] = hd.x;
        unpack_scales(hd.y, hd.z, hd.w, scw[r], mnw[r]);
        if (REPACK) {  // this thread's bytes [8t, 8t+8) of chunks 0..3, stored together
          const uint4 q01 = *reinterpret_cast<const uint4*>(rp + 16 + 32 * t);
          const uint4 q23 = *reinterpret_cast<const uint4*>(rp + 32 + 32 * t);
          qv[r][0] = make_uint2(q01.x, q01.y);
          qv[r][1] = make_uint2(q01.z, q01.w);
          qv[r][2] = make_uint2(q23.x, q23.y);
          qv[r][3] = make_uint2(q23.z, q23.w);
        } else {
#pragma unroll
          for (int c = 0; c < 4; ++c) qv[r][c] = *reinterpret_cast<const uint2*>(rp + QO + 32 * c + 8 * t);
        }
        if (Q5) qhv[r] = *reinterpret_cast<const uint2*>(rp + kQ5QhOff + 8 * t);
      }
      if (!Q80) {
        __syncwarp();
        if (lane == 0) mbar_arrive(wempty(sw));  // the weight tile is in registers: release it
      }
      if (++sw == SW) {
        sw = 0;
        pw ^= 1u;
      }
      mbar_wait(xfull(sx), px, abort_flag);
      const uint8_t* xb = xring + (size_t)sx * L::xstage;
      if (valid) {
        float C[TILES][MT][4];
        int IA[TILES][MT][4];  // Q8 lane: sum_j sc_j * (q_w . q_x) of the super-block, exact
#pragma unroll
        for (int tt = 0; tt < TILES; ++tt)
#pragma unroll
          for (int f = 0; f < MT; ++f)
#pragma unroll
            for (int e = 0; e < 4; ++e) IA[tt][f][e] = 0;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t qs8[R][2];  // words shifted by 8: bytes 1,3 in the positions of bytes 0,2
#pragma unroll
          for (int r = 0; r < R; ++r) {
            qs8[r][0] = qv[r][c].x >> 8;
            qs8[r][1] = qv[r][c].y >> 8;
          }
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int j = 2 * c + h;  // sub-block
            const uint32_t msk = h ? 0x00F000F0u : 0x000F000Fu;
            if (Q8X) {
              // Q8 lane: A = the sub-block's nibbles as bytes (k slots 4t.. from word x, 16+4t..
              // from word y, so B is the codes in natural order: eight bytes at 32j + 8t); one
              // integer MMA per token group, the six-bit scale applied in int32
              uint32_t A8[TILES][4];
              int sci[R];
#pragma unroll
              for (int r = 0; r < R; ++r) sci[r] = (int)((scw[r][j >> 2] >> (8 * (j & 3))) & 0xFFu);
#pragma unroll
              for (int tt = 0; tt < TILES; ++tt) {
                const int ra = 2 * tt, rb = 2 * tt + 1;
                const uint32_t sh = 4 * h;
                A8[tt][0] = (qv[ra][c].x >> sh) & 0x0F0F0F0Fu;
                A8[tt][1] = (qv[rb][c].x >> sh) & 0x0F0F0F0Fu;
                A8[tt][2] = (qv[ra][c].y >> sh) & 0x0F0F0F0Fu;
                A8[tt][3] = (qv[rb][c].y >> sh) & 0x0F0F0F0Fu;
              }
#pragma unroll
              for (int f = 0; f < MT; ++f) {
                if (GROUPED && 8 * f >= count) break;
                const uint2 bq = *reinterpret_cast<const uint2*>(xb + (8 * f + g) * kXRec + 32 * j + 8 * t);
#pragma unroll
                for (int tt = 0; tt < TILES; ++tt) {
                  int ci[4];
                  imma_16832(ci, A8[tt][0], A8[tt][1], A8[tt][2], A8[tt][3], bq.x, bq.y);
                  IA[tt][f][0] += sci[2 * tt] * ci[0];
                  IA[tt][f][1] += sci[2 * tt] * ci[1];
                  IA[tt][f][2] += sci[2 * tt + 1] * ci[2];
                  IA[tt][f][3] += sci[2 * tt + 1] * ci[3];
                }
              }
              continue;
            }
            // Q5: fifth bits of the four weights in bytes {0,2} (e = 0) and {1,3} (e = 1) of
            // each quant word, at bit 4 (low nibbles: q + 16*bit) or 8 (high: 16q + 256*bit)
            uint32_t hb[R][2][2];  // [row][k-step][byte pair]
#pragma unroll
            for (int r = 0; r < R; ++r)
#pragma unroll
              for (int st = 0; st < 2; ++st) {
                hb[r][st][0] = hb[r][st][1] = 0u;
                if (Q5) {
                  const uint32_t wq = st ? qhv[r].y : qhv[r].x;
                  hb[r][st][0] = fifth_bits(wq, j, 4 + 4 * h);
                  hb[r][st][1] = fifth_bits(wq >> 8, j, 4 + 4 * h);
                }
              }
            if (SUBN) {
              // A = the raw nibble field as fp16 bits: q * 2^-24 (low nibble) or 16q * 2^-24
              // (high), fp16 subnormals, which the tensor core multiplies exactly. The
              // sub-block's two k-steps accumulate on their own; its scale, sc (sc/16 for
              // high nibbles) as an exact fp32, is applied to the per-row results.
              float fs[R];
              uint32_t A[TILES][2][4];
              if (Q80) {
                // block j of this 256-wide column: fp16 d at byte 34j, q[8t .. 8t+7] at
                // 34j + 2 + 8t (4-byte aligned for odd j; for even j two funnel shifts
                // realign three aligned words), each byte's sign bit flipped: q + 128 in
                // 0..255, the low byte of 0x6400 = 1024 + (q + 128); one fp16 add of -1152
                // then leaves q itself, exact (the weight enters the MMA as the signed
                // integer: no offset term whose cancellation would cost accuracy)
                uint32_t xw[R][2];
#pragma unroll
                for (int r = 0; r < R; ++r) {
                  const uint8_t* rp = wt + (g + 8 * r) * L::pitch;
                  const uint32_t dw = *reinterpret_cast<const uint32_t*>(rp + ((34 * j) & ~3));
                  fs[r] = half_bits_to_float((j & 1) ? (dw >> 16) : (dw & 0xFFFFu));
                  const int base = 34 * j + 2 + 8 * t;
                  if (j & 1) {
                    xw[r][0] = *reinterpret_cast<const uint32_t*>(rp + base);
                    xw[r][1] = *reinterpret_cast<const uint32_t*>(rp + base + 4);
                  } else {
                    const uint32_t w0 = *reinterpret_cast<const uint32_t*>(rp + base - 2);
                    const uint32_t w1 = *reinterpret_cast<const uint32_t*>(rp + base + 2);
                    const uint32_t w2 = *reinterpret_cast<const uint32_t*>(rp + base + 6);
                    xw[r][0] = __funnelshift_r(w0, w1, 16);
                    xw[r][1] = __funnelshift_r(w1, w2, 16);
                  }
                  xw[r][0] ^= 0x80808080u;
                  xw[r][1] ^= 0x80808080u;
                }
#pragma unroll
                for (int tt = 0; tt < TILES; ++tt) {
                  const int ra = 2 * tt, rb = 2 * tt + 1;
#pragma unroll
                  for (int st = 0; st < 2; ++st) {  // bytes {0,2} and {1,3} into the low byte of each half
                    const __half2 off = __float2half2_rn(-1152.f);
                    A[tt][st][0] = h2_bits(__hadd2(bits_h2(__byte_perm(xw[ra][st], 0x64646464u, 0x4240u)), off));
                    A[tt][st][1] = h2_bits(__hadd2(bits_h2(__byte_perm(xw[rb][st], 0x64646464u, 0x4240u)), off));
                    A[tt][st][2] = h2_bits(__hadd2(bits_h2(__byte_perm(xw[ra][st], 0x64646464u, 0x4341u)), off));
                    A[tt][st][3] = h2_bits(__hadd2(bits_h2(__byte_perm(xw[rb][st], 0x64646464u, 0x4341u)), off));
                  }
                }
              } else {
#pragma unroll
                for (int r = 0; r < R; ++r) {  // 0x4B0000sc = 2^23 + sc; 0x490000sc = 2^19 + sc/16
                  const uint32_t bits = __byte_perm(scw[r][j >> 2], h ? 0x49000000u : 0x4B000000u,
                                                    0x7650u | (uint32_t)(j & 3));
                  fs[r] = __uint_as_float(bits) - (h ? 524288.f : 8388608.f);
                }
#pragma unroll
                for (int tt = 0; tt < TILES; ++tt) {
                  const int ra = 2 * tt, rb = 2 * tt + 1;
#pragma unroll
                  for (int st = 0; st < 2; ++st) {
                    A[tt][st][0] = and_or((st ? qv[ra][c].y : qv[ra][c].x), msk, hb[ra][st][0]);
                    A[tt][st][1] = and_or((st ? qv[rb][c].y : qv[rb][c].x), msk, hb[rb][st][0]);
                    A[tt][st][2] = and_or(qs8[ra][st], msk, hb[ra][st][1]);
                    A[tt][st][3] = and_or(qs8[rb][st], msk, hb[rb][st][1]);
                  }
                }
              }
#pragma unroll
              for (int f = 0; f < MT; ++f) {
                if (GROUPED && 8 * f >= count) break;  // token groups past this expert's rows
                const uint4 bx = *reinterpret_cast<const uint4*>(xb + (8 * f + g) * kXRec + (j * 4 + t) * 16);
#pragma unroll
                for (int tt = 0; tt < TILES; ++tt) {
                  float Cj[4];
                  mma_f16_16816(Cj, A[tt][0][0], A[tt][0][1], A[tt][0][2], A[tt][0][3], bx.x, bx.y, true);
                  mma_f16_16816(Cj, A[tt][1][0], A[tt][1][1], A[tt][1][2], A[tt][1][3], bx.z, bx.w, false);
                  const float fa = fs[2 * tt], fb = fs[2 * tt + 1];
                  if (j == 0) {
                    C[tt][f][0] = fa * Cj[0];
                    C[tt][f][1] = fa * Cj[1];
                    C[tt][f][2] = fb * Cj[2];
                    C[tt][f][3] = fb * Cj[3];
                  } else {
                    C[tt][f][0] = fmaf(fa, Cj[0], C[tt][f][0]);
                    C[tt][f][1] = fmaf(fa, Cj[1], C[tt][f][1]);
                    C[tt][f][2] = fmaf(fb, Cj[2], C[tt][f][2]);
                    C[tt][f][3] = fmaf(fb, Cj[3], C[tt][f][3]);
                  }
                }
              }
              continue;
            }
            // per row: multiplier (sc, or sc/16 for high nibbles) and bias -1024 * multiplier
            __half2 mul[R], cst[R];
#pragma unroll
            for (int r = 0; r < R; ++r) {
              const __half2 s1024 = bits_h2(bytes_1024(scw[r][j >> 2], j & 3, j & 3));
              mul[r] = h ? __hfma2(s1024, sixteenth, neg64) : __hadd2(s1024, neg1024);
              cst[r] = __hmul2(mul[r], neg1024);
            }
            uint32_t A[TILES][2][4];  // [tile][k-step][reg], fp16 q*sc
#pragma unroll
            for (int tt = 0; tt < TILES; ++tt) {
              const int ra = 2 * tt, rb = 2 * tt + 1;  // rows g(+16), g+8(+16)
#pragma unroll
              for (int st = 0; st < 2; ++st) {
                const uint32_t wa = st ? qv[ra][c].y : qv[ra][c].x, wb = st ? qv[rb][c].y : qv[rb][c].x;
                const uint32_t sa = qs8[ra][st], sbw = qs8[rb][st];
                A[tt][st][0] = h2_bits(__hfma2(bits_h2(and_or(wa, msk, 0x64006400u | hb[ra][st][0])), mul[ra], cst[ra]));
                A[tt][st][1] = h2_bits(__hfma2(bits_h2(and_or(wb, msk, 0x64006400u | hb[rb][st][0])), mul[rb], cst[rb]));
                A[tt][st][2] = h2_bits(__hfma2(bits_h2(and_or(sa, msk, 0x64006400u | hb[ra][st][1])), mul[ra], cst[ra]));
                A[tt][st][3] = h2_bits(__hfma2(bits_h2(and_or(sbw, msk, 0x64006400u | hb[rb][st][1])), mul[rb], cst[rb]));
              }
            }
#pragma unroll
            for (int f = 0; f < MT; ++f) {
              if (GROUPED && 8 * f >= count) break;  // token groups past this expert's rows
              const uint4 bx = *reinterpret_cast<const uint4*>(xb + (8 * f + g) * kXRec + (j * 4 + t) * 16);
#pragma unroll
              for (int tt = 0; tt < TILES; ++tt) {
                mma_f16_16816(C[tt][f], A[tt][0][0], A[tt][0][1], A[tt][0][2], A[tt][0][3], bx.x, bx.y,
                              j == 0);
                mma_f16_16816(C[tt][f], A[tt][1][0], A[tt][1][1], A[tt][1][2], A[tt][1][3], bx.z, bx.w,
                              false);
              }
            }
          }
        }
        if (Q8X) {  // the super-block's exact integer sums (|IA| < 2^31) as fp32
#pragma unroll
          for (int tt = 0; tt < TILES; ++tt)
#pragma unroll
            for (int f = 0; f < MT; ++f)
#pragma unroll
              for (int e = 0; e < 4; ++e) C[tt][f][e] = (float)IA[tt][f][e];
        }
        // min term: Cm = sum_j m_j * X_j (k = sub-block index; k >= 8 is zero)
        uint32_t am[R];
        const uint32_t mb = 2u * (t & 1);
#pragma unroll
        for (int r = 0; r < R; ++r) {
          if (Q80) {  // Q8_0 has no min term
            am[r] = 0u;
          } else {
            am[r] = h2_bits(__hadd2(bits_h2(bytes_1024((t >> 1) ? mnw[r][1] : mnw[r][0], mb, mb + 1)),
                                    neg1024));
          }
        }
        float dd[R], dn[R];
#pragma unroll
        for (int r = 0; r < R; ++r) {
          // the subnormal form's products carry 2^-24: fold 2^24 into d
          // (Q8_0: A is q itself and the block scales d_j are already in C)
          dd[r] = Q80 ? 1.f : (SUBN ? 16777216.f : 1.f) * half_bits_to_float(hdx[r]);
          dn[r] = Q80 ? 0.f : 64.f * half_bits_to_float(hdx[r] >> 16);
        }
#pragma unroll
        for (int f = 0; f < MT; ++f) {
          if (GROUPED && 8 * f >= count) break;
          const uint8_t* rg = xb + (8 * f + g) * kXRec;
          const uint32_t bh = *reinterpret_cast<const uint32_t*>(rg + 512 + 4 * t);
          const uint32_t bl = *reinterpret_cast<const uint32_t*>(rg + 528 + 4 * t);
          const float s0 = *reinterpret_cast<const float*>(xb + (8 * f + 2 * t) * kXRec + 544);
          const float s1 = *reinterpret_cast<const float*>(xb + (8 * f + 2 * t + 1) * kXRec + 544);
#pragma unroll
          for (int tt = 0; tt < TILES; ++tt) {
            float Cm[4] = {0.f, 0.f, 0.f, 0.f};
            if (!Q80) {
              mma_f16_16816(Cm, am[2 * tt], am[2 * tt + 1], 0u, 0u, bh, 0u, true);
              mma_f16_16816(Cm, am[2 * tt], am[2 * tt + 1], 0u, 0u, bl, 0u, false);
            }
            const float dA = dd[2 * tt], dB = dd[2 * tt + 1], mA = dn[2 * tt], mB = dn[2 * tt + 1];
            acc[tt][f][0] = fmaf(-mA * s0, Cm[0], fmaf(dA * s0, C[tt][f][0], acc[tt][f][0]));
            acc[tt][f][1] = fmaf(-mA * s1, Cm[1], fmaf(dA * s1, C[tt][f][1], acc[tt][f][1]));
            acc[tt][f][2] = fmaf(-mB * s0, Cm[2], fmaf(dB * s0, C[tt][f][2], acc[tt][f][2]));
            acc[tt][f][3] = fmaf(-mB * s1, Cm[3], fmaf(dB * s1, C[tt][f][3], acc[tt][f][3]));
          }
        }
      }
      if (Q80) {  // the weight stage was read until here
        __syncwarp();
        if (lane == 0) mbar_arrive(wempty(sw_cur));
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(xempty(sx));
      if (++sx == SX) {
        sx = 0;
        px ^= 1u;
      }
    }

    // ---- CTA partial -> shared memory, token-major: red[token][local row] ----
    // (in the weight ring for Q8_0: wait until every consumer warp is past its last stage)
    if (L::red_in_ring) asm volatile("bar.sync 1, %0;" ::"n"(32 * WARPS) : "memory");
#pragma unroll
    for (int tt = 0; tt < TILES; ++tt)
#pragma unroll
      for (int f = 0; f < MT; ++f) {
        const int lr = warp * WROWS + tt * 16 + g;
        const int i0 = 8 * f + 2 * t;
        red[(size_t)i0 * ROWS + lr] = acc[tt][f][0];
        red[(size_t)(i0 + 1) * ROWS + lr] = acc[tt][f][1];
        red[(size_t)i0 * ROWS + lr + 8] = acc[tt][f][2];
        red[(size_t)(i0 + 1) * ROWS + lr + 8] = acc[tt][f][3];
      }
  }

  cg::cluster_group cluster = cg::this_cluster();
  if (p.ksplit > 1) {
    cluster.sync();
  } else {
    __syncthreads();
  }

  // Cluster reduction, spread over the ranks: rank r sums a 1/ksplit slice of the
  // (token, 4 output rows) vectors over all ranks' partials, always in rank order
  // 0, 1, ..., so the result does not depend on which rank reduces it.
  {
    constexpr int OUTW = SWIGLU ? ROWS / 2 : ROWS;
    constexpr int VPT = OUTW / 4;  // float4 vectors per token
    const int nvec = count * VPT;
    const int per = (nvec + p.ksplit - 1) / p.ksplit;
    const int v0 = rank * per, v1 = min(nvec, v0 + per);
    for (int v = v0 + (int)threadIdx.x; v < v1; v += blockDim.x) {
      const int i = v / VPT, lr = (v % VPT) * 4;
      float4 g4 = make_float4(0.f, 0.f, 0.f, 0.f), u4 = g4;
      for (int r = 0; r < p.ksplit; ++r) {
        const float* rr = p.ksplit > 1 ? cluster.map_shared_rank(red, r) : red;
        const float4 a4 = *reinterpret_cast<const float4*>(rr + (size_t)i * ROWS + lr);
        g4.x += a4.x; g4.y += a4.y; g4.z += a4.z; g4.w += a4.w;
        if (SWIGLU) {
          const float4 b4 = *reinterpret_cast<const float4*>(rr + (size_t)i * ROWS + lr + ROWS / 2);
          u4.x += b4.x; u4.y += b4.y; u4.z += b4.z; u4.w += b4.w;
        }
      }
      if (SWIGLU) {
        const int half = p.N / 2;
        const int n = tile * (ROWS / 2) + lr;
        if (n < half) {  // half % 16 == 0, so all four are in range
          uint2 o;
          o.x = pack_bf16x2(silu_mul(g4.x, u4.x), silu_mul(g4.y, u4.y));
          o.y = pack_bf16x2(silu_mul(g4.z, u4.z), silu_mul(g4.w, u4.w));
          *reinterpret_cast<uint2*>(static_cast<uint16_t*>(p.out) + (int64_t)(row_base + i) * half + n) = o;
        }
      } else {
        const int n = tile * ROWS + lr;
        if (n < p.N) *reinterpret_cast<float4*>(static_cast<float*>(p.out) + (int64_t)(row_base + i) * p.N + n) = g4;
      }
    }
  }
  if (p.ksplit > 1) cluster.sync();  // keep every CTA's shared memory alive until all ranks are done
}

// Load-time repack (one thread per 8-byte unit of the output): row r of 128-row
// tile T, super-block kb lands at ((T*nkb + kb)*128 + r)*144; inside the 144
// bytes the header (units 0..1) stays and quant unit 2 + 4t + c takes the
// source's unit 2 + 4c + t (bytes [8t, 8t+8) of chunk c), so the eight bytes a
// GEMV thread t needs from each chunk follow one another. Rows past N are zero.
__global__ void __launch_bounds__(256) repack_kernel(const uint8_t* __restrict__ W, int N, int nkb,
                                                     uint8_t* __restrict__ Wr, int64_t units) {
  const int64_t row_bytes = (int64_t)nkb * BLOCK_BYTES;
  for (int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; u < units;
       u += (int64_t)gridDim.x * blockDim.x) {
    const int64_t blk = u / 18;  // output row-block, tile-major
    const int pu = (int)(u - blk * 18);
    const int r = (int)(blk % kRepackRows);
    const int64_t tk = blk / kRepackRows;
    const int kb = (int)(tk % nkb);
    const int64_t row = (tk / nkb) * kRepackRows + r;
    uint2 v = make_uint2(0u, 0u);
    if (row < N) {
      const int su = pu < 2 ? pu : 2 + 4 * ((pu - 2) & 3) + ((pu - 2) >> 2);
      v = *reinterpret_cast<const uint2*>(W + row * row_bytes + (int64_t)kb * BLOCK_BYTES + 8 * su);
    }
    *reinterpret_cast<uint2*>(Wr + blk * BLOCK_BYTES + 8 * pu) = v;
  }
}

inline int64_t repacked_bytes(int N, int K) {
  return (int64_t)((N + kRepackRows - 1) / kRepackRows) * kRepackRows * (K / QK) * BLOCK_BYTES;
}

// Raw Q4_K rows as bytes [rows][row_bytes], box 160 bytes x box_rows rows (one super-block
// per row plus 16 bytes of the next; past the end of a row the box reads zeros).
// elem_bytes 2 views the bytes as 16-bit elements, for boxes wider than the 256
// elements a box dimension may hold (the Q8_0 272-byte column); the kernel's x
// coordinates are then in those elements.
inline bool make_tmap_w_rowgroup(CUtensorMap* m, const void* base, int64_t rows, int64_t row_bytes,
                                 int box_rows, int box_bytes = kGemvPitch, int elem_bytes = 1) {
  auto enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)(row_bytes / elem_bytes), (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
  cuuint32_t box[2] = {(cuuint32_t)(box_bytes / elem_bytes), (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_UINT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
             const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Bytes of prepared-activation workspace for `rows` activation rows of K inputs.
inline size_t gemv_ws_bytes(int64_t rows, int K) {
  return (size_t)(K / QK) * (size_t)(rows + kXPadRows) * kXRec;
}

}  // namespace q4k
