// Q4_K decode GEMV (1..32 tokens) and its grouped mixture-of-experts form.
//
// Operation: Y[m][n] = sum_k w[n][k] * X[m][k] over Q4_K weights (hipEngine
// 0.3.0 README, "Quickstart": the GEMV-decode profile; hipster README claims
// table: "GEMV ... GB/s"). The weight stream from HBM is the roofline.
//
// Design (sm_100a):
//  * A producer warp streams the CTA's weight rows, one super-block column
//    (16 rows x 144 bytes per row group) per stage, into an S-deep shared
//    memory ring with TMA (cp.async.bulk.tensor) and mbarrier completion, so
//    many kilobytes per SM are in flight regardless of the compute loop.
//  * Consumer warps own 16 weight rows each. Weights are the 16-row A operand
//    of mma.sync m16n8k16 (bf16 in, fp32 accumulate); tokens are the 8-wide B
//    operand (MT fragments of 8 tokens).
//  * A nibble q ORed into the bf16 pattern 0x4300 is exactly 128+q, so two
//    weights become one bf16x2 register with a single mask/or. The bias is
//    removed per sub-block: with C = sum (128+q)*x and Sx = sum x,
//      sum_i w_i x_i = (d*sc) * C - (128*d*sc + dmin*m) * Sx,
//    applied with packed fp32x2 FMAs (one per pair of tokens).
//  * The k order inside a sub-block is free for a dot product, so each
//    thread takes the nibbles in the order the mask produces them, and the
//    activations staged in shared memory are stored in that same order.
//  * A CTA owns 16*WARPS weight rows and a contiguous range of super-blocks;
//    a thread-block cluster of KSPLIT CTAs covers the whole K range and its
//    partial sums are reduced in rank order through distributed shared memory
//    (deterministic, no atomics). The decomposition depends only on (N, K), so
//    a token's result never depends on the other tokens in the batch.
#pragma once
#include <cooperative_groups.h>

#include "common.cuh"
#include "gemm_tc.cuh"  // mbarrier / TMA wrappers

namespace q4k {

namespace cg = cooperative_groups;

constexpr uint32_t kBf16Bias2 = 0x43004300u;  // bf16x2 (128.0, 128.0)

__device__ __forceinline__ uint32_t nib2(uint32_t word, int shift) {
  return ((word >> shift) & 0x000F000Fu) | kBf16Bias2;
}

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1, bool zero_c) {
  if (zero_c) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%10,%10,%10,%10};"
        : "=f"(c[0]), "=f"(c[1]), "=f"(c[2]), "=f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(0.0f));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
}

// acc = fma(s, c, acc) on a pair of fp32 values with one packed instruction.
__device__ __forceinline__ void fma2(float& acc0, float& acc1, float s, float c0, float c1) {
  uint64_t a = (uint64_t)__float_as_uint(acc0) | ((uint64_t)__float_as_uint(acc1) << 32);
  const uint64_t sv = (uint64_t)__float_as_uint(s) | ((uint64_t)__float_as_uint(s) << 32);
  const uint64_t cv = (uint64_t)__float_as_uint(c0) | ((uint64_t)__float_as_uint(c1) << 32);
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(a) : "l"(sv), "l"(cv));
  acc0 = __uint_as_float((uint32_t)a);
  acc1 = __uint_as_float((uint32_t)(a >> 32));
}

__device__ __forceinline__ void consumer_sync(int nthreads) {
  asm volatile("bar.sync 1, %0;" ::"r"(nthreads) : "memory");
}

struct GemvParams {
  const uint8_t* W;          // dense: [N][nkb][144]; grouped: [E][N][nkb][144]
  const uint16_t* X;         // bf16 activations
  void* out;                 // fp32 [rows][N] or bf16 [rows][N/2] (SWIGLU)
  const int32_t* offsets;    // grouped: [E+1] rows per expert (device); dense: nullptr
  const int32_t* gather;     // grouped: optional sorted row -> X row
  int M;                     // dense: tokens; grouped: unused
  int N;                     // weight rows per matrix
  int K;
  int nkb;                   // K / 256
  int E;                     // grouped: experts
  int64_t expert_stride;     // bytes per expert matrix
  int ksplit;                // cluster size along K
  int kc;                    // super-blocks of activations staged per chunk (power of 2)
  int stages;                // weight ring depth
};

// Each consumer warp owns 32 weight rows (two 16-row MMA tiles). A stage of the
// weight ring holds, per warp, 32 rows x 160 bytes: one 144-byte super-block plus
// the first 16 bytes of the next (read and ignored) -- the 160-byte pitch makes the
// per-thread 8-byte quant reads bank-conflict-free.
constexpr int kGemvPitch = 160;
constexpr int kGemvWarpTile = 32 * kGemvPitch;  // 5120 B

// Shared memory layout (dynamic):
//   ring [stages][WARPS][32 rows][160 B]              weight tiles (TMA destination)
//   xs   [8*MT tokens][kc*8 sub-blocks][4][8] bf16    permuted activations of one chunk
//   xsum [kc*8][8*MT] fp32                            per sub-block sum of x
//   red  [32*WARPS rows][8*MT] fp32                   per-CTA partial result
//   bars [2*stages] mbarriers, abort flag
template <int MT, int WARPS>
struct GemvSmem {
  static constexpr size_t ring_stage = (size_t)WARPS * kGemvWarpTile;
  static __host__ __device__ size_t xs_off(int stages) { return (size_t)stages * ring_stage; }
  static __host__ __device__ size_t xsum_off(int stages, int kc) {
    return xs_off(stages) + (size_t)8 * MT * kc * 8 * 32 * 2;
  }
  static __host__ __device__ size_t red_off(int stages, int kc) {
    return xsum_off(stages, kc) + (size_t)kc * 8 * 8 * MT * 4;
  }
  static __host__ __device__ size_t bar_off(int stages, int kc) {
    return red_off(stages, kc) + (size_t)32 * WARPS * 8 * MT * 4;
  }
  static __host__ __device__ size_t total(int stages, int kc) { return bar_off(stages, kc) + 16 * stages + 16; }
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

// Byte b of `word` as the float 2^23 + byte (exact), by one byte permute.
__device__ __forceinline__ float byte_magic(uint32_t word, int b) {
  return __uint_as_float(__byte_perm(word, 0x4B000000u, 0x7650u | (uint32_t)b));
}

// GROUPED: blockIdx.y enumerates non-empty experts (the y-th expert with a
// non-zero row count); SWIGLU: the CTA's first WARPS/2 warps hold gate rows and
// the last WARPS/2 the matching up rows (at +N/2).
template <int MT, int WARPS, bool GROUPED, bool SWIGLU>
__global__ void __launch_bounds__(32 * (WARPS + 1)) gemv_kernel(const __grid_constant__ CUtensorMap tmap_w,
                                                                GemvParams p) {
  using L = GemvSmem<MT, WARPS>;
  constexpr int TOK = 8 * MT;
  constexpr int NCONS = 32 * WARPS;
  constexpr int ROWS = 32 * WARPS;  // weight rows per CTA
  extern __shared__ __align__(128) uint8_t smem[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int S = p.stages;

  const int rank = (int)(blockIdx.x % (unsigned)p.ksplit);
  const int tile = (int)(blockIdx.x / (unsigned)p.ksplit);
  const int kb0 = (int)((int64_t)rank * p.nkb / p.ksplit);
  const int kb1 = (int)((int64_t)(rank + 1) * p.nkb / p.ksplit);
  const int nk = kb1 - kb0;

  // ---- which tokens / matrix ----
  int expert = 0, row_base = 0, count = p.M;
  if (GROUPED) {
    // Find the blockIdx.y-th expert with a non-empty row range (every warp does
    // the same scan, so the result is uniform).
    const int want = (int)blockIdx.y;
    int found = -1, seen = 0;
    for (int e0 = 0; e0 < p.E && found < 0; e0 += 32) {
      const int e = e0 + lane;
      const bool ne = e < p.E && p.offsets[e + 1] > p.offsets[e];
      const unsigned bal = __ballot_sync(0xffffffffu, ne);
      const int n = __popc(bal);
      if (want < seen + n) {
        unsigned b = bal;
        for (int i = 0; i < want - seen; ++i) b &= b - 1;
        found = e0 + __ffs(b) - 1;
      }
      seen += n;
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

  uint16_t* xs = reinterpret_cast<uint16_t*>(smem + L::xs_off(S));
  float* xsum = reinterpret_cast<float*>(smem + L::xsum_off(S, p.kc));
  float* red = reinterpret_cast<float*>(smem + L::red_off(S, p.kc));
  const uint32_t bar0 = smem_u32(smem + L::bar_off(S, p.kc));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::bar_off(S, p.kc) + 16 * S);
  auto bar_full = [&](int s) { return bar0 + 8u * s; };
  auto bar_empty = [&](int s) { return bar0 + 8u * (S + s); };
  const int nsb = p.kc * 8;  // sub-blocks per staged chunk

  // First weight row (within the [E*N] row space) of warp w's 32 rows, and
  // whether those rows exist (N is a multiple of 16, so a warp's second
  // 16-row tile may be past the end while its first is not).
  auto warp_row = [&](int w) -> int {
    int r;
    if (SWIGLU) {
      r = (w < WARPS / 2 ? 0 : p.N / 2) + tile * (ROWS / 2) + 32 * (w % (WARPS / 2));
    } else {
      r = tile * ROWS + 32 * w;
    }
    return expert * p.N + r;
  };
  auto rows_left = [&](int w) -> int {  // rows of warp w's 32 that exist
    const int lim = SWIGLU ? p.N / 2 : p.N;
    const int r0 = SWIGLU ? tile * (ROWS / 2) + 32 * (w % (WARPS / 2)) : tile * ROWS + 32 * w;
    return max(0, min(32, lim - r0));
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(bar_full(s), 1);
      mbar_init(bar_empty(s), WARPS);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  // Token rows past `count` stay zero for the whole kernel.
  for (int it = threadIdx.x; it < (TOK - count) * nsb * 4; it += blockDim.x) {
    const int i = count + it / (nsb * 4), rest = it % (nsb * 4);
    *reinterpret_cast<uint4*>(xs + ((size_t)i * nsb * 4 + rest) * 8) = make_uint4(0u, 0u, 0u, 0u);
  }
  for (int it = threadIdx.x; it < nsb * TOK; it += blockDim.x)
    if (it % TOK >= count) xsum[it] = 0.f;
  __syncthreads();

  if (warp == WARPS) {
    // ---------------- producer: weight tiles by TMA ----------------
    if (lane == 0) {
      int issued = 0;
      for (int ks = 0; ks < nk; ++ks) {
        const int s = ks % S, u = ks / S;
        if (u >= 1) mbar_wait(bar_empty(s), (u - 1) & 1, abort_flag);
        if (*abort_flag) break;
        mbar_arrive_expect_tx(bar_full(s), (uint32_t)(WARPS * kGemvWarpTile));
        const uint32_t dst = smem_u32(smem) + (uint32_t)(s * L::ring_stage);
        const int x = (kb0 + ks) * BLOCK_BYTES;
#pragma unroll
        for (int w = 0; w < WARPS; ++w)
          tma_load_2d(dst + w * kGemvWarpTile, &tmap_w, x, warp_row(w), bar_full(s));
        ++issued;
      }
      // Every issued stage must land before the CTA exits (normally the
      // consumers have already waited for all of them).
      for (int ks = (issued > S ? issued - S : 0); ks < issued; ++ks)
        mbar_wait(bar_full(ks % S), (ks / S) & 1, abort_flag);
    }
  } else {
    // ---------------- consumers ----------------
    const int nrows = rows_left(warp);
    const bool valid = nrows > 0;
    float acc[2][MT][4];
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
      for (int f = 0; f < MT; ++f)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[r][f][e] = 0.f;

    for (int cb = kb0; cb < kb1;) {
      // chunk of kcn super-blocks: a power of two, at most kc
      int kcn = p.kc;
      while (kcn > kb1 - cb) kcn >>= 1;
      int lg = 5;  // log2 of the staging items per token (32 per super-block)
      while ((1 << lg) < 32 * kcn) ++lg;
      consumer_sync(NCONS);  // previous chunk fully consumed
      // Stage activations of super-blocks [cb, cb+kcn) for the real tokens: each run
      // of 8 consecutive k is stored permuted as (e0,e2),(e1,e3),(e4,e6),(e5,e7) to
      // match the A-fragment nibble order, plus the fp32 sum of every 32-wide
      // sub-block. Item = (token, sub-block, quarter of 8 k); a warp's 32 lanes take
      // 32 consecutive items of one token, so a sub-block's quarters are adjacent.
      auto row_of = [&](int i) -> const uint16_t* {
        int64_t xrow = i;
        if (GROUPED) xrow = p.gather ? p.gather[row_base + i] : (row_base + i);
        return p.X + xrow * p.K + (int64_t)cb * QK;
      };
      auto put = [&](int it, const uint4 v) {
        const int i = it >> lg, q = it & ((1 << lg) - 1);
        const int sidx = q >> 2, tq = q & 3;
        uint4 o;
        o.x = __byte_perm(v.x, v.y, 0x5410);  // (e0, e2)
        o.y = __byte_perm(v.x, v.y, 0x7632);  // (e1, e3)
        o.z = __byte_perm(v.z, v.w, 0x5410);  // (e4, e6)
        o.w = __byte_perm(v.z, v.w, 0x7632);  // (e5, e7)
        *reinterpret_cast<uint4*>(xs + (((size_t)i * nsb + sidx) * 4 + tq) * 8) = o;
        float sum = 0.f;
        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          sum += bf16_bits_to_float(w4[e] & 0xFFFFu);
          sum += bf16_bits_to_float(w4[e] >> 16);
        }
        sum += __shfl_xor_sync(0xffffffffu, sum, 1);
        sum += __shfl_xor_sync(0xffffffffu, sum, 2);
        if (tq == 0) xsum[(size_t)sidx * TOK + i] = sum;
      };
      const int total = count << lg;  // a multiple of 32: warps are fully in or out
      int it = threadIdx.x;
      for (; it + NCONS < total; it += 2 * NCONS) {  // two independent loads in flight
        const int q0 = it & ((1 << lg) - 1), q1 = (it + NCONS) & ((1 << lg) - 1);
        const uint4 v0 = ldg_u4(row_of(it >> lg) + (q0 >> 2) * 32 + (q0 & 3) * 8);
        const uint4 v1 = ldg_u4(row_of((it + NCONS) >> lg) + (q1 >> 2) * 32 + (q1 & 3) * 8);
        put(it, v0);
        put(it + NCONS, v1);
      }
      if (it < total) {
        const int q0 = it & ((1 << lg) - 1);
        put(it, ldg_u4(row_of(it >> lg) + (q0 >> 2) * 32 + (q0 & 3) * 8));
      }
      consumer_sync(NCONS);

      for (int kb = cb; kb < cb + kcn; ++kb) {
        const int ks = kb - kb0, s = ks % S;
        mbar_wait(bar_full(s), (ks / S) & 1, abort_flag);
        const uint8_t* wt = smem + s * L::ring_stage + warp * kGemvWarpTile;
        // rows g, g+8 (tile 0) and g+16, g+24 (tile 1) of this warp's 32
        uint4 hd[4];
        uint2 qv[4][4];  // [row][chunk]
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const uint8_t* rp = wt + (g + 8 * r) * kGemvPitch;
          hd[r] = *reinterpret_cast<const uint4*>(rp);
#pragma unroll
          for (int c = 0; c < 4; ++c) qv[r][c] = *reinterpret_cast<const uint2*>(rp + 16 + 32 * c + 8 * t);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_empty(s));  // the tile is in registers: release the slot
        if (!valid) continue;

        // Scales of the four rows: a_j = d*sc_j (exact), b_j = 128*a_j + dmin*m_j.
        uint32_t scw[4][2], mnw[4][2];
        float dd[4], dn[4], cd[4], cn[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          unpack_scales(hd[r].y, hd[r].z, hd[r].w, scw[r], mnw[r]);
          dd[r] = half_bits_to_float(hd[r].x);
          dn[r] = half_bits_to_float(hd[r].x >> 16);
          cd[r] = -8388608.f * dd[r];  // -2^23 d, exact
          cn[r] = -8388608.f * dn[r];
        }
        const int sb_base = (kb - cb) * 8;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int j = 2 * c + h;
            float a[4], b[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) {
              a[r] = fmaf(byte_magic(scw[r][j >> 2], j & 3), dd[r], cd[r]);  // d*sc, exact
              const float dm = fmaf(byte_magic(mnw[r][j >> 2], j & 3), dn[r], cn[r]);  // dmin*m, exact
              b[r] = fmaf(128.f, a[r], dm);
            }
            // A fragments of sub-block j for its two k-steps, both 16-row tiles.
            const int sh = 4 * h;
            uint32_t A[2][2][4];  // [tile][k-step][reg]
#pragma unroll
            for (int tt = 0; tt < 2; ++tt) {
              const uint2 lo = qv[2 * tt][c], hi = qv[2 * tt + 1][c];
              A[tt][0][0] = nib2(lo.x, sh);
              A[tt][0][1] = nib2(hi.x, sh);
              A[tt][0][2] = nib2(lo.x, sh + 8);
              A[tt][0][3] = nib2(hi.x, sh + 8);
              A[tt][1][0] = nib2(lo.y, sh);
              A[tt][1][1] = nib2(hi.y, sh);
              A[tt][1][2] = nib2(lo.y, sh + 8);
              A[tt][1][3] = nib2(hi.y, sh + 8);
            }
            const int sbi = sb_base + j;
#pragma unroll
            for (int f = 0; f < MT; ++f) {
              const uint4 bx = *reinterpret_cast<const uint4*>(
                  xs + (((size_t)(8 * f + g) * nsb + sbi) * 4 + t) * 8);
              const float2 sx = *reinterpret_cast<const float2*>(xsum + (size_t)sbi * TOK + 8 * f + 2 * t);
#pragma unroll
              for (int tt = 0; tt < 2; ++tt) {
                float cc[4];
                mma_bf16_16816(cc, A[tt][0], bx.x, bx.y, true);
                mma_bf16_16816(cc, A[tt][1], bx.z, bx.w, false);
                fma2(acc[tt][f][0], acc[tt][f][1], a[2 * tt], cc[0], cc[1]);
                fma2(acc[tt][f][0], acc[tt][f][1], -b[2 * tt], sx.x, sx.y);
                fma2(acc[tt][f][2], acc[tt][f][3], a[2 * tt + 1], cc[2], cc[3]);
                fma2(acc[tt][f][2], acc[tt][f][3], -b[2 * tt + 1], sx.x, sx.y);
              }
            }
          }
        }
      }
      cb += kcn;
    }

    // ---- CTA partial -> shared memory: red[local row][token] ----
#pragma unroll
    for (int tt = 0; tt < 2; ++tt)
#pragma unroll
      for (int f = 0; f < MT; ++f) {
        const int lr = warp * 32 + tt * 16 + g;
        red[(size_t)lr * TOK + 8 * f + 2 * t] = acc[tt][f][0];
        red[(size_t)lr * TOK + 8 * f + 2 * t + 1] = acc[tt][f][1];
        red[(size_t)(lr + 8) * TOK + 8 * f + 2 * t] = acc[tt][f][2];
        red[(size_t)(lr + 8) * TOK + 8 * f + 2 * t + 1] = acc[tt][f][3];
      }
  }

  cg::cluster_group cluster = cg::this_cluster();
  if (p.ksplit > 1) {
    cluster.sync();
  } else {
    __syncthreads();
  }

  if (rank == 0) {
    const int outw = SWIGLU ? ROWS / 2 : ROWS;
    for (int it = threadIdx.x; it < outw * TOK; it += blockDim.x) {
      const int i = it / outw;       // token
      const int lr = it % outw;      // local output row (consecutive threads -> consecutive n)
      if (i >= count) continue;
      float v = red[(size_t)lr * TOK + i];
      float u = SWIGLU ? red[(size_t)(lr + ROWS / 2) * TOK + i] : 0.f;
      for (int r = 1; r < p.ksplit; ++r) {
        const float* rr = cluster.map_shared_rank(red, r);
        v += rr[(size_t)lr * TOK + i];
        if (SWIGLU) u += rr[(size_t)(lr + ROWS / 2) * TOK + i];
      }
      if (SWIGLU) {
        const int half = p.N / 2;
        const int n = tile * (ROWS / 2) + lr;
        if (n < half) {
          const __nv_bfloat16 hb = __float2bfloat16_rn(silu_mul(v, u));
          static_cast<uint16_t*>(p.out)[(int64_t)(row_base + i) * half + n] = __bfloat16_as_ushort(hb);
        }
      } else {
        const int n = tile * ROWS + lr;
        if (n < p.N) static_cast<float*>(p.out)[(int64_t)(row_base + i) * p.N + n] = v;
      }
    }
  }
  if (p.ksplit > 1) cluster.sync();  // keep every CTA's shared memory alive until rank 0 is done
}

// Raw Q4_K rows as bytes [rows][row_bytes], box 160 bytes x 32 rows (one super-block per
// row plus 16 bytes of the next; past the end of a row the box reads zeros).
inline bool make_tmap_w_rowgroup(CUtensorMap* m, const void* base, int64_t rows, int64_t row_bytes) {
  auto enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)row_bytes, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
  cuuint32_t box[2] = {(cuuint32_t)kGemvPitch, 32};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace q4k
