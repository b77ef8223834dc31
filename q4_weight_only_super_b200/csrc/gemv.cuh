// Q4_K decode GEMV (1..32 tokens) and its grouped mixture-of-experts form.
//
// Operation: Y[m][n] = sum_k w[n][k] * X[m][k] over Q4_K weights (hipEngine
// 0.3.0 README, "Quickstart": the GEMV-decode profile; hipster README claims
// table: "GEMV ... GB/s"). The weight stream from HBM is the roofline.
//
// Design (sm_100a):
//  * Weights are the 16-row A operand of mma.sync m16n8k16 (bf16 in, fp32
//    accumulate); tokens are the 8-wide B operand (MT fragments of 8 tokens).
//  * A nibble q ORed into the bf16 pattern 0x4300 is exactly 128+q, so two
//    weights become one bf16x2 register with a single mask/or. The bias is
//    removed per sub-block: with C = sum (128+q)*x and Sx = sum x,
//      sum_i w_i x_i = (d*sc) * C - (128*d*sc + dmin*m) * Sx.
//  * The k order inside a sub-block is free for a dot product, so each
//    thread takes the nibbles in the order the mask produces them, and the
//    staged activations in shared memory are stored in that same order.
//  * A CTA owns 16*WARPS weight rows (one 16-row group per warp) and a
//    contiguous range of super-blocks; a thread-block cluster of KSPLIT CTAs
//    covers the whole K range and its partial sums are reduced in rank order
//    through distributed shared memory (deterministic, no atomics). The
//    decomposition depends only on (N, K), so a token's result never depends
//    on the other tokens in the batch.
#pragma once
#include <cooperative_groups.h>

#include "common.cuh"

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
  int kc;                    // super-blocks of activations staged per chunk
};

// Shared memory layout (dynamic):
//   xs   [8*MT tokens][kc*8 sub-blocks][4][8] bf16  (permuted activations of one chunk)
//   xsum [kc*8][8*MT] fp32                          (per sub-block sum of x)
//   red  [16*WARPS rows][8*MT] fp32                 (per-CTA partial result)
template <int MT, int WARPS>
__host__ __device__ constexpr size_t gemv_smem_bytes(int kc) {
  return (size_t)8 * MT * kc * 8 * 32 * 2 + (size_t)kc * 8 * 8 * MT * 4 +
         (size_t)16 * WARPS * 8 * MT * 4;
}

// GROUPED: blockIdx.y enumerates non-empty experts (the y-th expert with a
// non-zero row count); SWIGLU: the CTA's first WARPS/2 row groups are gate
// rows and the last WARPS/2 the matching up rows (at +N/2).
template <int MT, int WARPS, bool GROUPED, bool SWIGLU>
__global__ void __launch_bounds__(32 * WARPS) gemv_kernel(GemvParams p) {
  constexpr int TOK = 8 * MT;
  extern __shared__ __align__(16) uint8_t smem[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;

  const int rank = (int)(blockIdx.x % (unsigned)p.ksplit);
  const int tile = (int)(blockIdx.x / (unsigned)p.ksplit);
  const int kb0 = (int)((int64_t)rank * p.nkb / p.ksplit);
  const int kb1 = (int)((int64_t)(rank + 1) * p.nkb / p.ksplit);
  const int nk = kb1 - kb0;

  // ---- which tokens / matrix ----
  const uint8_t* W = p.W;
  int row_base = 0, count = p.M;
  if (GROUPED) {
    // Find the blockIdx.y-th expert with a non-empty row range.
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
    row_base = p.offsets[found];
    count = p.offsets[found + 1] - row_base;
    if (count > TOK) {
      if (threadIdx.x == 0 && rank == 0) latch_status(Q4K_ERR_DEVICE_BOUNDS);
      count = TOK;
    }
    W += (int64_t)found * p.expert_stride;
  }

  uint16_t* xs = reinterpret_cast<uint16_t*>(smem);
  float* xsum = reinterpret_cast<float*>(smem + (size_t)TOK * p.kc * 8 * 32 * 2);
  float* red = xsum + (size_t)p.kc * 8 * TOK;
  const int nsb = p.kc * 8;  // sub-blocks per staged chunk

  // Stage activations of super-blocks [c0, c0+kcn): each run of 8 consecutive k is stored
  // permuted as (e0,e2),(e1,e3),(e4,e6),(e5,e7) to match the A-fragment nibble order, plus
  // the fp32 sum of every 32-wide sub-block. Work item = (token i, sub-block s, quarter tq);
  // the quarter is the fastest index so a sub-block's four quarters are adjacent lanes.
  auto stage = [&](int c0, int kcn) {
    const int ns = kcn * 8;
    for (int it = threadIdx.x; it < TOK * ns * 4; it += blockDim.x) {
      const int tq = it & 3;
      const int s = (it >> 2) % ns;
      const int i = (it >> 2) / ns;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (i < count) {
        int64_t xrow = i;
        if (GROUPED) xrow = p.gather ? p.gather[row_base + i] : (row_base + i);
        v = ldg_u4(p.X + xrow * p.K + (int64_t)c0 * QK + s * 32 + tq * 8);
      }
      uint4 o;
      o.x = __byte_perm(v.x, v.y, 0x5410);  // (e0, e2)
      o.y = __byte_perm(v.x, v.y, 0x7632);  // (e1, e3)
      o.z = __byte_perm(v.z, v.w, 0x5410);  // (e4, e6)
      o.w = __byte_perm(v.z, v.w, 0x7632);  // (e5, e7)
      *reinterpret_cast<uint4*>(xs + (((size_t)i * nsb + s) * 4 + tq) * 8) = o;
      float sum = 0.f;
      const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        sum += bf16_bits_to_float(w4[e] & 0xFFFFu);
        sum += bf16_bits_to_float(w4[e] >> 16);
      }
      sum += __shfl_xor_sync(0xffffffffu, sum, 1);
      sum += __shfl_xor_sync(0xffffffffu, sum, 2);
      if (tq == 0) xsum[(size_t)s * TOK + i] = sum;
    }
  };

  // ---- per-warp row group ----
  int64_t row_g;  // row (within the matrix) of this thread's first A row
  bool valid;
  if (SWIGLU) {
    const int half = p.N / 2;
    const int tile_rows = 16 * (WARPS / 2);
    const int wg = warp % (WARPS / 2);
    const int r0 = tile * tile_rows + 16 * wg;
    valid = r0 < half;
    row_g = (warp < WARPS / 2 ? 0 : half) + r0 + g;
  } else {
    const int r0 = (tile * WARPS + warp) * 16;
    valid = r0 < p.N;
    row_g = r0 + g;
  }
  const int64_t row_bytes = (int64_t)p.nkb * BLOCK_BYTES;
  const uint8_t* wg_ptr = W + row_g * row_bytes;
  const uint8_t* wg8_ptr = wg_ptr + 8 * row_bytes;

  float acc[MT][4];
#pragma unroll
  for (int f = 0; f < MT; ++f)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[f][e] = 0.f;

  uint4 hg = make_uint4(0u, 0u, 0u, 0u), hg8 = hg;
  uint2 qg[4], qg8[4];
  auto load = [&](int kb) {
    const uint8_t* a = wg_ptr + (int64_t)kb * BLOCK_BYTES;
    const uint8_t* b = wg8_ptr + (int64_t)kb * BLOCK_BYTES;
    hg = ldg_stream_u4(a);
    hg8 = ldg_stream_u4(b);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      qg[c] = ldg_stream_u2(a + 16 + 32 * c + 8 * t);
      qg8[c] = ldg_stream_u2(b + 16 + 32 * c + 8 * t);
    }
  };
  if (valid && nk > 0) load(kb0);

  for (int cb = kb0; cb < kb1; cb += p.kc) {
    const int kcn = min(p.kc, kb1 - cb);
    __syncthreads();  // previous chunk fully consumed
    stage(cb, kcn);
    __syncthreads();
    if (!valid) continue;
    for (int kb = cb; kb < cb + kcn; ++kb) {
      const uint4 cg_ = hg, cg8 = hg8;
      uint2 cq[4], cq8[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) { cq[c] = qg[c]; cq8[c] = qg8[c]; }
      if (kb + 1 < kb1) load(kb + 1);  // prefetch, also across the chunk boundary

      // Thread t decodes pairs j = 2t, 2t+1 of both rows; the others come by shuffle.
      float a_own[2][2], b_own[2][2];  // [row g / g+8][h]
      {
        const uint4 hh[2] = {cg_, cg8};
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const float d = half_bits_to_float(hh[r].x), dmin = half_bits_to_float(hh[r].x >> 16);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t sc, m;
            scale_min(hh[r].y, hh[r].z, hh[r].w, 2 * t + h, sc, m);
            const float a = d * (float)sc;                  // exact
            a_own[r][h] = a;
            b_own[r][h] = fmaf(128.f, a, dmin * (float)m);  // exact terms, one rounding
          }
        }
      }
      const int sb_base = (kb - cb) * 8;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int src = (lane & ~3) | c;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const float ag = __shfl_sync(0xffffffffu, a_own[0][h], src);
          const float bg = __shfl_sync(0xffffffffu, b_own[0][h], src);
          const float ag8 = __shfl_sync(0xffffffffu, a_own[1][h], src);
          const float bg8 = __shfl_sync(0xffffffffu, b_own[1][h], src);
          // A fragments of sub-block j = 2c+h for its two k-steps of 16.
          const int sh = 4 * h;
          const uint32_t A0[4] = {nib2(cq[c].x, sh), nib2(cq8[c].x, sh), nib2(cq[c].x, sh + 8),
                                  nib2(cq8[c].x, sh + 8)};
          const uint32_t A1[4] = {nib2(cq[c].y, sh), nib2(cq8[c].y, sh), nib2(cq[c].y, sh + 8),
                                  nib2(cq8[c].y, sh + 8)};
          const int s = sb_base + 2 * c + h;
#pragma unroll
          for (int f = 0; f < MT; ++f) {
            const uint4 bx = *reinterpret_cast<const uint4*>(
                xs + (((size_t)(8 * f + g) * nsb + s) * 4 + t) * 8);
            float cc[4];
            mma_bf16_16816(cc, A0, bx.x, bx.y, true);
            mma_bf16_16816(cc, A1, bx.z, bx.w, false);
            const float2 sx = *reinterpret_cast<const float2*>(xsum + (size_t)s * TOK + 8 * f + 2 * t);
            acc[f][0] = fmaf(-bg, sx.x, fmaf(ag, cc[0], acc[f][0]));
            acc[f][1] = fmaf(-bg, sx.y, fmaf(ag, cc[1], acc[f][1]));
            acc[f][2] = fmaf(-bg8, sx.x, fmaf(ag8, cc[2], acc[f][2]));
            acc[f][3] = fmaf(-bg8, sx.y, fmaf(ag8, cc[3], acc[f][3]));
          }
        }
      }
    }
  }

  // ---- CTA partial -> shared memory: red[local row][token] ----
#pragma unroll
  for (int f = 0; f < MT; ++f) {
    const int lr = warp * 16 + g;
    red[(size_t)lr * TOK + 8 * f + 2 * t] = acc[f][0];
    red[(size_t)lr * TOK + 8 * f + 2 * t + 1] = acc[f][1];
    red[(size_t)(lr + 8) * TOK + 8 * f + 2 * t] = acc[f][2];
    red[(size_t)(lr + 8) * TOK + 8 * f + 2 * t + 1] = acc[f][3];
  }

  cg::cluster_group cluster = cg::this_cluster();
  if (p.ksplit > 1) {
    cluster.sync();
  } else {
    __syncthreads();
  }

  if (rank == 0) {
    constexpr int ROWS = 16 * WARPS;
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
          const float h = silu_mul(v, u);
          const __nv_bfloat16 hb = __float2bfloat16_rn(h);
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

}  // namespace q4k
