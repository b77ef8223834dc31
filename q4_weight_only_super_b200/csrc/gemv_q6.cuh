// Q6_K decode GEMV (1..32 tokens): Y[m][n] = sum_k w[n][k] * X[m][k] over Q6_K
// weights, the remaining large tensor family of a Q4_K_M file (hipEngine 0.3.0
// README, "GGUF Support": the tensor-family table lists Q6_K beside Q4_K, Q5_K and
// Q8_0).
//
// Q6_K super-block (llama.cpp-style K-quant, 256 weights in 210 bytes): ql[128]
// (low four bits), qh[64] (high two bits), sixteen signed byte scales, fp16 d.
// Weight i = 128n + 32u + l takes nibble u/2 of ql[64n + 32(u%2) + l] and bits
// 2u, 2u+1 of qh[32n + l]; q = those six bits - 32 in -32..31 and
// w = d * scale[i/16] * q.
//
// Design (sm_100a):
//  * 210-byte blocks leave rows only 2-byte aligned, out of reach of TMA and bulk
//    copies (16-byte rules), so each warp reads its weights from global memory
//    itself: every 4-byte word a thread needs comes from one aligned load, or two
//    and a funnel shift where the block starts 2 bytes off a word.
//  * A warp owns a 16-row tile and a part of K; eight warps per CTA cover
//    8/P tiles x P parts, and the CTA sums the parts in part order through shared
//    memory (deterministic). P is the smallest power of two that gives at least
//    8192 warps, so many loads are in flight and short matrices still fill the GPU.
//  * One mma.sync m16n8k16 per 16-weight sub-block (n, u, lh) and token group:
//    thread t takes the sub-block's weights 16lh + 4t + {0,1,2,3}, which makes its
//    four ql bytes, four qh bytes (and the activations) one word each. The six
//    bits are put into the low byte of 0x6400 = 1024 + (q + 32), and one fp16 add
//    of -1056 leaves q itself, exact: the weight enters the MMA as the signed
//    integer, with no offset term to cancel. The sub-block's signed scale is
//    applied to the fp32 MMA result, and d * 2^-k once per super-block.
//  * The activations are the GEMV pre-pass's records (fp16, scaled per 256-wide
//    column by a power of two, exact): the weights 16lh + 4t + {0..3} of
//    32-wide column 4n + u sit in one 8-byte half of one 16-byte record chunk.
#pragma once
#include "common.cuh"
#include "gemm_tc.cuh"
#include "gemv.cuh"  // mma_f16_16816, h2_bits, bits_h2, kXRec

namespace q4k {

constexpr int kQ6BlockBytes = 210;
constexpr int kQ6Warps = 8;

// The 4 bytes at a 2-byte-aligned global address, without reading past them when
// they are word-aligned (the last word of the matrix may end its allocation).
__device__ __forceinline__ uint32_t ld_word_a2(const uint8_t* p) {
  const uintptr_t a = reinterpret_cast<uintptr_t>(p);
  const uint32_t* q = reinterpret_cast<const uint32_t*>(a & ~static_cast<uintptr_t>(3));
  if (a & 2) return __funnelshift_r(__ldg(q), __ldg(q + 1), 16);
  return __ldg(q);
}

struct Q6Params {
  const uint8_t* W;      // [N][nkb][210]
  const uint8_t* xprep;  // pre-pass records [nkb][rows_pad][576]
  float* Y;              // fp32 [M][N]
  int M, N, nkb;
  int rows_pad;
  int P;                 // K parts per tile (1, 2, 4 or 8)
};

template <int MT>
__global__ void __launch_bounds__(32 * kQ6Warps) q6k_gemv_kernel(const Q6Params p) {
  __shared__ float red[kQ6Warps][8 * MT][17];  // per warp: [token][row], padded
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int T = kQ6Warps / p.P;
  const int tile = (int)blockIdx.x * T + warp / p.P, part = warp % p.P;
  const int kb0 = (int)((int64_t)part * p.nkb / p.P), kb1 = (int)((int64_t)(part + 1) * p.nkb / p.P);
  const bool live = tile * 16 < p.N;
  // the records come from the pre-pass, launched just before this kernel
  asm volatile("griddepcontrol.wait;" ::: "memory");

  float acc[MT][4];
#pragma unroll
  for (int f = 0; f < MT; ++f) acc[f][0] = acc[f][1] = acc[f][2] = acc[f][3] = 0.f;
  const int64_t row_bytes = (int64_t)p.nkb * kQ6BlockBytes;
  const uint8_t* r0 = p.W + (int64_t)(tile * 16 + g) * row_bytes;
  const uint8_t* r1 = r0 + 8 * row_bytes;
  for (int kb = kb0; live && kb < kb1; ++kb) {
    const uint8_t* b0 = r0 + (int64_t)kb * kQ6BlockBytes;
    const uint8_t* b1 = r1 + (int64_t)kb * kQ6BlockBytes;
    // scales (16 signed bytes at 192) and d (fp16 at 208) of rows g and g+8
    uint32_t sc0[4], sc1[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      sc0[i] = ld_word_a2(b0 + 192 + 4 * i);
      sc1[i] = ld_word_a2(b1 + 192 + 4 * i);
    }
    const float d0 = __half2float(__ldg(reinterpret_cast<const __half*>(b0 + 208)));
    const float d1 = __half2float(__ldg(reinterpret_cast<const __half*>(b1 + 208)));
    const uint8_t* xk = p.xprep + (int64_t)kb * p.rows_pad * kXRec;
    float C[MT][4];
#pragma unroll
    for (int n = 0; n < 2; ++n) {
#pragma unroll
      for (int lh = 0; lh < 2; ++lh) {
        // this thread's words for weights 16lh + 4t + {0..3} of half n: ql for u = 0, 2
        // (v = 0) and u = 1, 3 (v = 1), and qh for all four quarters
        const int o = 64 * n + 16 * lh + 4 * t;
        const uint32_t l0a = ld_word_a2(b0 + o), l0b = ld_word_a2(b0 + o + 32);
        const uint32_t l1a = ld_word_a2(b1 + o), l1b = ld_word_a2(b1 + o + 32);
        const uint32_t h0 = ld_word_a2(b0 + 128 + 32 * n + 16 * lh + 4 * t);
        const uint32_t h1 = ld_word_a2(b1 + 128 + 32 * n + 16 * lh + 4 * t);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int si = 8 * n + 2 * u + lh;  // scale index (i / 16)
          const uint32_t w0 = (u & 1) ? l0b : l0a, w1 = (u & 1) ? l1b : l1a;
          // six-bit values q + 32 of the four weights, one per byte
          const uint32_t v0 = ((w0 >> (4 * (u >> 1))) & 0x0F0F0F0Fu) | (((h0 >> (2 * u)) & 0x03030303u) << 4);
          const uint32_t v1 = ((w1 >> (4 * (u >> 1))) & 0x0F0F0F0Fu) | (((h1 >> (2 * u)) & 0x03030303u) << 4);
          // A: rows g (regs 0, 2), g+8 (regs 1, 3); weights {0,2} then {1,3}, as q in fp16
          const __half2 off = __float2half2_rn(-1056.f);
          const uint32_t a0 = h2_bits(__hadd2(bits_h2(__byte_perm(v0, 0x64646464u, 0x4240u)), off));
          const uint32_t a2 = h2_bits(__hadd2(bits_h2(__byte_perm(v0, 0x64646464u, 0x4341u)), off));
          const uint32_t a1 = h2_bits(__hadd2(bits_h2(__byte_perm(v1, 0x64646464u, 0x4240u)), off));
          const uint32_t a3 = h2_bits(__hadd2(bits_h2(__byte_perm(v1, 0x64646464u, 0x4341u)), off));
          const float s0 = (float)(int8_t)((sc0[si >> 2] >> (8 * (si & 3))) & 0xFFu);
          const float s1 = (float)(int8_t)((sc1[si >> 2] >> (8 * (si & 3))) & 0xFFu);
          // activations: weights 16lh + 4t + {0..3} of 32-wide column 4n + u are chunk
          // (4(4n+u) + 2lh + t/2), half t%2 of each token's record
          const int boff = (4 * (4 * n + u) + 2 * lh + (t >> 1)) * 16 + 8 * (t & 1);
#pragma unroll
          for (int f = 0; f < MT; ++f) {
            const uint2 bx = __ldg(reinterpret_cast<const uint2*>(xk + (int64_t)(8 * f + g) * kXRec + boff));
            float Cj[4];
            mma_f16_16816(Cj, a0, a1, a2, a3, bx.x, bx.y, true);
            if (n == 0 && lh == 0 && u == 0) {
              C[f][0] = s0 * Cj[0];
              C[f][1] = s0 * Cj[1];
              C[f][2] = s1 * Cj[2];
              C[f][3] = s1 * Cj[3];
            } else {
              C[f][0] = fmaf(s0, Cj[0], C[f][0]);
              C[f][1] = fmaf(s0, Cj[1], C[f][1]);
              C[f][2] = fmaf(s1, Cj[2], C[f][2]);
              C[f][3] = fmaf(s1, Cj[3], C[f][3]);
            }
          }
        }
      }
    }
    // y += d * 2^-k * C (2^-k of tokens 2t and 2t+1 of each group, from the records)
#pragma unroll
    for (int f = 0; f < MT; ++f) {
      const float k0 = __ldg(reinterpret_cast<const float*>(xk + (int64_t)(8 * f + 2 * t) * kXRec + 544));
      const float k1 = __ldg(reinterpret_cast<const float*>(xk + (int64_t)(8 * f + 2 * t + 1) * kXRec + 544));
      acc[f][0] = fmaf(d0 * k0, C[f][0], acc[f][0]);
      acc[f][1] = fmaf(d0 * k1, C[f][1], acc[f][1]);
      acc[f][2] = fmaf(d1 * k0, C[f][2], acc[f][2]);
      acc[f][3] = fmaf(d1 * k1, C[f][3], acc[f][3]);
    }
  }
  // parts of each tile summed in part order
#pragma unroll
  for (int f = 0; f < MT; ++f) {
    red[warp][8 * f + 2 * t][g] = acc[f][0];
    red[warp][8 * f + 2 * t + 1][g] = acc[f][1];
    red[warp][8 * f + 2 * t][g + 8] = acc[f][2];
    red[warp][8 * f + 2 * t + 1][g + 8] = acc[f][3];
  }
  __syncthreads();
  if (part == 0 && live) {
    for (int o = lane; o < 16 * p.M; o += 32) {
      const int tok = o >> 4, row = o & 15;
      float v = 0.f;
      for (int q = 0; q < p.P; ++q) v += red[warp + q][tok][row];
      p.Y[(int64_t)tok * p.N + tile * 16 + row] = v;
    }
  }
}

// K parts per tile: the smallest power of two (at most 8) giving 8192 warps or more.
// The warps' word loads are the bound (long-scoreboard stalls), so more of them in
// flight is the lever: gate+up (2176 tiles) with four parts instead of one took
// 89.4 -> 78.6 us at 1 token and 209 -> 175 us at 32 (eight parts: no better at 1
// token, 205 us at 32).
inline int q6_parts(int N, int nkb) {
  const int tiles = N / 16;
  int P = 1;
  while (P < 8 && (int64_t)tiles * P < 8192 && P * 2 <= nkb) P *= 2;
  return P;
}

}  // namespace q4k
