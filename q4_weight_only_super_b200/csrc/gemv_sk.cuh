// Q4_K decode GEMV for 1..8 tokens with super-block-stationary warps.
//
// Operation: Y[m][n] = sum_k w[n][k] * X[m][k] over Q4_K weights, the GEMV half of
// the WMMA-prefill / GEMV-decode session profile (hipEngine 0.3.0 README,
// "Quickstart"; hipster README claims table: "GEMV ... GB/s"). The weight stream
// from HBM is the roofline.
//
// Design (sm_100a):
//  * Work unit = 16 weight rows (one mma.sync tile) x the super-blocks of one K
//    part. The unit's row pieces are contiguous runs of the row-major matrix
//    (whole rows when K is not split: a unit is then one contiguous 16-row block),
//    fetched with one 1-D bulk copy per row into a ring of shared-memory stages:
//    long runs keep DRAM pages open, unlike a walk down a 144-byte column of many
//    rows at once.
//  * One persistent CTA per SM (a thread-block cluster of P CTAs when K is split
//    into P parts, rank = part). Units are dealt round-robin: cluster c takes row
//    tiles c, c + C, c + 2C, ..., so the whole GPU streams one window of memory.
//  * Consumer warp w owns super-blocks kb0 + KPW*w .. kb0 + KPW*w + KPW-1 of its
//    part for the whole kernel: their activation fragments (for each, the 256
//    values of each of up to 8 tokens, scaled by
//    a power of two so the column's largest magnitude lands in [2^14, 2^15) --
//    exact -- rounded to fp16 in mma fragment order, plus the eight sub-block sums
//    as fp16 hi + lo pairs) are computed once from X and live in registers. No
//    activation pre-pass and no activation traffic per unit.
//  * Per unit each consumer warp multiplies its KPW 16 x 256 weight blocks (the KPW
//    blocks share the per-unit waits, releases and partial): the A
//    operand is the raw nibble field read as fp16 subnormals (q * 2^-24, or
//    16q * 2^-24 for high nibbles -- exact on the tensor core), two m16n8k16 MMAs
//    per 32-weight sub-block accumulate on their own and are scaled by the exact
//    six-bit scale afterwards; the min term is one more MMA pair (A = m_j, B = the
//    sub-block sums); y = d*2^-k*C - dmin*2^-k*Cm (2^24 and 64 folded in).
//  * An epilogue warp sums the consumer warps' partials of a unit in warp (= K)
//    order and writes Y; with P > 1 it keeps the part's partial per unit, and
//    after all units the cluster sums the parts in rank order through distributed
//    shared memory. No floating-point atomics: the order of every sum is fixed by
//    (N, K) and the device, so a token's result does not depend on the other
//    tokens in the batch (1..8 tokens).
//  * Every wait is bounded (g_wait_limit_ns); on expiry the kernel latches
//    Q4K_ERR_DEVICE_TIMEOUT, all roles stop, the producer drains its own copies
//    and the kernel returns.
#pragma once
#include <cooperative_groups.h>

#include "common.cuh"
#include "gemm_tc.cuh"  // mbarrier and clock helpers
#include "gemv.cuh"     // mma_f16_16816, and_or, h2_bits, bulk_copy_g2s, unpack_scales

namespace q4k {

constexpr int kSkRows = 16;          // weight rows per unit (one MMA tile)
constexpr int kSkRedSlots = 2;       // reduction slots between consumers and the epilogue
constexpr int kSkTokStride = 20;     // floats per token in a partial (16 rows + 4: no bank conflicts)
constexpr int kSkPartial = 8 * kSkTokStride;  // floats per warp partial (8 tokens)
constexpr int kSkMaxUnitSlots = 64;  // per-CTA unit results kept for the cluster reduction (at most)
constexpr int kSkUnitFloats = kSkRows * 8;    // one unit's result: 16 rows x 8 tokens

// Super-blocks a consumer warp owns (KPW) and consumer warps at most: one super-block
// a warp, up to 18 warps (20 with the producer and epilogue warps: 96 registers a
// thread); two, up to 10 warps (12 warps, 168 registers: room for both activation
// sets; measured the faster of the two on the decode projections).
template <int KPW>
struct SkMax {
  static constexpr int warps = KPW == 1 ? 18 : 10;
  static constexpr int KU = warps * KPW;  // super-blocks of a K part
  static constexpr int threads = 32 * (warps + 2);
};

struct SkParams {
  const uint8_t* W;    // [N][nkb][144]
  const uint16_t* X;   // bf16 [M][K]
  float* Y;            // fp32 [M][N]
  int M, N, K, nkb;
  int P;               // K parts = cluster size
  int KU;              // super-blocks per part (at most)
  int CW;              // consumer warps = ceil(KU / KPW)
  int units;           // N / 16 row units
  int pitch;           // shared-memory bytes per staged row (>= KU * 144)
  int stages;          // weight ring depth
  int uslots;          // P > 1: unit results kept per CTA (>= units per cluster)
};

// Shared-memory layout (dynamic; every piece a multiple of 16 bytes).
struct SkSmem {
  static __host__ __device__ size_t stage_bytes(int pitch) { return (size_t)kSkRows * pitch; }
  static __host__ __device__ size_t red_off(int pitch, int stages) { return (size_t)stages * stage_bytes(pitch); }
  static __host__ __device__ size_t unit_off(int pitch, int stages, int CW) {
    return red_off(pitch, stages) + (size_t)kSkRedSlots * CW * kSkPartial * 4;
  }
  static __host__ __device__ size_t bar_off(int pitch, int stages, int CW, int uslots) {
    return unit_off(pitch, stages, CW) + (size_t)uslots * kSkUnitFloats * 4;
  }
  static __host__ __device__ size_t total(int pitch, int stages, int CW, int uslots) {
    return bar_off(pitch, stages, CW, uslots) + 8 * (2 * stages + 2 * kSkRedSlots) + 16;
  }
};

// Row pitch in shared memory: the run of KU super-blocks, padded so that a warp's
// 8-byte quant reads (rows g = 0..7 at g * pitch, four threads 8 bytes apart) fall
// into distinct banks: pitch = 32 or 96 modulo 128.
inline int sk_pitch(int KU) {
  int p = KU * BLOCK_BYTES;
  while ((p & 127) != 32 && (p & 127) != 96) p += 16;
  return p;
}

// Activation fragments of one 256-wide column for token g of the warp's MMA
// (lanes 4g..4g+3): the values scaled by 2^k (largest |x| in [2^14, 2^15), exact)
// as fp16 pairs in the order the nibble masks produce the weights, the sub-block
// sums (2t, 2t+1) as fp16 hi + lo pairs for the min term, and 2^-k of the result
// columns' tokens 2t and 2t+1.
struct SkAct {
  uint4 bx[8];
  uint32_t bh, bl;
  float s0, s1;
};

__device__ __forceinline__ void sk_load_act(SkAct& a, const uint16_t* xr, bool mine, int t) {
  uint32_t amax = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    a.bx[j] = mine ? ldg_u4(xr + 32 * j) : make_uint4(0u, 0u, 0u, 0u);
    amax = __vmaxu2(amax, a.bx[j].x & 0x7FFF7FFFu);
    amax = __vmaxu2(amax, a.bx[j].y & 0x7FFF7FFFu);
    amax = __vmaxu2(amax, a.bx[j].z & 0x7FFF7FFFu);
    amax = __vmaxu2(amax, a.bx[j].w & 0x7FFF7FFFu);
  }
  amax = max(amax & 0xFFFFu, amax >> 16);  // bf16 bit order = magnitude order for |x|
  amax = max(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
  amax = max(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
  int k = 0;
  if (amax != 0) {
    const int E = max(1, (int)(amax >> 7));  // biased exponent of the largest |x|
    k = min(126, max(-126, 141 - E));       // largest |x| * 2^k in [2^14, 2^15)
  }
  const float f = __uint_as_float((uint32_t)(127 + k) << 23);
  const float kinv = __uint_as_float((uint32_t)(127 - k) << 23);
  float sa = 0.f, sb = 0.f;  // sums of sub-blocks 2t and 2t+1 (the min-term operand)
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const uint32_t wv[4] = {a.bx[j].x, a.bx[j].y, a.bx[j].z, a.bx[j].w};
    float xs[8];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      xs[2 * e] = bf16_bits_to_float(wv[e] & 0xFFFFu) * f;  // exact
      xs[2 * e + 1] = bf16_bits_to_float(wv[e] >> 16) * f;
    }
    float sum = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) sum += xs[e];
    sum += __shfl_xor_sync(0xffffffffu, sum, 1);
    sum += __shfl_xor_sync(0xffffffffu, sum, 2);
    sum *= 0.015625f;  // 2^-6: |sum| < 2^14
    if ((j >> 1) == t) {
      if (j & 1)
        sb = sum;
      else
        sa = sum;
    }
    // fragment order (e0,e2),(e1,e3),(e4,e6),(e5,e7), as the nibble masks produce them
    a.bx[j].x = h2_bits(__floats2half2_rn(xs[0], xs[2]));
    a.bx[j].y = h2_bits(__floats2half2_rn(xs[1], xs[3]));
    a.bx[j].z = h2_bits(__floats2half2_rn(xs[4], xs[6]));
    a.bx[j].w = h2_bits(__floats2half2_rn(xs[5], xs[7]));
  }
  const __half ha = __float2half_rn(sa), hb = __float2half_rn(sb);
  const __half la = __float2half_rn(sa - __half2float(ha)), lb = __float2half_rn(sb - __half2float(hb));
  a.bh = h2_bits(__halves2half2(ha, hb));
  a.bl = h2_bits(__halves2half2(la, lb));
  // 2^-k of tokens 2t and 2t+1 (held by lanes 8t and 8t + 4)
  a.s0 = __shfl_sync(0xffffffffu, kinv, 8 * t);
  a.s1 = __shfl_sync(0xffffffffu, kinv, 8 * t + 4);
}

// One 16 x 256 block (rows g, g+8 at r0p, r1p) times the warp's activation fragments,
// added to c: c[0..1] row g, tokens 2t, 2t+1; c[2..3] row g+8.
__device__ __forceinline__ void sk_block(float (&c)[4], const uint8_t* r0p, const uint8_t* r1p, const SkAct& a,
                                         int t, uint32_t mb) {
  uint32_t sc0[2], sc1[2], am0, am1;
  float dA, dB, mA, mB;
  {
    const uint4 h0 = *reinterpret_cast<const uint4*>(r0p);
    const uint4 h1 = *reinterpret_cast<const uint4*>(r1p);
    uint32_t mn0[2], mn1[2];
    unpack_scales(h0.y, h0.z, h0.w, sc0, mn0);
    unpack_scales(h1.y, h1.z, h1.w, sc1, mn1);
    // min-term A operand: (m_2t, m_2t+1) of rows g and g+8, exact in fp16
    am0 = h2_bits(__hadd2(bits_h2(bytes_1024((t >> 1) ? mn0[1] : mn0[0], mb, mb + 1)), __float2half2_rn(-1024.f)));
    am1 = h2_bits(__hadd2(bits_h2(bytes_1024((t >> 1) ? mn1[1] : mn1[0], mb, mb + 1)), __float2half2_rn(-1024.f)));
    // the subnormal operand's products carry 2^-24: 2^24 folds into d; 64 undoes the
    // sums' 2^-6
    dA = 16777216.f * half_bits_to_float(h0.x);
    dB = 16777216.f * half_bits_to_float(h1.x);
    mA = 64.f * half_bits_to_float(h0.x >> 16);
    mB = 64.f * half_bits_to_float(h1.x >> 16);
  }
  float C[4];
#pragma unroll
  for (int cc = 0; cc < 4; ++cc) {
    // this thread's quant bytes [8t, 8t+8) of chunk cc for rows g and g+8
    const uint2 q0 = *reinterpret_cast<const uint2*>(r0p + 16 + 32 * cc + 8 * t);
    const uint2 q1 = *reinterpret_cast<const uint2*>(r1p + 16 + 32 * cc + 8 * t);
    const uint32_t q0x8 = q0.x >> 8, q1x8 = q1.x >> 8, q0y8 = q0.y >> 8, q1y8 = q1.y >> 8;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int j = 2 * cc + h;
      const uint32_t msk = h ? 0x00F000F0u : 0x000F000Fu;
      // sub-block scale sc_j (sc_j / 16 for high nibbles) as an exact fp32:
      // 0x4B0000sc = 2^23 + sc, 0x490000sc = 2^19 + sc/16
      const float fa = __uint_as_float(__byte_perm(sc0[j >> 2], h ? 0x49000000u : 0x4B000000u,
                                                   0x7650u | (uint32_t)(j & 3))) -
                       (h ? 524288.f : 8388608.f);
      const float fb = __uint_as_float(__byte_perm(sc1[j >> 2], h ? 0x49000000u : 0x4B000000u,
                                                   0x7650u | (uint32_t)(j & 3))) -
                       (h ? 524288.f : 8388608.f);
      // A: rows g (regs 0, 2) and g+8 (regs 1, 3); k-step 0 from word x, 1 from word y;
      // bytes {0,2} straight, bytes {1,3} after an 8-bit shift
      float Cj[4];
      mma_f16_16816(Cj, q0.x & msk, q1.x & msk, q0x8 & msk, q1x8 & msk, a.bx[j].x, a.bx[j].y, true);
      mma_f16_16816(Cj, q0.y & msk, q1.y & msk, q0y8 & msk, q1y8 & msk, a.bx[j].z, a.bx[j].w, false);
      if (j == 0) {
        C[0] = fa * Cj[0];
        C[1] = fa * Cj[1];
        C[2] = fb * Cj[2];
        C[3] = fb * Cj[3];
      } else {
        C[0] = fmaf(fa, Cj[0], C[0]);
        C[1] = fmaf(fa, Cj[1], C[1]);
        C[2] = fmaf(fb, Cj[2], C[2]);
        C[3] = fmaf(fb, Cj[3], C[3]);
      }
    }
  }
  // min term: Cm = sum_j m_j * X_j (k = sub-block index; k >= 8 is zero)
  float Cm[4];
  mma_f16_16816(Cm, am0, am1, 0u, 0u, a.bh, 0u, true);
  mma_f16_16816(Cm, am0, am1, 0u, 0u, a.bl, 0u, false);
  c[0] = fmaf(-mA * a.s0, Cm[0], fmaf(dA * a.s0, C[0], c[0]));
  c[1] = fmaf(-mA * a.s1, Cm[1], fmaf(dA * a.s1, C[1], c[1]));
  c[2] = fmaf(-mB * a.s0, Cm[2], fmaf(dB * a.s0, C[2], c[2]));
  c[3] = fmaf(-mB * a.s1, Cm[3], fmaf(dB * a.s1, C[3], c[3]));
}

template <int KPW>
__global__ void __launch_bounds__(SkMax<KPW>::threads, 1) gemv_sk_kernel(const SkParams p) {
  using L = SkSmem;
  extern __shared__ __align__(128) uint8_t smem[];
  namespace cg = cooperative_groups;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int CW = p.CW, S = p.stages;
  const int rank = (int)(blockIdx.x % (unsigned)p.P);
  const int cid = (int)(blockIdx.x / (unsigned)p.P), ncl = (int)(gridDim.x / (unsigned)p.P);
  const int kb0 = (int)((int64_t)rank * p.nkb / p.P);
  const int kup = (int)((int64_t)(rank + 1) * p.nkb / p.P) - kb0;  // super-blocks of this part
  const int nunits = cid < p.units ? (p.units - 1 - cid) / ncl + 1 : 0;
  const uint32_t stage_bytes = (uint32_t)L::stage_bytes(p.pitch);
  const uint64_t limit = *const_cast<volatile unsigned long long*>(&g_wait_limit_ns);

  float* red = reinterpret_cast<float*>(smem + L::red_off(p.pitch, S));
  float* upart = reinterpret_cast<float*>(smem + L::unit_off(p.pitch, S, CW));
  const uint32_t bar0 = smem_u32(smem + L::bar_off(p.pitch, S, CW, p.uslots));
  volatile int* abort_flag =
      reinterpret_cast<volatile int*>(smem + L::bar_off(p.pitch, S, CW, p.uslots) + 8 * (2 * S + 2 * kSkRedSlots));
  auto full = [&](int s) { return bar0 + 8u * s; };
  auto empty = [&](int s) { return bar0 + 8u * (S + s); };
  auto redfull = [&](int r) { return bar0 + 8u * (2 * S + r); };
  auto redempty = [&](int r) { return bar0 + 8u * (2 * S + kSkRedSlots + r); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), CW);
    }
    for (int r = 0; r < kSkRedSlots; ++r) {
      mbar_init(redfull(r), CW);
      mbar_init(redempty(r), 1);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  // Dependents may launch now: each of them waits (griddepcontrol.wait) for this
  // grid to complete before it reads or writes anything this grid touches.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  if (warp == CW) {
    // ---------------- producer: one bulk copy per staged row ----------------
    const int drop = g_test_drop_stage;  // test hook; -1 in normal use
    const uint32_t run = (uint32_t)kup * BLOCK_BYTES;
    const int64_t row_bytes = (int64_t)p.nkb * BLOCK_BYTES;
    const uint8_t* src = p.W + ((int64_t)cid * kSkRows + (lane & 15)) * row_bytes + (int64_t)kb0 * BLOCK_BYTES;
    const int64_t src_step = (int64_t)ncl * kSkRows * row_bytes;
    const uint32_t dst0 = smem_u32(smem) + (uint32_t)((lane & 15) * p.pitch);
    int s = 0;
    uint32_t ph = 0, soff = 0;
    int done = 0;  // loop iterations passed (stages issued, the dropped one included)
    for (int i = 0; i < nunits; ++i) {
      int ok = 1;
      if (lane == 0) ok = (i < S || mbar_wait_l(empty(s), ph ^ 1u, abort_flag, limit)) && !*abort_flag;
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      ++done;
      if (i != drop) {
        if (lane == 0) mbar_arrive_expect_tx(full(s), (uint32_t)kSkRows * run);
        __syncwarp();
        if (lane < kSkRows) bulk_copy_g2s(dst0 + soff, src, run, full(s));
      }
      src += src_step;
      soff += stage_bytes;
      if (++s == S) {
        s = 0;
        soff = 0;
        ph ^= 1u;
      }
    }
    // every issued stage must land before the CTA exits, abort or not
    if (lane == 0)
      for (int i = (done > S ? done - S : 0); i < done; ++i)
        if (i != drop) mbar_wait_drain(full(i % S), (uint32_t)(i / S) & 1u);
  } else if (warp == CW + 1) {
    // ---------------- epilogue: sum the warps' partials in K order ----------------
    // output o = token * 16 + row; lane handles o = lane + 32 q
    constexpr int WMAX = SkMax<KPW>::warps;
    int r = 0;
    uint32_t rph = 0;
    const int nout = kSkRows * p.M;
    for (int i = 0; i < nunits; ++i) {
      if (!mbar_wait_l(redfull(r), rph, abort_flag, limit)) break;
      const int unit = cid + i * ncl;
      const float* rs = red + (size_t)r * CW * kSkPartial;
      float v[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int o = lane + 32 * q;
        v[q] = 0.f;
        if (q * 32 < nout) {  // uniform over the warp
          const float* rp = rs + (o >> 4) * kSkTokStride + (o & 15);
          float pv[WMAX];
#pragma unroll
          for (int w = 0; w < WMAX; ++w) pv[w] = (w < CW && o < nout) ? rp[w * kSkPartial] : 0.f;
          float acc = 0.f;
#pragma unroll
          for (int w = 0; w < WMAX; ++w) acc += pv[w];  // in K order
          v[q] = acc;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(redempty(r));
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int o = lane + 32 * q;
        if (o < nout) {
          if (p.P == 1)
            p.Y[(int64_t)(o >> 4) * p.N + unit * kSkRows + (o & 15)] = v[q];
          else
            upart[i * kSkUnitFloats + o] = v[q];
        }
      }
      if (++r == kSkRedSlots) {
        r = 0;
        rph ^= 1u;
      }
    }
  } else {
    // ---------------- consumers: warp w owns super-blocks kb0 + KPW*w + (0..KPW-1) ----------------
    const int w = warp;
    // activation fragments of token g (rows of X may come from the previous kernel)
    asm volatile("griddepcontrol.wait;" ::: "memory");
    SkAct act[KPW];
    bool has[KPW];
#pragma unroll
    for (int kk = 0; kk < KPW; ++kk) {
      const int kl = KPW * w + kk;  // super-block within the part
      has[kk] = kl < kup;
      sk_load_act(act[kk], p.X + (int64_t)g * p.K + (int64_t)(kb0 + kl) * QK + 8 * t, has[kk] && g < p.M, t);
    }
    const uint32_t mb = 2u * (t & 1);
    const uint8_t* rowp = smem + g * p.pitch + KPW * w * BLOCK_BYTES;  // row g, first owned block
    const int p8 = 8 * p.pitch;
    float* redw = red + (size_t)w * kSkPartial + 2 * t * kSkTokStride + g;  // this lane's partial slots
    const size_t red_slot = (size_t)CW * kSkPartial;
    const bool st0 = 2 * t < p.M, st1 = 2 * t + 1 < p.M;
    int s = 0, r = 0;
    uint32_t ph = 0, rph = 0, soff = 0;
    for (int i = 0; i < nunits; ++i) {
      if (!mbar_wait_l(full(s), ph, abort_flag, limit)) break;
      float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int kk = 0; kk < KPW; ++kk) {
        const uint8_t* r0p = rowp + soff + kk * BLOCK_BYTES;
        if (has[kk]) sk_block(c, r0p, r0p + p8, act[kk], t, mb);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty(s));  // the stage has been read: release it
      soff += stage_bytes;
      if (++s == S) {
        s = 0;
        soff = 0;
        ph ^= 1u;
      }
      // partial -> reduction slot r: [token][row], tokens >= M not written
      if (i >= kSkRedSlots && !mbar_wait_l(redempty(r), rph ^ 1u, abort_flag, limit)) break;
      float* rp = redw + r * red_slot;
      if (st0) {
        rp[0] = c[0];
        rp[8] = c[2];
      }
      if (st1) {
        rp[kSkTokStride] = c[1];
        rp[kSkTokStride + 8] = c[3];
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(redfull(r));
      if (++r == kSkRedSlots) {
        r = 0;
        rph ^= 1u;
      }
    }
  }

  if (p.P > 1) {
    // the parts of every unit, summed in rank order through distributed shared memory
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();
    const int nout = kSkRows * p.M;
    for (int i = rank; i < nunits; i += p.P) {
      const int unit = cid + i * ncl;
      for (int o = (int)threadIdx.x; o < nout; o += (int)blockDim.x) {
        float acc = 0.f;
        for (int q = 0; q < p.P; ++q) acc += cluster.map_shared_rank(upart, q)[i * kSkUnitFloats + o];
        p.Y[(int64_t)(o >> 4) * p.N + unit * kSkRows + (o & 15)] = acc;
      }
    }
    cluster.sync();  // keep every CTA's shared memory alive until all ranks have read it
  }
}

// Launch shape for the stationary GEMV. KPW = super-blocks a consumer warp owns: two
// from 11 super-blocks on (per-unit costs over two blocks), else one.
// P = the number of K parts (the cluster size, at most 8) so that a part has at most
// SkMax<KPW>::KU super-blocks; KU = ceil(nkb / P); CW = ceil(KU / KPW) consumer warps;
// one CTA per SM; `clusters` = how many clusters of P such CTAs are resident at once
// (from the occupancy query), capped by the row units; the ring as deep as the shared
// memory allows (at least 2 stages).
struct SkCfg {
  int kpw;
  int P, KU, CW, pitch, stages, grid, uslots, units;
  size_t smem;
};

constexpr size_t kSkSmemBudget = 227 * 1024;

inline bool sk_shape(int N, int nkb, SkCfg* c) {
  c->kpw = nkb > 10 ? 2 : 1;
  const int KUmax = c->kpw == 2 ? SkMax<2>::KU : SkMax<1>::KU;
  c->P = (nkb + KUmax - 1) / KUmax;
  if (c->P > 8) return false;
  c->KU = (nkb + c->P - 1) / c->P;
  c->CW = (c->KU + c->kpw - 1) / c->kpw;
  c->pitch = sk_pitch(c->KU);
  c->units = N / kSkRows;
  return true;
}

inline bool sk_finish(int clusters, SkCfg* c) {
  clusters = std::max(1, std::min(c->units, clusters));
  c->uslots = c->P > 1 ? (c->units + clusters - 1) / clusters : 0;
  if (c->uslots > kSkMaxUnitSlots) return false;
  int st = 6;
  while (st > 2 && SkSmem::total(c->pitch, st, c->CW, c->uslots) > kSkSmemBudget) --st;
  c->stages = st;
  c->smem = SkSmem::total(c->pitch, st, c->CW, c->uslots);
  if (c->smem > kSkSmemBudget) return false;
  c->grid = clusters * c->P;
  return true;
}

}  // namespace q4k
