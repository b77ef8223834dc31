// Q6_K decode GEMV for 1..8 tokens with super-block-stationary warps: the Q6_K form of
// the stationary Q4_K GEMV (same roles, rings, reductions and launch shapes), for the
// remaining large tensor family of a Q4_K_M file (hipEngine 0.3.0 README, "GGUF
// Support": the tensor-family table lists Q6_K beside Q4_K, Q5_K and Q8_0).
//
// Q6_K super-block (256 weights in 210 bytes): ql[128] (low four bits), qh[64] (high
// two bits), sixteen signed byte scales, fp16 d. Weight i = 128n + 32u + l takes nibble
// u/2 of ql[64n + 32(u%2) + l] and bits 2u, 2u+1 of qh[32n + l]; q = those six bits - 32
// and w = d * scale[i/16] * q.
//
// Design (sm_100a):
//  * Rows of 210-byte blocks are only 2-byte aligned, so the producer copies a 16-byte-
//    aligned superset of each row run (start rounded down, end rounded up; the matrix
//    is a multiple of 16 bytes long, so nothing past it is read) and the consumers index
//    each row from its own offset. A 4-byte word at a 2-byte-aligned shared-memory
//    address is two aligned loads and a funnel shift.
//  * One mma.sync m16n8k16 per 16-weight sub-block (n, u, lh): thread t takes weights
//    16lh + 4t + {0..3}, so its ql and qh data are one word each per row; the six bits
//    go into the low byte of 0x6400 = 1024 + (q + 32) and one fp16 add of -1056 leaves q,
//    exact. The signed scale multiplies the fp32 MMA result, d * 2^-k the super-block.
//  * Activations in registers, formed once per warp from X: for sub-block (n, u, lh) and
//    token g, thread t holds x[128n + 32u + 16lh + 4t + {0, 2}] and [.. + {1, 3}] as fp16
//    pairs (the B fragment matching the A byte order), the 256-wide column scaled by 2^k
//    so its largest |x| lies in [2^14, 2^15) (exact).
#pragma once
#include "gemv_sk.cuh"

namespace q4k {

// Row pitch in shared memory for runs of KU super-blocks: the aligned superset (up to
// 30 bytes more), padded to 32 or 96 modulo 128 (rows g = 0..7 in distinct banks) with
// 8 bytes of slack for the second load of the last word.
inline int sk6_pitch(int KU) {
  int p = ((KU * kQ6BB + 30 + 8) + 15) & ~15;
  while ((p & 127) != 32 && (p & 127) != 96) p += 16;
  return p;
}

// Activation fragments of one 256-wide column for token g (lanes 4g..4g+3): b[si] =
// (x[4t], x[4t+2]), (x[4t+1], x[4t+3]) of sub-block si = 8n + 2u + lh (16-wide column
// 128n + 32u + 16lh), scaled by 2^k, and 2^-k of the result columns' tokens 2t, 2t+1.
struct Sk6Act {
  uint2 b[16];
  float s0, s1;
};

__device__ __forceinline__ void sk6_load_act(Sk6Act& a, const uint16_t* xc, bool mine, int t) {
  uint32_t amax = 0;
#pragma unroll
  for (int si = 0; si < 16; ++si) {
    // sub-block si = 8n + 2u + lh starts at 128n + 32u + 16lh = 16 * si
    a.b[si] = mine ? *reinterpret_cast<const uint2*>(xc + 16 * si + 4 * t) : make_uint2(0u, 0u);
    amax = __vmaxu2(amax, a.b[si].x & 0x7FFF7FFFu);
    amax = __vmaxu2(amax, a.b[si].y & 0x7FFF7FFFu);
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
#pragma unroll
  for (int si = 0; si < 16; ++si) {
    const float x0 = bf16_bits_to_float(a.b[si].x & 0xFFFFu) * f;  // exact
    const float x1 = bf16_bits_to_float(a.b[si].x >> 16) * f;
    const float x2 = bf16_bits_to_float(a.b[si].y & 0xFFFFu) * f;
    const float x3 = bf16_bits_to_float(a.b[si].y >> 16) * f;
    a.b[si].x = h2_bits(__floats2half2_rn(x0, x2));  // k = 2t, 2t+1: weights 4t, 4t+2
    a.b[si].y = h2_bits(__floats2half2_rn(x1, x3));  // k = 2t+8, 2t+9: weights 4t+1, 4t+3
  }
  a.s0 = __shfl_sync(0xffffffffu, kinv, 8 * t);
  a.s1 = __shfl_sync(0xffffffffu, kinv, 8 * t + 4);
}

// One 16 x 256 Q6_K block (rows g, g+8 start at b0, b1 in shared memory, 2-byte aligned)
// times the warp's activation fragments, added to c: c[0..1] row g, tokens 2t, 2t+1;
// c[2..3] row g+8.
__device__ __forceinline__ void sk6_block(float (&c)[4], const uint8_t* b0, const uint8_t* b1, const Sk6Act& a,
                                          int t) {
  uint32_t sc0[4], sc1[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    sc0[i] = lds_word_a2(b0 + 192 + 4 * i);
    sc1[i] = lds_word_a2(b1 + 192 + 4 * i);
  }
  const float d0 = __half2float(*reinterpret_cast<const __half*>(b0 + 208));
  const float d1 = __half2float(*reinterpret_cast<const __half*>(b1 + 208));
  const __half2 off = __float2half2_rn(-1056.f);
  float C[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int n = 0; n < 2; ++n) {
#pragma unroll
    for (int lh = 0; lh < 2; ++lh) {
      const int o = 64 * n + 16 * lh + 4 * t;
      const uint32_t l0a = lds_word_a2(b0 + o), l0b = lds_word_a2(b0 + o + 32);
      const uint32_t l1a = lds_word_a2(b1 + o), l1b = lds_word_a2(b1 + o + 32);
      const uint32_t h0 = lds_word_a2(b0 + 128 + 32 * n + 16 * lh + 4 * t);
      const uint32_t h1 = lds_word_a2(b1 + 128 + 32 * n + 16 * lh + 4 * t);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int si = 8 * n + 2 * u + lh;
        const uint32_t w0 = (u & 1) ? l0b : l0a, w1 = (u & 1) ? l1b : l1a;
        // six-bit values q + 32 of the four weights, one per byte
        const uint32_t v0 = ((w0 >> (4 * (u >> 1))) & 0x0F0F0F0Fu) | (((h0 >> (2 * u)) & 0x03030303u) << 4);
        const uint32_t v1 = ((w1 >> (4 * (u >> 1))) & 0x0F0F0F0Fu) | (((h1 >> (2 * u)) & 0x03030303u) << 4);
        const uint32_t a0 = h2_bits(__hadd2(bits_h2(__byte_perm(v0, 0x64646464u, 0x4240u)), off));
        const uint32_t a2 = h2_bits(__hadd2(bits_h2(__byte_perm(v0, 0x64646464u, 0x4341u)), off));
        const uint32_t a1 = h2_bits(__hadd2(bits_h2(__byte_perm(v1, 0x64646464u, 0x4240u)), off));
        const uint32_t a3 = h2_bits(__hadd2(bits_h2(__byte_perm(v1, 0x64646464u, 0x4341u)), off));
        const float s0 = s8_to_f32(sc0[si >> 2], si & 3);
        const float s1 = s8_to_f32(sc1[si >> 2], si & 3);
        float Cj[4];
        mma_f16_16816(Cj, a0, a1, a2, a3, a.b[si].x, a.b[si].y, true);
        C[0] = fmaf(s0, Cj[0], C[0]);
        C[1] = fmaf(s0, Cj[1], C[1]);
        C[2] = fmaf(s1, Cj[2], C[2]);
        C[3] = fmaf(s1, Cj[3], C[3]);
      }
    }
  }
  c[0] = fmaf(d0 * a.s0, C[0], c[0]);
  c[1] = fmaf(d0 * a.s1, C[1], c[1]);
  c[2] = fmaf(d1 * a.s0, C[2], c[2]);
  c[3] = fmaf(d1 * a.s1, C[3], c[3]);
}

template <int KPW>
__global__ void __launch_bounds__(SkMax<KPW>::threads, 1) gemv_sk6_kernel(const SkParams p) {
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
  const int64_t row_bytes = (int64_t)p.nkb * kQ6BB;
  // offset of row r's run inside its 16-byte-aligned superset: the same for every unit
  // (16 rows are a multiple of 16 bytes)
  auto run_off = [&](int r) { return (int)(((int64_t)r * row_bytes + (int64_t)kb0 * kQ6BB) & 15); };

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
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  if (warp == CW) {
    // ---------------- producer: one bulk copy per staged row (an aligned superset) ----------------
    const int drop = g_test_drop_stage;  // test hook; -1 in normal use
    const int r = lane & 15;
    const int off = run_off(r);
    const uint32_t len = (uint32_t)((off + kup * kQ6BB + 15) & ~15);
    const uint32_t tx = __reduce_add_sync(0xffffffffu, lane < kSkRows ? len : 0u);
    const uint8_t* src = p.W + ((int64_t)cid * kSkRows + r) * row_bytes + (int64_t)kb0 * kQ6BB - off;
    const int64_t src_step = (int64_t)ncl * kSkRows * row_bytes;
    const uint32_t dst0 = smem_u32(smem) + (uint32_t)(r * p.pitch);
    int s = 0;
    uint32_t ph = 0, soff = 0;
    int done = 0;
    for (int i = 0; i < nunits; ++i) {
      int ok = 1;
      if (lane == 0) ok = (i < S || mbar_wait_l(empty(s), ph ^ 1u, abort_flag, limit)) && !*abort_flag;
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      ++done;
      if (i != drop) {
        if (lane == 0) mbar_arrive_expect_tx(full(s), tx);
        __syncwarp();
        if (lane < kSkRows) bulk_copy_g2s(dst0 + soff, src, len, full(s));
      }
      src += src_step;
      soff += stage_bytes;
      if (++s == S) {
        s = 0;
        soff = 0;
        ph ^= 1u;
      }
    }
    if (lane == 0)
      for (int i = (done > S ? done - S : 0); i < done; ++i)
        if (i != drop) mbar_wait_drain(full(i % S), (uint32_t)(i / S) & 1u);
  } else if (warp == CW + 1) {
    // ---------------- epilogue: sum the warps' partials in K order ----------------
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
    asm volatile("griddepcontrol.wait;" ::: "memory");  // X may come from the previous kernel
    Sk6Act act[KPW];
    bool has[KPW];
#pragma unroll
    for (int kk = 0; kk < KPW; ++kk) {
      const int kl = KPW * w + kk;  // super-block within the part
      has[kk] = kl < kup;
      sk6_load_act(act[kk], p.X + (int64_t)g * p.K + (int64_t)(kb0 + kl) * QK, has[kk] && g < p.M, t);
    }
    // rows g and g+8 of a stage, at their runs' offsets, at this warp's first block
    const uint8_t* row0 = smem + g * p.pitch + run_off(g) + KPW * w * kQ6BB;
    const uint8_t* row1 = smem + (g + 8) * p.pitch + run_off(g + 8) + KPW * w * kQ6BB;
    float* redw = red + (size_t)w * kSkPartial + 2 * t * kSkTokStride + g;
    const size_t red_slot = (size_t)CW * kSkPartial;
    const bool st0 = 2 * t < p.M, st1 = 2 * t + 1 < p.M;
    int s = 0, r = 0;
    uint32_t ph = 0, rph = 0, soff = 0;
    for (int i = 0; i < nunits; ++i) {
      if (!mbar_wait_l(full(s), ph, abort_flag, limit)) break;
      float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int kk = 0; kk < KPW; ++kk)
        if (has[kk]) sk6_block(c, row0 + soff + kk * kQ6BB, row1 + soff + kk * kQ6BB, act[kk], t);
      __syncwarp();
      if (lane == 0) mbar_arrive(empty(s));  // the stage has been read: release it
      soff += stage_bytes;
      if (++s == S) {
        s = 0;
        soff = 0;
        ph ^= 1u;
      }
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
    cluster.sync();
  }
}

// Launch shape: as the stationary Q4_K GEMV's (sk_shape / sk_finish) with the Q6_K row
// pitch.
inline bool sk6_shape(int N, int nkb, SkCfg* c) {
  if (!sk_shape(N, nkb, c)) return false;
  c->pitch = sk6_pitch(c->KU);
  return true;
}

}  // namespace q4k
