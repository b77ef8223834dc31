// Grouped (mixture-of-experts) Q4_K decode GEMV with super-block-stationary warps:
// out[r] = A[gather(r)] * W_e^T for the rows r of every expert e, the decode form of
// the grouped expert matmul (hipEngine 0.3.0 README, "Core principles": MoE experts
// in Q4_K; the routed-expert FFN of the Qwen3.6-35B-A3B decode workload). The weight
// stream of the experts the routing touched is the roofline.
//
// Design (sm_100a), built on the dense stationary GEMV's block arithmetic (sk_block,
// sk_load_act: same operands, same per-warp K ownership, same summation order):
//  * No activation pre-pass: each consumer warp forms its activation fragments from
//    the bf16 rows of A itself, once per (expert, token group) it meets.
//  * Work unit = (expert e, token group tg of 8 of e's rows, 16 weight rows u). The
//    units of the non-empty experts are numbered in (e, tg, u) order -- a table of
//    per-expert unit starts is built in shared memory from the expert offsets -- and
//    each of the G CTAs takes a contiguous run of T/G or T/G + 1 of the T units, so
//    a CTA meets few (expert, token group) pairs and reloads few activations; its
//    roles step from unit to unit without a search. An expert with more than 8 rows
//    streams its weights once per token group.
//  * SwiGLU: unit u of the fused [gate; up] matrix stages gate rows 8u..8u+7 in tile
//    rows 0..7 and the matching up rows N/2 + 8u.. in tile rows 8..15, so the
//    epilogue holds g and u of one output side by side and writes SiLU(g) * u as
//    bf16 (the MMA treats every row alike, so g and u are bit-identical to the
//    plain output's).
//  * K is not split across CTAs (at most SkMax<KPW>::KU super-blocks a row); the
//    consumer warps' partials are summed in warp (= K) order by an epilogue warp.
//    A row's result depends only on (N, K) and the device: not on the batch, the
//    expert's other rows, or the grid.
//  * Every wait is bounded (g_wait_limit_ns); offsets that are not a non-decreasing
//    sequence inside [0, rows] latch Q4K_ERR_DEVICE_BOUNDS and nothing is computed.
#pragma once
#include "gemv_sk.cuh"
#include "moe.cuh"  // route_tile, route_scan_place_one (the routing prologue)

namespace q4k {

struct SkgParams {
  const uint8_t* W;        // [E][N][nkb][144]
  const uint16_t* A;       // bf16 activation rows [*][K]
  const int32_t* gather;   // nullable: A row of sorted row r = gather[r]
  const int32_t* offsets;  // [E+1] sorted-row range of each expert
  void* out;               // fp32 [rows][N], or bf16 [rows][N/2] (SwiGLU)
  int E, N, K, nkb, rows;
  int CW;                  // consumer warps = ceil(nkb / KPW)
  int pitch;               // shared-memory bytes per staged row (>= nkb * 144)
  int stages;              // weight ring depth
  // routing prologue (PL > 0): top-k routing and permutation of the M <= 32 tokens
  // in every CTA; CTA 0 writes the routing outputs (offsets and gather come from it)
  const float* logits;     // fp32 [M][E]
  int M, topk;
  int32_t* topk_ids;       // [M][topk]
  float* topk_w;           // [M][topk]
  int32_t* offsets_out;    // [E+1]
  int32_t* perm;           // [rows]
  int32_t* inv_perm;       // [rows]
  int32_t* row_token;      // [rows]
};

// Warps that route in the routing prologue (route_tile deals the <= 32 tokens to them).
constexpr int kSkgRouteWarps = 8;

// Shared memory: ring [stages][16][pitch], partials [2][CW][8 tokens x 20], the
// expert offsets [E+1] and unit starts [E+2] (each padded to 16 B), with the routing
// prologue its arrays (per-expert totals, starts and token masks [E], warp sums [32],
// the tile's expert ids and the sorted rows' tokens [32 x 16] each), barriers, abort flag.
struct SkgSmem {
  static __host__ __device__ size_t red_off(int pitch, int stages) { return (size_t)stages * kSkRows * pitch; }
  static __host__ __device__ size_t tab_off(int pitch, int stages, int CW) {
    return red_off(pitch, stages) + (size_t)kSkRedSlots * CW * kSkPartial * 4;
  }
  static __host__ __device__ size_t tab_bytes(int E) { return ((size_t)(E + 2) * 4 + 15) & ~(size_t)15; }
  static __host__ __device__ size_t route_off(int pitch, int stages, int CW, int E) {
    return tab_off(pitch, stages, CW) + 2 * tab_bytes(E);
  }
  static __host__ __device__ size_t route_bytes(int E) {
    return (size_t)3 * ((E * 4 + 15) & ~15) + 128 + (size_t)2 * kRouteTokPerCta * kMaxTopk * 4;
  }
  static __host__ __device__ size_t bar_off(int pitch, int stages, int CW, int E, bool route) {
    return route_off(pitch, stages, CW, E) + (route ? route_bytes(E) : 0);
  }
  static __host__ __device__ size_t total(int pitch, int stages, int CW, int E, bool route = false) {
    return bar_off(pitch, stages, CW, E, route) + 8 * (2 * stages + 2 * kSkRedSlots) + 16;
  }
};

// Largest e with ustart[e] <= x; with x < ustart[E] that expert is non-empty.
__device__ __forceinline__ int skg_expert(const int* ustart, int E, int x) {
  int lo = 0, hi = E;  // ustart[lo] <= x < ustart[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (ustart[mid] <= x)
      lo = mid;
    else
      hi = mid;
  }
  return lo;
}

// Position of a unit: expert e, unit u of its token group, the group's first sorted
// row r0, its rows nr (<= 8) and the expert's end row oe.
struct SkgPos {
  int e, u, r0, nr, oe;
};

// The position of unit x (a binary search; once per CTA and role). `eoff` holds the
// expert offsets (shared memory).
__device__ __forceinline__ void skg_first(SkgPos& s, const int* ustart, const int* eoff, int E, int U, int x) {
  s.e = skg_expert(ustart, E, x);
  const int loc = x - ustart[s.e];
  const int tg = loc / U;
  s.u = loc - tg * U;
  s.r0 = eoff[s.e] + 8 * tg;
  s.oe = eoff[s.e + 1];
  s.nr = min(8, s.oe - s.r0);
}

// From unit x to unit x + 1, which must exist: the next unit of the group, else the
// next token group of the expert, else the first group of the next non-empty expert.
__device__ __forceinline__ void skg_next(SkgPos& s, const int* ustart, const int* eoff, int U) {
  if (++s.u < U) return;
  s.u = 0;
  s.r0 += 8;
  if (s.r0 >= s.oe) {
    do {
      ++s.e;
    } while (ustart[s.e + 1] == ustart[s.e]);
    s.r0 = eoff[s.e];
    s.oe = eoff[s.e + 1];
  }
  s.nr = min(8, s.oe - s.r0);
}

// PL > 0: the routing prologue (route_tile with PL logits per lane, E <= 32 * PL),
// run by every CTA with the same code and order as the one-CTA routing kernel, so its
// results are bit-identical to moe_route_permute's.
template <int KPW, bool SWIGLU, int PL = 0>
__global__ void __launch_bounds__(SkMax<KPW>::threads, 1) gemv_skg_kernel(const SkgParams p) {
  using L = SkgSmem;
  constexpr bool ROUTE = PL > 0;
  extern __shared__ __align__(128) uint8_t smem[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int CW = p.CW, S = p.stages, E = p.E;
  const int U = p.N / kSkRows;  // units per (expert, token group)
  const uint32_t stage_bytes = (uint32_t)kSkRows * p.pitch;
  // global words read up front, so that their latency overlaps the set-up
  const uint64_t limit = *const_cast<volatile unsigned long long*>(&g_wait_limit_ns);
  const int drop = *const_cast<volatile int*>(&g_test_drop_stage);  // test hook; -1 in normal use

  float* red = reinterpret_cast<float*>(smem + L::red_off(p.pitch, S));
  int* eoff = reinterpret_cast<int*>(smem + L::tab_off(p.pitch, S, CW));  // expert offsets [E+1]
  int* ustart = eoff + L::tab_bytes(E) / 4;  // unit starts [E+1], then the unit total
  const uint32_t bar0 = smem_u32(smem + L::bar_off(p.pitch, S, CW, E, ROUTE));
  volatile int* abort_flag =
      reinterpret_cast<volatile int*>(smem + L::bar_off(p.pitch, S, CW, E, ROUTE) + 8 * (2 * S + 2 * kSkRedSlots));
  // routing prologue arrays (ROUTE)
  uint8_t* rbase = smem + L::route_off(p.pitch, S, CW, E);
  const size_t ea = (size_t)((E * 4 + 15) & ~15);
  int* r_total = reinterpret_cast<int*>(rbase);
  int* r_start = reinterpret_cast<int*>(rbase + ea);
  unsigned* r_tmask = reinterpret_cast<unsigned*>(rbase + 2 * ea);
  int* r_wsum = reinterpret_cast<int*>(rbase + 3 * ea);
  int* r_sids = reinterpret_cast<int*>(rbase + 3 * ea + 128);
  int* r_rtok = r_sids + kRouteTokPerCta * kMaxTopk;  // token of each sorted row
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
  // Dependents may launch now; each waits (griddepcontrol.wait) for this grid to
  // complete before it touches anything this grid reads or writes.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // the offsets, the gather indices (or the logits) and A come from the previous kernels
  asm volatile("griddepcontrol.wait;" ::: "memory");

  if (ROUTE) {
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
      r_total[e] = 0;
      r_tmask[e] = 0u;
    }
    __syncthreads();
    const bool out = blockIdx.x == 0;  // CTA 0 writes the routing outputs
    if (warp < kSkgRouteWarps)
      route_tile<(ROUTE ? PL : 1), kSkgRouteWarps>(p.logits, p.M, E, p.topk, out ? p.topk_ids : nullptr,
                                                   out ? p.topk_w : nullptr, r_total, r_sids, r_tmask, 0);
    __syncthreads();
    route_scan_place_one(r_total, r_start, r_wsum, E, p.M, p.topk, r_sids, r_tmask, out ? p.offsets_out : nullptr,
                         out ? p.perm : nullptr, out ? p.inv_perm : nullptr, out ? p.row_token : nullptr, eoff,
                         r_rtok);
    __syncthreads();
  }

  if (warp == 0) {
    // unit starts: ustart[e] = U * (token groups of experts 0..e-1); the checks
    // make every later index lie inside [0, rows)
    if (!ROUTE) {
#pragma unroll 4
      for (int e = lane; e <= E; e += 32) eoff[e] = __ldg(p.offsets + e);  // all loads in flight at once
    }
    __syncwarp();
    bool bad = false;
    for (int e = lane; e < E; e += 32) {  // token groups of expert e, in ustart[e + 1] for now
      const int a = eoff[e], b = eoff[e + 1];
      bad |= a < 0 || b < a || b > p.rows;
      ustart[e + 1] = b > a ? (b - a + 7) >> 3 : 0;
    }
    int base = 0;
    for (int e0 = 0; e0 < E; e0 += 32) {  // each lane reads and rewrites its own entry
      const int e = e0 + lane;
      int sc = e < E ? ustart[e + 1] : 0;  // inclusive scan over the warp
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, sc, d);
        if (lane >= d) sc += v;
      }
      if (e < E) ustart[e + 1] = (base + sc) * U;
      base += __shfl_sync(0xffffffffu, sc, 31);
    }
    bad = __any_sync(0xffffffffu, bad);
    if (lane == 0) {
      ustart[0] = 0;
      ustart[E + 1] = bad ? 0 : base * U;  // the unit total
      if (bad) latch_status(Q4K_ERR_DEVICE_BOUNDS);
    }
  }
  __syncthreads();

  const int T = ustart[E + 1];
  const int G = (int)gridDim.x, cid = (int)blockIdx.x;
  // CTA cid takes units [x0, x0 + nunits): T / G each, one more for the first T % G
  const int per = T / G, extra = T - per * G;
  const int x0 = cid * per + min(cid, extra);
  const int nunits = per + (cid < extra ? 1 : 0);
  const int64_t row_bytes = (int64_t)p.nkb * BLOCK_BYTES;
  SkgPos pos;
  if (nunits > 0) skg_first(pos, ustart, eoff, E, U, x0);

  if (warp == CW) {
    // ---------------- producer: one bulk copy per staged row ----------------
    const uint32_t run = (uint32_t)p.nkb * BLOCK_BYTES;
    const int r = lane & 15;
    // tile row r holds matrix row 16u + r, or (SwiGLU) gate row 8u + r / up row N/2 + 8u + r - 8
    const int rofs = SWIGLU ? (r < 8 ? r : p.N / 2 + r - 8) : r;
    const int ustep = SWIGLU ? 8 : kSkRows;
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
        const uint8_t* src = p.W + ((int64_t)pos.e * p.N + (int64_t)pos.u * ustep + rofs) * row_bytes;
        if (lane == 0) mbar_arrive_expect_tx(full(s), (uint32_t)kSkRows * run);
        __syncwarp();
        if (lane < kSkRows) bulk_copy_g2s(dst0 + soff, src, run, full(s));
      }
      if (i + 1 < nunits) skg_next(pos, ustart, eoff, U);
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
    for (int i = 0; i < nunits; ++i) {
      if (!mbar_wait_l(redfull(r), rph, abort_flag, limit)) break;
      const int nout = kSkRows * pos.nr;
      const float* rs = red + (size_t)r * CW * kSkPartial;
      float v[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {  // output o = token * 16 + row, o = lane + 32 q
        const int o = lane + 32 * q;
        const float* rp = rs + (o >> 4) * kSkTokStride + (o & 15);
        float pv[WMAX];
#pragma unroll
        for (int w = 0; w < WMAX; ++w) pv[w] = w < CW ? rp[w * kSkPartial] : 0.f;
        float acc = 0.f;
#pragma unroll
        for (int w = 0; w < WMAX; ++w) acc += pv[w];  // in K order
        v[q] = acc;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(redempty(r));
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int o = lane + 32 * q;
        const int tok = o >> 4, row = o & 15;
        if (SWIGLU) {
          const float up = __shfl_down_sync(0xffffffffu, v[q], 8);  // row + 8 of the same token
          if (row < 8 && o < nout) {
            const __nv_bfloat16 h = __float2bfloat16_rn(silu_mul(v[q], up));
            static_cast<__nv_bfloat16*>(p.out)[(int64_t)(pos.r0 + tok) * (p.N / 2) + 8 * pos.u + row] = h;
          }
        } else if (o < nout) {
          static_cast<float*>(p.out)[(int64_t)(pos.r0 + tok) * p.N + kSkRows * pos.u + row] = v[q];
        }
      }
      if (i + 1 < nunits) skg_next(pos, ustart, eoff, U);
      if (++r == kSkRedSlots) {
        r = 0;
        rph ^= 1u;
      }
    }
  } else {
    // ---------------- consumers: warp w owns super-blocks KPW*w .. KPW*w + KPW-1 ----------------
    const int w = warp;
    bool has[KPW];
#pragma unroll
    for (int kk = 0; kk < KPW; ++kk) has[kk] = KPW * w + kk < p.nkb;
    SkAct act[KPW];
    int cur = -1;  // first sorted row of the token group whose fragments are loaded
    const uint32_t mb = 2u * (t & 1);
    const uint8_t* rowp = smem + g * p.pitch + KPW * w * BLOCK_BYTES;
    const int p8 = 8 * p.pitch;
    float* redw = red + (size_t)w * kSkPartial + 2 * t * kSkTokStride + g;
    const size_t red_slot = (size_t)CW * kSkPartial;
    int s = 0, r = 0;
    uint32_t ph = 0, rph = 0, soff = 0;
    for (int i = 0; i < nunits; ++i) {
      if (pos.r0 != cur) {  // a new token group: its fragments, from A rows (gathered)
        cur = pos.r0;
        const bool mine = g < pos.nr;
        const int64_t arow =
            mine ? (ROUTE ? r_rtok[pos.r0 + g] : (p.gather ? __ldg(p.gather + pos.r0 + g) : pos.r0 + g)) : 0;
#pragma unroll
        for (int kk = 0; kk < KPW; ++kk)
          sk_load_act(act[kk], p.A + arow * p.K + (int64_t)(KPW * w + kk) * QK + 8 * t, has[kk] && mine, t);
      }
      if (i + 1 < nunits) skg_next(pos, ustart, eoff, U);
      if (!mbar_wait_l(full(s), ph, abort_flag, limit)) break;
      float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int kk = 0; kk < KPW; ++kk) {
        const uint8_t* r0p = rowp + soff + kk * BLOCK_BYTES;
        if (has[kk]) sk_block(c, r0p, r0p + p8, act[kk], t, mb);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty(s));
      soff += stage_bytes;
      if (++s == S) {
        s = 0;
        soff = 0;
        ph ^= 1u;
      }
      if (i >= kSkRedSlots && !mbar_wait_l(redempty(r), rph ^ 1u, abort_flag, limit)) break;
      float* rp = redw + r * red_slot;  // [token][row]; tokens past the group read as zero
      rp[0] = c[0];
      rp[8] = c[2];
      rp[kSkTokStride] = c[1];
      rp[kSkTokStride + 8] = c[3];
      __syncwarp();
      if (lane == 0) mbar_arrive(redfull(r));
      if (++r == kSkRedSlots) {
        r = 0;
        rph ^= 1u;
      }
    }
  }
}

// Launch shape: KPW as the dense stationary GEMV picks it (two super-blocks a warp
// from 11 on), one K part only; the ring as deep as the budget allows, between 2 and
// 8 stages. `smem_budget` is the shared memory one CTA may take.
struct SkgCfg {
  int kpw, CW, pitch, stages;
  size_t smem;
};

inline bool skg_shape(int nkb, int E, size_t smem_budget, SkgCfg* c, bool route = false) {
  c->kpw = nkb > 10 ? 2 : 1;
  const int KU = c->kpw == 2 ? SkMax<2>::KU : SkMax<1>::KU;
  if (nkb > KU) return false;
  c->CW = (nkb + c->kpw - 1) / c->kpw;
  c->pitch = sk_pitch(nkb);
  int st = 8;
  while (st > 2 && SkgSmem::total(c->pitch, st, c->CW, E, route) > smem_budget) --st;
  c->stages = st;
  c->smem = SkgSmem::total(c->pitch, st, c->CW, E, route);
  return c->smem <= smem_budget;
}

}  // namespace q4k
