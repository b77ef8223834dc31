// Mixture-of-experts routing, token permutation and weighted combine
// (hipEngine 0.3.0 README, "Architecture at a glance": the moe kernel family;
// "Core principles": the gate_combine_residual composite).
#pragma once
#include "common.cuh"

namespace q4k {

constexpr int kRouteWarps = 8;
constexpr int kRouteTokPerWarp = 4;
constexpr int kRouteTokPerCta = kRouteWarps * kRouteTokPerWarp;  // tokens per histogram tile
constexpr int kMaxE = 1024;
constexpr int kMaxTopk = 16;

// Is (va, ia) ranked before (vb, ib)? Higher logit first; equal logits -> lower id.
__device__ __forceinline__ bool ranks_before(float va, int ia, float vb, int ib) {
  return va > vb || (va == vb && ia < ib);
}

// Unsigned key with the order of the fp32 value (finite values; -0 and +0
// equal, as in the float comparison).
__device__ __forceinline__ uint32_t order_key(float v) {
  const uint32_t u = __float_as_uint(v == 0.f ? 0.f : v);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// Routing of one tile of kRouteTokPerCta tokens: a warp per token, tokens
// dealt round-robin over the NW warps of the CTA. Iterated arg-max over the E logits (each
// lane holds PL <= 32 of them, E <= 32*PL): per round each lane takes its best
// remaining (logit, id), the warp takes the largest logit (a reduce-max over
// order keys) and, among lanes holding it, the smallest id (a reduce-min) --
// the order "higher logit first, equal logits to the lower id". Softmax over
// the selected logits in fp32 (lane k holds winner k: one exp per lane, the sum
// over the lanes in a fixed butterfly order). `hist` (shared, E entries, zeroed by the caller)
// receives the tile's expert histogram; `sids` (shared, or nullptr) a copy of
// the tile's ids [token in tile][topk]; `tmask` (shared, or nullptr) bit t of
// entry e set when token t of the tile selected expert e.
template <int PL, int NW>
__device__ __forceinline__ void route_tile(const float* __restrict__ logits, int M, int E, int topk,
                                           int32_t* __restrict__ ids, float* __restrict__ wts, int* hist,
                                           int* sids, unsigned* tmask, int tile) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  static_assert(kRouteTokPerCta % NW == 0, "whole tokens per warp");
  constexpr int TPW = kRouteTokPerCta / NW;  // tokens per warp
  if constexpr (TPW == 1) {
    // One token a warp (the one-CTA routing kernel): its logits loaded at once, the
    // selection rounds unrolled where the registers allow. Winner k is kept by lane k.
    float v[TPW][PL];
    uint32_t taken[TPW];
    float my_v[TPW];
    int my_i[TPW];
#pragma unroll
    for (int tt = 0; tt < TPW; ++tt) {
      const int tok = tile * kRouteTokPerCta + tt * NW + warp;
      const float* row = logits + (int64_t)tok * E;
#pragma unroll
      for (int i = 0; i < PL; ++i) {
        const int e = i * 32 + lane;
        v[tt][i] = (tok < M && e < E) ? row[e] : 0.f;
      }
      taken[tt] = 0u;
      my_v[tt] = 0.f;
      my_i[tt] = 0;
    }
    // this warp's tokens in the tile (tokens past M take no rounds)
    const int ntok = min(TPW, max(0, (M - tile * kRouteTokPerCta - warp + NW - 1) / NW));
    auto round = [&](int k) {
#pragma unroll
      for (int tt = 0; tt < TPW; ++tt) {
        if (tt >= ntok) break;  // uniform per warp
        float bv = -INFINITY;  // a lane with no candidate left never wins
        int bi = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < PL; ++i) {
          const int e = i * 32 + lane;
          if (e < E && !((taken[tt] >> i) & 1u) && ranks_before(v[tt][i], e, bv, bi)) {
            bv = v[tt][i];
            bi = e;
          }
        }
        const uint32_t key = bi == 0x7fffffff ? 0u : order_key(bv);
        const uint32_t kmax = __reduce_max_sync(0xffffffffu, key);
        const int wi = (int)__reduce_min_sync(0xffffffffu, key == kmax ? (uint32_t)bi : 0x7fffffffu);
        if ((wi & 31) == lane) taken[tt] |= 1u << (wi >> 5);
        if (lane == k) {
          my_v[tt] = key_value(kmax);
          my_i[tt] = wi;
        }
      }
    };
    if constexpr (PL <= 8) {  // the rounds unrolled (few logits a lane: registers to spare)
#pragma unroll
      for (int k = 0; k < kMaxTopk; ++k) {
        if (k >= topk) break;
        round(k);
      }
    } else {
      for (int k = 0; k < topk; ++k) round(k);
    }
    // softmax over each token's selected logits (lane 0 holds the largest): one exp
    // per lane, the sum over the lanes in a fixed butterfly order
#pragma unroll
    for (int tt = 0; tt < TPW; ++tt) {
      const int tl = tt * NW + warp;  // token within the tile
      const int tok = tile * kRouteTokPerCta + tl;
      if (tok >= M) break;  // uniform per warp
      const float v0 = __shfl_sync(0xffffffffu, my_v[tt], 0);
      const float ek = lane < topk ? expf(my_v[tt] - v0) : 0.f;
      float den = ek;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
      if (lane < topk) {
        const int id = my_i[tt];
        if (ids) ids[(int64_t)tok * topk + lane] = id;  // (null: not written)
        if (wts) wts[(int64_t)tok * topk + lane] = ek / den;
        if (sids) sids[tl * topk + lane] = id;
        if (tmask) atomicOr(&tmask[id], 1u << tl);
        atomicAdd(&hist[id], 1);
      }
    }
  } else {
    // Several tokens a warp: one after another (the next token's logits load while the
    // warp routes the current one; one copy of the rounds, so the code stays small).
    float nxt[PL];
    auto load = [&](int tt) {
      const int tok = tile * kRouteTokPerCta + tt * NW + warp;
      const float* row = logits + (int64_t)tok * E;
#pragma unroll
      for (int i = 0; i < PL; ++i) {
        const int e = i * 32 + lane;
        nxt[i] = (tok < M && e < E) ? row[e] : 0.f;
      }
    };
    load(0);
#pragma unroll 1
    for (int tt = 0; tt < TPW; ++tt) {
      const int tl = tt * NW + warp;  // token within the tile
      const int tok = tile * kRouteTokPerCta + tl;
      if (tok >= M) break;  // uniform per warp
      float v[PL];
      uint32_t taken = 0;
#pragma unroll
      for (int i = 0; i < PL; ++i) v[i] = nxt[i];
      if (tt + 1 < TPW) load(tt + 1);
      float my_v = 0.f;
      int my_i = 0;
      for (int k = 0; k < topk; ++k) {
        float bv = -INFINITY;
        int bi = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < PL; ++i) {
          const int e = i * 32 + lane;
          if (e < E && !((taken >> i) & 1u) && ranks_before(v[i], e, bv, bi)) {
            bv = v[i];
            bi = e;
          }
        }
        const uint32_t key = bi == 0x7fffffff ? 0u : order_key(bv);
        const uint32_t kmax = __reduce_max_sync(0xffffffffu, key);
        const int wi = (int)__reduce_min_sync(0xffffffffu, key == kmax ? (uint32_t)bi : 0x7fffffffu);
        if ((wi & 31) == lane) taken |= 1u << (wi >> 5);
        if (lane == k) {
          my_v = key_value(kmax);
          my_i = wi;
        }
      }
      const float v0 = __shfl_sync(0xffffffffu, my_v, 0);
      const float ek = lane < topk ? expf(my_v - v0) : 0.f;
      float den = ek;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
      if (lane < topk) {
        const int id = my_i;
        if (ids) ids[(int64_t)tok * topk + lane] = id;
        if (wts) wts[(int64_t)tok * topk + lane] = ek / den;
        if (sids) sids[tl * topk + lane] = id;
        if (tmask) atomicOr(&tmask[id], 1u << tl);
        atomicAdd(&hist[id], 1);
      }
    }
  }
}

// Routing of any number of tokens: CTA b routes token tile b and writes its
// expert histogram to counts[b][E]. The logits may come from the previous
// kernel (programmatic dependent launch: wait first, then let the permutation
// kernel launch).
template <int PL>
__global__ void __launch_bounds__(32 * kRouteWarps)
route_kernel(const float* __restrict__ logits, int M, int E, int topk, int32_t* __restrict__ ids,
             float* __restrict__ wts, int32_t* __restrict__ counts) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  __shared__ int hist[kMaxE];
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  route_tile<PL, kRouteWarps>(logits, M, E, topk, ids, wts, hist, nullptr, nullptr, blockIdx.x);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) counts[(int64_t)blockIdx.x * E + e] = hist[e];
}

// Exclusive scan of the per-expert totals (E <= 1024, 256 threads): expert e's
// rows start at the running sum of the totals before it. base[e] (holding this
// tile's offset inside expert e) gets that start added; the CTA with
// `write_offsets` stores expert_offsets[0..E]. Then warp 0 places the tile's
// (token, slot) pairs f in [f0, f1) in flat-index order (stable sort by expert),
// their experts read from `sids` (shared, indexed f - f0) when given, else from ids.
__device__ __forceinline__ void scan_and_place(int* base, const int* total, int* warp_sums, int E,
                                               bool write_offsets, int32_t* __restrict__ expert_offsets,
                                               const int32_t* ids, const int* sids, int f0, int f1, int topk,
                                               int32_t* __restrict__ perm, int32_t* __restrict__ inv_perm,
                                               int32_t* __restrict__ row_token) {
  {
    const int per = (E + blockDim.x - 1) / blockDim.x;
    const int e0 = threadIdx.x * per;
    int run = 0;
    for (int e = e0; e < e0 + per && e < E; ++e) run += total[e];
    // block-wide exclusive scan of run
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = run;
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += o;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const int nw = blockDim.x / 32;
      int ws = lane < nw ? warp_sums[lane] : 0;
      for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, ws, off);
        if (lane >= off) ws += o;
      }
      if (lane < nw) warp_sums[lane] = ws;  // inclusive
    }
    __syncthreads();
    int excl = incl - run + (warp > 0 ? warp_sums[warp - 1] : 0);
    for (int e = e0; e < e0 + per && e < E; ++e) {
      const int tot = total[e];
      if (write_offsets) expert_offsets[e] = excl;
      base[e] += excl;
      excl += tot;
    }
    if (write_offsets && threadIdx.x == blockDim.x - 1) expert_offsets[E] = excl;  // grand total
  }
  __syncthreads();
  // stable placement by warp 0, 32 pairs at a time in flat-index order
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    for (int fs = f0; fs < f1; fs += 32) {
      const int f = fs + lane;
      const bool act = f < f1;
      // (from L2 when global: they may be this kernel's own stores)
      const int e = act ? (sids ? sids[f - f0] : __ldcg(ids + f)) : -1 - lane;
      const bool ok = !act || (e >= 0 && e < E);
      if (!ok) latch_status(Q4K_ERR_DEVICE_BOUNDS);
      const unsigned peers = __match_any_sync(0xffffffffu, e);
      const int rank = __popc(peers & ((1u << lane) - 1u));
      if (act && ok) {
        const int pos = base[e] + rank;
        perm[pos] = f;
        inv_perm[f] = pos;
        row_token[pos] = f / topk;
      }
      __syncwarp();
      if (act && ok && rank == __popc(peers) - 1) base[e] += __popc(peers);
      __syncwarp();
    }
  }
}

// Permutation: CTA b places the (token, slot) pairs of its token tile. Its
// base position for expert e is offsets[e] + (rows of e in tiles < b).
__global__ void __launch_bounds__(256)
permute_kernel(const int32_t* __restrict__ ids, const int32_t* __restrict__ counts, int M, int E,
               int topk, int ntiles, int32_t* __restrict__ expert_offsets, int32_t* __restrict__ perm,
               int32_t* __restrict__ inv_perm, int32_t* __restrict__ row_token) {
  asm volatile("griddepcontrol.wait;" ::: "memory");  // ids and counts come from route_kernel
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  __shared__ int base[kMaxE];
  __shared__ int total[kMaxE];
  __shared__ int warp_sums[32];
  const int b = blockIdx.x;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int before = 0, all = 0;
    for (int bb = 0; bb < ntiles; ++bb) {
      const int c = counts[(int64_t)bb * E + e];
      all += c;
      if (bb < b) before += c;
    }
    total[e] = all;
    base[e] = before;
  }
  __syncthreads();
  scan_and_place(base, total, warp_sums, E, b == 0, expert_offsets, ids, nullptr, b * kRouteTokPerCta * topk,
                 min(M, (b + 1) * kRouteTokPerCta) * topk, topk, perm, inv_perm, row_token);
}

// After route_tile over a CTA's single tile (all threads of the CTA call this): the
// exclusive scan of the per-expert totals into the expert offsets and each expert's
// start, then the stable place of every (token, slot) pair f = t*topk + j: a token
// selects an expert at most once, so f's rank among expert e's pairs is the number of
// earlier tokens that selected e (the popcount of e's token mask below bit t). Each of
// the outputs may be null (not written): global (g_*) and shared-memory copies (s_offsets
// [E+1], s_row_token [M*topk]).
__device__ __forceinline__ void route_scan_place_one(const int* total, int* start, int* warp_sums, int E, int M,
                                                     int topk, const int* sids, const unsigned* tmask,
                                                     int32_t* __restrict__ g_offsets, int32_t* __restrict__ g_perm,
                                                     int32_t* __restrict__ g_inv_perm,
                                                     int32_t* __restrict__ g_row_token, int* s_offsets,
                                                     int* s_row_token) {
  {
    const int per = (E + blockDim.x - 1) / blockDim.x;
    const int e0 = threadIdx.x * per;
    int run = 0;
    for (int e = e0; e < e0 + per && e < E; ++e) run += total[e];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = run;
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += o;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const int nw = blockDim.x / 32;
      int ws = lane < nw ? warp_sums[lane] : 0;
      for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, ws, off);
        if (lane >= off) ws += o;
      }
      if (lane < nw) warp_sums[lane] = ws;
    }
    __syncthreads();
    int excl = incl - run + (warp > 0 ? warp_sums[warp - 1] : 0);
    for (int e = e0; e < e0 + per && e < E; ++e) {
      if (g_offsets) g_offsets[e] = excl;
      if (s_offsets) s_offsets[e] = excl;
      start[e] = excl;
      excl += total[e];
    }
    if (threadIdx.x == blockDim.x - 1) {
      if (g_offsets) g_offsets[E] = excl;
      if (s_offsets) s_offsets[E] = excl;
    }
  }
  __syncthreads();
  for (int f = threadIdx.x; f < M * topk; f += blockDim.x) {
    const int t = f / topk;
    const int e = sids[f];
    if (e < 0 || e >= E) {
      latch_status(Q4K_ERR_DEVICE_BOUNDS);
      continue;
    }
    const int pos = start[e] + __popc(tmask[e] & ((1u << t) - 1u));
    if (g_perm) g_perm[pos] = f;
    if (g_inv_perm) g_inv_perm[f] = pos;
    if (g_row_token) g_row_token[pos] = t;
    if (s_row_token) s_row_token[pos] = t;
  }
}

// Routing and permutation of at most kRouteTokPerCta tokens in one CTA (one
// launch instead of two; the histogram, the ids and the per-expert token masks
// stay in shared memory). A token selects an expert at most once, so the rank
// of pair f = t*topk + j among expert e's pairs in flat order is the number of
// earlier tokens that selected e: the popcount of e's mask below bit t. Every
// pair is placed by its own thread.
constexpr int kRouteOneWarps = kRouteTokPerCta;  // one warp per token

template <int PL>
__global__ void __launch_bounds__(32 * kRouteOneWarps)
route_permute_one_kernel(const float* __restrict__ logits, int M, int E, int topk, int32_t* __restrict__ ids,
                         float* __restrict__ wts, int32_t* __restrict__ expert_offsets,
                         int32_t* __restrict__ perm, int32_t* __restrict__ inv_perm,
                         int32_t* __restrict__ row_token) {
  static_assert(kRouteTokPerCta <= 32, "one mask bit per token of the tile");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  __shared__ int total[kMaxE];
  __shared__ int start[kMaxE];
  __shared__ unsigned tmask[kMaxE];
  __shared__ int warp_sums[32];
  __shared__ int sids[kRouteTokPerCta * kMaxTopk];
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    total[e] = 0;
    tmask[e] = 0u;
  }
  __syncthreads();
  route_tile<PL, kRouteOneWarps>(logits, M, E, topk, ids, wts, total, sids, tmask, 0);
  __syncthreads();
  route_scan_place_one(total, start, warp_sums, E, M, topk, sids, tmask, expert_offsets, perm, inv_perm,
                       row_token, nullptr, nullptr);
}

// y[t][h] = sum_j w[t][j] * O[inv_perm[t*topk + j]][h], j in increasing order.
// Slots are taken eight at a time: their row indices and weights are loaded
// first, then their O rows, then they are added in slot order (two memory
// latencies per eight slots, at a register count that keeps the large-M case
// bandwidth-bound).
// RESID: y = residual + (the weighted sum), one final fp32 add (the
// gate_combine_residual composite); residual may be Y itself (each thread reads
// its four values before it writes them).
template <bool RESID>
__global__ void __launch_bounds__(256)
combine_kernel(const float* __restrict__ O, const int32_t* __restrict__ inv_perm,
               const float* __restrict__ w, int M, int topk, int H, const float* residual, float* Y) {
  asm volatile("griddepcontrol.wait;" ::: "memory");  // O comes from the expert GEMV
  const int t = blockIdx.y;
  const int h4 = blockIdx.x * blockDim.x + threadIdx.x;  // index of a float4
  if (h4 * 4 >= H) return;
  const int rows = M * topk;
  constexpr int B = 8;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int j0 = 0; j0 < topk; j0 += B) {
    int r[B];
    float wj[B];
#pragma unroll
    for (int j = 0; j < B; ++j) {
      r[j] = -1;
      wj[j] = 0.f;
      if (j0 + j < topk) {
        r[j] = __ldg(inv_perm + (int64_t)t * topk + j0 + j);
        wj[j] = __ldg(w + (int64_t)t * topk + j0 + j);
      }
    }
    float4 o[B];
#pragma unroll
    for (int j = 0; j < B; ++j) {
      o[j] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (j0 + j < topk && r[j] >= 0 && r[j] < rows)
        o[j] = *reinterpret_cast<const float4*>(O + (int64_t)r[j] * H + 4 * h4);
    }
#pragma unroll
    for (int j = 0; j < B; ++j) {
      if (j0 + j >= topk) break;
      if (r[j] < 0 || r[j] >= rows) {
        latch_status(Q4K_ERR_DEVICE_BOUNDS);
        continue;
      }
      acc.x = fmaf(wj[j], o[j].x, acc.x);
      acc.y = fmaf(wj[j], o[j].y, acc.y);
      acc.z = fmaf(wj[j], o[j].z, acc.z);
      acc.w = fmaf(wj[j], o[j].w, acc.w);
    }
  }
  if (RESID) {
    const float4 rv = *reinterpret_cast<const float4*>(residual + (int64_t)t * H + 4 * h4);
    acc.x = rv.x + acc.x;
    acc.y = rv.y + acc.y;
    acc.z = rv.z + acc.z;
    acc.w = rv.w + acc.w;
  }
  *reinterpret_cast<float4*>(Y + (int64_t)t * H + 4 * h4) = acc;
}

// Router logits: logits[t][e] = sum_k X[t][k] * Wr[e][k] (bf16 x bf16, fp32
// accumulation; the products are exact in fp32). CTA (t, eb) computes experts
// 32*eb .. 32*eb+31 of token t, four per warp: each lane sums its 8-wide slices
// in increasing k, then the warp adds the lanes in a fixed tree.
__global__ void __launch_bounds__(256)
router_logits_kernel(const uint16_t* __restrict__ X, const uint16_t* __restrict__ Wr, int M, int E, int H,
                     float* __restrict__ logits) {
  asm volatile("griddepcontrol.wait;" ::: "memory");  // X may come from the previous kernel
  const int t = blockIdx.x, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint16_t* x = X + (int64_t)t * H;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int e = blockIdx.y * 32 + warp * 4 + i;
    if (e >= E) break;  // uniform per warp
    const uint16_t* w = Wr + (int64_t)e * H;
    float acc = 0.f;
    for (int k8 = lane * 8; k8 < H; k8 += 256) {
      const uint4 xv = ldg_u4(x + k8), wv = ldg_u4(w + k8);
      const uint32_t xa[4] = {xv.x, xv.y, xv.z, xv.w}, wa[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        acc = fmaf(bf16_bits_to_float(xa[j] & 0xFFFFu), bf16_bits_to_float(wa[j] & 0xFFFFu), acc);
        acc = fmaf(bf16_bits_to_float(xa[j] >> 16), bf16_bits_to_float(wa[j] >> 16), acc);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) logits[(int64_t)t * E + e] = acc;
  }
}

}  // namespace q4k
