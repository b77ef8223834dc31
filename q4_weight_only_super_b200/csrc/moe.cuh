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

// Routing of one tile of kRouteTokPerCta tokens: one warp per token. Iterated
// arg-max over the E logits (each lane holds PL <= 32 of them, E <= 32*PL),
// softmax over the selected logits in fp32. `hist` (shared, E entries, zeroed
// by the caller) receives the tile's expert histogram; `sids` (shared, or
// nullptr) a copy of the tile's ids, [token in tile][topk].
template <int PL>
__device__ __forceinline__ void route_tile(const float* __restrict__ logits, int M, int E, int topk,
                                           int32_t* __restrict__ ids, float* __restrict__ wts, int* hist,
                                           int* sids, int tile) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int tt = 0; tt < kRouteTokPerWarp; ++tt) {
    const int tl = warp * kRouteTokPerWarp + tt;  // token within the tile
    const int tok = tile * kRouteTokPerCta + tl;
    if (tok >= M) break;  // uniform per warp
    const float* row = logits + (int64_t)tok * E;
    float v[PL];
    uint32_t taken = 0;
#pragma unroll
    for (int i = 0; i < PL; ++i) {
      const int e = i * 32 + lane;
      v[i] = e < E ? row[e] : 0.f;
    }
    float sel_v[kMaxTopk];
    int sel_i[kMaxTopk];
    for (int k = 0; k < topk; ++k) {
      float bv = -INFINITY;  // a lane with no candidate left never wins
      int bi = 0x7fffffff;
#pragma unroll
      for (int i = 0; i < PL; ++i) {
        const int e = i * 32 + lane;
        if (e < E && !((taken >> i) & 1u) && ranks_before(v[i], e, bv, bi)) {
          bv = v[i];
          bi = e;
        }
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
        if (ranks_before(ov, oi, bv, bi)) { bv = ov; bi = oi; }
      }
      if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
      sel_v[k] = bv;
      sel_i[k] = bi;
    }
    // softmax over the selected logits; sel_v[0] is the largest
    float den = 0.f;
    for (int k = 0; k < topk; ++k) den += expf(sel_v[k] - sel_v[0]);
    if (lane < topk) {
      float num = 0.f;
      int id = 0;
      for (int k = 0; k < topk; ++k)
        if (k == lane) { num = expf(sel_v[k] - sel_v[0]); id = sel_i[k]; }
      ids[(int64_t)tok * topk + lane] = id;
      wts[(int64_t)tok * topk + lane] = num / den;
      if (sids) sids[tl * topk + lane] = id;
      atomicAdd(&hist[id], 1);
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
  route_tile<PL>(logits, M, E, topk, ids, wts, hist, nullptr, blockIdx.x);
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

// Routing and permutation of at most kRouteTokPerCta tokens in one CTA (one
// launch instead of two; the histogram and the ids stay in shared memory).
template <int PL>
__global__ void __launch_bounds__(256)
route_permute_one_kernel(const float* __restrict__ logits, int M, int E, int topk, int32_t* __restrict__ ids,
                         float* __restrict__ wts, int32_t* __restrict__ expert_offsets,
                         int32_t* __restrict__ perm, int32_t* __restrict__ inv_perm,
                         int32_t* __restrict__ row_token) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  __shared__ int base[kMaxE];
  __shared__ int total[kMaxE];
  __shared__ int warp_sums[32];
  __shared__ int sids[kRouteTokPerCta * kMaxTopk];
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    total[e] = 0;
    base[e] = 0;
  }
  __syncthreads();
  route_tile<PL>(logits, M, E, topk, ids, wts, total, sids, 0);
  __syncthreads();
  scan_and_place(base, total, warp_sums, E, true, expert_offsets, ids, sids, 0, M * topk, topk, perm, inv_perm,
                 row_token);
}

// y[t][h] = sum_j w[t][j] * O[inv_perm[t*topk + j]][h], j in increasing order.
__global__ void __launch_bounds__(256)
combine_kernel(const float* __restrict__ O, const int32_t* __restrict__ inv_perm,
               const float* __restrict__ w, int M, int topk, int H, float* __restrict__ Y) {
  asm volatile("griddepcontrol.wait;" ::: "memory");  // O comes from the expert GEMV
  const int t = blockIdx.y;
  const int h4 = blockIdx.x * blockDim.x + threadIdx.x;  // index of a float4
  if (h4 * 4 >= H) return;
  const int rows = M * topk;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int j = 0; j < topk; ++j) {
    const int r = inv_perm[(int64_t)t * topk + j];
    if (r < 0 || r >= rows) {
      latch_status(Q4K_ERR_DEVICE_BOUNDS);
      continue;
    }
    const float wj = w[(int64_t)t * topk + j];
    const float4 o = *reinterpret_cast<const float4*>(O + (int64_t)r * H + 4 * h4);
    acc.x = fmaf(wj, o.x, acc.x);
    acc.y = fmaf(wj, o.y, acc.y);
    acc.z = fmaf(wj, o.z, acc.z);
    acc.w = fmaf(wj, o.w, acc.w);
  }
  *reinterpret_cast<float4*>(Y + (int64_t)t * H + 4 * h4) = acc;
}

}  // namespace q4k
