// Q4_K block dequantisation (the Q4_K "quant reader" of the hipEngine 0.3.0
// README, section "GGUF Support"): 144-byte super-block -> 256 weights,
// w = d*sc*q - dmin*m, rounded once to fp32 (and optionally then to bf16).
#pragma once
#include "common.cuh"

namespace q4k {

// One thread per 8 consecutive weights; 32 threads per block.
// Thread s of a block: chunk c = s/8, half h = (s/4)%2, lanes l0 = 8*(s%4) .. +7.
template <bool BF16>
__global__ void __launch_bounds__(256) dequant_kernel(const uint8_t* __restrict__ W, int64_t nblocks,
                                                      void* __restrict__ out) {
  const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t b = tid >> 5;
  if (b >= nblocks) return;
  const int s = (int)(tid & 31);
  const int c = s >> 3, h = (s >> 2) & 1, l0 = (s & 3) * 8;
  const uint8_t* blk = W + b * BLOCK_BYTES;
  const uint4 hdr = ldg_u4(blk);
  const uint2 qv = *reinterpret_cast<const uint2*>(blk + 16 + 32 * c + l0);
  const float d = half_bits_to_float(hdr.x), dmin = half_bits_to_float(hdr.x >> 16);
  uint32_t sc, m;
  scale_min(hdr.y, hdr.z, hdr.w, 2 * c + h, sc, m);
  const float ds = d * (float)sc;    // exact: 11-bit x 6-bit significands
  const float dm = dmin * (float)m;  // exact
  float w[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const uint32_t word = e < 4 ? qv.x : qv.y;
    const uint32_t q = (word >> (8 * (e & 3) + 4 * h)) & 15u;
    w[e] = fmaf((float)q, ds, -dm);  // one rounding of the exact value
  }
  const int64_t i0 = b * QK + 64 * c + 32 * h + l0;
  if (BF16) {
    uint4 o;
    uint32_t* op = &o.x;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const __nv_bfloat162 p = __floats2bfloat162_rn(w[2 * e], w[2 * e + 1]);
      op[e] = *reinterpret_cast<const uint32_t*>(&p);
    }
    *reinterpret_cast<uint4*>(static_cast<uint16_t*>(out) + i0) = o;
  } else {
    float4* o = reinterpret_cast<float4*>(static_cast<float*>(out) + i0);
    o[0] = make_float4(w[0], w[1], w[2], w[3]);
    o[1] = make_float4(w[4], w[5], w[6], w[7]);
  }
}

}  // namespace q4k
