// Shared device helpers for the Q4_K kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "q4k.h"

namespace q4k {

constexpr int QK = 256;           // weights per super-block
constexpr int BLOCK_BYTES = 144;  // bytes per super-block

// Device status word: 0 = no error latched. Kernels latch the first error.
__device__ int g_status;

// Limit of every bounded device-side wait, in ns of %globaltimer: 2 s by default,
// far beyond any legal wait. A test may shorten it (q4k_test_wait_fault).
__device__ unsigned long long g_wait_limit_ns = 2000000000ull;
// Test hook (q4k_test_wait_fault): when >= 0, the weight producer of every CTA of the
// prefill GEMM and the decode GEMVs skips its stage with this index -- neither the
// copy nor the arrival happens -- so the roles waiting for that stage run into the
// wait limit. -1 (the default) disables it.
__device__ int g_test_drop_stage = -1;

__device__ __forceinline__ void latch_status(int code) { atomicCAS(&g_status, 0, code); }

// ---- loads ---------------------------------------------------------------

// Streaming read-only 8-byte load that does not allocate in L1.
__device__ __forceinline__ uint2 ldg_stream_u2(const void* p) {
  uint2 v;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];"
               : "=r"(v.x), "=r"(v.y) : "l"(p));
  return v;
}

__device__ __forceinline__ uint4 ldg_stream_u4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

__device__ __forceinline__ uint4 ldg_u4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

// ---- Q4_K field decode ----------------------------------------------------

__device__ __forceinline__ float half_bits_to_float(uint32_t h16) {
  return __half2float(__ushort_as_half((unsigned short)(h16 & 0xFFFFu)));
}

// Six-bit (scale, min) pair j of a block, from the 12 packed bytes held as
// three little-endian words s0 = bytes 0..3, s1 = bytes 4..7, s2 = bytes 8..11.
__device__ __forceinline__ void scale_min(uint32_t s0, uint32_t s1, uint32_t s2, int j,
                                          uint32_t& sc, uint32_t& m) {
  if (j < 4) {
    sc = (s0 >> (8 * j)) & 63u;
    m = (s1 >> (8 * j)) & 63u;
  } else {
    const int b = 8 * (j - 4);
    const uint32_t lo = (s2 >> b) & 0xFFu;
    sc = (lo & 15u) | (((s0 >> (b + 6)) & 3u) << 4);
    m = (lo >> 4) | (((s1 >> (b + 6)) & 3u) << 4);
  }
}

__device__ __forceinline__ float bf16_bits_to_float(uint32_t b) {
  return __uint_as_float(b << 16);
}

// SiLU(g) * u with the logistic function evaluated on exp(-|g|), which never
// overflows: for g >= 0, g / (1 + e^-g); for g < 0, g * e^g / (1 + e^g).
__device__ __forceinline__ float silu_mul(float g, float u) {
  const float e = expf(-fabsf(g));
  const float sig = g >= 0.f ? 1.0f / (1.0f + e) : e / (1.0f + e);
  return g * sig * u;
}

}  // namespace q4k
