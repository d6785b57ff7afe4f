// Shared device helpers of libmsa (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#define MSA_FULL_MASK 0xffffffffu

namespace msa {

// ---------------------------------------------------------------------------
// Element loads: every kernel computes in fp32 whatever the stored type.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ float to_f32(__nv_fp8_e4m3 x) { return float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Loads N consecutive elements starting at p into fp32 registers, in the widest
// chunks (16, 8 or 4 bytes) that N * sizeof(T) allows; p must be aligned to
// that chunk size (callers pass rows whose offsets are multiples of N).
template <typename T, int N>
__device__ __forceinline__ void load_vec(const T* __restrict__ p, float (&out)[N]) {
  constexpr int bytes = N * int(sizeof(T));
  if constexpr (bytes % 16 == 0) {
    constexpr int per = 16 / sizeof(T);
#pragma unroll
    for (int c = 0; c < N / per; ++c) {
      const uint4 u = *reinterpret_cast<const uint4*>(p + c * per);
      const T* e = reinterpret_cast<const T*>(&u);
#pragma unroll
      for (int i = 0; i < per; ++i) out[c * per + i] = to_f32(e[i]);
    }
  } else if constexpr (bytes % 8 == 0) {
    constexpr int per = 8 / sizeof(T);
#pragma unroll
    for (int c = 0; c < N / per; ++c) {
      const uint2 u = *reinterpret_cast<const uint2*>(p + c * per);
      const T* e = reinterpret_cast<const T*>(&u);
#pragma unroll
      for (int i = 0; i < per; ++i) out[c * per + i] = to_f32(e[i]);
    }
  } else {
#pragma unroll
    for (int i = 0; i < N; ++i) out[i] = to_f32(p[i]);
  }
}

// ---------------------------------------------------------------------------
// Total order on block scores.  The key of block c with score s is
//   (orderable(s) << 32) | (0xffffffff - c)
// so a larger key means a higher score, and among equal scores the lower block
// id.  -0.0 is folded into +0.0 so that equal scores compare equal.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t orderable(float s) {
  if (s == 0.0f) s = 0.0f;
  uint32_t u = __float_as_uint(s);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ uint64_t block_key(float s, int c) {
  return (uint64_t(orderable(s)) << 32) | uint64_t(0xffffffffu - uint32_t(c));
}

__device__ __forceinline__ int key_block(uint64_t key) {
  return int(0xffffffffu - uint32_t(key & 0xffffffffu));
}

// Warp-wide maximum of 64-bit keys: the maximum high word, then the maximum
// low word among the lanes holding that high word (two redux instructions).
__device__ __forceinline__ uint64_t warp_max_u64(uint64_t v) {
  const uint32_t hi = uint32_t(v >> 32), lo = uint32_t(v);
  const uint32_t mh = __reduce_max_sync(MSA_FULL_MASK, hi);
  const uint32_t ml = __reduce_max_sync(MSA_FULL_MASK, hi == mh ? lo : 0u);
  return (uint64_t(mh) << 32) | ml;
}

__device__ __forceinline__ float warp_max_f32(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(MSA_FULL_MASK, v, o));
  return v;
}

__device__ __forceinline__ float warp_sum_f32(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(MSA_FULL_MASK, v, o);
  return v;
}

// Ascending bitonic sort of one int per lane across the warp.
__device__ __forceinline__ int warp_sort_asc(int v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      int other = __shfl_xor_sync(MSA_FULL_MASK, v, stride);
      bool up = (lane & size) == 0 || size == 32;
      bool lower = (lane & stride) == 0;
      v = (lower == up) ? min(v, other) : max(v, other);
    }
  }
  return v;
}

}  // namespace msa
