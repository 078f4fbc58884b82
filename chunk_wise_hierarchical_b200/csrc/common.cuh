// Shared device helpers for the HiLS kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/hils.h"

namespace hils {

constexpr int kChunk = 64;        // B: keys per chunk (the only supported value)
constexpr int kMaxTopK = 64;

// Error word bits written by kernels into the first 8 bytes of a workspace.
constexpr unsigned kErrBadPage = 1u;
constexpr unsigned kErrTimeout = 2u;

// Polls of the waits that drain an abort path (copies and MMAs already issued
// finish before shared and tensor memory are released).  They use this bound
// whatever limit the caller set for ordinary waits.
constexpr uint32_t kDrainPolls = HILS_DEFAULT_WAIT_LIMIT;

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Loads 4 consecutive elements (16-byte aligned for float, 8-byte for bf16) as floats.
__device__ __forceinline__ float4 load4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ float4 load4(const __nv_bfloat16* p) {
  uint2 u = *reinterpret_cast<const uint2*>(p);
  __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162*>(&u.x);
  __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162*>(&u.y);
  float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
  return make_float4(fa.x, fa.y, fb.x, fb.y);
}

// Total order on floats mapped to unsigned ints (larger float -> larger key).
// NaN is mapped like -inf so that it never wins a selection.
__device__ __forceinline__ uint32_t orderable(float f) {
  if (f != f) f = -INFINITY;
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float unorderable(uint32_t u) {
  return __uint_as_float((u & 0x80000000u) ? (u & 0x7fffffffu) : ~u);
}
// Selection key: score in the high word, (0xffffffff - chunk) in the low word,
// so that the larger key is the higher score and, on equal scores, the lower
// chunk index.  Every valid key is > 0; 0 marks "none".
__device__ __forceinline__ unsigned long long pack_key(float score, int chunk) {
  return ((unsigned long long)orderable(score) << 32) | (unsigned long long)(0xffffffffu - (uint32_t)chunk);
}
__device__ __forceinline__ int key_chunk(unsigned long long key) {
  return (int)(0xffffffffu - (uint32_t)(key & 0xffffffffull));
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ unsigned long long warp_max_u64(unsigned long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    unsigned long long w = __shfl_xor_sync(0xffffffffu, v, o);
    v = w > v ? w : v;
  }
  return v;
}

__device__ __forceinline__ void set_error(unsigned* err, unsigned bit) {
  if (err) atomicOr(err, bit);
}

// Remote candidate chunks of the query at position i: the complete chunks before its
// local branch, c < floor(i / B) + 1 - n_local (n_local = 1: the own chunk only; a
// sliding window of W keys spans n_local = W / B chunks), capped at the C complete
// chunks.
__host__ __device__ __forceinline__ int n_candidates(int i, int n_local, int n_chunks) {
  const int c = i / kChunk + 1 - n_local;
  return c < 0 ? 0 : (c < n_chunks ? c : n_chunks);
}

}  // namespace hils
