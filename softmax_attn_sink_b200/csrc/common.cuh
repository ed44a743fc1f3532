// Shared device helpers for the sink-attention kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "launch.h"

namespace attn_sink {

constexpr float kNegInf = -__builtin_huge_valf();
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ float to_float(float x) { return x; }
__device__ __forceinline__ float to_float(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ float to_float(__half x) { return __half2float(x); }

template <typename T> __device__ __forceinline__ T from_float(float x);
template <> __device__ __forceinline__ float from_float<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_float<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}
template <> __device__ __forceinline__ __half from_float<__half>(float x) { return __float2half_rn(x); }

// Two floats rounded to nearest-even into one 32-bit pair of T (low half = lo).
template <typename T> __device__ __forceinline__ uint32_t pack2(float lo, float hi);
template <> __device__ __forceinline__ uint32_t pack2<__nv_bfloat16>(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
template <> __device__ __forceinline__ uint32_t pack2<__half>(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// Key range [lo, hi) visible from query row i of a sequence with sq queries and sk keys,
// bottom-right aligned: pos = i + sk - sq; visible iff pos - left <= j <= pos + right.
// left / right >= kUnbounded mean no bound on that side (causal already folded into right).
__device__ __forceinline__ void row_key_range(long long i, long long sq, long long sk, int left,
                                              int right, long long& lo, long long& hi) {
  const long long pos = i + sk - sq;
  lo = (left >= kUnbounded) ? 0 : pos - left;
  hi = (right >= kUnbounded) ? sk : pos + right + 1;
  lo = lo < 0 ? 0 : lo;
  hi = hi > sk ? sk : hi;
}

// Query range [lo, hi) that sees key j (the inverse of row_key_range).
__device__ __forceinline__ void key_query_range(long long j, long long sq, long long sk, int left,
                                                int right, long long& lo, long long& hi) {
  const long long off = sk - sq;
  // j <= i + off + right  <=>  i >= j - off - right ;  j >= i + off - left  <=>  i <= j - off + left
  lo = (right >= kUnbounded) ? 0 : j - off - right;
  hi = (left >= kUnbounded) ? sq : j - off + left + 1;
  lo = lo < 0 ? 0 : lo;
  hi = hi > sq ? sq : hi;
}

__device__ __forceinline__ bool visible(long long i, long long j, long long sq, long long sk,
                                        int left, int right) {
  const long long pos = i + sk - sq;
  if (j < 0 || j >= sk) return false;
  if (right < kUnbounded && j > pos + right) return false;
  if (left < kUnbounded && j < pos - left) return false;
  return true;
}

__device__ __forceinline__ void set_status(unsigned* status, unsigned bit) {
  if (status) atomicOr(status, bit);
}

}  // namespace attn_sink
