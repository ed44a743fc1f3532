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

// Philox4x32 with 10 rounds (Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As Easy
// as 1, 2, 3", SC 2011): counter c0..c3, key k0 k1; returns the four 32-bit output words.
__device__ __forceinline__ uint4 philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3, uint32_t k0,
                                               uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint32_t hi0 = __umulhi(0xD2511F53u, c0), lo0 = 0xD2511F53u * c0;
    const uint32_t hi1 = __umulhi(0xCD9E8D57u, c2), lo1 = 0xCD9E8D57u * c2;
    c0 = hi1 ^ c1 ^ k0;
    c1 = lo1;
    c2 = hi0 ^ c3 ^ k1;
    c3 = lo0;
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
  return make_uint4(c0, c1, c2, c3);
}

// The 16 keep bytes of keys 16 kb .. 16 kb + 15 for packed row r, head h.
__device__ __forceinline__ uint4 dropout_bytes(const Dropout& d, uint32_t kb, uint32_t r, uint32_t h) {
  return philox4x32_10(kb, r, h, d.offset, d.seed_lo, d.seed_hi);
}

// Drop flags of the four keep bytes in x: bit 7 of byte b of the result is set iff byte b of
// x is >= T (the element is dropped); the other bits are unspecified.  t4 = (T - 1) in every
// byte, t4h = t4 | 0x80808080.  Per byte, d = (T - 1 | 0x80) - (x & 0x7F) cannot borrow from
// the next byte, and its bit 7 says (T - 1) mod 128 >= x mod 128; combined with the top bits
// of x and T - 1 that decides T - 1 < x.  Valid for every 1 <= T <= 256.
__device__ __forceinline__ uint32_t drop_flags4(uint32_t x, uint32_t t4, uint32_t t4h) {
  const uint32_t d = t4h - (x & 0x7F7F7F7Fu);
  return (~t4 & x) | (~(x ^ t4) & ~d);
}

// prmt.b32 with sign replication: selector nibble 8 | b fills the result byte with bit 7 of
// byte b of `a`.  Used to widen drop flags into element masks.
template <uint32_t SEL>
__device__ __forceinline__ uint32_t prmt_sign(uint32_t a) {
  uint32_t r;
  asm("prmt.b32 %0, %1, 0, %2;" : "=r"(r) : "r"(a), "n"(SEL));
  return r;
}

__device__ __forceinline__ uint32_t prmt_sign_r(uint32_t a, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, 0, %2;" : "=r"(r) : "r"(a), "r"(sel));
  return r;
}

// Drop flags for a kernel whose compute thread owns a key (a Philox call covers 16 keys of one
// query).  For a tile of 64 queries x 128 keys, 64 producer threads draw the 512 calls (thread
// rt: key block rt / 8, queries u + 16 k for u in {rt % 8, rt % 8 + 8}, k = 0..3) and store
// the flags transposed: word [block][key tk][u] holds, in byte k, the flag of query u + 16 k
// for key 16 block + tk; + 16 words per block put blocks 2w and 2w + 1 in other banks.
constexpr int kFlagWords64 = 16 * 16 + 16;
constexpr int kFlagBytes64 = 4 * 8 * kFlagWords64;

// rt's share of the tile whose first key block is key_block0 and first packed row row0, as
// flag words in registers (fw[uh][4 k + word]: queries rt % 8 + 8 uh + 16 k).
__device__ __forceinline__ void draw_flag_words64(const Dropout& d, int rt, long long key_block0, long long row0,
                                                  int h, uint32_t (&fw)[2][16]) {
  const int blk = rt >> 3, u0 = rt & 7;
  const uint32_t t4 = (d.threshold - 1u) * 0x01010101u, t4h = t4 | 0x80808080u;
#pragma unroll
  for (int uh = 0; uh < 2; ++uh)
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint4 w = dropout_bytes(d, (uint32_t)(key_block0 + blk), (uint32_t)(row0 + u0 + 8 * uh + 16 * k),
                                    (uint32_t)h);
      fw[uh][4 * k] = drop_flags4(w.x, t4, t4h);
      fw[uh][4 * k + 1] = drop_flags4(w.y, t4, t4h);
      fw[uh][4 * k + 2] = drop_flags4(w.z, t4, t4h);
      fw[uh][4 * k + 3] = drop_flags4(w.w, t4, t4h);
    }
}

// Stores rt's flag words transposed into the tile's buffer at zbuf.
__device__ __forceinline__ void store_flag_words64(uint32_t zbuf, int rt, const uint32_t (&fw)[2][16]) {
  const int blk = rt >> 3, u0 = rt & 7;
#pragma unroll
  for (int uh = 0; uh < 2; ++uh)
#pragma unroll
    for (int tk = 0; tk < 16; ++tk) {
      // flag byte of key tk of query u + 16 k is byte tk % 4 of fw[uh][4 k + tk / 4]
      const uint32_t sel = (uint32_t)(tk & 3) | ((uint32_t)(4 + (tk & 3)) << 4);
      const uint32_t lo2 = __byte_perm(fw[uh][tk >> 2], fw[uh][4 + (tk >> 2)], sel);
      const uint32_t hi2 = __byte_perm(fw[uh][8 + (tk >> 2)], fw[uh][12 + (tk >> 2)], sel);
      asm volatile("st.shared.u32 [%0], %1;" ::"r"(zbuf + 4u * (blk * kFlagWords64 + tk * 16 + u0 + 8 * uh)),
                   "r"(__byte_perm(lo2, hi2, 0x5410))
                   : "memory");
    }
}

__device__ __forceinline__ void draw_flags64(const Dropout& d, uint32_t zbuf, int rt, long long key_block0,
                                             long long row0, int h) {
  uint32_t fw[2][16];
  draw_flag_words64(d, rt, key_block0, row0, h, fw);
  store_flag_words64(zbuf, rt, fw);
}

// The 16 flag words of key r of the tile (word u: queries u + 16 k in byte k).
__device__ __forceinline__ void read_flags64(uint32_t zbuf, int r, uint32_t (&zb)[16]) {
  const uint32_t src = zbuf + 4u * ((r >> 4) * kFlagWords64 + (r & 15) * 16);
#pragma unroll
  for (int v4 = 0; v4 < 4; ++v4)
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(zb[4 * v4]), "=r"(zb[4 * v4 + 1]), "=r"(zb[4 * v4 + 2]), "=r"(zb[4 * v4 + 3])
                 : "r"(src + 16u * v4)
                 : "memory");
}

// All-ones mask if query q (0..63) of the tile is dropped for this key, else 0.
__device__ __forceinline__ uint32_t flag_mask64(const uint32_t (&zb)[16], int q) {
  return prmt_sign_r(zb[q & 15], (8u | (uint32_t)(q >> 4)) * 0x1111u);
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

// Debug builds (compiled with -DATTN_SINK_DEBUG) check the element range [first, last] of a
// global store against its tensor's element count n: a range outside it sets
// kStatusDebugBounds in the device status word and the store is skipped.  This stands in
// for a memory checker on machines where none can run.  Release builds compile it away.
__device__ __forceinline__ bool store_ok(long long first, long long last, long long n, unsigned* status) {
#ifdef ATTN_SINK_DEBUG
  if (first >= 0 && first <= last && last < n) return true;
  set_status(status, kStatusDebugBounds);
  return false;
#else
  (void)first; (void)last; (void)n; (void)status;
  return true;
#endif
}

}  // namespace attn_sink
