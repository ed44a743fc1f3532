// Sink-attention forward at head dim 256 on the sm_100a tensor cores (bf16 or fp16 in, fp32
// accumulation).  Same result as the d <= 128 kernel (Huawei CANN ops-transformer flash_attn
// doc, "Function", the formula after "After adding sink"; softmax_lse formula):
//   S = scale * Q K^T,  m = max(sink, max S),
//   out = sum e^{S-m} V / (sum e^{S-m} + e^{sink-m}),   lse = log sum e^{S}  (no sink).
// The CANN doc lists head dims 64, 128 and 256 for q, k and v.
//
// At d = 256 the fp32 O accumulator of one 128-row query unit takes 256 of the 512 TMEM
// columns, so a CTA runs one unit.  Q is kept in TMEM as the A operand of S = Q K^T (128
// columns of packed 16-bit pairs), which frees shared memory for a 3-stage ring of 64-key
// K / V tiles (32 KB each) and keeps the S MMAs compute-bound at N = 64: each K = 16 step
// reads only the 2 KB K slice from shared memory.
//
// TMEM columns: Q [0,128), S/P buffer 0 [128,192), buffer 1 [192,256), O [256,512).
// Warps: 0 TMA producer (K / V ring), 1 TMEM allocation and MMA issuer (the warp runs the loop
// in step; elect.sync over the full warp picks the same issuing lane every time), 2-3 idle,
// 4-7 softmax (thread t = query row t = TMEM lane t), which first copy their Q rows into TMEM
// and finally write out and lse.
// MMA issue order: S(0), S(1), then per tile j: PV(j), S(j+2).  S(j+2) goes into the buffer
// that holds P(j); MMAs from one thread execute in issue order, so PV(j) has read P(j) by
// then.  The softmax of tile j+1 overlaps PV(j) and S(j+2) on the tensor pipe.
// The running max starts at the sink (log2 domain; the sink is in post-scale units), the
// running sum counts keys only, and O is rescaled lazily, only when a row's max grows by more
// than 2^8.  Every mbarrier wait is bounded; a timeout sets the status word and the CTA
// drains and frees its TMEM instead of hanging.
#include <cuda.h>

#include <type_traits>

#include "sm100_ptx.cuh"
#include "tma_map.h"

namespace attn_sink {
namespace {

using namespace sm100;

constexpr int D = 256;
constexpr int kBM = 128;                    // query rows per CTA
constexpr int kBN = 64;                     // keys per tile
constexpr int kStages = 3;                  // K / V ring depth
constexpr int kThreads = 256;
constexpr int kBox = kBN * 128;             // one TMA box: 64 rows x 64 columns (128 bytes)
constexpr int kTileBytes = (D / 64) * kBox; // a K or V tile: 4 boxes
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColQ = 0, kColO = 256;
constexpr float kRescaleThreshold = 8.0f;   // log2 units

__host__ __device__ constexpr uint32_t col_S(int b) { return 128u + 64u * (uint32_t)b; }

constexpr int kOffK = 0;
constexpr int kOffV = kOffK + kStages * kTileBytes;
constexpr int kOffBar = kOffV + kStages * kTileBytes;
// q_full, k_full[S], k_empty[S], v_full[S], v_empty[S], s_full[2], p_full[2], pv_done, drain,
// o_done
constexpr int kNumBars = 1 + 4 * kStages + 7;
constexpr int kOffSlot = kOffBar + kNumBars * 8;
constexpr int kSmem = kOffSlot + 16 + 1024;  // + slack to align the base to 1 KB

struct Bars {
  uint32_t base;
  __device__ __forceinline__ uint32_t q_full() const { return base; }
  __device__ __forceinline__ uint32_t k_full(int s) const { return base + 8u * (1 + s); }
  __device__ __forceinline__ uint32_t k_empty(int s) const { return base + 8u * (1 + kStages + s); }
  __device__ __forceinline__ uint32_t v_full(int s) const { return base + 8u * (1 + 2 * kStages + s); }
  __device__ __forceinline__ uint32_t v_empty(int s) const { return base + 8u * (1 + 3 * kStages + s); }
  __device__ __forceinline__ uint32_t s_full(int b) const { return base + 8u * (1 + 4 * kStages + b); }
  __device__ __forceinline__ uint32_t p_full(int b) const { return base + 8u * (3 + 4 * kStages + b); }
  __device__ __forceinline__ uint32_t pv_done() const { return base + 8u * (5 + 4 * kStages); }
  __device__ __forceinline__ uint32_t drain() const { return base + 8u * (6 + 4 * kStages); }
  // after the last PV only: the epilogue cannot use pv_done's parity, because when the last
  // S is ready PV(n - 2) may still be running (S(j) is issued behind PV(j - 2), not PV(j - 1))
  __device__ __forceinline__ uint32_t o_done() const { return base + 8u * (7 + 4 * kStages); }
};

// CTA -> (sequence b, row tile z, q head h): sequence by sequence, within a sequence the
// deepest row tiles first (under a causal mask they see the most keys), heads fastest so
// that the CTAs of one GQA group run together.  The CTAs resident at any time then read the
// K / V of one or two sequences, which stay in L2 while every row tile of those sequences
// reads them; the hardware hands out CTAs in this order as SMs free up, which keeps the
// load balanced.  False for a row tile the sequence does not have.
__device__ __forceinline__ bool item_of(const FwdArgs& a, int zmax, int& z, int& b, int& h) {
  const long long id = blockIdx.x;
  const long long per_seq = (long long)zmax * a.hq;
  b = (int)(id / per_seq);
  const int rem = (int)(id - (long long)b * per_seq);
  const int zr = rem / a.hq;
  z = zmax - 1 - zr;
  h = rem - zr * a.hq;
  return (long long)z * kBM < (long long)(a.cu_q[b + 1] - a.cu_q[b]);
}

template <typename T, bool DROP>
__global__ void __launch_bounds__(kThreads, 1)
fwd_d256_sm100_kernel(const FwdArgs a, int zmax, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v) {
  extern __shared__ unsigned char smem_raw[];
  int z, b, h;
  if (!item_of(a, zmax, z, b, h)) return;   // before taking any resource
  const int q0 = a.cu_q[b], sq = a.cu_q[b + 1] - q0;
  const int k0 = a.cu_k[b], sk = a.cu_k[b + 1] - k0;
  const int m0 = z * kBM;
  const int nrows = (sq - m0 < kBM) ? sq - m0 : kBM;
  const int g = h / (a.hq / a.hkv);
  long long l1, h1, l2, h2;
  row_key_range(m0, sq, sk, a.left, a.right, l1, h1);
  row_key_range(m0 + nrows - 1, sq, sk, a.left, a.right, l2, h2);
  int lo = (int)l1;
  const int hi = (int)(h2 < l1 ? l1 : h2);   // ranges move right with the row: the union
  if (DROP && hi > lo) lo &= ~15;            // dropout draws keep bytes for 16-key blocks
  const int n = hi > lo ? (hi - lo + kBN - 1) / kBN : 0;

  const uint32_t base_u32 = (smem_addr(smem_raw) + 1023u) & ~1023u;
  unsigned char* smem = smem_raw + (base_u32 - smem_addr(smem_raw));
  const uint32_t sK = base_u32 + kOffK, sV = base_u32 + kOffV;
  const Bars bar{base_u32 + kOffBar};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffSlot);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(bar.q_full(), 4);   // one arrival per softmax warp, after its Q rows are in TMEM
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar.k_full(s), 1);
      mbar_init(bar.k_empty(s), 1);
      mbar_init(bar.v_full(s), 1);
      mbar_init(bar.v_empty(s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar.s_full(s), 1);
      mbar_init(bar.p_full(s), 4);
    }
    mbar_init(bar.pv_done(), 1);
    mbar_init(bar.drain(), 1);
    mbar_init(bar.o_done(), 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ================================ TMA producer ======================================
    if (lane == 0 && n > 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      int nk = 0, nv = 0;   // tiles whose K / V loads were issued
      for (int j = 0; j < n; ++j) {
        const int st = j % kStages;
        const uint32_t par = ((j / kStages) & 1) ^ 1;
        const int row = k0 + lo + j * kBN;
        if (!mbar_wait(bar.k_empty(st), par, a.status)) break;
        mbar_arrive_expect_tx(bar.k_full(st), kTileBytes);
        for (int hf = 0; hf < D / 64; ++hf)
          tma_load_3d(sK + st * kTileBytes + hf * kBox, &tm_k, bar.k_full(st), hf * 64, g, row);
        nk = j + 1;
        if (!mbar_wait(bar.v_empty(st), par, a.status)) break;
        mbar_arrive_expect_tx(bar.v_full(st), kTileBytes);
        for (int hf = 0; hf < D / 64; ++hf)
          tma_load_3d(sV + st * kTileBytes + hf * kBox, &tm_v, bar.v_full(st), hf * 64, g, row);
        nv = j + 1;
      }
      // make sure no copy is still landing in shared memory when the CTA exits
      for (int p = nk - kStages < 0 ? 0 : nk - kStages; p < nk; ++p)
        mbar_wait(bar.k_full(p % kStages), (p / kStages) & 1, a.status);
      for (int p = nv - kStages < 0 ? 0 : nv - kStages; p < nv; ++p)
        mbar_wait(bar.v_full(p % kStages), (p / kStages) & 1, a.status);
    }
  } else if (warp == 1) {
    // ================================ MMA issuer =========================================
    // The whole warp runs the issue loop in step; elect.sync picks the issuing lane.
    if (n > 0) {
      constexpr uint32_t idesc_s = idesc_of<T>(kBM, kBN, 0, 0);   // Q (TMEM) x K (K-major)
      constexpr uint32_t idesc_pv = idesc_of<T>(kBM, D, 0, 1);    // P (TMEM) x V (MN-major)
      // Shared-memory descriptors, built once; an address offset adds to the start field.
      const uint64_t dK0 = smem_desc(sK, 16, 1024, kLayoutSwizzle128B);
      const uint64_t dV0 = smem_desc(sV, kBox, 1024, kLayoutSwizzle128B);   // LBO: next 64 columns
      // S(j) = Q K_j^T into buffer j % 2, then K_j's stage is free
      auto issue_s = [&](int j) -> bool {
        const int st = j % kStages;
        if (!mbar_wait_warp(bar.k_full(st), (j / kStages) & 1, a.status)) return false;
        tc_fence_after();
        const uint64_t dk = dK0 + (uint64_t)((st * kTileBytes) >> 4);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t off16 = ((ks >> 2) * kBox + (ks & 3) * 32) >> 4;
          mma_ts_elect(tmem + col_S(j & 1), tmem + kColQ + ks * 8, dk + off16, idesc_s, ks > 0 ? 1u : 0u);
        }
        mma_commit_elect(bar.s_full(j & 1));
        mma_commit_elect(bar.k_empty(st));
        return true;
      };
      bool ok = mbar_wait_warp(bar.q_full(), 0, a.status);
      tc_fence_after();
      if (ok) ok = issue_s(0);
      if (ok && n > 1) ok = issue_s(1);
      for (int j = 0; j < n && ok; ++j) {
        const int st = j % kStages;
        if (!(ok = mbar_wait_warp(bar.p_full(j & 1), (j >> 1) & 1, a.status))) break;
        if (!(ok = mbar_wait_warp(bar.v_full(st), (j / kStages) & 1, a.status))) break;
        tc_fence_after();
        const uint64_t dv = dV0 + (uint64_t)((st * kTileBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk)
          mma_ts_elect(tmem + kColO, tmem + col_S(j & 1) + kk * 8, dv + (uint64_t)((kk * 2048) >> 4), idesc_pv,
                 (j > 0 || kk > 0) ? 1u : 0u);
        mma_commit_elect(bar.pv_done());
        mma_commit_elect(bar.v_empty(st));
        if (j + 2 < n) ok = issue_s(j + 2);
      }
      if (ok) mma_commit_elect(bar.o_done());
      // every MMA must be complete before the TMEM is freed
      mma_commit_elect(bar.drain());
      mbar_wait_warp(bar.drain(), 0, a.status);
    }
  } else if (warp >= 4) {
    // ================================ softmax warps ======================================
    const int lg = warp & 3;                      // TMEM lane quarter this warp may access
    const int r = lg * 32 + lane;
    const uint32_t lane_off = (uint32_t)(lg * 32) << 16;
    const int i = m0 + r;
    const bool row_ok = i < sq;
    // Q row i into TMEM columns [0, 128) as packed pairs (zeros past the sequence end); all
    // 32 loads of the row are issued before the first store (one memory round trip)
    {
      const uint4* qrow = reinterpret_cast<const uint4*>(static_cast<const T*>(a.q) +
                                                         ((long long)(q0 + (row_ok ? i : 0)) * a.hq + h) * D);
      uint32_t w[4][32];
#pragma unroll
      for (int v = 0; v < 32; ++v) {
        const uint4 x = row_ok ? qrow[v] : make_uint4(0u, 0u, 0u, 0u);
        w[v >> 3][4 * (v & 7)] = x.x;
        w[v >> 3][4 * (v & 7) + 1] = x.y;
        w[v >> 3][4 * (v & 7) + 2] = x.z;
        w[v >> 3][4 * (v & 7) + 3] = x.w;
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_st32(tmem + lane_off + kColQ + c * 32, w[c]);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar.q_full());
    }
    // this row's visible keys relative to the first key of the loop: [rlo, rhi)
    int rlo = 0, rhi = 0;
    if (row_ok) {
      long long l_, h_;
      row_key_range(i, sq, sk, a.left, a.right, l_, h_);
      rlo = (int)(l_ - lo);
      rhi = (int)(h_ - lo);
    }
    const float scale2 = a.scale * kLog2e;
    float m = a.sink ? a.sink[h] * kLog2e : kNegInf, l = 0.f;
    const uint32_t t4 = (a.drop.threshold - 1u) * 0x01010101u, t4h = t4 | 0x80808080u;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      if (!__all_sync(0xffffffffu, mbar_wait(bar.s_full(j & 1), (j >> 1) & 1, a.status))) { ok = false; break; }
      tc_fence_after();
      const uint32_t tS = tmem + lane_off + col_S(j & 1);
      uint32_t sr[kBN];
      tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      tmem_wait_ld();
      const int klo = rlo - j * kBN, khi = rhi - j * kBN;   // visible columns [klo, khi)
      if (!(klo <= 0 && khi >= kBN)) {
#pragma unroll
        for (int c = 0; c < kBN; ++c)
          if (c < klo || c >= khi) sr[c] = __float_as_uint(kNegInf);
      }
      // row max over 8 independent chains of three-input maxima
      float mxv[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) mxv[e] = fmaxf(__uint_as_float(sr[e]), __uint_as_float(sr[8 + e]));
#pragma unroll
      for (int c = 16; c < kBN; c += 16)
#pragma unroll
        for (int e = 0; e < 8; ++e) mxv[e] = fmax3(mxv[e], __uint_as_float(sr[c + e]), __uint_as_float(sr[c + 8 + e]));
      const float mx = fmax3(fmax3(mxv[0], mxv[1], mxv[2]), fmax3(mxv[3], mxv[4], mxv[5]), fmaxf(mxv[6], mxv[7]));
      const float m_tile = mx * scale2;
      const bool need = m_tile > m + kRescaleThreshold;
      float alpha = 1.f;
      if (need) {
        alpha = (m == kNegInf) ? 0.f : ex2(m - m_tile);
        m = m_tile;
      }
      const bool any_rescale = __any_sync(0xffffffffu, need);
      // P = 2^{S scale log2e - m}, packed over S's first 32 columns; masked scores are -inf
      // (2^-inf = +0); m = -inf only when every score is -inf (neg_m = 0 then avoids NaN)
      const float neg_m = (m == kNegInf) ? 0.f : -m;
      const float2 sc2 = make_float2(scale2, scale2), nm2 = make_float2(neg_m, neg_m);
      float2 sv[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
      // dropout: drop flags of the tile's four 16-key blocks; the row sum keeps every
      // probability, the P V operand only the kept ones (256 / T is applied to the output)
      uint32_t fl[DROP ? 16 : 1];
      if constexpr (DROP) {
        const uint32_t kb0 = (uint32_t)(lo + j * kBN) >> 4;
#pragma unroll
        for (int gq = 0; gq < 4; ++gq) {
          const uint4 w = dropout_bytes(a.drop, kb0 + gq, (uint32_t)(q0 + i), (uint32_t)h);
          fl[4 * gq] = drop_flags4(w.x, t4, t4h);
          fl[4 * gq + 1] = drop_flags4(w.y, t4, t4h);
          fl[4 * gq + 2] = drop_flags4(w.z, t4, t4h);
          fl[4 * gq + 3] = drop_flags4(w.w, t4, t4h);
        }
      }
      uint32_t pk[kBN / 2];
#pragma unroll
      for (int c = 0; c < kBN / 2; ++c) {
        const float2 x = ffma2(make_float2(__uint_as_float(sr[2 * c]), __uint_as_float(sr[2 * c + 1])), sc2, nm2);
        const float2 pp = make_float2(ex2(x.x), ex2(x.y));
        sv[c & 1] = fadd2(sv[c & 1], pp);
        pk[c] = pack2<T>(pp.x, pp.y);
        if constexpr (DROP) {
          // keys 2c, 2c + 1 are bytes 0-1 (c even) or 2-3 (c odd) of flag word c / 2
          const uint32_t mask = (c & 1) ? prmt_sign<0xBBAA>(fl[c >> 1]) : prmt_sign<0x9988>(fl[c >> 1]);
          pk[c] &= ~mask;
        }
      }
      tmem_st32(tS, pk);
      l = l * alpha + ((sv[0].x + sv[0].y) + (sv[1].x + sv[1].y));
      if (any_rescale && j > 0) {
        // O holds sum of the earlier P V: wait for the last of those MMAs, then scale rows
        if (!__all_sync(0xffffffffu, mbar_wait(bar.pv_done(), (j - 1) & 1, a.status))) { ok = false; break; }
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tmem + lane_off + kColO + c * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(tmem + lane_off + kColO + c * 32, o);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar.p_full(j & 1));
    }
    // ---- epilogue: out = O / (l + 2^{sink2 - m}),  lse = (m + log2 l) ln 2 ----------------
    if (ok && n > 0) ok = __all_sync(0xffffffffu, mbar_wait(bar.o_done(), 0, a.status));
    if (ok) {
      tc_fence_after();
      const float sink2 = a.sink ? a.sink[h] * kLog2e : kNegInf;
      const float e_sink = (sink2 == kNegInf || m == kNegInf) ? 0.f : ex2(sink2 - m);
      const float den = l + e_sink;
      // with dropout, O summed the kept probabilities unscaled: the 256 / T factor goes here
      const float inv = den > 0.f ? (DROP ? a.drop.scale : 1.f) / den : 0.f;
      uint4* orow = reinterpret_cast<uint4*>(static_cast<T*>(a.out) + ((long long)(q0 + i) * a.hq + h) * D);
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        if (n > 0) {
          tmem_ld32(tmem + lane_off + kColO + c * 32, o);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = 0u;
        }
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[e] = pack2<T>(__uint_as_float(o[2 * e]) * inv, __uint_as_float(o[2 * e + 1]) * inv);
        const long long ob = ((long long)(q0 + i) * a.hq + h) * D + c * 32;
        if (row_ok && store_ok(ob, ob + 31, (long long)a.total_q * a.hq * D, a.status)) {
#pragma unroll
          for (int v = 0; v < 4; ++v) orow[c * 4 + v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
        }
      }
      // lse is [Hq, total_q]: the row itself must lie inside total_q
      if (row_ok && a.lse && store_ok((long long)q0 + i, (long long)q0 + i, a.total_q, a.status))
        a.lse[(long long)h * a.total_q + q0 + i] = l > 0.f ? (m + __log2f(l)) * kLn2 : kNegInf;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---- host ----------------------------------------------------------------------------------

long long grid_of(const FwdArgs& a) {
  const long long zmax = (a.max_sq + kBM - 1) / kBM;
  return zmax * a.batch * a.hq;
}

template <typename T>
cudaError_t launch_typed(const FwdArgs& a, cudaStream_t s) {
  const int zmax = (a.max_sq + kBM - 1) / kBM;
  if (zmax <= 0) return cudaSuccess;
  constexpr CUtensorMapDataType dt = tma_dtype<T>();
  CUtensorMap tk, tv;
  if (!make_map_3d(&tk, a.k, D, a.hkv, a.total_k, kBN, dt) || !make_map_3d(&tv, a.v, D, a.hkv, a.total_k, kBN, dt))
    return cudaErrorInvalidValue;
  auto kernel = a.drop.threshold ? fwd_d256_sm100_kernel<T, true> : fwd_d256_sm100_kernel<T, false>;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (e != cudaSuccess) return e;
  kernel<<<(unsigned)grid_of(a), kThreads, kSmem, s>>>(a, zmax, tk, tv);
  return cudaGetLastError();
}

}  // namespace

bool fwd_d256_sm100_supported(const FwdArgs& a, int dtype) {
  if ((dtype != 0 && dtype != 2) || a.cu_q == nullptr) return false;
  if (a.dk != D || a.dv != D) return false;
  if (grid_of(a) > 0x7fffffffLL) return false;   // 1-D grid
  return encode_fn() != nullptr;
}

cudaError_t launch_fwd_d256_sm100(const FwdArgs& a, int dtype, cudaStream_t s) {
  return dtype == 2 ? launch_typed<__half>(a, s) : launch_typed<__nv_bfloat16>(a, s);
}

}  // namespace attn_sink
