// Sink-attention backward at head dim 256 on the sm_100a tensor cores (bf16 or fp16 in, fp32
// accumulation), after the preprocess pass (D = dout . out, lse_tot = logaddexp(lse, sink),
// dsink).  Gradient of the loss sum(dout * out) (slime learnable_softmax_attention.py,
// class docstring and ``backward``; the forward of CANN flash_attn doc, "Function"):
//   P = e^{S scale - lse_tot},  dP = dout V^T,  dS = P (dP - D),
//   dq = scale dS K,  dk = scale dS^T Q,  dv = P^T dout.
//
// At d = 256 the fp32 dK and dV accumulators of one 128-key tile fill all 512 TMEM columns,
// so the gradient is computed by three kernels, each holding its stationary operand in TMEM
// as the A operand of the score MMAs (128 columns of packed 16-bit pairs, copied there by the
// compute warps) and streaming the other side through a shared-memory ring:
//   dQ  query-stationary (128 queries of one q head); TMEM Q [0,128) S [128,192)
//       dP [192,256) dQ [256,512); per 64-key tile: S = Q K^T (TS), dP = dout V^T (SS),
//       dS over S's columns, dQ += dS K (TS, K read N-major).
//   dV  key-stationary (128 keys of one kv head, every q head of its group); TMEM K [0,128)
//       S^T buffers [128,192) and [192,256), dV [256,512); per 64-query tile:
//       S^T = K Q^T (TS), P^T over S^T's columns, dV += P^T dout (TS); S^T(t+2) is issued
//       behind dV(t), so the exponentials of tile t+1 overlap the tensor pipe.
//   dK  key-stationary; V whole in shared memory; TMEM K [0,128) S^T [128,192)
//       dP^T [192,256) dK [256,512); per 64-query tile: S^T = K Q^T (TS),
//       dP^T = V dout^T (SS), dS^T over S^T's columns, dK += dS^T Q (TS).
// None of them needs atomics, so the result is the same bits on every run.  Warps: 0 TMA
// producer, 1 TMEM allocation and MMA issuer (the warp in step, one elected lane issuing),
// 2-3 idle, 4-7 compute (thread t =
// stationary row t = TMEM lane t).  Every mbarrier wait is bounded; a timeout sets the status
// word and the CTA drains and frees its TMEM instead of hanging.  Named barriers (the per-tile
// lse_tot / D staging of the key-stationary kernels) are passed by every compute warp in
// every iteration, also after a timed-out wait.
#include <cuda.h>

#include <type_traits>

#include "sm100_ptx.cuh"
#include "tma_map.h"

namespace attn_sink {
namespace {

using namespace sm100;

constexpr int D = 256;
constexpr int kThreads = 256;
constexpr uint32_t kTmemCols = 512;
constexpr int kBox64 = 64 * 128;     // TMA box of 64 rows x 64 columns (128 bytes)
constexpr int kBox128 = 128 * 128;   // TMA box of 128 rows x 64 columns
constexpr int kTile64 = 4 * kBox64;  // 64 rows x 256 columns: 32 KB
constexpr int kTile128 = 4 * kBox128;

// K-major operand of 64 / 128-row boxes: offset of k-step ks (16 columns) in 16-byte units
__device__ __forceinline__ uint64_t kmaj_off(int ks, int box) { return (uint64_t)(((ks >> 2) * box + (ks & 3) * 32) >> 4); }

// The calling thread's 256-element row into TMEM columns [col, col + 128) of its lane as
// packed pairs (zeros when !ok), then this warp's arrival on `bar`.  All 32 loads are issued
// before the first store (one memory round trip).
template <typename T>
__device__ __forceinline__ void stage_row(const T* row, bool ok, uint32_t taddr, uint32_t bar, int lane) {
  const uint4* src = reinterpret_cast<const uint4*>(row);
  uint32_t w[4][32];
#pragma unroll
  for (int v = 0; v < 32; ++v) {
    const uint4 x = ok ? src[v] : make_uint4(0u, 0u, 0u, 0u);
    w[v >> 3][4 * (v & 7)] = x.x;
    w[v >> 3][4 * (v & 7) + 1] = x.y;
    w[v >> 3][4 * (v & 7) + 2] = x.z;
    w[v >> 3][4 * (v & 7) + 3] = x.w;
  }
#pragma unroll
  for (int c = 0; c < 4; ++c) tmem_st32(taddr + c * 32, w[c]);
  tmem_wait_st();
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(bar);
}

// The calling thread's fp32 TMEM row [col, col + 256) times `mul`, rounded, to global memory.
template <typename T>
__device__ __forceinline__ void store_row(uint32_t taddr, bool have, float mul, T* dst, bool ok) {
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll 1
  for (int c = 0; c < D / 32; ++c) {
    uint32_t v[32];
    if (have) {
      tmem_ld32(taddr + c * 32, v);
      tmem_wait_ld();
    }
    uint32_t pk[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const float x0 = have ? __uint_as_float(v[2 * e]) * mul : 0.f;
      const float x1 = have ? __uint_as_float(v[2 * e + 1]) * mul : 0.f;
      pk[e] = pack2<T>(x0, x1);
    }
    if (ok) {
#pragma unroll
      for (int u = 0; u < 4; ++u) d4[c * 4 + u] = make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
    }
  }
}

__device__ __forceinline__ void named_bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// ============================================================================================
// dQ: query-stationary
// ============================================================================================
namespace dq {
constexpr int kBM = 128, kBN = 64, kStages = 2;
constexpr int kOffO = 0;                            // dout tile, 4 boxes of 128 rows
constexpr int kOffK = kOffO + kTile128;             // K ring
constexpr int kOffV = kOffK + kStages * kTile64;    // V ring
constexpr int kOffBar = kOffV + kStages * kTile64;
constexpr int kNumBars = 2 + 2 * kStages + 5;       // o_full, q_full, kv_full[S], kv_empty[S], sdp_full, ds_full, dq_done, drain
constexpr int kOffSlot = kOffBar + kNumBars * 8;
constexpr int kSmem = kOffSlot + 16 + 1024;
constexpr uint32_t kColQ = 0, kColS = 128, kColP = 192, kColDQ = 256;
struct Bars {
  uint32_t base;
  __device__ __forceinline__ uint32_t o_full() const { return base; }
  __device__ __forceinline__ uint32_t q_full() const { return base + 8u; }
  __device__ __forceinline__ uint32_t kv_full(int s) const { return base + 8u * (2 + s); }
  __device__ __forceinline__ uint32_t kv_empty(int s) const { return base + 8u * (2 + kStages + s); }
  __device__ __forceinline__ uint32_t sdp_full() const { return base + 8u * (2 + 2 * kStages); }
  __device__ __forceinline__ uint32_t ds_full() const { return base + 8u * (3 + 2 * kStages); }
  __device__ __forceinline__ uint32_t dq_done() const { return base + 8u * (4 + 2 * kStages); }
  __device__ __forceinline__ uint32_t drain() const { return base + 8u * (5 + 2 * kStages); }
};
}  // namespace dq

template <typename T, bool DROP>
__global__ void __launch_bounds__(kThreads, 1)
bwd_dq_d256_kernel(const BwdArgs a, int mtiles, int band, const __grid_constant__ CUtensorMap tm_o,
                   const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v) {
  using namespace dq;
  extern __shared__ unsigned char smem_raw[];
  // CTA -> (row tile, sequence, q head), in bands of `band` (sequence, kv head) groups whose
  // K / V fit in L2 together; within a band the deepest row tiles first, then the groups and
  // their q heads
  const int group = a.hq / a.hkv, G = a.batch * a.hkv;
  const long long per_band = (long long)band * group * mtiles;
  const int bi = (int)(blockIdx.x / per_band);
  const int first = bi * band, members = (G - first < band) ? G - first : band;
  const long long rem = blockIdx.x - (long long)bi * per_band;
  const int zr = (int)(rem / ((long long)members * group));
  const int r2 = (int)(rem - (long long)zr * members * group);
  const int grp = first + r2 / group;
  const int m = mtiles - 1 - zr, b = grp / a.hkv;
  const int h = (grp - b * a.hkv) * group + r2 % group;
  const int q0 = a.cu_q[b], sq = a.cu_q[b + 1] - q0;
  const int k0 = a.cu_k[b], sk = a.cu_k[b + 1] - k0;
  const int m0 = m * kBM;
  if (m0 >= sq) return;
  const int g = h / (a.hq / a.hkv);
  const int nrows = (sq - m0 < kBM) ? sq - m0 : kBM;
  long long l1, h1, l2, h2;
  row_key_range(m0, sq, sk, a.left, a.right, l1, h1);
  row_key_range(m0 + nrows - 1, sq, sk, a.left, a.right, l2, h2);
  int lo = (int)l1;
  const int hi = (int)(h2 < l1 ? l1 : h2);
  if (DROP && hi > lo) lo &= ~15;   // dropout draws keep bytes for 16-key blocks
  const int n = hi > lo ? (hi - lo + kBN - 1) / kBN : 0;

  const uint32_t base_u32 = (smem_addr(smem_raw) + 1023u) & ~1023u;
  unsigned char* smem = smem_raw + (base_u32 - smem_addr(smem_raw));
  const uint32_t sO = base_u32 + kOffO, sK = base_u32 + kOffK, sV = base_u32 + kOffV;
  const Bars bar{base_u32 + kOffBar};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffSlot);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(bar.o_full(), 1);
    mbar_init(bar.q_full(), 4);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar.kv_full(s), 1);
      mbar_init(bar.kv_empty(s), 1);
    }
    mbar_init(bar.sdp_full(), 1);
    mbar_init(bar.ds_full(), 4);
    mbar_init(bar.dq_done(), 1);
    mbar_init(bar.drain(), 1);
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
    if (lane == 0 && n > 0) {
      tma_prefetch_desc(&tm_o);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      mbar_arrive_expect_tx(bar.o_full(), kTile128);
      for (int hf = 0; hf < 4; ++hf) tma_load_3d(sO + hf * kBox128, &tm_o, bar.o_full(), hf * 64, h, q0 + m0);
      int issued = 0;
      for (int j = 0; j < n; ++j) {
        const int st = j % kStages;
        if (!mbar_wait(bar.kv_empty(st), ((j / kStages) & 1) ^ 1, a.status)) break;
        const int row = k0 + lo + j * kBN;
        mbar_arrive_expect_tx(bar.kv_full(st), 2 * kTile64);
        for (int hf = 0; hf < 4; ++hf) {
          tma_load_3d(sK + st * kTile64 + hf * kBox64, &tm_k, bar.kv_full(st), hf * 64, g, row);
          tma_load_3d(sV + st * kTile64 + hf * kBox64, &tm_v, bar.kv_full(st), hf * 64, g, row);
        }
        issued = j + 1;
      }
      mbar_wait(bar.o_full(), 0, a.status);
      for (int p = issued - kStages < 0 ? 0 : issued - kStages; p < issued; ++p)
        mbar_wait(bar.kv_full(p % kStages), (p / kStages) & 1, a.status);
    }
  } else if (warp == 1) {
    // The whole warp runs the issue loop in step; elect.sync picks the issuing lane.
    if (n > 0) {
      constexpr uint32_t id_s = idesc_of<T>(kBM, kBN, 0, 0);   // S, dP: K-major B
      constexpr uint32_t id_q = idesc_of<T>(kBM, D, 0, 1);     // dS (TMEM) x K (N-major)
      const uint64_t kO = smem_desc(sO, 16, 1024, kLayoutSwizzle128B);
      const uint64_t kK = smem_desc(sK, 16, 1024, kLayoutSwizzle128B);
      const uint64_t mK = smem_desc(sK, kBox64, 1024, kLayoutSwizzle128B);
      const uint64_t kV = smem_desc(sV, 16, 1024, kLayoutSwizzle128B);
      bool ok = mbar_wait_warp(bar.q_full(), 0, a.status) && mbar_wait_warp(bar.o_full(), 0, a.status);
      for (int j = 0; j < n && ok; ++j) {
        const int st = j % kStages;
        if (!(ok = mbar_wait_warp(bar.kv_full(st), (j / kStages) & 1, a.status))) break;
        tc_fence_after();
        const uint64_t so = (uint64_t)((st * kTile64) >> 4);
        // S = Q K^T (A = Q from TMEM); dS(j - 1) in S's columns was read by dQ(j - 1), issued
        // earlier by this thread
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks)
          mma_ts_elect(tmem + kColS, tmem + kColQ + ks * 8, kK + so + kmaj_off(ks, kBox64), id_s, ks > 0 ? 1u : 0u);
        // dP = dout V^T
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks)
          mma_ss_elect(tmem + kColP, kO + kmaj_off(ks, kBox128), kV + so + kmaj_off(ks, kBox64), id_s, ks > 0 ? 1u : 0u);
        mma_commit_elect(bar.sdp_full());
        if (!(ok = mbar_wait_warp(bar.ds_full(), j & 1, a.status))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk)
          mma_ts_elect(tmem + kColDQ, tmem + kColS + kk * 8, mK + so + (uint64_t)((kk * 2048) >> 4), id_q,
                 (j > 0 || kk > 0) ? 1u : 0u);
        mma_commit_elect(bar.kv_empty(st));
      }
      if (ok) mma_commit_elect(bar.dq_done());
      mma_commit_elect(bar.drain());
      mbar_wait_warp(bar.drain(), 0, a.status);
    }
  } else if (warp >= 4) {
    const int lg = warp & 3;
    const int r = lg * 32 + lane;
    const uint32_t lane_off = (uint32_t)(lg * 32) << 16;
    const int i = m0 + r;
    const bool row_ok = i < sq;
    stage_row(static_cast<const T*>(a.q) + ((long long)(q0 + (row_ok ? i : 0)) * a.hq + h) * D, row_ok,
              tmem + lane_off + kColQ, bar.q_full(), lane);
    int rlo = 0, rhi = 0;
    float neg_lt = 0.f, Dr = 0.f;
    if (row_ok) {
      long long l_, h_;
      row_key_range(i, sq, sk, a.left, a.right, l_, h_);
      rlo = (int)(l_ - lo);
      rhi = (int)(h_ - lo);
      const long long idx = (long long)h * a.total_q + q0 + i;
      const float lt2 = a.lse_tot[idx] * kLog2e;
      neg_lt = (lt2 == kNegInf) ? 0.f : -lt2;   // no key and no sink: every score is -inf, P = 0
      Dr = a.D[idx];
    }
    const float scale2 = a.scale * kLog2e;
    const uint32_t t4 = (a.drop.threshold - 1u) * 0x01010101u, t4h = t4 | 0x80808080u;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      // dropout: drop flags of this row's 64 keys of the tile (4 Philox calls, drawn before
      // the wait so that they overlap the tensor pipe); dS = P (Z dP - D)
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
      if (!__all_sync(0xffffffffu, mbar_wait(bar.sdp_full(), j & 1, a.status))) { ok = false; break; }
      tc_fence_after();
      const int klo = rlo - j * kBN, khi = rhi - j * kBN;   // visible columns [klo, khi)
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t sv[32], pv[32];
        tmem_ld32(tmem + lane_off + kColS + c * 32, sv);
        tmem_ld32(tmem + lane_off + kColP + c * 32, pv);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int c0 = c * 32 + 2 * e;
          const float s0 = (c0 >= klo && c0 < khi) ? __uint_as_float(sv[2 * e]) : kNegInf;
          const float s1 = (c0 + 1 >= klo && c0 + 1 < khi) ? __uint_as_float(sv[2 * e + 1]) : kNegInf;
          const float p0 = ex2(fmaf(s0, scale2, neg_lt)), p1 = ex2(fmaf(s1, scale2, neg_lt));
          if constexpr (DROP) {
            // keys c0, c0 + 1: bytes 0-1 (e even) or 2-3 (e odd) of flag word c0 / 4
            const uint32_t w = fl[c0 >> 2];
            const uint32_t d0 = (e & 1) ? prmt_sign<0xAAAA>(w) : prmt_sign<0x8888>(w);
            const uint32_t d1 = (e & 1) ? prmt_sign<0xBBBB>(w) : prmt_sign<0x9999>(w);
            pk[e] = pack2<T>(p0 * fmaf(__uint_as_float(pv[2 * e] & ~d0), a.drop.scale, -Dr),
                             p1 * fmaf(__uint_as_float(pv[2 * e + 1] & ~d1), a.drop.scale, -Dr));
          } else {
            pk[e] = pack2<T>(p0 * (__uint_as_float(pv[2 * e]) - Dr), p1 * (__uint_as_float(pv[2 * e + 1]) - Dr));
          }
        }
        // dS of keys [32 c, 32 c + 32) over S columns [16 c, 16 c + 16), already read
        tmem_st16(tmem + lane_off + kColS + c * 16, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar.ds_full());
    }
    bool have = ok && n > 0;
    if (have) have = __all_sync(0xffffffffu, mbar_wait(bar.dq_done(), 0, a.status));
    tc_fence_after();
    if (ok)
      store_row<T>(tmem + lane_off + kColDQ, have, a.scale,
                   static_cast<T*>(a.grad_q) + ((long long)(q0 + i) * a.hq + h) * D,
                   row_ok && store_ok(((long long)(q0 + i) * a.hq + h) * D, ((long long)(q0 + i) * a.hq + h) * D + D - 1,
                                      (long long)a.total_q * a.hq * D, a.status));
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ============================================================================================
// dK and dV: key-stationary
// ============================================================================================
namespace ks {
constexpr int kBN = 128;   // keys per CTA
constexpr int kBM = 64;    // queries per tile
// CTA -> (key tile, sequence, kv head).  Under a bottom-right causal mask the first key tiles
// are seen by the most queries, so they go first.
// In bands of `band` (sequence, kv head) groups whose Q / dout fit in L2 together; within a
// band key tiles in increasing order, then the groups.
struct Tile {
  int b, g, q0, sq, k0, sk, n0, nkeys, qlo, n_m, T;
};
__device__ __forceinline__ bool tile_of(const BwdArgs& a, int ntiles, int band, Tile& t) {
  const int G = a.batch * a.hkv;
  const long long per_band = (long long)band * ntiles;
  const int bi = (int)(blockIdx.x / per_band);
  const int first = bi * band, members = (G - first < band) ? G - first : band;
  const long long rem = blockIdx.x - (long long)bi * per_band;
  const int nt = (int)(rem / members);
  const int grp = first + (int)(rem - (long long)nt * members);
  t.b = grp / a.hkv;
  t.g = grp - t.b * a.hkv;
  t.q0 = a.cu_q[t.b];
  t.sq = a.cu_q[t.b + 1] - t.q0;
  t.k0 = a.cu_k[t.b];
  t.sk = a.cu_k[t.b + 1] - t.k0;
  t.n0 = nt * kBN;
  if (t.n0 >= t.sk) return false;
  t.nkeys = (t.sk - t.n0 < kBN) ? t.sk - t.n0 : kBN;
  long long ql, qh, ql1, qh1;
  key_query_range(t.n0, t.sq, t.sk, a.left, a.right, ql, qh);
  key_query_range(t.n0 + t.nkeys - 1, t.sq, t.sk, a.left, a.right, ql1, qh1);
  t.qlo = (int)ql;
  const int qhi = (int)qh1;   // query ranges move right with the key: the union
  t.n_m = qhi > t.qlo ? (qhi - t.qlo + kBM - 1) / kBM : 0;
  t.T = t.n_m * (a.hq / a.hkv);
  return true;
}
// Dropout in the key-stationary kernels: warps 2-3 draw each 64-query tile's flags
// (draw_flags64) into stage t % 2 of a two-stage buffer, and they meet the compute warps on named
// barrier 3 + t % 2 once per tile (64 + 128 threads).  The producer passes the barrier of tile
// t - 1 only after the compute warps are done with tile t - 2, whose stage tile t reuses.
}  // namespace ks

// ---- dV --------------------------------------------------------------------------------------
namespace dvk {
constexpr int kStages = 3;
constexpr int kOffQ = 0;                           // Q ring
constexpr int kOffO = kOffQ + kStages * kTile64;   // dout ring
constexpr int kOffLT = kOffO + kStages * kTile64;  // -lse_tot log2e of the tile's queries [2][64]
constexpr int kOffZ = kOffLT + 2 * 64 * 4;         // dropout flags, 2 stages
constexpr int kOffBar = kOffZ + 2 * kFlagBytes64;
constexpr int kNumBars = 1 + 2 * kStages + 6;      // k_full, qd_full[S], qd_empty[S], s_full[2], p_full[2], dv_done, drain
constexpr int kOffSlot = kOffBar + kNumBars * 8;
constexpr int kSmem = kOffSlot + 16 + 1024;
constexpr uint32_t kColK = 0, kColDV = 256;
__host__ __device__ constexpr uint32_t col_S(int b) { return 128u + 64u * (uint32_t)b; }
struct Bars {
  uint32_t base;
  __device__ __forceinline__ uint32_t k_full() const { return base; }
  __device__ __forceinline__ uint32_t qd_full(int s) const { return base + 8u * (1 + s); }
  __device__ __forceinline__ uint32_t qd_empty(int s) const { return base + 8u * (1 + kStages + s); }
  __device__ __forceinline__ uint32_t s_full(int b) const { return base + 8u * (1 + 2 * kStages + b); }
  __device__ __forceinline__ uint32_t p_full(int b) const { return base + 8u * (3 + 2 * kStages + b); }
  __device__ __forceinline__ uint32_t dv_done() const { return base + 8u * (5 + 2 * kStages); }
  __device__ __forceinline__ uint32_t drain() const { return base + 8u * (6 + 2 * kStages); }
};
}  // namespace dvk

template <typename T, bool DROP>
__global__ void __launch_bounds__(kThreads, 1)
bwd_dv_d256_kernel(const BwdArgs a, int ntiles, int band, const __grid_constant__ CUtensorMap tm_q,
                   const __grid_constant__ CUtensorMap tm_o) {
  using namespace dvk;
  using ks::kBM;
  extern __shared__ unsigned char smem_raw[];
  ks::Tile tl;
  if (!ks::tile_of(a, ntiles, band, tl)) return;
  const int group = a.hq / a.hkv, T_ = tl.T;
  auto head_of = [&](int t) { return tl.g * group + t / tl.n_m; };
  auto qbase_of = [&](int t) { return tl.qlo + (t % tl.n_m) * kBM; };

  const uint32_t base_u32 = (smem_addr(smem_raw) + 1023u) & ~1023u;
  unsigned char* smem = smem_raw + (base_u32 - smem_addr(smem_raw));
  const uint32_t sQ = base_u32 + kOffQ, sO = base_u32 + kOffO;
  float* s_nlt = reinterpret_cast<float*>(smem + kOffLT);
  const uint32_t sZ = base_u32 + kOffZ;
  const Bars bar{base_u32 + kOffBar};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffSlot);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(bar.k_full(), 4);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar.qd_full(s), 1);
      mbar_init(bar.qd_empty(s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar.s_full(s), 1);
      mbar_init(bar.p_full(s), 4);
    }
    mbar_init(bar.dv_done(), 1);
    mbar_init(bar.drain(), 1);
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
    if (lane == 0 && T_ > 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_o);
      int issued = 0;
      for (int t = 0; t < T_; ++t) {
        const int st = t % kStages;
        if (!mbar_wait(bar.qd_empty(st), ((t / kStages) & 1) ^ 1, a.status)) break;
        const int h = head_of(t), row = tl.q0 + qbase_of(t);
        mbar_arrive_expect_tx(bar.qd_full(st), 2 * kTile64);
        for (int hf = 0; hf < 4; ++hf) {
          tma_load_3d(sQ + st * kTile64 + hf * kBox64, &tm_q, bar.qd_full(st), hf * 64, h, row);
          tma_load_3d(sO + st * kTile64 + hf * kBox64, &tm_o, bar.qd_full(st), hf * 64, h, row);
        }
        issued = t + 1;
      }
      for (int p = issued - kStages < 0 ? 0 : issued - kStages; p < issued; ++p)
        mbar_wait(bar.qd_full(p % kStages), (p / kStages) & 1, a.status);
    }
  } else if (warp == 1) {
    // The whole warp runs the issue loop in step; elect.sync picks the issuing lane.
    if (T_ > 0) {
      constexpr uint32_t id_s = idesc_of<T>(ks::kBN, kBM, 0, 0);   // K (TMEM) x Q (K-major)
      constexpr uint32_t id_v = idesc_of<T>(ks::kBN, D, 0, 1);     // P^T (TMEM) x dout (N-major)
      const uint64_t kQ = smem_desc(sQ, 16, 1024, kLayoutSwizzle128B);
      const uint64_t mO = smem_desc(sO, kBox64, 1024, kLayoutSwizzle128B);
      auto issue_s = [&](int t) -> bool {
        const int st = t % kStages;
        if (!mbar_wait_warp(bar.qd_full(st), (t / kStages) & 1, a.status)) return false;
        tc_fence_after();
        const uint64_t so = (uint64_t)((st * kTile64) >> 4);
#pragma unroll
        for (int k = 0; k < D / 16; ++k)
          mma_ts_elect(tmem + col_S(t & 1), tmem + kColK + k * 8, kQ + so + kmaj_off(k, kBox64), id_s, k > 0 ? 1u : 0u);
        mma_commit_elect(bar.s_full(t & 1));
        return true;
      };
      bool ok = mbar_wait_warp(bar.k_full(), 0, a.status);
      tc_fence_after();
      if (ok) ok = issue_s(0);
      if (ok && T_ > 1) ok = issue_s(1);
      for (int t = 0; t < T_ && ok; ++t) {
        const int st = t % kStages;
        if (!(ok = mbar_wait_warp(bar.p_full(t & 1), (t >> 1) & 1, a.status))) break;
        tc_fence_after();
        const uint64_t so = (uint64_t)((st * kTile64) >> 4);
#pragma unroll
        for (int kk = 0; kk < kBM / 16; ++kk)
          mma_ts_elect(tmem + kColDV, tmem + col_S(t & 1) + kk * 8, mO + so + (uint64_t)((kk * 2048) >> 4), id_v,
                 (t > 0 || kk > 0) ? 1u : 0u);
        mma_commit_elect(bar.qd_empty(st));
        if (t + 2 < T_) ok = issue_s(t + 2);
      }
      if (ok) mma_commit_elect(bar.dv_done());
      mma_commit_elect(bar.drain());
      mbar_wait_warp(bar.drain(), 0, a.status);
    }
  } else if (DROP && warp < 4) {
    // warps 2-3: the dropout flags of every tile, a tile ahead of the compute warps
    const int rt = (warp - 2) * 32 + lane;
    for (int t = 0; t < T_; ++t) {
      draw_flags64(a.drop, sZ + (t & 1) * kFlagBytes64, rt, tl.n0 >> 4, (long long)tl.q0 + qbase_of(t), head_of(t));
      named_bar_sync(3 + (t & 1), 192);
    }
  } else if (warp >= 4) {
    const int lg = warp & 3;
    const int r = lg * 32 + lane;
    const uint32_t lane_off = (uint32_t)(lg * 32) << 16;
    const int j = tl.n0 + r;
    const bool key_ok = j < tl.sk;
    stage_row(static_cast<const T*>(a.k) + ((long long)(tl.k0 + (key_ok ? j : 0)) * a.hkv + tl.g) * D, key_ok,
              tmem + lane_off + kColK, bar.k_full(), lane);
    long long qa_, qb_;
    key_query_range(j, tl.sq, tl.sk, a.left, a.right, qa_, qb_);
    const int jlo = key_ok ? (int)qa_ : 0, jhi = key_ok ? (int)qb_ : 0;   // queries that see key j
    const float scale2 = a.scale * kLog2e;
    // -lse_tot log2e of query r of tile t (threads r < 64), loaded a tile ahead
    auto fetch = [&](int t) -> float {
      const int i = qbase_of(t) + r;
      if (r >= kBM || i >= tl.sq) return 0.f;
      const float lt2 = a.lse_tot[(long long)head_of(t) * a.total_q + tl.q0 + i] * kLog2e;
      return lt2 == kNegInf ? 0.f : -lt2;
    };
    float pf = T_ > 0 ? fetch(0) : 0.f;
    bool ok = true;
    for (int t = 0; t < T_; ++t) {
      if (r < kBM) s_nlt[(t & 1) * kBM + r] = pf;
      named_bar_sync(1, 128);   // buffer t & 1 was last read in tile t - 2
      if (t + 1 < T_) pf = fetch(t + 1);
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar.s_full(t & 1), (t >> 1) & 1, a.status));
      if constexpr (DROP) named_bar_sync(3 + (t & 1), 192);   // this tile's flags are written
      if (!ok) continue;   // keep passing the named barriers with the other warps
      tc_fence_after();
      const int c_lo = jlo - qbase_of(t), c_hi = jhi - qbase_of(t);   // visible columns
      const uint32_t tS = tmem + lane_off + col_S(t & 1);
      const float* nl = s_nlt + (t & 1) * kBM;
      uint32_t zb[DROP ? 16 : 1];
      if constexpr (DROP) read_flags64(sZ + (t & 1) * kFlagBytes64, r, zb);
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t sv[32];
        tmem_ld32(tS + c * 32, sv);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int c0 = c * 32 + 2 * e;
          const float2 n2 = *reinterpret_cast<const float2*>(nl + c0);
          const float s0 = (c0 >= c_lo && c0 < c_hi) ? __uint_as_float(sv[2 * e]) : kNegInf;
          const float s1 = (c0 + 1 >= c_lo && c0 + 1 < c_hi) ? __uint_as_float(sv[2 * e + 1]) : kNegInf;
          float p0 = ex2(fmaf(s0, scale2, n2.x)), p1 = ex2(fmaf(s1, scale2, n2.y));
          if constexpr (DROP) {   // dV takes the kept probabilities (256 / T is applied to dV)
            p0 = __uint_as_float(__float_as_uint(p0) & ~flag_mask64(zb, c0));
            p1 = __uint_as_float(__float_as_uint(p1) & ~flag_mask64(zb, c0 + 1));
          }
          pk[e] = pack2<T>(p0, p1);
        }
        tmem_st16(tS + c * 16, pk);   // P^T over S^T columns already read
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar.p_full(t & 1));
    }
    bool have = ok && T_ > 0;
    if (have) have = __all_sync(0xffffffffu, mbar_wait(bar.dv_done(), 0, a.status));
    tc_fence_after();
    if (ok)
      store_row<T>(tmem + lane_off + kColDV, have, DROP ? a.drop.scale : 1.f,
                   static_cast<T*>(a.grad_v) + ((long long)(tl.k0 + j) * a.hkv + tl.g) * D,
                   key_ok && store_ok(((long long)(tl.k0 + j) * a.hkv + tl.g) * D,
                                      ((long long)(tl.k0 + j) * a.hkv + tl.g) * D + D - 1,
                                      (long long)a.total_k * a.hkv * D, a.status));
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---- dK --------------------------------------------------------------------------------------
namespace dkk {
constexpr int kStages = 2;
constexpr int kOffV = 0;                           // V, 4 boxes of 128 rows
constexpr int kOffQ = kOffV + kTile128;            // Q ring
constexpr int kOffO = kOffQ + kStages * kTile64;   // dout ring
constexpr int kOffLT = kOffO + kStages * kTile64;  // -lse_tot log2e [2][64], D [2][64]
constexpr int kOffZ = kOffLT + 4 * 64 * 4;         // dropout flags, 2 stages
constexpr int kOffBar = kOffZ + 2 * kFlagBytes64;
constexpr int kNumBars = 2 + 2 * kStages + 4;      // k_full, v_full, qd_full[S], qd_empty[S], sdp_full, ds_full, dk_done, drain
constexpr int kOffSlot = kOffBar + kNumBars * 8;
constexpr int kSmem = kOffSlot + 16 + 1024;
constexpr uint32_t kColK = 0, kColS = 128, kColP = 192, kColDK = 256;
struct Bars {
  uint32_t base;
  __device__ __forceinline__ uint32_t k_full() const { return base; }
  __device__ __forceinline__ uint32_t v_full() const { return base + 8u; }
  __device__ __forceinline__ uint32_t qd_full(int s) const { return base + 8u * (2 + s); }
  __device__ __forceinline__ uint32_t qd_empty(int s) const { return base + 8u * (2 + kStages + s); }
  __device__ __forceinline__ uint32_t sdp_full() const { return base + 8u * (2 + 2 * kStages); }
  __device__ __forceinline__ uint32_t ds_full() const { return base + 8u * (3 + 2 * kStages); }
  __device__ __forceinline__ uint32_t dk_done() const { return base + 8u * (4 + 2 * kStages); }
  __device__ __forceinline__ uint32_t drain() const { return base + 8u * (5 + 2 * kStages); }
};
}  // namespace dkk

template <typename T, bool DROP>
__global__ void __launch_bounds__(kThreads, 1)
bwd_dk_d256_kernel(const BwdArgs a, int ntiles, int band, const __grid_constant__ CUtensorMap tm_q,
                   const __grid_constant__ CUtensorMap tm_o, const __grid_constant__ CUtensorMap tm_v) {
  using namespace dkk;
  using ks::kBM;
  extern __shared__ unsigned char smem_raw[];
  ks::Tile tl;
  if (!ks::tile_of(a, ntiles, band, tl)) return;
  const int group = a.hq / a.hkv, T_ = tl.T;
  auto head_of = [&](int t) { return tl.g * group + t / tl.n_m; };
  auto qbase_of = [&](int t) { return tl.qlo + (t % tl.n_m) * kBM; };

  const uint32_t base_u32 = (smem_addr(smem_raw) + 1023u) & ~1023u;
  unsigned char* smem = smem_raw + (base_u32 - smem_addr(smem_raw));
  const uint32_t sV = base_u32 + kOffV, sQ = base_u32 + kOffQ, sO = base_u32 + kOffO;
  float* s_nlt = reinterpret_cast<float*>(smem + kOffLT);
  float* s_D = s_nlt + 2 * kBM;
  const uint32_t sZ = base_u32 + kOffZ;
  const Bars bar{base_u32 + kOffBar};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffSlot);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(bar.k_full(), 4);
    mbar_init(bar.v_full(), 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar.qd_full(s), 1);
      mbar_init(bar.qd_empty(s), 1);
    }
    mbar_init(bar.sdp_full(), 1);
    mbar_init(bar.ds_full(), 4);
    mbar_init(bar.dk_done(), 1);
    mbar_init(bar.drain(), 1);
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
    if (lane == 0 && T_ > 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_o);
      tma_prefetch_desc(&tm_v);
      mbar_arrive_expect_tx(bar.v_full(), kTile128);
      for (int hf = 0; hf < 4; ++hf) tma_load_3d(sV + hf * kBox128, &tm_v, bar.v_full(), hf * 64, tl.g, tl.k0 + tl.n0);
      int issued = 0;
      for (int t = 0; t < T_; ++t) {
        const int st = t % kStages;
        if (!mbar_wait(bar.qd_empty(st), ((t / kStages) & 1) ^ 1, a.status)) break;
        const int h = head_of(t), row = tl.q0 + qbase_of(t);
        mbar_arrive_expect_tx(bar.qd_full(st), 2 * kTile64);
        for (int hf = 0; hf < 4; ++hf) {
          tma_load_3d(sQ + st * kTile64 + hf * kBox64, &tm_q, bar.qd_full(st), hf * 64, h, row);
          tma_load_3d(sO + st * kTile64 + hf * kBox64, &tm_o, bar.qd_full(st), hf * 64, h, row);
        }
        issued = t + 1;
      }
      mbar_wait(bar.v_full(), 0, a.status);
      for (int p = issued - kStages < 0 ? 0 : issued - kStages; p < issued; ++p)
        mbar_wait(bar.qd_full(p % kStages), (p / kStages) & 1, a.status);
    }
  } else if (warp == 1) {
    // The whole warp runs the issue loop in step; elect.sync picks the issuing lane.
    if (T_ > 0) {
      constexpr uint32_t id_s = idesc_of<T>(ks::kBN, kBM, 0, 0);   // S^T, dP^T: K-major B
      constexpr uint32_t id_k = idesc_of<T>(ks::kBN, D, 0, 1);     // dS^T (TMEM) x Q (N-major)
      const uint64_t kV = smem_desc(sV, 16, 1024, kLayoutSwizzle128B);
      const uint64_t kQ = smem_desc(sQ, 16, 1024, kLayoutSwizzle128B);
      const uint64_t mQ = smem_desc(sQ, kBox64, 1024, kLayoutSwizzle128B);
      const uint64_t kO = smem_desc(sO, 16, 1024, kLayoutSwizzle128B);
      bool ok = mbar_wait_warp(bar.k_full(), 0, a.status) && mbar_wait_warp(bar.v_full(), 0, a.status);
      for (int t = 0; t < T_ && ok; ++t) {
        const int st = t % kStages;
        if (!(ok = mbar_wait_warp(bar.qd_full(st), (t / kStages) & 1, a.status))) break;
        tc_fence_after();
        const uint64_t so = (uint64_t)((st * kTile64) >> 4);
        // S^T = K Q^T (A = K from TMEM); dS^T(t - 1) in S^T's columns was read by dK(t - 1)
#pragma unroll
        for (int k = 0; k < D / 16; ++k)
          mma_ts_elect(tmem + kColS, tmem + kColK + k * 8, kQ + so + kmaj_off(k, kBox64), id_s, k > 0 ? 1u : 0u);
        // dP^T = V dout^T
#pragma unroll
        for (int k = 0; k < D / 16; ++k)
          mma_ss_elect(tmem + kColP, kV + kmaj_off(k, kBox128), kO + so + kmaj_off(k, kBox64), id_s, k > 0 ? 1u : 0u);
        mma_commit_elect(bar.sdp_full());
        if (!(ok = mbar_wait_warp(bar.ds_full(), t & 1, a.status))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kBM / 16; ++kk)
          mma_ts_elect(tmem + kColDK, tmem + kColS + kk * 8, mQ + so + (uint64_t)((kk * 2048) >> 4), id_k,
                 (t > 0 || kk > 0) ? 1u : 0u);
        mma_commit_elect(bar.qd_empty(st));
      }
      if (ok) mma_commit_elect(bar.dk_done());
      mma_commit_elect(bar.drain());
      mbar_wait_warp(bar.drain(), 0, a.status);
    }
  } else if (DROP && warp < 4) {
    // warps 2-3: the dropout flags of every tile, a tile ahead of the compute warps
    const int rt = (warp - 2) * 32 + lane;
    for (int t = 0; t < T_; ++t) {
      draw_flags64(a.drop, sZ + (t & 1) * kFlagBytes64, rt, tl.n0 >> 4, (long long)tl.q0 + qbase_of(t), head_of(t));
      named_bar_sync(3 + (t & 1), 192);
    }
  } else if (warp >= 4) {
    const int lg = warp & 3;
    const int r = lg * 32 + lane;
    const uint32_t lane_off = (uint32_t)(lg * 32) << 16;
    const int j = tl.n0 + r;
    const bool key_ok = j < tl.sk;
    stage_row(static_cast<const T*>(a.k) + ((long long)(tl.k0 + (key_ok ? j : 0)) * a.hkv + tl.g) * D, key_ok,
              tmem + lane_off + kColK, bar.k_full(), lane);
    long long qa_, qb_;
    key_query_range(j, tl.sq, tl.sk, a.left, a.right, qa_, qb_);
    const int jlo = key_ok ? (int)qa_ : 0, jhi = key_ok ? (int)qb_ : 0;
    const float scale2 = a.scale * kLog2e;
    // -lse_tot log2e and D of query r of tile t (threads r < 64), loaded a tile ahead
    float pf_l = 0.f, pf_d = 0.f;
    auto fetch = [&](int t) {
      const int i = qbase_of(t) + r;
      pf_l = pf_d = 0.f;
      if (r >= kBM || i >= tl.sq) return;
      const long long idx = (long long)head_of(t) * a.total_q + tl.q0 + i;
      const float lt2 = a.lse_tot[idx] * kLog2e;
      pf_l = lt2 == kNegInf ? 0.f : -lt2;
      pf_d = a.D[idx];
    };
    if (T_ > 0) fetch(0);
    bool ok = true;
    for (int t = 0; t < T_; ++t) {
      if (r < kBM) {
        s_nlt[(t & 1) * kBM + r] = pf_l;
        s_D[(t & 1) * kBM + r] = pf_d;
      }
      named_bar_sync(1, 128);   // buffer t & 1 was last read in tile t - 2
      if (t + 1 < T_) fetch(t + 1);
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar.sdp_full(), t & 1, a.status));
      if constexpr (DROP) named_bar_sync(3 + (t & 1), 192);   // this tile's flags are written
      if (!ok) continue;   // keep passing the named barriers with the other warps
      tc_fence_after();
      const int c_lo = jlo - qbase_of(t), c_hi = jhi - qbase_of(t);
      const float* nl = s_nlt + (t & 1) * kBM;
      const float* dd = s_D + (t & 1) * kBM;
      uint32_t zb[DROP ? 16 : 1];
      if constexpr (DROP) read_flags64(sZ + (t & 1) * kFlagBytes64, r, zb);
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t sv[32], pv[32];
        tmem_ld32(tmem + lane_off + kColS + c * 32, sv);
        tmem_ld32(tmem + lane_off + kColP + c * 32, pv);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int c0 = c * 32 + 2 * e;
          const float2 n2 = *reinterpret_cast<const float2*>(nl + c0);
          const float2 d2 = *reinterpret_cast<const float2*>(dd + c0);
          const float s0 = (c0 >= c_lo && c0 < c_hi) ? __uint_as_float(sv[2 * e]) : kNegInf;
          const float s1 = (c0 + 1 >= c_lo && c0 + 1 < c_hi) ? __uint_as_float(sv[2 * e + 1]) : kNegInf;
          const float p0 = ex2(fmaf(s0, scale2, n2.x)), p1 = ex2(fmaf(s1, scale2, n2.y));
          if constexpr (DROP) {   // dS = P (Z dP - D)
            const uint32_t m0 = flag_mask64(zb, c0), m1 = flag_mask64(zb, c0 + 1);
            pk[e] = pack2<T>(p0 * fmaf(__uint_as_float(pv[2 * e] & ~m0), a.drop.scale, -d2.x),
                             p1 * fmaf(__uint_as_float(pv[2 * e + 1] & ~m1), a.drop.scale, -d2.y));
          } else {
            pk[e] = pack2<T>(p0 * (__uint_as_float(pv[2 * e]) - d2.x), p1 * (__uint_as_float(pv[2 * e + 1]) - d2.y));
          }
        }
        tmem_st16(tmem + lane_off + kColS + c * 16, pk);   // dS^T over S^T columns already read
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar.ds_full());
    }
    bool have = ok && T_ > 0;
    if (have) have = __all_sync(0xffffffffu, mbar_wait(bar.dk_done(), 0, a.status));
    tc_fence_after();
    if (ok)
      store_row<T>(tmem + lane_off + kColDK, have, a.scale,
                   static_cast<T*>(a.grad_k) + ((long long)(tl.k0 + j) * a.hkv + tl.g) * D,
                   key_ok && store_ok(((long long)(tl.k0 + j) * a.hkv + tl.g) * D,
                                      ((long long)(tl.k0 + j) * a.hkv + tl.g) * D + D - 1,
                                      (long long)a.total_k * a.hkv * D, a.status));
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---- host ------------------------------------------------------------------------------------

long long dq_grid(const BwdArgs& a) { return (long long)((a.max_sq + dq::kBM - 1) / dq::kBM) * a.batch * a.hq; }
long long ks_grid(const BwdArgs& a) { return (long long)((a.max_sk + ks::kBN - 1) / ks::kBN) * a.batch * a.hkv; }

// (sequence, kv head) groups per band: as many as fit `per_group` bytes each in about half of
// the 126 MB L2
int band_of(const BwdArgs& a, long long per_group) {
  long long s = (64LL << 20) / (per_group > 0 ? per_group : 1);
  const long long G = (long long)a.batch * a.hkv;
  if (s < 1) s = 1;
  if (s > G) s = G;
  return (int)s;
}

template <typename T>
cudaError_t launch_typed(const BwdArgs& a, cudaStream_t s) {
  constexpr CUtensorMapDataType dt = tma_dtype<T>();
  CUtensorMap q64, o64, o128, k64, v64, v128;
  if (!make_map_3d(&q64, a.q, D, a.hq, a.total_q, 64, dt) || !make_map_3d(&o64, a.dout, D, a.hq, a.total_q, 64, dt) ||
      !make_map_3d(&o128, a.dout, D, a.hq, a.total_q, 128, dt) || !make_map_3d(&k64, a.k, D, a.hkv, a.total_k, 64, dt) ||
      !make_map_3d(&v64, a.v, D, a.hkv, a.total_k, 64, dt) || !make_map_3d(&v128, a.v, D, a.hkv, a.total_k, 128, dt))
    return cudaErrorInvalidValue;
  cudaError_t e;
  const bool drop = a.drop.threshold != 0;
  auto kq = drop ? bwd_dq_d256_kernel<T, true> : bwd_dq_d256_kernel<T, false>;
  auto kv = drop ? bwd_dv_d256_kernel<T, true> : bwd_dv_d256_kernel<T, false>;
  auto kk = drop ? bwd_dk_d256_kernel<T, true> : bwd_dk_d256_kernel<T, false>;
  if ((e = cudaFuncSetAttribute(kq, cudaFuncAttributeMaxDynamicSharedMemorySize, dq::kSmem)) ||
      (e = cudaFuncSetAttribute(kv, cudaFuncAttributeMaxDynamicSharedMemorySize, dvk::kSmem)) ||
      (e = cudaFuncSetAttribute(kk, cudaFuncAttributeMaxDynamicSharedMemorySize, dkk::kSmem)))
    return e;
  const int mtiles = (a.max_sq + dq::kBM - 1) / dq::kBM, ntiles = (a.max_sk + ks::kBN - 1) / ks::kBN;
  const int group = a.hq / a.hkv;
  // per group: K and V of the sequence (dQ); Q and dout of the group's q heads (dK, dV)
  const int band_q = band_of(a, (long long)(a.max_sk > 0 ? a.max_sk : 1) * 2 * D * 2);
  const int band_k = band_of(a, (long long)(a.max_sq > 0 ? a.max_sq : 1) * group * 2 * D * 2);
  if (mtiles > 0) {
    kq<<<(unsigned)dq_grid(a), kThreads, dq::kSmem, s>>>(a, mtiles, band_q, o128, k64, v64);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (ks_grid(a) > 0) {
    kk<<<(unsigned)ks_grid(a), kThreads, dkk::kSmem, s>>>(a, ntiles, band_k, q64, o64, v128);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    kv<<<(unsigned)ks_grid(a), kThreads, dvk::kSmem, s>>>(a, ntiles, band_k, q64, o64);
  }
  return cudaGetLastError();
}

}  // namespace

bool bwd_d256_sm100_supported(const BwdArgs& a, int dtype) {
  if (dtype != 0 && dtype != 2) return false;
  if (a.dk != D || a.dv != D) return false;
  if (dq_grid(a) > 0x7fffffffLL || ks_grid(a) > 0x7fffffffLL) return false;   // 1-D grids
  return encode_fn() != nullptr;
}

cudaError_t launch_bwd_d256_sm100(const BwdArgs& a, int dtype, cudaStream_t s) {
  return dtype == 2 ? launch_typed<__half>(a, s) : launch_typed<__nv_bfloat16>(a, s);
}

}  // namespace attn_sink
