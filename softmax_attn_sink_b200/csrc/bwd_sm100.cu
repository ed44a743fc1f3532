// Sink-attention backward on the sm_100a tensor cores (bf16 in, fp32 accumulation).
//
// Gradient of the sink forward for the loss sum(dout * out).  With lse_tot =
// logaddexp(lse, sink) (from the preprocess pass) the probabilities are
// P_ij = e^{S_ij - lse_tot_i}; then dS = P * (dout V^T - D) with D_i = dout_i . out_i,
// dq = scale dS K, dk = scale dS^T Q, dv = P^T dout.  slime's learnable_softmax_attention.py
// writes the same gradient as dS = P_van * s * (D - s * di) with s = sigmoid(lse - offset)
// (class docstring); P = s P_van and D_i = s di make the two forms equal.
//
// One CTA owns a 128-key tile of one (sequence, kv head) and loops over every q head of
// the GQA group and every 128-query tile that can see those keys, so dK and dV
// accumulate in TMEM with no atomics.  Per query tile t:
//   S^T  = K Q^T        (M = keys, N = queries)        -> TMEM R0
//   dP^T = V dout^T                                    -> TMEM R1
//   compute warps (thread = key row): P^T = 2^{S^T scale log2e - lse_tot log2e} (masked),
//     dS^T = P^T (dP^T - D); P^T as bf16 back into R0 (TMEM A operand), dS^T as bf16 into
//     a 128-byte-swizzled shared tile
//   dV += P^T dout      (A = P^T from TMEM, B = dout MN-major)
//   dK += dS^T Q        (A = dS^T K-major from shared memory, B = Q MN-major)
//   dQ_t = dS K         (A = the same dS^T tile read MN-major, B = K MN-major) -> TMEM R1
//   dQ warps (thread = query row) read dQ_t and add scale * dQ_t into an fp32 workspace
//     with vector atomics; a final pass converts it to bf16.
// TMEM columns: dK [0,128) dV [128,256) R0 [256,384) R1 [384,512).
// The next tile's S^T overwrites R0, which the dV MMA reads as P^T: the MMA thread waits
// for a commit of that dV MMA first (it is issued ahead of dK and dQ, so the tensor pipe
// stays busy meanwhile).  All mbarrier waits are bounded.
#include <cuda.h>

#include "sm100_ptx.cuh"
#include "tma_map.h"

namespace attn_sink {

cudaError_t launch_bwd_preprocess(const BwdArgs& a, int dtype, cudaStream_t s);

namespace {

// Work order of the key-tile CTAs (1-D grid).  The (sequence, kv head) groups are taken in
// bands of a.band_groups; inside a band the CTAs go key tile by key tile (tile 0, which sees
// the most queries under a causal mask, first), cycling through the band's groups.  So the
// CTAs resident at any time reduce into the dq_acc rows and read the Q / dO tiles of a few
// groups only, a working set the launcher sizes to stay in L2: fp32 reductions into
// L2-resident lines run about 1.7x faster than into lines that spill to DRAM.
__device__ __forceinline__ void bwd_tile_of(const BwdArgs& a, int ntiles, int& g, int& b, int& nt) {
  const long long id = blockIdx.x;
  const int G = a.batch * a.hkv, S = a.band_groups;
  const long long per_band = (long long)S * ntiles;
  const int band = (int)(id / per_band);
  const int first = band * S, members = (G - first < S) ? G - first : S;
  const long long rem = id - (long long)band * per_band;
  nt = (int)(rem / members);
  const int grp = first + (int)(rem - (long long)nt * members);
  b = grp / a.hkv;
  g = grp - b * a.hkv;
}

// Groups per band: as many (sequence, kv head) groups as fit, with their dq_acc rows and
// Q / dO tiles, in about half of the 126 MB L2.
inline int bwd_band_groups(const BwdArgs& a) {
  const long long per_group = (long long)(a.max_sq > 0 ? a.max_sq : 1) * (a.hq / a.hkv) *
                              ((long long)a.dk * 4 + (long long)(a.dk + a.dv) * 2);
  long long s = (64LL << 20) / (per_group > 0 ? per_group : 1);
  const long long G = (long long)a.batch * a.hkv;
  if (s < 1) s = 1;
  if (s > G) s = G;
  return (int)s;
}

using namespace sm100;

__device__ __forceinline__ void named_bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

constexpr int kBN = 128;  // keys per CTA
constexpr int kBM = 128;  // queries per inner tile
constexpr int kThreads = 320;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColDK = 0, kColDV = 128, kColR0 = 256, kColR1 = 384;

// Dropout flags of a 128-query x 128-key tile, transposed for the compute threads (one key
// each): word [block][key tk][w][u] holds, in byte m, the drop flag of query u + 16 (4 w + m);
// + 16 words per block so that blocks 2x and 2x + 1 start in different banks.
constexpr int kFlagBlockWords = 16 * 32 + 16;
constexpr int kFlagBytes = 4 * 8 * kFlagBlockWords;

template <int DK, int DV, bool DROP = false>
struct BLayout {
  static constexpr int KH = DK / 64, VH = DV / 64;
  static constexpr int kHalf = 128 * 128;                  // 128 rows x 128 bytes
  static constexpr int kKBytes = KH * kHalf, kVBytes = VH * kHalf;
  static constexpr int kQBytes = KH * kHalf, kOBytes = VH * kHalf;
  static constexpr int kDSBytes = 2 * kHalf;               // 128 keys x 128 queries bf16
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kOffK + kKBytes;
  static constexpr int kOffQ = kOffV + kVBytes;            // 2 stages
  static constexpr int kOffO = kOffQ + 2 * kQBytes;        // 2 stages (dout)
  static constexpr int kOffDS = kOffO + 2 * kOBytes;
  static constexpr int kOffZ = kOffDS + kDSBytes;          // dropout flags, 2 stages
  static constexpr int kOffBar = kOffZ + (DROP ? 2 * kFlagBytes : 0);
  static constexpr int kNumBars = 12;
  static constexpr int kOffSlot = kOffBar + kNumBars * 8;
  static constexpr int kSmem = kOffSlot + 16 + 1024;
};

struct BBars {
  uint32_t base;
  __device__ __forceinline__ uint32_t kv_full() const { return base; }
  __device__ __forceinline__ uint32_t qd_full(int s) const { return base + 8u * (1 + s); }
  __device__ __forceinline__ uint32_t qd_empty(int s) const { return base + 8u * (3 + s); }
  __device__ __forceinline__ uint32_t sdp_full() const { return base + 8u * 5; }
  __device__ __forceinline__ uint32_t compute_done() const { return base + 8u * 6; }
  __device__ __forceinline__ uint32_t dv_done() const { return base + 8u * 7; }
  __device__ __forceinline__ uint32_t dq_full() const { return base + 8u * 8; }
  __device__ __forceinline__ uint32_t dq_free() const { return base + 8u * 9; }
  __device__ __forceinline__ uint32_t ds_free() const { return base + 8u * 10; }
  __device__ __forceinline__ uint32_t drain() const { return base + 8u * 11; }
};

// DVO <= DV is the width of v, dout and dv in memory (DV that of the tiles and products):
// with DVO = 32 the V and dout tiles are 64-column boxes over 32-column tensors, whose
// columns 32-63 the copies fill with zeros, so dP is exact and dV's columns 32-63 stay zero.
template <typename Elem, int DK, int DV, bool DQ, bool DROP = false, int DVO = DV>
__global__ void __launch_bounds__(kThreads, 1)
bwd_sm100_kernel(const BwdArgs a, const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do) {
  static_assert(!(DQ && DROP), "dropout runs with the dQ pass of the deterministic backward");
  using L = BLayout<DK, DV, DROP>;
  extern __shared__ unsigned char smem_raw[];

  // ---- work unit: key tile nt of (sequence b, kv head g) ---------------------------------
  int g, b, nt;
  bwd_tile_of(a, (a.max_sk + kBN - 1) / kBN, g, b, nt);
  const long long q0 = a.cu_q[b], sq = a.cu_q[b + 1] - q0;
  const long long k0 = a.cu_k[b], sk = a.cu_k[b + 1] - k0;
  const long long n0 = (long long)nt * kBN;
  if (n0 >= sk) return;
  const int group = a.hq / a.hkv;
  const long long nkeys = (sk - n0 < kBN) ? sk - n0 : kBN;
  long long qlo, qhi, qlo1, qhi1;
  key_query_range(n0, sq, sk, a.left, a.right, qlo, qhi);
  key_query_range(n0 + nkeys - 1, sq, sk, a.left, a.right, qlo1, qhi1);
  qhi = qhi1;  // query ranges move right with the key, so the union is [qlo(first), qhi(last))
  const int n_m = qhi > qlo ? (int)((qhi - qlo + kBM - 1) / kBM) : 0;
  const int T = n_m * group;

  const uint32_t base_u32 = (smem_addr(smem_raw) + 1023u) & ~1023u;
  unsigned char* smem = smem_raw + (base_u32 - smem_addr(smem_raw));
  const uint32_t sK = base_u32 + L::kOffK, sV = base_u32 + L::kOffV, sQ = base_u32 + L::kOffQ,
                 sO = base_u32 + L::kOffO, sDS = base_u32 + L::kOffDS, sZ = base_u32 + L::kOffZ;
  const BBars bar{base_u32 + L::kOffBar};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kOffSlot);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(bar.kv_full(), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar.qd_full(s), 1);
      mbar_init(bar.qd_empty(s), 1);
    }
    mbar_init(bar.sdp_full(), 1);
    mbar_init(bar.compute_done(), 4);
    mbar_init(bar.dv_done(), 1);
    mbar_init(bar.dq_full(), 1);
    mbar_init(bar.dq_free(), 4);
    mbar_init(bar.ds_free(), 1);
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

  auto head_of = [&](int t) { return g * group + t / n_m; };
  auto qbase_of = [&](int t) { return qlo + (long long)(t % n_m) * kBM; };

  if (warp == 0) {
    // ================================ TMA producer ======================================
    if (lane == 0 && T > 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      mbar_arrive_expect_tx(bar.kv_full(), L::kKBytes + L::kVBytes);
      for (int hf = 0; hf < L::KH; ++hf)
        tma_load_3d(sK + hf * L::kHalf, &tm_k, bar.kv_full(), hf * 64, g, (int)(k0 + n0));
      for (int hf = 0; hf < L::VH; ++hf)
        tma_load_3d(sV + hf * L::kHalf, &tm_v, bar.kv_full(), hf * 64, g, (int)(k0 + n0));
      int issued = 0;
      for (int t = 0; t < T; ++t) {
        const int st = t & 1;
        if (!mbar_wait(bar.qd_empty(st), ((t >> 1) & 1) ^ 1, a.status)) break;
        const int h = head_of(t);
        const int row = (int)(q0 + qbase_of(t));
        mbar_arrive_expect_tx(bar.qd_full(st), L::kQBytes + L::kOBytes);
        for (int hf = 0; hf < L::KH; ++hf)
          tma_load_3d(sQ + st * L::kQBytes + hf * L::kHalf, &tm_q, bar.qd_full(st), hf * 64, h, row);
        for (int hf = 0; hf < L::VH; ++hf)
          tma_load_3d(sO + st * L::kOBytes + hf * L::kHalf, &tm_do, bar.qd_full(st), hf * 64, h, row);
        issued = t + 1;
      }
      mbar_wait(bar.kv_full(), 0, a.status);
      for (int t = issued - 2 < 0 ? 0 : issued - 2; t < issued; ++t)
        mbar_wait(bar.qd_full(t & 1), (t >> 1) & 1, a.status);
    }
  } else if (warp == 1) {
    // ================================ MMA issuer =========================================
    // The whole warp runs the issue loop in step and elect.sync picks the issuing lane
    // (an MMA costs the warp 5-10 cycles this way, against about 50 from a lone lane).
    if (T > 0) {
      constexpr uint32_t id_s = idesc_of<Elem>(kBN, kBM, 0, 0);   // S^T, dP^T: K-major A and B
      constexpr uint32_t id_dv = idesc_of<Elem>(kBN, DV, 0, 1);   // A from TMEM, B = dout MN-major
      constexpr uint32_t id_dk = idesc_of<Elem>(kBN, DK, 0, 1);   // A = dS^T K-major, B = Q MN-major
      constexpr uint32_t id_dq = idesc_of<Elem>(kBM, DK, 1, 1);   // A = dS MN-major, B = K MN-major
      bool ok = mbar_wait_warp(bar.kv_full(), 0, a.status);
      for (int t = 0; t < T && ok; ++t) {
        const int st = t & 1;
        const uint32_t q_s = sQ + st * L::kQBytes, o_s = sO + st * L::kOBytes;
        ok = mbar_wait_warp(bar.qd_full(st), (t >> 1) & 1, a.status);
        if (ok && t >= 1) ok = mbar_wait_warp(bar.dv_done(), (t - 1) & 1, a.status);   // R0 free
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < DK / 16; ++ks) {
          const uint32_t off = (ks >> 2) * L::kHalf + (ks & 3) * 32;
          mma_ss_elect(tmem + kColR0, smem_desc(sK + off, 16, 1024, kLayoutSwizzle128B),
                 smem_desc(q_s + off, 16, 1024, kLayoutSwizzle128B), id_s, ks > 0);
        }
        if (DQ && t >= 1 && !(ok = mbar_wait_warp(bar.dq_free(), (t - 1) & 1, a.status))) break;   // R1 free
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < DV / 16; ++ks) {
          const uint32_t off = (ks >> 2) * L::kHalf + (ks & 3) * 32;
          mma_ss_elect(tmem + kColR1, smem_desc(sV + off, 16, 1024, kLayoutSwizzle128B),
                 smem_desc(o_s + off, 16, 1024, kLayoutSwizzle128B), id_s, ks > 0);
        }
        mma_commit_elect(bar.sdp_full());
        if (!(ok = mbar_wait_warp(bar.compute_done(), t & 1, a.status))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kBM / 16; ++kk)
          mma_ts_elect(tmem + kColDV, tmem + kColR0 + kk * 8,
                 smem_desc(o_s + kk * 2048, L::kHalf, 1024, kLayoutSwizzle128B), id_dv, (t > 0 || kk > 0));
        mma_commit_elect(bar.dv_done());
#pragma unroll
        for (int kk = 0; kk < kBM / 16; ++kk)
          mma_ss_elect(tmem + kColDK, smem_desc(sDS + (kk >> 2) * L::kHalf + (kk & 3) * 32, 16, 1024, kLayoutSwizzle128B),
                 smem_desc(q_s + kk * 2048, L::kHalf, 1024, kLayoutSwizzle128B), id_dk, (t > 0 || kk > 0));
        if (DQ) {
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk)
            mma_ss_elect(tmem + kColR1, smem_desc(sDS + kk * 2048, L::kHalf, 1024, kLayoutSwizzle128B),
                   smem_desc(sK + kk * 2048, L::kHalf, 1024, kLayoutSwizzle128B), id_dq, kk > 0);
          mma_commit_elect(bar.dq_full());
        }
        mma_commit_elect(bar.ds_free());
        mma_commit_elect(bar.qd_empty(st));
      }
      mma_commit_elect(bar.drain());
      mbar_wait_warp(bar.drain(), 0, a.status);
    }
  } else if (warp < 6) {
    // ================================ compute warps (thread = key row) ===================
    const int lg = warp & 3;
    const int r = lg * 32 + lane;
    const uint32_t lane_off = (uint32_t)(lg * 32) << 16;
    const long long j = n0 + r;                       // key index in the sequence
    const bool key_ok = j < sk;
    const float scale2 = a.scale * kLog2e;
    const long long off = sk - sq;
    bool ok = true;
    for (int t = 0; t < T; ++t) {
      const int h = head_of(t);
      const long long i0 = qbase_of(t);
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar.sdp_full(), t & 1, a.status));
      if (ok && t >= 1) ok = __all_sync(0xffffffffu, mbar_wait(bar.ds_free(), (t - 1) & 1, a.status));
      // with dropout the flag producers (warps 6-9) meet these warps on a named barrier once
      // per tile, so after a timed-out wait these warps keep passing it instead of leaving
      if constexpr (DROP) named_bar_sync(3 + (t & 1), 256);
      if (!ok) {
        if constexpr (DROP) continue;
        else break;
      }
      tc_fence_after();
      const float* lt_row = a.lse_tot + (long long)h * a.total_q + q0;
      const float* D_row = a.D + (long long)h * a.total_q + q0;
      // dropout: this key's flags for the tile's 128 queries, words [w][u] (query u + 16 (4 w + m)
      // in byte m)
      uint32_t zb[DROP ? 32 : 1];
      if constexpr (DROP) {
        const uint32_t src = sZ + (t & 1) * kFlagBytes + 4u * ((r >> 4) * kFlagBlockWords + (r & 15) * 32);
#pragma unroll
        for (int v4 = 0; v4 < 8; ++v4)
          asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(zb[4 * v4]), "=r"(zb[4 * v4 + 1]), "=r"(zb[4 * v4 + 2]), "=r"(zb[4 * v4 + 3])
                       : "r"(src + 16u * v4)
                       : "memory");
      }
#pragma unroll 1
      for (int c = 0; c < kBM / 32; ++c) {
        uint32_t sv[32], dpv[32];
        tmem_ld32(tmem + lane_off + kColR0 + c * 32, sv);
        tmem_ld32(tmem + lane_off + kColR1 + c * 32, dpv);
        tmem_wait_ld();
        // queries 32 c + e: word (c / 2) * 16 + e % 16, byte 2 (c % 2) + e / 16
        uint32_t zh[DROP ? 16 : 1];
        if constexpr (DROP) {
#pragma unroll
          for (int w = 0; w < 16; ++w) zh[w] = (c >> 1) ? zb[16 + w] : zb[w];
        }
        uint32_t pk[16], dk_[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          float pp[2], dd[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const long long qi = i0 + c * 32 + e + u;
            bool vis = key_ok && qi < sq;
            const long long d = j - (qi + off);       // key offset from the query's diagonal
            if (a.right < kUnbounded) vis = vis && d <= a.right;
            if (a.left < kUnbounded) vis = vis && d >= -(long long)a.left;
            float p = 0.f, ds = 0.f;
            if (vis) {
              const float lt = __ldg(lt_row + qi);
              p = ex2(fmaf(__uint_as_float(sv[e + u]), scale2, -lt * kLog2e));
              if constexpr (DROP) {
                // dV takes the kept probabilities (256 / T is applied to dV), dS = P (Z dP - D)
                const uint32_t byte = (uint32_t)(2 * (c & 1) + ((e + u) >> 4));
                const uint32_t m = prmt_sign_r(zh[(e + u) & 15], (8u | byte) * 0x1111u);
                ds = p * fmaf(__uint_as_float(dpv[e + u] & ~m), a.drop.scale, -__ldg(D_row + qi));
                p = __uint_as_float(__float_as_uint(p) & ~m);
              } else {
                ds = p * (__uint_as_float(dpv[e + u]) - __ldg(D_row + qi));
              }
            }
            pp[u] = p;
            dd[u] = ds;
          }
          pk[e >> 1] = pack2<Elem>(pp[0], pp[1]);
          dk_[e >> 1] = pack2<Elem>(dd[0], dd[1]);
        }
        // P^T chunk -> TMEM R0 (its S^T columns were already read)
        tmem_st16(tmem + lane_off + kColR0 + c * 16, pk);
        // dS^T chunk -> shared tile, row r, queries [32c, 32c + 32): 4 swizzled 16-byte chunks
        const uint32_t half = sDS + (c >> 1) * L::kHalf + r * 128;
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const int ch = (c & 1) * 4 + v;
          st_shared_v4(half + ((ch ^ (r & 7)) << 4), dk_[4 * v], dk_[4 * v + 1], dk_[4 * v + 2], dk_[4 * v + 3]);
        }
      }
      tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar.compute_done());
    }
    // ---- epilogue: dK = scale * acc, dV = acc, bf16, this thread's key row -----------------
    const bool have = __all_sync(0xffffffffu, ok && T > 0 && mbar_wait(bar.ds_free(), (T - 1) & 1, a.status));
    tc_fence_after();
    Elem* dkp = static_cast<Elem*>(a.grad_k) + ((k0 + j) * a.hkv + g) * DK;
    Elem* dvp = static_cast<Elem*>(a.grad_v) + ((k0 + j) * a.hkv + g) * DVO;
#pragma unroll
    for (int pass = 0; pass < 2; ++pass) {
      const int ncol = pass == 0 ? DK : DVO;
      const uint32_t col = pass == 0 ? kColDK : kColDV;
      const float mul = pass == 0 ? a.scale : (DROP ? a.drop.scale : 1.f);
      uint4* dst = reinterpret_cast<uint4*>(pass == 0 ? dkp : dvp);
      for (int c = 0; c < ncol / 32; ++c) {
        uint32_t v[32];
        if (T > 0) {
          tmem_ld32(tmem + lane_off + col + c * 32, v);
          tmem_wait_ld();
        }
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float x0 = (T > 0 && have) ? __uint_as_float(v[2 * e]) * mul : 0.f;
          const float x1 = (T > 0 && have) ? __uint_as_float(v[2 * e + 1]) * mul : 0.f;
          pk[e] = pack2<Elem>(x0, x1);
        }
        const long long e0 = ((k0 + j) * a.hkv + g) * ncol + c * 32;
        if (key_ok && store_ok(e0, e0 + 31, (long long)a.total_k * a.hkv * ncol, a.status)) {
#pragma unroll
          for (int u = 0; u < 4; ++u) dst[c * 4 + u] = make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
        }
      }
    }
  } else if (DROP) {
    // ================================ dropout flags (warps 6-9) ============================
    // Thread rt draws key block rt / 16 for queries u0 + 16 m (u0 = rt % 16, m = 0..7) of
    // tile t: 8 Philox calls, a tile ahead of the compute warps, written transposed into
    // stage t % 2; the compute warps are done with tile t - 2 (the stage's previous use)
    // once this thread has passed the barrier of tile t - 1.
    const int rt = (warp - 6) * 32 + lane, blk = rt >> 4, u0 = rt & 15;
    const uint32_t t4 = (a.drop.threshold - 1u) * 0x01010101u, t4h = t4 | 0x80808080u;
    for (int t = 0; t < T; ++t) {
      uint32_t fw[8][4];   // [m][word]
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const uint4 w = dropout_bytes(a.drop, (uint32_t)((n0 >> 4) + blk), (uint32_t)(q0 + qbase_of(t) + u0 + 16 * m),
                                      (uint32_t)head_of(t));
        fw[m][0] = drop_flags4(w.x, t4, t4h);
        fw[m][1] = drop_flags4(w.y, t4, t4h);
        fw[m][2] = drop_flags4(w.z, t4, t4h);
        fw[m][3] = drop_flags4(w.w, t4, t4h);
      }
      const uint32_t stage = sZ + (t & 1) * kFlagBytes;
#pragma unroll
      for (int tk = 0; tk < 16; ++tk) {
        const uint32_t sel = (uint32_t)(tk & 3) | ((uint32_t)(4 + (tk & 3)) << 4);
#pragma unroll
        for (int w = 0; w < 2; ++w) {
          // bytes m = 0..3 of this word: queries u0 + 16 (4 w + m), key tk
          const uint32_t lo2 = __byte_perm(fw[4 * w][tk >> 2], fw[4 * w + 1][tk >> 2], sel);
          const uint32_t hi2 = __byte_perm(fw[4 * w + 2][tk >> 2], fw[4 * w + 3][tk >> 2], sel);
          asm volatile("st.shared.u32 [%0], %1;" ::"r"(stage + 4u * (blk * kFlagBlockWords + tk * 32 + w * 16 + u0)),
                       "r"(__byte_perm(lo2, hi2, 0x5410))
                       : "memory");
        }
      }
      named_bar_sync(3 + (t & 1), 256);
    }
  } else {
    // ================================ dQ warps (thread = query row) =======================
    const int lg = warp & 3;
    const int r = lg * 32 + lane;
    const uint32_t lane_off = (uint32_t)(lg * 32) << 16;
    for (int t = 0; t < (DQ ? T : 0); ++t) {
      if (!__all_sync(0xffffffffu, mbar_wait(bar.dq_full(), t & 1, a.status))) break;
      tc_fence_after();
      uint32_t v[DK];
#pragma unroll
      for (int c = 0; c < DK / 32; ++c) {
        uint32_t (&chunk)[32] = *reinterpret_cast<uint32_t(*)[32]>(&v[c * 32]);
        tmem_ld32(tmem + lane_off + kColR1 + c * 32, chunk);
      }
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar.dq_free());
      const long long qi = qbase_of(t) + r;
      const long long a0 = ((q0 + qi) * a.hq + head_of(t)) * DK;
      if (qi < sq && store_ok(a0, a0 + DK - 1, (long long)a.total_q * a.hq * DK, a.status)) {
        float* dst = a.dq_acc + a0;
#pragma unroll
        for (int e = 0; e < DK; e += 4)
          red_add_v4(dst + e, __uint_as_float(v[e]) * a.scale, __uint_as_float(v[e + 1]) * a.scale,
                     __uint_as_float(v[e + 2]) * a.scale, __uint_as_float(v[e + 3]) * a.scale);
      }
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

// ---- head dim 128: query tile in two 64-query halves, software-pipelined -----------------
//
// Same gradient as above.  Each 128-query tile is processed as two halves a/b so that the
// tensor pipe works on one half while the compute warps work on the other:
//   MMA order per tile t:  [wait compute_a] dV_a dK_a dQ^T_a  [wait compute_b]
//                          S_a(t+1) dP_a(t+1)  dV_b dK_b dQ^T_b  S_b(t+1) dP_b(t+1)
// dQ is produced transposed, dQ^T = K^T dS^T (M = head dim), so a dQ warp thread owns one
// head-dim index and each warp-wide reduction covers 128 contiguous bytes of a dQ row.
// TMEM: dK [0,128) dV [128,256) S_a [256,320) dP_a [320,384) S_b [384,448) dP_b [448,512);
// P^T of a half is written over its S columns, dQ^T of a half over its dP columns.
constexpr uint32_t kColSa = 256, kColDPa = 320, kColSb = 384, kColDPb = 448;
// 12 warps: warp 0 TMA, warp 1 MMA, warps 2-3 idle, warps 4-7 compute, warps 8-11 dQ.
// Launched at 168 registers (384 x 168 = 64512); the first warpgroup (whose MMA issuer keeps
// nine descriptors live) drops to 136, compute and dQ take 184: 128 x 136 + 256 x 184 = 64512.
constexpr int kThreadsP = 384;
constexpr int kRegsLow = 136, kRegsHigh = 184;
static_assert(128 * kRegsLow + 256 * kRegsHigh <= kThreadsP * 168, "register split");

template <int DV>
struct PLayout {   // head dim 128: K and Q tiles are two 64-column boxes
  static constexpr int VH = DV / 64;
  static constexpr int kHalf = 128 * 128;
  static constexpr int kKBytes = 2 * kHalf, kVBytes = VH * kHalf;
  static constexpr int kQBytes = 2 * kHalf, kOBytes = VH * kHalf;
  static constexpr int kDSBytes = 2 * kHalf;
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kOffK + kKBytes;
  static constexpr int kOffQ = kOffV + kVBytes;
  static constexpr int kOffO = kOffQ + 2 * kQBytes;
  static constexpr int kOffDS = kOffO + 2 * kOBytes;
  static constexpr int kOffLD = kOffDS + kDSBytes;         // lse_tot * log2e [128], D [128]
  static constexpr int kOffBar = kOffLD + 1024;
  static constexpr int kNumBars = 18;
  static constexpr int kOffSlot = kOffBar + kNumBars * 8;
  static constexpr int kSmem = kOffSlot + 16 + 1024;
};

struct PBars {
  uint32_t base;
  __device__ __forceinline__ uint32_t kv_full() const { return base; }
  __device__ __forceinline__ uint32_t qd_full(int s) const { return base + 8u * (1 + s); }
  __device__ __forceinline__ uint32_t qd_empty(int s) const { return base + 8u * (3 + s); }
  __device__ __forceinline__ uint32_t sdp_full(int h) const { return base + 8u * (5 + h); }
  __device__ __forceinline__ uint32_t compute_done(int h) const { return base + 8u * (7 + h); }
  __device__ __forceinline__ uint32_t dv_done(int h) const { return base + 8u * (9 + h); }
  __device__ __forceinline__ uint32_t dq_full(int h) const { return base + 8u * (11 + h); }
  __device__ __forceinline__ uint32_t dq_free(int h) const { return base + 8u * (13 + h); }
  __device__ __forceinline__ uint32_t ds_free(int h) const { return base + 8u * (15 + h); }
  __device__ __forceinline__ uint32_t drain() const { return base + 8u * 17; }
};



template <typename Elem, int DV, bool DQ, bool DROP, int DVO = DV>
__global__ void __launch_bounds__(kThreadsP, 1)
bwd_sm100_d128_kernel(const BwdArgs a, const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                      const __grid_constant__ CUtensorMap tm_do) {
  using L = PLayout<DV>;
  constexpr int DK = 128;
  extern __shared__ unsigned char smem_raw[];

  int g, b, nt;
  bwd_tile_of(a, (a.max_sk + kBN - 1) / kBN, g, b, nt);
  const long long q0 = a.cu_q[b], sq = a.cu_q[b + 1] - q0;
  const long long k0 = a.cu_k[b], sk = a.cu_k[b + 1] - k0;
  const long long n0 = (long long)nt * kBN;
  if (n0 >= sk) return;
  const int group = a.hq / a.hkv;
  const long long nkeys = (sk - n0 < kBN) ? sk - n0 : kBN;
  long long qlo, qhi, qlo1, qhi1;
  key_query_range(n0, sq, sk, a.left, a.right, qlo, qhi);
  key_query_range(n0 + nkeys - 1, sq, sk, a.left, a.right, qlo1, qhi1);
  qhi = qhi1;
  const int n_m = qhi > qlo ? (int)((qhi - qlo + kBM - 1) / kBM) : 0;
  const int T = n_m * group;

  const uint32_t base_u32 = (smem_addr(smem_raw) + 1023u) & ~1023u;
  unsigned char* smem = smem_raw + (base_u32 - smem_addr(smem_raw));
  const uint32_t sK = base_u32 + L::kOffK, sV = base_u32 + L::kOffV, sQ = base_u32 + L::kOffQ,
                 sO = base_u32 + L::kOffO, sDS = base_u32 + L::kOffDS;
  float* s_lt = reinterpret_cast<float*>(smem + L::kOffLD);
  float* s_D = s_lt + 128;
  const PBars bar{base_u32 + L::kOffBar};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kOffSlot);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(bar.kv_full(), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar.qd_full(s), 1);
      mbar_init(bar.qd_empty(s), 1);
      mbar_init(bar.sdp_full(s), 1);
      mbar_init(bar.compute_done(s), 4);
      mbar_init(bar.dv_done(s), 1);
      mbar_init(bar.dq_full(s), 1);
      mbar_init(bar.dq_free(s), 4);
      mbar_init(bar.ds_free(s), 1);
    }
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

  auto head_of = [&](int t) { return g * group + t / n_m; };
  auto qbase_of = [&](int t) { return qlo + (long long)(t % n_m) * kBM; };

  if (warp == 0) {
    // ================================ TMA producer ======================================
    regs_dec<kRegsLow>();
    if (lane == 0 && T > 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      mbar_arrive_expect_tx(bar.kv_full(), L::kKBytes + L::kVBytes);
      for (int hf = 0; hf < 2; ++hf) tma_load_3d(sK + hf * L::kHalf, &tm_k, bar.kv_full(), hf * 64, g, (int)(k0 + n0));
      for (int hf = 0; hf < L::VH; ++hf)
        tma_load_3d(sV + hf * L::kHalf, &tm_v, bar.kv_full(), hf * 64, g, (int)(k0 + n0));
      int issued = 0;
      for (int t = 0; t < T; ++t) {
        const int st = t & 1;
        if (!mbar_wait(bar.qd_empty(st), ((t >> 1) & 1) ^ 1, a.status)) break;
        const int h = head_of(t);
        const int row = (int)(q0 + qbase_of(t));
        mbar_arrive_expect_tx(bar.qd_full(st), L::kQBytes + L::kOBytes);
        for (int hf = 0; hf < 2; ++hf)
          tma_load_3d(sQ + st * L::kQBytes + hf * L::kHalf, &tm_q, bar.qd_full(st), hf * 64, h, row);
        for (int hf = 0; hf < L::VH; ++hf)
          tma_load_3d(sO + st * L::kOBytes + hf * L::kHalf, &tm_do, bar.qd_full(st), hf * 64, h, row);
        issued = t + 1;
      }
      mbar_wait(bar.kv_full(), 0, a.status);
      for (int t = issued - 2 < 0 ? 0 : issued - 2; t < issued; ++t)
        mbar_wait(bar.qd_full(t & 1), (t >> 1) & 1, a.status);
    }
  } else if (warp == 1) {
    // ================================ MMA issuer =========================================
    regs_dec<kRegsLow>();
    // Without the dQ part the whole warp runs the issue loop in step and elect.sync picks the
    // issuing lane (an MMA costs the warp 5-10 cycles this way, against about 50 from a lone
    // lane): +1.5-3% on the deterministic and dropout backward.  With dQ (the atomic
    // backward) that measured 0.5-1% slower, so there one lane issues.
    constexpr bool kElect = !DQ;
    if ((kElect || lane == 0) && T > 0) {
      auto wait_ = [&](uint32_t b, uint32_t par) -> bool {
        return kElect ? mbar_wait_warp(b, par, a.status) : mbar_wait(b, par, a.status);
      };
      auto mma_ss_ = [&](uint32_t d, uint32_t al, uint32_t bl, uint32_t hi, uint32_t id, uint32_t acc) {
        if constexpr (kElect) mma_ss_lo_elect(d, al, bl, hi, id, acc);
        else mma_ss_lo(d, al, bl, hi, id, acc);
      };
      auto mma_ts_ = [&](uint32_t d, uint32_t at, uint32_t bl, uint32_t hi, uint32_t id, uint32_t acc) {
        if constexpr (kElect) mma_ts_lo_elect(d, at, bl, hi, id, acc);
        else mma_ts_lo(d, at, bl, hi, id, acc);
      };
      auto commit_ = [&](uint32_t b) {
        if constexpr (kElect) mma_commit_elect(b);
        else mma_commit(b);
      };
      constexpr uint32_t id_s = idesc_of<Elem>(kBN, 64, 0, 0);    // S_h, dP_h: 128 keys x 64 queries
      constexpr uint32_t id_dv = idesc_of<Elem>(kBN, DV, 0, 1);   // P^T_h (TMEM) x dout_h (MN-major)
      constexpr uint32_t id_dk = idesc_of<Elem>(kBN, DK, 0, 1);   // dS^T_h (K-major) x Q_h (MN-major)
      constexpr uint32_t id_dq = idesc_of<Elem>(DK, 64, 1, 1);    // K^T (MN-major) x dS^T_h (MN-major)
      // S_h(t) = K Q_h^T -> S columns; dP_h(t) = V dout_h^T -> dP columns
      // Shared-memory descriptors, built once: an address offset is an addition to the start
      // field (addresses stay below 2^18 bytes, so the 14-bit field never carries).  "k" =
      // K-major view (LBO unused), "m" = MN-major view (LBO = the 16 KB between 64-column halves).
      // Start address and LBO sit in the low word; every descriptor shares the high word
      // (1024-byte stride, SW128), kept once in desc_hi, so each costs one register.
      const uint32_t desc_hi = (uint32_t)(smem_desc(sK, 16, 1024, kLayoutSwizzle128B) >> 32);
      const uint32_t kK = (uint32_t)smem_desc(sK, 16, 1024, kLayoutSwizzle128B);
      const uint32_t mK = (uint32_t)smem_desc(sK, L::kHalf, 1024, kLayoutSwizzle128B);
      const uint32_t kV = (uint32_t)smem_desc(sV, 16, 1024, kLayoutSwizzle128B);
      const uint32_t kQ = (uint32_t)smem_desc(sQ, 16, 1024, kLayoutSwizzle128B);
      const uint32_t mQ = (uint32_t)smem_desc(sQ, L::kHalf, 1024, kLayoutSwizzle128B);
      const uint32_t kO = (uint32_t)smem_desc(sO, 16, 1024, kLayoutSwizzle128B);
      const uint32_t mO = (uint32_t)smem_desc(sO, L::kHalf, 1024, kLayoutSwizzle128B);
      const uint32_t kDS = (uint32_t)smem_desc(sDS, 16, 1024, kLayoutSwizzle128B);
      const uint32_t mDS = (uint32_t)smem_desc(sDS, L::kHalf, 1024, kLayoutSwizzle128B);
      auto issue_sdp = [&](int t, int hh) -> bool {
        const int st = t & 1;
        const uint32_t qoff = (uint32_t)((st * L::kQBytes + hh * 8192) >> 4);
        const uint32_t ooff = (uint32_t)((st * L::kOBytes + hh * 8192) >> 4);
        const uint32_t cS = tmem + (hh ? kColSb : kColSa), cP = tmem + (hh ? kColDPb : kColDPa);
        if (hh == 0 && !wait_(bar.qd_full(st), (t >> 1) & 1)) return false;
        if (t >= 1 && !wait_(bar.dv_done(hh), (t - 1) & 1)) return false;   // P^T_h read
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < DK / 16; ++ks) {
          const uint32_t off16 = ((ks >> 2) * L::kHalf + (ks & 3) * 32) >> 4;
          mma_ss_(cS, kK + off16, kQ + qoff + off16, desc_hi, id_s, ks > 0);
        }
        if (DQ && t >= 1 && !wait_(bar.dq_free(hh), (t - 1) & 1)) return false;   // dQ^T_h read
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < DV / 16; ++ks) {
          const uint32_t off16 = ((ks >> 2) * L::kHalf + (ks & 3) * 32) >> 4;
          mma_ss_(cP, kV + off16, kO + ooff + off16, desc_hi, id_s, ks > 0);
        }
        commit_(bar.sdp_full(hh));
        return true;
      };
      auto issue_grads = [&](int t, int hh) {
        const int st = t & 1;
        const uint32_t qoff = (uint32_t)((st * L::kQBytes) >> 4), ooff = (uint32_t)((st * L::kOBytes) >> 4);
        const uint32_t dsoff = (uint32_t)((hh * L::kHalf) >> 4);
        const uint32_t cS = tmem + (hh ? kColSb : kColSa), cP = tmem + (hh ? kColDPb : kColDPa);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ts_(tmem + kColDV, cS + kk * 8, mO + ooff + (uint32_t)(((4 * hh + kk) * 2048) >> 4), desc_hi,
                          id_dv, (t > 0 || hh > 0 || kk > 0));
        commit_(bar.dv_done(hh));
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ss_(tmem + kColDK, kDS + dsoff + (uint32_t)((kk * 32) >> 4),
                          mQ + qoff + (uint32_t)(((4 * hh + kk) * 2048) >> 4), desc_hi, id_dk, (t > 0 || hh > 0 || kk > 0));
        if (DQ) {
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk)
            mma_ss_(cP, mK + (uint32_t)((kk * 2048) >> 4), mDS + dsoff + (uint32_t)((kk * 2048) >> 4), desc_hi, id_dq,
                            kk > 0);
          commit_(bar.dq_full(hh));
        }
        commit_(bar.ds_free(hh));
      };
      bool ok = wait_(bar.kv_full(), 0);
      if (ok) ok = issue_sdp(0, 0) && issue_sdp(0, 1);
      for (int t = 0; t < T && ok; ++t) {
        if (!(ok = wait_(bar.compute_done(0), t & 1))) break;
        tc_fence_after();
        issue_grads(t, 0);
        if (!(ok = wait_(bar.compute_done(1), t & 1))) break;
        tc_fence_after();
        if (t + 1 < T && !(ok = issue_sdp(t + 1, 0))) break;
        issue_grads(t, 1);
        commit_(bar.qd_empty(t & 1));
        if (t + 1 < T && !(ok = issue_sdp(t + 1, 1))) break;
      }
      commit_(bar.drain());
      wait_(bar.drain(), 0);
    }
  } else if (warp < 4) {
    regs_dec<kRegsLow>();   // warps 2-3: dropout keep flags (below), else no role
    if constexpr (DROP) {
      // Each half's 64 queries x 128 keys take 512 Philox calls (a call gives the bytes of 16
      // keys for one query).  Thread rt draws block blk = rt / 8 for queries u + 16 k,
      // u in {rt % 8, rt % 8 + 8}, k = 0..3, a half ahead of the compute warps, turns them
      // into drop flags and, once the half's dS staging area is free, writes there the
      // words [block][key tk][u] (byte k: query u + 16 k), then syncs on named barrier
      // 3 + half with the compute warps (64 + 128 threads).  Both sides take that barrier
      // exactly once per half, also after a timed-out wait, so its generations always pair
      // up; while the compute warps work on a half these warps draw the next one.
      const int rt = (warp - 2) * 32 + lane;
      bool ok = true;
      for (int t = 0; t < T; ++t) {
        const int h = head_of(t);
#pragma unroll 1
        for (int hh = 0; hh < 2; ++hh) {
          uint32_t fw[2][16];
          draw_flag_words64(a.drop, rt, n0 >> 4, q0 + qbase_of(t) + 64 * hh, h, fw);
          if (ok && t >= 1) ok = __all_sync(0xffffffffu, mbar_wait(bar.ds_free(hh), (t - 1) & 1, a.status));
          if (ok) store_flag_words64(sDS + hh * L::kHalf, rt, fw);
          named_bar_sync(3 + hh, 192);
        }
      }
    }
  } else if (warp < 8) {
    // ================================ compute warps (thread = key row) ===================
    regs_inc<kRegsHigh>();
    const int lg = warp & 3;
    const int r = lg * 32 + lane;
    const uint32_t lane_off = (uint32_t)(lg * 32) << 16;
    const long long j = n0 + r;
    const bool key_ok = j < sk;
    const float scale2 = a.scale * kLog2e;
    const long long off = sk - sq;
    bool ok = true;
    // lse_tot * log2e and D of query r of tile t, loaded one tile ahead
    float pf_lt = 0.f, pf_D = 0.f;
    auto prefetch = [&](int t) {
      const long long qi = qbase_of(t) + r;
      const long long idx = (long long)head_of(t) * a.total_q + q0 + qi;
      pf_lt = qi < sq ? a.lse_tot[idx] * kLog2e : 0.f;
      pf_D = qi < sq ? a.D[idx] : 0.f;
    };
    if (T > 0) prefetch(0);
    // The two named barriers below are hardware waits with no time limit, so every compute
    // warp passes both in every iteration: after a timed-out mbarrier wait a warp stops
    // working (ok = false) but never leaves the loop.
    for (int t = 0; t < T; ++t) {
      const int h = head_of(t);
      const long long i0 = qbase_of(t);
      // stage -lse_tot * log2e and -D of this tile's 128 queries (all 128 compute threads);
      // negated so that P's exponent and dP - D are single fused / packed operations
      named_bar_sync(1, 128);
      s_lt[r] = -pf_lt;
      s_D[r] = -pf_D;
      named_bar_sync(1, 128);
      if (t + 1 < T) prefetch(t + 1);   // in flight while this tile is computed
#pragma unroll 1
      for (int hh = 0; hh < 2; ++hh) {
        const uint32_t cS = hh ? kColSb : kColSa, cP = hh ? kColDPb : kColDPa;
        const long long qa = i0 + 64 * hh;
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar.sdp_full(hh), t & 1, a.status));
        if (ok && t >= 1) ok = __all_sync(0xffffffffu, mbar_wait(bar.ds_free(hh), (t - 1) & 1, a.status));
        if (ok) tc_fence_after();
        // The drop flags of this half, written by warps 2-3 into the (now free) dS staging
        // area: word [block][key t][u] holds, in byte k, the flag byte of query u + 16 k for
        // key t.  Both barriers are passed by every compute warp, also after a timed-out wait
        // (ok = false), like the named barriers of the tile loop.
        uint32_t zb[DROP ? 16 : 1];
        if constexpr (DROP) {
          named_bar_sync(3 + hh, 192);   // warps 2-3 have written this half's flags
          if (ok) read_flags64(sDS + hh * L::kHalf, r, zb);
          named_bar_sync(2, 128);   // every thread has its bytes before dS overwrites the area
        }
        if (!ok) continue;
        // every (key, query) pair of this half visible?  (then skip the per-element mask)
        bool full = (nkeys == kBN) && (qa + 63 < sq);
        if (a.right < kUnbounded) full = full && (n0 + kBN - 1 <= qa + off + a.right);
        if (a.left < kUnbounded) full = full && (n0 >= qa + 63 + off - a.left);
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
          uint32_t sv[32], dpv[32];
          tmem_ld32(tmem + lane_off + cS + c * 32, sv);
          tmem_ld32(tmem + lane_off + cP + c * 32, dpv);
          tmem_wait_ld();
          const int qc = 64 * hh + 32 * c;           // first query of the chunk within the tile
          float nlt[32], nd[32];   // -lse_tot * log2e, -D
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            const float4 x = *reinterpret_cast<const float4*>(s_lt + qc + e);
            const float4 y = *reinterpret_cast<const float4*>(s_D + qc + e);
            nlt[e] = x.x; nlt[e + 1] = x.y; nlt[e + 2] = x.z; nlt[e + 3] = x.w;
            nd[e] = y.x; nd[e + 1] = y.y; nd[e + 2] = y.z; nd[e + 3] = y.w;
          }
          float p[32], ds[32];
          if (full) {
            const float2 sc2 = make_float2(scale2, scale2);
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              const float2 x = ffma2(make_float2(__uint_as_float(sv[e]), __uint_as_float(sv[e + 1])), sc2,
                                     make_float2(nlt[e], nlt[e + 1]));
              p[e] = ex2(x.x);
              p[e + 1] = ex2(x.y);
            }
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const long long qi = i0 + qc + e;
              bool vis = key_ok && qi < sq;
              const long long d = j - (qi + off);
              if (a.right < kUnbounded) vis = vis && d <= a.right;
              if (a.left < kUnbounded) vis = vis && d >= -(long long)a.left;
              p[e] = vis ? ex2(fmaf(__uint_as_float(sv[e]), scale2, nlt[e])) : 0.f;
            }
          }
          if constexpr (DROP) {
            // dropout: dV takes the kept probabilities (its 256 / T scale is applied to the
            // result), dS = P (Z dP - D).  Query 32 c + e of the half is byte 2 c + e / 16 of
            // word e % 16; its flag widened to 32 bits clears a dropped element.
            const uint32_t sel0 = (8u | (2u * c)) * 0x1111u, sel1 = (8u | (2u * c + 1u)) * 0x1111u;
            const float zs = a.drop.scale;
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const uint32_t drop = prmt_sign_r(zb[e & 15], (e >> 4) ? sel1 : sel0);
              ds[e] = p[e] * fmaf(__uint_as_float(dpv[e] & ~drop), zs, nd[e]);
              p[e] = __uint_as_float(__float_as_uint(p[e]) & ~drop);
            }
          } else {
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              const float2 d = fmul2(make_float2(p[e], p[e + 1]),
                                     fadd2(make_float2(__uint_as_float(dpv[e]), __uint_as_float(dpv[e + 1])),
                                           make_float2(nd[e], nd[e + 1])));
              ds[e] = d.x;
              ds[e + 1] = d.y;
            }
          }
          uint32_t pk[16], dk_[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            pk[e] = pack2<Elem>(p[2 * e], p[2 * e + 1]);
            dk_[e] = pack2<Elem>(ds[2 * e], ds[2 * e + 1]);
          }
          tmem_st16(tmem + lane_off + cS + c * 16, pk);
          const uint32_t rowp = sDS + hh * L::kHalf + r * 128;
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const int ch = c * 4 + v;
            st_shared_v4(rowp + ((ch ^ (r & 7)) << 4), dk_[4 * v], dk_[4 * v + 1], dk_[4 * v + 2], dk_[4 * v + 3]);
          }
        }
        tmem_wait_st();
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar.compute_done(hh));
      }
    }
    // ---- epilogue: dK = scale * acc, dV = acc -------------------------------------------
    const bool have = __all_sync(0xffffffffu, ok && T > 0 && mbar_wait(bar.ds_free(1), (T - 1) & 1, a.status));
    tc_fence_after();
    Elem* dkp = static_cast<Elem*>(a.grad_k) + ((k0 + j) * a.hkv + g) * DK;
    Elem* dvp = static_cast<Elem*>(a.grad_v) + ((k0 + j) * a.hkv + g) * DVO;
#pragma unroll
    for (int pass = 0; pass < 2; ++pass) {
      const int ncol = pass == 0 ? DK : DVO;
      const uint32_t col = pass == 0 ? kColDK : kColDV;
      const float mul = pass == 0 ? a.scale : (DROP ? a.drop.scale : 1.f);
      uint4* dst = reinterpret_cast<uint4*>(pass == 0 ? dkp : dvp);
      for (int c = 0; c < ncol / 32; ++c) {
        uint32_t v[32];
        if (T > 0) {
          tmem_ld32(tmem + lane_off + col + c * 32, v);
          tmem_wait_ld();
        }
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float x0 = (T > 0 && have) ? __uint_as_float(v[2 * e]) * mul : 0.f;
          const float x1 = (T > 0 && have) ? __uint_as_float(v[2 * e + 1]) * mul : 0.f;
          pk[e] = pack2<Elem>(x0, x1);
        }
        const long long e0 = ((k0 + j) * a.hkv + g) * ncol + c * 32;
        if (key_ok && store_ok(e0, e0 + 31, (long long)a.total_k * a.hkv * ncol, a.status)) {
#pragma unroll
          for (int u = 0; u < 4; ++u) dst[c * 4 + u] = make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
        }
      }
    }
  } else {
    // ================================ dQ warps (thread = head-dim index) ==================
    regs_inc<kRegsHigh>();
    const int lg = warp & 3;
    const int d = lg * 32 + lane;                     // TMEM lane = head-dim index of dQ^T
    const uint32_t lane_off = (uint32_t)(lg * 32) << 16;
    bool ok = true;
    for (int t = 0; t < (DQ ? T : 0) && ok; ++t) {
      const int h = head_of(t);
      const long long i0 = qbase_of(t);
      for (int hh = 0; hh < 2; ++hh) {
        if (!__all_sync(0xffffffffu, mbar_wait(bar.dq_full(hh), t & 1, a.status))) { ok = false; break; }
        tc_fence_after();
        uint32_t v[64];
        tmem_ld32(tmem + lane_off + (hh ? kColDPb : kColDPa), *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
        tmem_ld32(tmem + lane_off + (hh ? kColDPb : kColDPa) + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar.dq_free(hh));
        // dq_acc is head-major, [hq][total_q][128]: consecutive queries of a head are 512
        // bytes apart, a compile-time stride that folds into each reduction's address.
        const long long qa = i0 + 64 * hh;
        const long long left = sq - qa;
        const int nval = left < 64 ? (int)left : 64;
        float* dst = a.dq_acc + ((long long)h * a.total_q + q0 + qa) * DK + d;
        const long long a0 = ((long long)h * a.total_q + q0 + qa) * DK + d;
        if (nval > 0 && !store_ok(a0, a0 + (long long)(nval - 1) * DK, (long long)a.hq * a.total_q * DK, a.status))
          continue;
#pragma unroll
        for (int e = 0; e < 64; ++e)
          if (e < nval) atomicAdd(dst + e * DK, __uint_as_float(v[e]) * a.scale);
      }
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

// dq = bf16(dq_acc), 8 elements per thread
template <typename T>
__global__ void dq_convert_kernel(const float* __restrict__ acc, T* __restrict__ dq, long long n8) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n8) return;
  const float4 x = reinterpret_cast<const float4*>(acc)[2 * i];
  const float4 y = reinterpret_cast<const float4*>(acc)[2 * i + 1];
  uint4 o;
  o.x = pack2<T>(x.x, x.y);
  o.y = pack2<T>(x.z, x.w);
  o.z = pack2<T>(y.x, y.y);
  o.w = pack2<T>(y.z, y.w);
  reinterpret_cast<uint4*>(dq)[i] = o;
}

// dq[t][h][:] = bf16(dq_acc[h][t][:]) for the head-major accumulator, 8 elements per thread.
template <typename T>
__global__ void dq_convert_hmajor_kernel(const float* __restrict__ acc, T* __restrict__ dq, int total_q,
                                         int hq, long long n8) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n8) return;
  const int c = (int)(i & 15);                      // 8-element chunk of the 128 dims
  const long long th = i >> 4;                      // t * hq + h (output order)
  const long long t = th / hq, h = th % hq;
  const float* src = acc + ((h * total_q + t) * 128 + c * 8);
  const float4 x = reinterpret_cast<const float4*>(src)[0];
  const float4 y = reinterpret_cast<const float4*>(src)[1];
  uint4 o;
  o.x = pack2<T>(x.x, x.y);
  o.y = pack2<T>(x.z, x.w);
  o.z = pack2<T>(y.x, y.y);
  o.w = pack2<T>(y.z, y.w);
  reinterpret_cast<uint4*>(dq)[i] = o;
}

template <typename T> constexpr int dtype_code();
template <> constexpr int dtype_code<__nv_bfloat16>() { return 0; }
template <> constexpr int dtype_code<__half>() { return 2; }

template <typename T, int DV, int DVO = DV>
cudaError_t launch_d128(const BwdArgs& a, cudaStream_t s) {
  using L = PLayout<DV>;
  constexpr CUtensorMapDataType dt = tma_dtype<T>();
  CUtensorMap tq, tk, tv, to;
  if (!make_map_3d(&tq, a.q, 128, a.hq, a.total_q, 128, dt) || !make_map_3d(&tk, a.k, 128, a.hkv, a.total_k, 128, dt) ||
      !make_map_3d(&tv, a.v, DVO, a.hkv, a.total_k, 128, dt) || !make_map_3d(&to, a.dout, DVO, a.hq, a.total_q, 128, dt))
    return cudaErrorInvalidValue;
  const bool dq = a.dq_acc != nullptr;
  cudaError_t e = dq ? cudaMemsetAsync(a.dq_acc, 0, (size_t)a.total_q * a.hq * 128 * sizeof(float), s) : cudaSuccess;
  if (e != cudaSuccess) return e;
  if ((e = launch_bwd_preprocess(a, dtype_code<T>(), s)) != cudaSuccess) return e;
  auto kernel = dq ? bwd_sm100_d128_kernel<T, DV, true, false, DVO>
                  : (a.drop.threshold ? bwd_sm100_d128_kernel<T, DV, false, true, DVO>
                                      : bwd_sm100_d128_kernel<T, DV, false, false, DVO>);
  if ((e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmem)) != cudaSuccess)
    return e;
  BwdArgs ab = a;
  ab.band_groups = bwd_band_groups(a);
  const long long ctas = (long long)a.hkv * a.batch * ((a.max_sk + kBN - 1) / kBN);
  kernel<<<(unsigned)ctas, kThreadsP, L::kSmem, s>>>(ab, tq, tk, tv, to);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (!dq) return cudaSuccess;
  const long long n8 = (long long)a.total_q * a.hq * 128 / 8;
  dq_convert_hmajor_kernel<T><<<(unsigned)((n8 + 255) / 256), 256, 0, s>>>(
      a.dq_acc, static_cast<T*>(a.grad_q), a.total_q, a.hq, n8);
  return cudaGetLastError();
}

template <typename T, int DK, int DV, int DVO = DV>
cudaError_t launch_typed(const BwdArgs& a, cudaStream_t s) {
  constexpr CUtensorMapDataType dt = tma_dtype<T>();
  CUtensorMap tq, tk, tv, to;
  if (!make_map_3d(&tq, a.q, DK, a.hq, a.total_q, 128, dt) || !make_map_3d(&tk, a.k, DK, a.hkv, a.total_k, 128, dt) ||
      !make_map_3d(&tv, a.v, DVO, a.hkv, a.total_k, 128, dt) || !make_map_3d(&to, a.dout, DVO, a.hq, a.total_q, 128, dt))
    return cudaErrorInvalidValue;
  const bool dq = a.dq_acc != nullptr;
  cudaError_t e = dq ? cudaMemsetAsync(a.dq_acc, 0, (size_t)a.total_q * a.hq * DK * sizeof(float), s) : cudaSuccess;
  if (e != cudaSuccess) return e;
  if ((e = launch_bwd_preprocess(a, dtype_code<T>(), s)) != cudaSuccess) return e;
  const bool drop = !dq && a.drop.threshold != 0;
  auto kernel = dq ? bwd_sm100_kernel<T, DK, DV, true, false, DVO>
                   : (drop ? bwd_sm100_kernel<T, DK, DV, false, true, DVO> : bwd_sm100_kernel<T, DK, DV, false, false, DVO>);
  const int smem = drop ? BLayout<DK, DV, true>::kSmem : BLayout<DK, DV>::kSmem;
  if ((e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) != cudaSuccess)
    return e;
  BwdArgs ab = a;
  ab.band_groups = bwd_band_groups(a);
  const long long ctas = (long long)a.hkv * a.batch * ((a.max_sk + kBN - 1) / kBN);
  kernel<<<(unsigned)ctas, kThreads, smem, s>>>(ab, tq, tk, tv, to);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (!dq) return cudaSuccess;
  const long long n8 = (long long)a.total_q * a.hq * DK / 8;
  dq_convert_kernel<T><<<(unsigned)((n8 + 255) / 256), 256, 0, s>>>(a.dq_acc, static_cast<T*>(a.grad_q), n8);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_dims(const BwdArgs& a, cudaStream_t s) {
  if (a.dk == 128 && a.dv == 128) return launch_d128<T, 128>(a, s);
  if (a.dk == 128 && a.dv == 64) return launch_d128<T, 64>(a, s);
  if (a.dk == 64 && a.dv == 64) return launch_typed<T, 64, 64>(a, s);
  if (a.dk == 64 && a.dv == 128) return launch_typed<T, 64, 128>(a, s);
  // dv = 32: 64-wide V / dout tiles over zero-filled columns
  if (a.dk == 128 && a.dv == 32) return launch_d128<T, 64, 32>(a, s);
  if (a.dk == 64 && a.dv == 32) return launch_typed<T, 64, 64, 32>(a, s);
  return cudaErrorInvalidValue;
}

}  // namespace

bool bwd_sm100_supported(const BwdArgs& a, int dtype) {
  if (dtype != 0 && dtype != 2) return false;
  if (!((a.dk == 64 || a.dk == 128) && (a.dv == 32 || a.dv == 64 || a.dv == 128))) return false;
  if ((long long)a.batch * a.hkv * ((a.max_sk + kBN - 1) / kBN) > 0x7fffffffLL) return false;  // 1-D grid
  return encode_fn() != nullptr;
}

cudaError_t launch_bwd_sm100(const BwdArgs& a, int dtype, cudaStream_t s) {
  return dtype == 2 ? launch_dims<__half>(a, s) : launch_dims<__nv_bfloat16>(a, s);
}

}  // namespace attn_sink
