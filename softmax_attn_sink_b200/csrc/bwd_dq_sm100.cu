// Query-stationary dQ for the deterministic backward on the sm_100a tensor cores.
//
// The gradient with respect to q of the sink attention (Huawei CANN ops-transformer
// flash_attn doc, "Function", the formula after "After adding sink"; its exact gradient,
// which the slime learnable_softmax_attention.py docstring states as
// dS = P * s * (D - s * di) with s = sigmoid(lse - sink)) is
//   dq_i = scale * sum_j dS_ij k_j,   dS_ij = P_ij (dP_ij - D_i),
//   P_ij = e^{scale q_i.k_j - lse_tot_i},  dP_ij = dout_i . v_j,  D_i = dout_i . out_i,
// with lse_tot = logaddexp(lse, sink) from the preprocess pass.  The key-stationary kernel
// adds dQ contributions of different key tiles with fp32 atomics, whose order varies from
// run to run.  Here one CTA owns a 128-row query tile of one q head and walks its visible
// key tiles in increasing order, accumulating dQ in TMEM, so every run adds the same
// numbers in the same order.
//
// Per key tile j (128 keys):
//   MMA thread:   S_j = Q K_j^T (SS, K-major) into S buffer j % 2, dP = dout V_j^T into
//                 the dP columns, and, once the compute warps wrote dS_j over S_j,
//                 dQ += dS_j K_j (A = dS from TMEM, B = K_j read MN-major from the same
//                 shared-memory tile).  Issue order: S(0), dP(0), then per tile
//                 S(j+1), [dS(j) written], dP(j+1), dQ(j): S(j+1) runs while the compute
//                 warps work on tile j, and they start on tile j+1 as soon as dP(j+1) is
//                 done, while dQ(j) runs.  K tiles go through a 3-stage ring (2 with
//                 dropout, whose keep-byte ring takes the room), V tiles through 2 stages.
//   compute warps (thread = query row, TMEM lane): two 64-key halves; P = 2^{S scale log2e
//                 - lse_tot log2e} (masked scores are -inf, so P = 0), dS = P (dP - D),
//                 rounded to the input type and written over the S columns of its half.
// TMEM columns: S buffer 0 [0,128), dP [128,256), dQ [256,256+DK), S buffer 1 [384,512).
// dS(j) sits in S buffer j % 2 until dQ(j) has read it; S(j+2) into the same buffer is
// issued after dQ(j) by the same thread, and MMAs from one thread execute in issue order.
// dP(j+1) overwrites dP(j) after the compute warps have signalled dS(j), so after their
// last read of it.  Every mbarrier wait is bounded; a timeout sets the
// status word and the CTA drains and frees its TMEM instead of hanging.
#include <cuda.h>

#include <type_traits>

#include "sm100_ptx.cuh"
#include "tma_map.h"

namespace attn_sink {
namespace {

using namespace sm100;

constexpr int kBM = 128;       // query rows per CTA
constexpr int kBN = 128;       // keys per tile
constexpr int kThreads = 256;  // warp 0 TMA, warp 1 MMA, warps 2-3 idle, warps 4-7 compute
// With dropout a fourth warpgroup (warps 8-11, one warp per SM sub-partition) draws the keep
// bytes of each key tile one tile ahead of the compute warps, into a two-stage shared-memory
// ring.  Launched at 168 registers (384 x 168 = 64512): the first warpgroup drops to 136, the
// dropout warpgroup to 120, the compute warps take 248 (128 x (136 + 120 + 248) = 64512; no
// spills, where 136 / 136 / 232 spilled 24 bytes).
constexpr int kThreadsDrop = 384;
constexpr int kRegsLowD = 136, kRegsFlagD = 120, kRegsHighD = 248;
static_assert(128 * (kRegsLowD + kRegsFlagD + kRegsHighD) <= kThreadsDrop * 168, "register split");
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColP = 128, kColQ = 256;
__host__ __device__ constexpr uint32_t col_S(int b) { return b ? 384u : 0u; }

template <int DK, int DV, bool DROP>
struct DqLayout {
  static constexpr int KH = DK / 64, VH = DV / 64;     // 64-element (128-byte) column halves
  static constexpr int kHalf = 128 * 128;              // one 128-row x 64-column box
  static constexpr int kQBytes = KH * kHalf, kOBytes = VH * kHalf;
  static constexpr int kKBytes = KH * kHalf, kVBytes = VH * kHalf;
  static constexpr int KS = DROP ? 2 : 3;              // K ring depth
  static constexpr int kOffQ = 0;
  static constexpr int kOffO = kOffQ + kQBytes;
  static constexpr int kOffK = kOffO + kOBytes;        // K ring, KS stages
  static constexpr int kOffV = kOffK + KS * kKBytes;   // V ring, 2 stages
  // dropout keep bytes, 2 stages x 128 rows x 128 keys; row r's 16-byte block u sits at
  // slot u ^ (r % 8), so that the compute warps' 16-byte row reads hit distinct banks
  static constexpr int kZStage = 128 * 128;
  static constexpr int kOffZ = kOffV + 2 * kVBytes;
  static constexpr int kOffBar = kOffZ + (DROP ? 2 * kZStage : 0);
  // qd_full, k_full[3], k_empty[3], v_full[2], v_empty[2], sdp_full, ds_full, dq_done, drain
  // (+ rng_full[2], rng_empty[2] with dropout)
  static constexpr int kNumBars = DROP ? 19 : 15;
  static constexpr int kOffSlot = kOffBar + kNumBars * 8;
  // + slack to align the base to 1 KB; at least 116 KB so two CTAs never share an SM (each
  // holds all 512 TMEM columns)
  static constexpr int kSmem = (kOffSlot + 16 + 1024) > 118784 ? (kOffSlot + 16 + 1024) : 118784;
};

struct DqBars {
  uint32_t base;
  __device__ __forceinline__ uint32_t qd_full() const { return base; }
  __device__ __forceinline__ uint32_t k_full(int s) const { return base + 8u * (1 + s); }
  __device__ __forceinline__ uint32_t k_empty(int s) const { return base + 8u * (4 + s); }
  __device__ __forceinline__ uint32_t v_full(int s) const { return base + 8u * (7 + s); }
  __device__ __forceinline__ uint32_t v_empty(int s) const { return base + 8u * (9 + s); }
  __device__ __forceinline__ uint32_t sdp_full() const { return base + 8u * 11; }
  __device__ __forceinline__ uint32_t ds_full() const { return base + 8u * 12; }
  __device__ __forceinline__ uint32_t dq_done() const { return base + 8u * 13; }
  __device__ __forceinline__ uint32_t drain() const { return base + 8u * 14; }
  __device__ __forceinline__ uint32_t rng_full(int s) const { return base + 8u * (15 + s); }
  __device__ __forceinline__ uint32_t rng_empty(int s) const { return base + 8u * (17 + s); }
};

// CTA -> (row tile m, sequence b, q head h): the deepest row tiles first (under a causal mask
// they see the most keys), heads fastest so the CTAs resident together share K/V tiles.
__device__ __forceinline__ void dq_tile_of(const BwdArgs& a, int mtiles, int& m, int& b, int& h) {
  const long long id = blockIdx.x;
  const long long per_level = (long long)a.batch * a.hq;
  const int zr = (int)(id / per_level);
  const int rem = (int)(id - (long long)zr * per_level);
  m = mtiles - 1 - zr;
  b = rem / a.hq;
  h = rem - b * a.hq;
}

template <typename Elem, int DK, int DV, bool DROP>
__global__ void __launch_bounds__(DROP ? kThreadsDrop : kThreads, 1)
bwd_dq_sm100_kernel(const BwdArgs a, const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_do) {
  using L = DqLayout<DK, DV, DROP>;
  extern __shared__ unsigned char smem_raw[];

  int m, b, h;
  dq_tile_of(a, (a.max_sq + kBM - 1) / kBM, m, b, h);
  const long long q0 = a.cu_q[b], sq = a.cu_q[b + 1] - q0;
  const long long k0 = a.cu_k[b], sk = a.cu_k[b + 1] - k0;
  const long long m0 = (long long)m * kBM;
  if (m0 >= sq) return;
  const int g = h / (a.hq / a.hkv);
  const long long nrows = (sq - m0 < kBM) ? sq - m0 : kBM;
  long long lo, hi, l2, h2;
  row_key_range(m0, sq, sk, a.left, a.right, lo, hi);
  row_key_range(m0 + nrows - 1, sq, sk, a.left, a.right, l2, h2);
  hi = h2 > lo ? h2 : lo;   // key ranges move right with the row: the union is [lo(first), hi(last))
  if (DROP && hi > lo) lo &= ~15LL;   // dropout draws keep bytes for 16-key blocks
  const int n = hi > lo ? (int)((hi - lo + kBN - 1) / kBN) : 0;

  const uint32_t base_u32 = (smem_addr(smem_raw) + 1023u) & ~1023u;
  unsigned char* smem = smem_raw + (base_u32 - smem_addr(smem_raw));
  const uint32_t sQ = base_u32 + L::kOffQ, sO = base_u32 + L::kOffO, sK = base_u32 + L::kOffK,
                 sV = base_u32 + L::kOffV, sZ = base_u32 + L::kOffZ;
  const DqBars bar{base_u32 + L::kOffBar};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kOffSlot);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(bar.qd_full(), 1);
    for (int s = 0; s < L::KS; ++s) {
      mbar_init(bar.k_full(s), 1);
      mbar_init(bar.k_empty(s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar.v_full(s), 1);
      mbar_init(bar.v_empty(s), 1);
    }
    mbar_init(bar.sdp_full(), 1);
    mbar_init(bar.ds_full(), 4);   // one arrival per compute warp
    mbar_init(bar.dq_done(), 1);
    mbar_init(bar.drain(), 1);
    if (DROP) {
      for (int s = 0; s < 2; ++s) {
        mbar_init(bar.rng_full(s), 128);    // every dropout thread, after storing its row
        mbar_init(bar.rng_empty(s), 128);   // every compute thread, after reading its row
      }
    }
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
    if constexpr (DROP) regs_dec<kRegsLowD>();
    if (lane == 0 && n > 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      const int row = (int)(q0 + m0);
      mbar_arrive_expect_tx(bar.qd_full(), L::kQBytes + L::kOBytes);
      for (int hf = 0; hf < L::KH; ++hf) tma_load_3d(sQ + hf * L::kHalf, &tm_q, bar.qd_full(), hf * 64, h, row);
      for (int hf = 0; hf < L::VH; ++hf) tma_load_3d(sO + hf * L::kHalf, &tm_do, bar.qd_full(), hf * 64, h, row);
      int nk = 0, nv = 0;   // tiles whose K / V loads were issued
      for (int j = 0; j < n; ++j) {
        const int sk_ = j % L::KS, sv_ = j & 1;
        const int krow = (int)(k0 + lo + (long long)j * kBN);
        if (!mbar_wait(bar.k_empty(sk_), ((j / L::KS) & 1) ^ 1, a.status)) break;
        mbar_arrive_expect_tx(bar.k_full(sk_), L::kKBytes);
        for (int hf = 0; hf < L::KH; ++hf)
          tma_load_3d(sK + sk_ * L::kKBytes + hf * L::kHalf, &tm_k, bar.k_full(sk_), hf * 64, g, krow);
        nk = j + 1;
        if (!mbar_wait(bar.v_empty(sv_), ((j >> 1) & 1) ^ 1, a.status)) break;
        mbar_arrive_expect_tx(bar.v_full(sv_), L::kVBytes);
        for (int hf = 0; hf < L::VH; ++hf)
          tma_load_3d(sV + sv_ * L::kVBytes + hf * L::kHalf, &tm_v, bar.v_full(sv_), hf * 64, g, krow);
        nv = j + 1;
      }
      // make sure no copy is still landing in shared memory when the CTA exits
      mbar_wait(bar.qd_full(), 0, a.status);
      for (int p = nk - L::KS < 0 ? 0 : nk - L::KS; p < nk; ++p)
        mbar_wait(bar.k_full(p % L::KS), (p / L::KS) & 1, a.status);
      for (int p = nv - 2 < 0 ? 0 : nv - 2; p < nv; ++p) mbar_wait(bar.v_full(p & 1), (p >> 1) & 1, a.status);
    }
  } else if (warp == 1) {
    // ================================ MMA issuer =========================================
    if constexpr (DROP) regs_dec<kRegsLowD>();
    // The whole warp runs the issue loop in step; elect.sync picks the issuing lane.
    if (n > 0) {
      constexpr uint32_t id_s = idesc_of<Elem>(kBM, kBN, 0, 0);   // S, dP: K-major A and B
      constexpr uint32_t id_q = idesc_of<Elem>(kBM, DK, 0, 1);    // dS (TMEM) x K (MN-major)
      // Shared-memory descriptors, built once; offsets add to the start field.  "k" = K-major
      // view, "m" = MN-major view (LBO = the 16 KB between 64-column halves).
      const uint64_t kQ = smem_desc(sQ, 16, 1024, kLayoutSwizzle128B);
      const uint64_t kO = smem_desc(sO, 16, 1024, kLayoutSwizzle128B);
      const uint64_t kK = smem_desc(sK, 16, 1024, kLayoutSwizzle128B);
      const uint64_t mK = smem_desc(sK, L::kHalf, 1024, kLayoutSwizzle128B);
      const uint64_t kV = smem_desc(sV, 16, 1024, kLayoutSwizzle128B);
      // S(j) = Q K_j^T into S buffer j % 2; that buffer's dS(j - 2) was read by dQ(j - 2),
      // issued earlier by this thread
      auto issue_s = [&](int j) -> bool {
        const int sk_ = j % L::KS;
        if (!mbar_wait_warp(bar.k_full(sk_), (j / L::KS) & 1, a.status)) return false;
        tc_fence_after();
        const uint64_t koff = (uint64_t)((sk_ * L::kKBytes) >> 4);
#pragma unroll
        for (int ks = 0; ks < DK / 16; ++ks) {
          const uint32_t off16 = ((ks >> 2) * L::kHalf + (ks & 3) * 32) >> 4;
          mma_ss_elect(tmem + col_S(j & 1), kQ + off16, kK + koff + off16, id_s, ks > 0);
        }
        return true;
      };
      // dP(j) = dout V_j^T; then V_j's stage is free and tile j's S and dP are announced
      auto issue_p = [&](int j) -> bool {
        const int sv_ = j & 1;
        if (!mbar_wait_warp(bar.v_full(sv_), (j >> 1) & 1, a.status)) return false;
        tc_fence_after();
        const uint64_t voff = (uint64_t)((sv_ * L::kVBytes) >> 4);
#pragma unroll
        for (int ks = 0; ks < DV / 16; ++ks) {
          const uint32_t off16 = ((ks >> 2) * L::kHalf + (ks & 3) * 32) >> 4;
          mma_ss_elect(tmem + kColP, kO + off16, kV + voff + off16, id_s, ks > 0);
        }
        mma_commit_elect(bar.v_empty(sv_));
        mma_commit_elect(bar.sdp_full());
        return true;
      };
      bool ok = mbar_wait_warp(bar.qd_full(), 0, a.status);
      if (ok) ok = issue_s(0) && issue_p(0);
      for (int j = 0; j < n && ok; ++j) {
        if (j + 1 < n && !(ok = issue_s(j + 1))) break;   // overlaps the compute warps' tile j
        // the compute warps have written dS(j) and are done reading dP(j)
        if (!(ok = mbar_wait_warp(bar.ds_full(), j & 1, a.status))) break;
        tc_fence_after();
        if (j + 1 < n && !(ok = issue_p(j + 1))) break;
        // dQ += dS(j) K_j, then K_j's stage is free
        const int sk_ = j % L::KS;
        const uint64_t koff = (uint64_t)((sk_ * L::kKBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk)
          mma_ts_elect(tmem + kColQ, tmem + col_S(j & 1) + kk * 8, mK + koff + (uint64_t)((kk * 2048) >> 4), id_q,
                 (j > 0 || kk > 0) ? 1u : 0u);
        mma_commit_elect(bar.k_empty(sk_));
      }
      if (ok) mma_commit_elect(bar.dq_done());
      // every MMA must be complete before the TMEM is freed
      mma_commit_elect(bar.drain());
      mbar_wait_warp(bar.drain(), 0, a.status);
    }
  } else if (warp < 4) {
    if constexpr (DROP) regs_dec<kRegsLowD>();   // warps 2-3: no role, but part of the first warpgroup
  } else if (warp < 8) {
    // ================================ compute warps (thread = query row) =================
    if constexpr (DROP) regs_inc<kRegsHighD>();
    const int lg = warp & 3;
    const int r = lg * 32 + lane;
    const uint32_t lane_off = (uint32_t)(lg * 32) << 16;
    const long long i = m0 + r;
    const bool row_ok = i < sq;
    int rlo = 0, rhi = 0;   // visible keys of this row relative to the first key of the loop
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
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      if (!__all_sync(0xffffffffu, mbar_wait(bar.sdp_full(), j & 1, a.status))) { ok = false; break; }
      if (DROP && !__all_sync(0xffffffffu, mbar_wait(bar.rng_full(j & 1), (j >> 1) & 1, a.status))) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t sv[64], pv[64];
        tmem_ld32(tmem + lane_off + col_S(j & 1) + hh * 64, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
        tmem_ld32(tmem + lane_off + col_S(j & 1) + hh * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
        tmem_ld32(tmem + lane_off + kColP + hh * 64, *reinterpret_cast<uint32_t(*)[32]>(&pv[0]));
        tmem_ld32(tmem + lane_off + kColP + hh * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&pv[32]));
        tmem_wait_ld();
        const int klo = rlo - j * kBN - hh * 64, khi = rhi - j * kBN - hh * 64;   // visible [klo, khi)
        if (!(klo <= 0 && khi >= 64)) {
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (c < klo || c >= khi) sv[c] = __float_as_uint(kNegInf);
        }
        uint32_t pk[32];
        // dropout: dS = P (Z dP - D) with Z = 256 / T for kept keys and 0 otherwise; the drop
        // flags of this row's keys [64 hh, 64 hh + 64), drawn by the dropout warps
        uint4 kb4[DROP ? 4 : 1];
        if constexpr (DROP) {
          const uint32_t zrow = sZ + (j & 1) * L::kZStage + r * 128;
#pragma unroll
          for (int gq = 0; gq < 4; ++gq)
            asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(kb4[gq].x), "=r"(kb4[gq].y), "=r"(kb4[gq].z), "=r"(kb4[gq].w)
                         : "r"(zrow + (((4 * hh + gq) ^ (r & 7)) << 4))
                         : "memory");
          if (hh == 1) mbar_arrive(bar.rng_empty(j & 1));
        }
        const float2 sc2 = make_float2(scale2, scale2), nlt2 = make_float2(neg_lt, neg_lt);
        const float2 nD2 = make_float2(-Dr, -Dr);
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          // P's exponent for two keys in one packed fused multiply-add
          const float2 x = ffma2(make_float2(__uint_as_float(sv[2 * c]), __uint_as_float(sv[2 * c + 1])), sc2, nlt2);
          const float p0 = ex2(x.x);
          const float p1 = ex2(x.y);
          if constexpr (DROP) {
            // keys 2c, 2c + 1: bytes 0-1 (c even) or 2-3 (c odd) of flag word c / 2
            const uint4 w4 = kb4[c >> 3];
            const int t = ((2 * c) & 15) >> 2;
            const uint32_t w = t == 0 ? w4.x : t == 1 ? w4.y : t == 2 ? w4.z : w4.w;
            const uint32_t d0 = (c & 1) ? prmt_sign<0xAAAA>(w) : prmt_sign<0x8888>(w);
            const uint32_t d1 = (c & 1) ? prmt_sign<0xBBBB>(w) : prmt_sign<0x9999>(w);
            pk[c] = pack2<Elem>(p0 * fmaf(__uint_as_float(pv[2 * c] & ~d0), a.drop.scale, -Dr),
                                p1 * fmaf(__uint_as_float(pv[2 * c + 1] & ~d1), a.drop.scale, -Dr));
          } else {
            const float2 d = fmul2(make_float2(p0, p1),
                                   fadd2(make_float2(__uint_as_float(pv[2 * c]), __uint_as_float(pv[2 * c + 1])), nD2));
            pk[c] = pack2<Elem>(d.x, d.y);
          }
        }
        // dS of keys [64 hh, 64 hh + 64) over S columns [32 hh, 32 hh + 32): half 0 goes over
        // S columns already read, half 1 over half 0's S columns
        tmem_st32(tmem + lane_off + col_S(j & 1) + hh * 32, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar.ds_full());
    }
    // ---- epilogue: dq = scale * dQ ------------------------------------------------------
    const bool have = __all_sync(0xffffffffu, ok && n > 0 && mbar_wait(bar.dq_done(), 0, a.status));
    tc_fence_after();
    Elem* dqp = static_cast<Elem*>(a.grad_q) + ((q0 + i) * a.hq + h) * DK;
#pragma unroll
    for (int c = 0; c < DK / 32; ++c) {
      uint32_t v[32];
      if (n > 0) {
        tmem_ld32(tmem + lane_off + kColQ + c * 32, v);
        tmem_wait_ld();
      }
      uint32_t pk[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float x0 = (n > 0 && have) ? __uint_as_float(v[2 * e]) * a.scale : 0.f;
        const float x1 = (n > 0 && have) ? __uint_as_float(v[2 * e + 1]) * a.scale : 0.f;
        pk[e] = pack2<Elem>(x0, x1);
      }
      const long long e0 = ((q0 + i) * a.hq + h) * DK + c * 32;
      if (row_ok && store_ok(e0, e0 + 31, (long long)a.total_q * a.hq * DK, a.status)) {
        uint4* dst = reinterpret_cast<uint4*>(dqp) + c * 4;
#pragma unroll
        for (int u = 0; u < 4; ++u) dst[u] = make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
      }
    }
  } else if constexpr (DROP) {
    // ================================ dropout warps (thread = query row) =================
    // Philox keep bytes of row r for the 8 16-key blocks of key tile j (counter: key block,
    // packed row, q head, offset), turned into drop flags (bit 7 of a byte set = dropped) and
    // stored for the compute thread of the same row.
    regs_dec<kRegsFlagD>();
    const int r = (warp - 8) * 32 + lane;
    const uint32_t row = (uint32_t)(q0 + m0 + r);
    const uint32_t t4 = (a.drop.threshold - 1u) * 0x01010101u, t4h = t4 | 0x80808080u;
    for (int j = 0; j < n; ++j) {
      const int st = j & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(bar.rng_empty(st), ((j >> 1) & 1) ^ 1, a.status))) break;
      const uint32_t kb0 = (uint32_t)((lo + (long long)j * kBN) >> 4);
      const uint32_t zrow = sZ + st * L::kZStage + r * 128;
#pragma unroll
      for (int gq = 0; gq < 8; ++gq) {
        const uint4 w = dropout_bytes(a.drop, kb0 + gq, row, (uint32_t)h);
        st_shared_v4(zrow + ((gq ^ (r & 7)) << 4), drop_flags4(w.x, t4, t4h), drop_flags4(w.y, t4, t4h),
                     drop_flags4(w.z, t4, t4h), drop_flags4(w.w, t4, t4h));
      }
      mbar_arrive(bar.rng_full(st));
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

// ---- host -----------------------------------------------------------------------------------

// DVO <= DV: the width of v and dout in memory; with DVO = 32 their tiles are 64-column boxes
// whose columns 32-63 the copies fill with zeros, which leaves dP = dout V^T exact.
template <typename Elem, int DK, int DV, int DVO = DV>
cudaError_t launch_typed(const BwdArgs& a, cudaStream_t s) {
  constexpr CUtensorMapDataType dt = tma_dtype<Elem>();
  CUtensorMap tq, tk, tv, to;
  if (!make_map_3d(&tq, a.q, DK, a.hq, a.total_q, 128, dt) || !make_map_3d(&tk, a.k, DK, a.hkv, a.total_k, 128, dt) ||
      !make_map_3d(&tv, a.v, DVO, a.hkv, a.total_k, 128, dt) || !make_map_3d(&to, a.dout, DVO, a.hq, a.total_q, 128, dt))
    return cudaErrorInvalidValue;
  const bool drop = a.drop.threshold != 0;
  auto kernel = drop ? bwd_dq_sm100_kernel<Elem, DK, DV, true> : bwd_dq_sm100_kernel<Elem, DK, DV, false>;
  const int smem = drop ? DqLayout<DK, DV, true>::kSmem : DqLayout<DK, DV, false>::kSmem;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const long long ctas = (long long)((a.max_sq + kBM - 1) / kBM) * a.batch * a.hq;
  kernel<<<(unsigned)ctas, drop ? kThreadsDrop : kThreads, smem, s>>>(a, tq, tk, tv, to);
  return cudaGetLastError();
}

template <typename Elem>
cudaError_t launch_dims(const BwdArgs& a, cudaStream_t s) {
  if (a.dk == 128 && a.dv == 128) return launch_typed<Elem, 128, 128>(a, s);
  if (a.dk == 128 && a.dv == 64) return launch_typed<Elem, 128, 64>(a, s);
  if (a.dk == 64 && a.dv == 64) return launch_typed<Elem, 64, 64>(a, s);
  if (a.dk == 64 && a.dv == 128) return launch_typed<Elem, 64, 128>(a, s);
  if (a.dk == 128 && a.dv == 32) return launch_typed<Elem, 128, 64, 32>(a, s);
  if (a.dk == 64 && a.dv == 32) return launch_typed<Elem, 64, 64, 32>(a, s);
  return cudaErrorInvalidValue;
}

}  // namespace

bool bwd_dq_sm100_supported(const BwdArgs& a, int dtype) {
  if (dtype != 0 && dtype != 2) return false;
  if (!((a.dk == 64 || a.dk == 128) && (a.dv == 32 || a.dv == 64 || a.dv == 128))) return false;
  if ((long long)((a.max_sq + kBM - 1) / kBM) * a.batch * a.hq > 0x7fffffffLL) return false;  // 1-D grid
  return encode_fn() != nullptr;
}

cudaError_t launch_bwd_dq_sm100(const BwdArgs& a, int dtype, cudaStream_t s) {
  return dtype == 2 ? launch_dims<__half>(a, s) : launch_dims<__nv_bfloat16>(a, s);
}

}  // namespace attn_sink
