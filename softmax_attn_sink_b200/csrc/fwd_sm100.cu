// Sink-attention forward on the sm_100a tensor cores (bf16 in, fp32 accumulation).
//
// What it computes (Huawei CANN ops-transformer flash_attn doc, "Function", the formula
// after "After adding sink"; softmax_lse formula of the same section):
//   S = scale * Q K^T,  m = max(sink, max S),
//   out = sum e^{S-m} V / (sum e^{S-m} + e^{sink-m}),   lse = log sum e^{S}  (no sink).
//
// A CTA owns two 128-row query units, A and B, that read the same K/V tiles: two q heads
// of one GQA group at the same row tile when the group size is even (identical key ranges),
// otherwise two adjacent row tiles of one head.  Keys are streamed in 128-key tiles over the
// union of the two units' visible ranges (bottom-right causal / sliding window, PyTorch
// issue #108108 "Proposal"; slime wrapper docstring "window_size"); each unit only takes the
// tiles that meet its own range.  Warp roles:
//   warp 0      TMA producer: Q_A, Q_B once, then K and V tiles into a 2-stage ring.
//   warp 1      TMEM allocation and the MMA issuer (one thread), in the order
//                 PV_A(j), QK_A(j+1), PV_B(j), QK_B(j+1)
//               so the tensor core works for one unit while the other unit's softmax runs.
//               QK: S_U = Q_U K^T (A, B from shared memory); PV: O_U += P_U V (P from TMEM).
//   warps 4-7   softmax of unit A, warps 8-11 softmax of unit B: thread t owns query row t
//               (TMEM lane t).  The running max starts at the sink (log2 domain, the sink is
//               in post-scale units); the running sum counts keys only and e^{sink-m} joins
//               the denominator in the epilogue, so the vanilla lse is m + log sum.  O is
//               rescaled lazily, only when a row's max grows by more than 2^8 (exact: O and
//               the sum share the stale reference).
// TMEM columns: S_A [0,128) O_A [128,256) S_B [256,384) O_B [384,512); P_U (bf16) is written
// over the first 64 columns of S_U once S_U has been read; the next QK_U into S_U is issued
// after the PV_U that reads it, and MMAs from one thread execute in issue order.  Because a
// commit tracks every earlier MMA of the thread, S_U(j) being ready also means PV_U(j-1) is
// done.  Every mbarrier wait is bounded; a timeout sets the status word and the CTA drains
// and frees its TMEM instead of hanging.
#include <cuda.h>

#include "sm100_ptx.cuh"

namespace attn_sink {
namespace {

using namespace sm100;

constexpr int kBM = 128;       // query rows per unit
constexpr int kBN = 128;       // keys per tile
constexpr int kStages = 2;     // K / V ring depth
constexpr int kThreads = 384;  // 3 warpgroups
// Registers: launched at 168 per thread (384 x 168 = 64512); the TMA/MMA warpgroup gives
// back down to 72 and the two softmax warpgroups take 216: 128 x 72 + 256 x 216 = 64512.
constexpr int kRegsLaunch = 168, kRegsProducer = 72, kRegsSoftmax = 216;
static_assert(128 * kRegsProducer + 256 * kRegsSoftmax <= kThreads * kRegsLaunch, "register split");
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

__host__ __device__ constexpr uint32_t col_S(int u) { return u ? 256u : 0u; }
__host__ __device__ constexpr uint32_t col_O(int u) { return u ? 384u : 128u; }

template <int DK, int DV>
struct Layout {
  static constexpr int KH = DK / 64, VH = DV / 64;           // 64-element (128-byte) column halves
  static constexpr int kHalfBytes = kBM * 128;               // one 128-row x 64-column box
  static constexpr int kQBytes = KH * kHalfBytes;
  static constexpr int kKBytes = KH * kHalfBytes;
  static constexpr int kVBytes = VH * kHalfBytes;
  static constexpr int kOffQ = 0;                             // Q_A, Q_B
  static constexpr int kOffK = kOffQ + 2 * kQBytes;
  static constexpr int kOffV = kOffK + kStages * kKBytes;
  static constexpr int kOffBar = kOffV + kStages * kVBytes;
  // q_full, k_full[S], k_empty[S], v_full[S], v_empty[S], s_full[2], p_full[2], pv_done[2], drain
  static constexpr int kNumBars = 1 + 4 * kStages + 6 + 1;
  static constexpr int kOffTmemSlot = kOffBar + kNumBars * 8;
  static constexpr int kBytes = kOffTmemSlot + 16;
  // + slack to align the base to 1 KB; at least 116 KB so that two CTAs never share an SM
  // (each CTA holds all 512 TMEM columns)
  static constexpr int kSmem = (kBytes + 1024) > 118784 ? (kBytes + 1024) : 118784;
};

// mbarrier addresses, laid out back to back from `base`.
struct Bars {
  uint32_t base;
  __device__ __forceinline__ uint32_t q_full() const { return base; }
  __device__ __forceinline__ uint32_t k_full(int s) const { return base + 8u * (1 + s); }
  __device__ __forceinline__ uint32_t k_empty(int s) const { return base + 8u * (1 + kStages + s); }
  __device__ __forceinline__ uint32_t v_full(int s) const { return base + 8u * (1 + 2 * kStages + s); }
  __device__ __forceinline__ uint32_t v_empty(int s) const { return base + 8u * (1 + 3 * kStages + s); }
  __device__ __forceinline__ uint32_t s_full(int u) const { return base + 8u * (1 + 4 * kStages + u); }
  __device__ __forceinline__ uint32_t p_full(int u) const { return base + 8u * (3 + 4 * kStages + u); }
  __device__ __forceinline__ uint32_t pv_done(int u) const { return base + 8u * (5 + 4 * kStages + u); }
  __device__ __forceinline__ uint32_t drain() const { return base + 8u * (7 + 4 * kStages); }
};

// One query unit of the CTA: q head, first row, rows, visible key range and the tiles of
// the CTA's key loop that meet it, [j0, j1).
struct Unit {
  int h;
  long long m0, nrows, lo, hi;
  int j0, j1;
  bool valid;
};

template <int DK, int DV>
__global__ void __launch_bounds__(kThreads, 1)
fwd_sm100_kernel(const FwdArgs a, const __grid_constant__ CUtensorMap tm_q,
                 const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v) {
  using L = Layout<DK, DV>;
  extern __shared__ unsigned char smem_raw[];

  // ---- work: two units; heaviest (largest) row tiles launch first ------------------------
  const int group = a.hq / a.hkv;
  const int b = blockIdx.y;
  const int zr = (int)gridDim.z - 1 - (int)blockIdx.z;
  int hA, hB, mA, mB;
  if ((group & 1) == 0) {
    const int g_ = blockIdx.x / (group / 2), p_ = blockIdx.x % (group / 2);
    hA = g_ * group + 2 * p_;
    hB = hA + 1;
    mA = mB = zr;
  } else {
    hA = hB = blockIdx.x;
    mA = 2 * zr;
    mB = 2 * zr + 1;
  }
  const long long q0 = a.cu_q[b], sq = a.cu_q[b + 1] - q0;
  const long long k0 = a.cu_k[b], sk = a.cu_k[b + 1] - k0;
  if ((long long)mA * kBM >= sq) return;  // unit B is never valid without unit A
  const int g = hA / group;

  Unit un[2];
  {
    const int hs[2] = {hA, hB}, ms[2] = {mA, mB};
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      Unit& x = un[u];
      x.h = hs[u];
      x.m0 = (long long)ms[u] * kBM;
      x.valid = x.m0 < sq;
      x.nrows = x.valid ? ((sq - x.m0 < kBM) ? sq - x.m0 : kBM) : 0;
      x.lo = x.hi = 0;
      if (x.valid) {
        long long l1, h1, l2, h2;
        row_key_range(x.m0, sq, sk, a.left, a.right, l1, h1);
        row_key_range(x.m0 + x.nrows - 1, sq, sk, a.left, a.right, l2, h2);
        x.lo = l1;
        x.hi = h2;  // ranges move right with the row: the union is [lo(first), hi(last))
        if (x.hi < x.lo) x.hi = x.lo;
      }
    }
  }
  long long lo = un[0].lo, hi = un[0].hi;
  if (un[1].valid && un[1].hi > un[1].lo) {
    if (hi <= lo) { lo = un[1].lo; hi = un[1].hi; }
    else { lo = lo < un[1].lo ? lo : un[1].lo; hi = hi > un[1].hi ? hi : un[1].hi; }
  }
  const int n_tiles = hi > lo ? (int)((hi - lo + kBN - 1) / kBN) : 0;
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    Unit& x = un[u];
    if (x.valid && x.hi > x.lo) {
      x.j0 = (int)((x.lo - lo) / kBN);
      x.j1 = (int)((x.hi - lo + kBN - 1) / kBN);
    } else {
      x.j0 = x.j1 = 0;
    }
  }

  const uint32_t base_u32 = (smem_addr(smem_raw) + 1023u) & ~1023u;
  unsigned char* smem = smem_raw + (base_u32 - smem_addr(smem_raw));
  const uint32_t sQ = base_u32 + L::kOffQ, sK = base_u32 + L::kOffK, sV = base_u32 + L::kOffV;
  const Bars bar{base_u32 + L::kOffBar};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kOffTmemSlot);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(bar.q_full(), 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar.k_full(s), 1);
      mbar_init(bar.k_empty(s), 1);
      mbar_init(bar.v_full(s), 1);
      mbar_init(bar.v_empty(s), 1);
    }
    for (int u = 0; u < 2; ++u) {
      mbar_init(bar.s_full(u), 1);
      mbar_init(bar.p_full(u), 4);   // one arrival per softmax warp of the unit
      mbar_init(bar.pv_done(u), 1);
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
  if (warp == 0) {
    // ================================ TMA producer ======================================
    regs_dec<kRegsProducer>();
    if (lane == 0 && n_tiles > 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      const int nq = un[1].valid ? 2 : 1;
      mbar_arrive_expect_tx(bar.q_full(), nq * L::kQBytes);
      for (int hf = 0; hf < L::KH; ++hf)
        tma_load_3d(sQ + hf * L::kHalfBytes, &tm_q, bar.q_full(), hf * 64, un[0].h, (int)(q0 + un[0].m0));
      if (nq == 2)
        for (int hf = 0; hf < L::KH; ++hf)
          tma_load_3d(sQ + L::kQBytes + hf * L::kHalfBytes, &tm_q, bar.q_full(), hf * 64, un[1].h,
                      (int)(q0 + un[1].m0));
      int issued = 0;
      for (int j = 0; j < n_tiles; ++j) {
        const int st = j % kStages;
        const uint32_t par = ((j / kStages) & 1) ^ 1;
        const int row = (int)(k0 + lo + (long long)j * kBN);
        if (!mbar_wait(bar.k_empty(st), par, a.status)) break;
        mbar_arrive_expect_tx(bar.k_full(st), L::kKBytes);
        for (int hf = 0; hf < L::KH; ++hf)
          tma_load_3d(sK + st * L::kKBytes + hf * L::kHalfBytes, &tm_k, bar.k_full(st), hf * 64, g, row);
        issued = j + 1;
        if (!mbar_wait(bar.v_empty(st), par, a.status)) break;
        mbar_arrive_expect_tx(bar.v_full(st), L::kVBytes);
        for (int hf = 0; hf < L::VH; ++hf)
          tma_load_3d(sV + st * L::kVBytes + hf * L::kHalfBytes, &tm_v, bar.v_full(st), hf * 64, g, row);
      }
      // make sure no copy is still landing in shared memory when the CTA exits
      mbar_wait(bar.q_full(), 0, a.status);
      for (int j = issued - kStages < 0 ? 0 : issued - kStages; j < issued; ++j) {
        mbar_wait(bar.k_full(j % kStages), (j / kStages) & 1, a.status);
        mbar_wait(bar.v_full(j % kStages), (j / kStages) & 1, a.status);
      }
    }
  } else if (warp == 1) {
    // ================================ MMA issuer =========================================
    regs_dec<kRegsProducer>();
    if (lane == 0 && n_tiles > 0) {
      constexpr uint32_t idesc_qk = idesc_bf16(kBM, kBN, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16(kBM, DV, 0, 1);
      bool ok = mbar_wait(bar.q_full(), 0, a.status);
      int k_waited = -1;  // last key tile whose K load we waited for
      // Shared-memory descriptors, built once: an address offset is an addition to the start
      // field (addresses stay below 2^18 bytes, so the 14-bit field never carries).
      const uint64_t dQ0 = smem_desc(sQ, 16, 1024, kLayoutSwizzle128B);
      const uint64_t dQ1 = dQ0 + (uint64_t)(L::kQBytes >> 4);
      const uint64_t dK0 = smem_desc(sK, 16, 1024, kLayoutSwizzle128B);
      const uint64_t dV0 = smem_desc(sV, L::kHalfBytes, 1024, kLayoutSwizzle128B);
      const int jA0 = un[0].j0, jA1 = un[0].j1, jB0 = un[1].j0, jB1 = un[1].j1;
      auto j0_of = [&](int u) { return u ? jB0 : jA0; };
      // S_u(j) = Q_u K_j^T
      auto issue_qk = [&](int u, int j) -> bool {
        const int st = j % kStages, jj = j - j0_of(u);
        if (k_waited < j) {
          if (!mbar_wait(bar.k_full(st), (j / kStages) & 1, a.status)) return false;
          k_waited = j;
        }
        (void)jj;
        // S_u is overwritten while P_u (inside S_u) was read by the previous PV_u: MMAs issued
        // by one thread execute in issue order, so that read is done before this write.
        tc_fence_after();
        const uint64_t dq = u ? dQ1 : dQ0, dk = dK0 + (uint64_t)(st * (L::kKBytes >> 4));
        const uint32_t dS = tmem + col_S(u);
#pragma unroll
        for (int ks = 0; ks < DK / 16; ++ks) {
          const uint32_t off16 = ((ks >> 2) * L::kHalfBytes + (ks & 3) * 32) >> 4;
          mma_ss(dS, dq + off16, dk + off16, idesc_qk, ks > 0);
        }
        mma_commit(bar.s_full(u));
        return true;
      };
      // O_u += P_u(j) V_j
      auto issue_pv = [&](int u, int j) -> bool {
        const int st = j % kStages, jj = j - j0_of(u);
        if (!mbar_wait(bar.p_full(u), jj & 1, a.status)) return false;
        tc_fence_after();
        const uint64_t dv = dV0 + (uint64_t)(st * (L::kVBytes >> 4));
        const uint32_t dO = tmem + col_O(u), aP = tmem + col_S(u);
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk)
          mma_ts(dO, aP + kk * 8, dv + (uint64_t)(kk * (2048 >> 4)), idesc_pv, (jj > 0 || kk > 0) ? 1u : 0u);
        mma_commit(bar.pv_done(u));
        return true;
      };
      auto active = [&](int u, int j) { return u ? (j >= jB0 && j < jB1) : (j >= jA0 && j < jA1); };
      for (int u = 0; u < 2 && ok; ++u)
        if (active(u, 0)) ok = issue_qk(u, 0);
      if (ok) mma_commit(bar.k_empty(0));
      for (int j = 0; j < n_tiles && ok; ++j) {
        const int st = j % kStages;
        if (!(ok = mbar_wait(bar.v_full(st), (j / kStages) & 1, a.status))) break;
        for (int u = 0; u < 2 && ok; ++u) {
          if (active(u, j)) ok = issue_pv(u, j);
          if (ok && j + 1 < n_tiles && active(u, j + 1)) ok = issue_qk(u, j + 1);
        }
        if (!ok) break;
        mma_commit(bar.v_empty(st));
        if (j + 1 < n_tiles) {
          // a tile no unit needs still has to be consumed for the producer's accounting
          if (k_waited < j + 1) {
            if (!(ok = mbar_wait(bar.k_full((j + 1) % kStages), ((j + 1) / kStages) & 1, a.status))) break;
            k_waited = j + 1;
          }
          mma_commit(bar.k_empty((j + 1) % kStages));
        }
      }
      // every MMA must be complete before the TMEM is freed
      mma_commit(bar.drain());
      mbar_wait(bar.drain(), 0, a.status);
    }
  } else if (warp < 4) {
    regs_dec<kRegsProducer>();   // warps 2-3: no role, but part of the first warpgroup
  } else {
    // ================================ softmax warpgroups =================================
    regs_inc<kRegsSoftmax>();
    const int u = warp < 8 ? 0 : 1;
    const Unit x = u ? un[1] : un[0];
    const int lg = warp & 3;                      // TMEM lane quarter this warp may access
    const int r = lg * 32 + lane;                 // row within the unit
    const uint32_t lane_off = (uint32_t)(lg * 32) << 16;
    const uint32_t tS = tmem + lane_off + col_S(u), tO = tmem + lane_off + col_O(u);
    const long long i = x.m0 + r;
    const bool row_ok = x.valid && i < sq;
    // this row's visible keys relative to the CTA's first key: [rlo, rhi) (empty if no row)
    int rlo = 0, rhi = 0;
    if (row_ok) {
      long long l_, h_;
      row_key_range(i, sq, sk, a.left, a.right, l_, h_);
      rlo = (int)(l_ - lo);
      rhi = (int)(h_ - lo);
    }
    const float sink2 = a.sink ? a.sink[x.h] * kLog2e : kNegInf;
    const float scale2 = a.scale * kLog2e;
    float m = sink2, l = 0.f;
    bool ok = true;
    const int nU = x.j1 - x.j0;

    for (int jj = 0; jj < nU; ++jj) {
      const int j = x.j0 + jj;
      if (!__all_sync(0xffffffffu, mbar_wait(bar.s_full(u), jj & 1, a.status))) { ok = false; break; }
      tc_fence_after();
      const int klo = rlo - j * kBN, khi = rhi - j * kBN;   // visible columns [klo, khi)
      const bool full = klo <= 0 && khi >= kBN;
      // the whole S row in one read (one TMEM round trip on the critical path)
      uint32_t sr[kBN];
#pragma unroll
      for (int c = 0; c < kBN / 32; ++c) tmem_ld32(tS + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
      tmem_wait_ld();
      if (!full) {
#pragma unroll
        for (int c = 0; c < kBN; ++c)
          if (c < klo || c >= khi) sr[c] = __float_as_uint(kNegInf);
      }
      // row max over 8 independent chains (a single chain would be 128 dependent steps)
      float mxv[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) mxv[e] = __uint_as_float(sr[e]);
#pragma unroll
      for (int c = 8; c < kBN; ++c) mxv[c & 7] = fmaxf(mxv[c & 7], __uint_as_float(sr[c]));
#pragma unroll
      for (int w = 4; w > 0; w >>= 1)
#pragma unroll
        for (int e = 0; e < w; ++e) mxv[e] = fmaxf(mxv[e], mxv[e + w]);
      const float mx = mxv[0];
      const float m_tile = mx * scale2;
      const bool need = m_tile > m + kRescaleThreshold;
      float alpha = 1.f;
      if (need) {
        alpha = (m == kNegInf) ? 0.f : ex2(m - m_tile);
        m = m_tile;
      }
      const bool any_rescale = __any_sync(0xffffffffu, need);
      // P = 2^{S scale log2e - m} as bf16, over S columns already read, 64 keys at a time.
      // Masked scores are -inf and 2^-inf = +0, so they need no test; m = -inf only when
      // every score is -inf (then neg_m = 0 keeps the argument -inf, not NaN).
      const float neg_m = (m == kNegInf) ? 0.f : -m;
      float sv[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t pk[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const float p0 = ex2(fmaf(__uint_as_float(sr[hh * 64 + 2 * c]), scale2, neg_m));
          const float p1 = ex2(fmaf(__uint_as_float(sr[hh * 64 + 2 * c + 1]), scale2, neg_m));
          sv[c & 3] += p0 + p1;
          pk[c] = pack_bf16x2(p0, p1);
        }
        tmem_st32(tS + hh * 32, pk);
      }
      const float sum = (sv[0] + sv[1]) + (sv[2] + sv[3]);
      l = l * alpha + sum;

      if (any_rescale && jj >= 1) {
        // O holds sum of the earlier P V: wait for the last of those MMAs, then scale rows
        if (!__all_sync(0xffffffffu, mbar_wait(bar.pv_done(u), (jj - 1) & 1, a.status))) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < DV / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + c * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(tO + c * 32, o);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar.p_full(u));
    }

    // ---- epilogue: out = O / (l + 2^{sink2 - m}),  lse = (m + log2 l) ln 2 -----------------
    const bool have_o = __all_sync(0xffffffffu, ok && nU > 0 &&
                                   mbar_wait(bar.pv_done(u), (nU - 1) & 1, a.status));
    tc_fence_after();
    const float e_sink = (sink2 == kNegInf || m == kNegInf) ? 0.f : ex2(sink2 - m);
    const float den = l + e_sink;
    const float inv = (den > 0.f && have_o) ? 1.f / den : 0.f;
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(a.out);
    uint4* orow = reinterpret_cast<uint4*>(out + ((q0 + i) * a.hq + x.h) * DV);
#pragma unroll
    for (int c = 0; c < DV / 32; ++c) {
      uint32_t o[32];
      if (nU > 0) {
        tmem_ld32(tO + c * 32, o);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) o[e] = 0u;
      }
      uint32_t pk[16];
#pragma unroll
      for (int e = 0; e < 16; ++e)
        pk[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv, __uint_as_float(o[2 * e + 1]) * inv);
      if (row_ok) {
#pragma unroll
        for (int v = 0; v < 4; ++v)
          orow[c * 4 + v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
      }
    }
    if (row_ok && a.lse)
      a.lse[(long long)x.h * a.total_q + q0 + i] = (l > 0.f && have_o) ? (m + __log2f(l)) * kLn2 : kNegInf;
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---- host: tensor maps and launch ----------------------------------------------------------

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// [rows, heads, d] bf16 viewed as a 3-D tensor (d innermost); boxes of 128 rows x 1 head x
// 64 columns (128 bytes), 128-byte swizzle; rows past the end read as zero.
bool make_map(CUtensorMap* map, const void* base, int d, int heads, int rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)heads, (cuuint64_t)rows};
  const cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)d * 2 * heads};
  const cuuint32_t box[3] = {64, 1, 128};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int DK, int DV>
cudaError_t launch_typed(const FwdArgs& a, cudaStream_t s) {
  using L = Layout<DK, DV>;
  CUtensorMap tq, tk, tv;
  if (!make_map(&tq, a.q, DK, a.hq, a.total_q) || !make_map(&tk, a.k, DK, a.hkv, a.total_k) ||
      !make_map(&tv, a.v, DV, a.hkv, a.total_k))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(fwd_sm100_kernel<DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       L::kSmem);
  if (e != cudaSuccess) return e;
  const int mtiles = (a.max_sq + kBM - 1) / kBM;
  const int group = a.hq / a.hkv;
  // two units per CTA: head pairs of a GQA group (even group size) or row-tile pairs
  dim3 grid = (group % 2 == 0) ? dim3(a.hq / 2, a.batch, mtiles) : dim3(a.hq, a.batch, (mtiles + 1) / 2);
  fwd_sm100_kernel<DK, DV><<<grid, kThreads, L::kSmem, s>>>(a, tq, tk, tv);
  return cudaGetLastError();
}

}  // namespace

bool fwd_sm100_supported(const FwdArgs& a, int dtype) {
  if (dtype != 0 || a.cu_q == nullptr) return false;
  if (!((a.dk == 64 || a.dk == 128) && (a.dv == 64 || a.dv == 128))) return false;
  if (a.batch > 65535 || (a.max_sq + kBM - 1) / kBM > 65535 || a.hq > 65535) return false;
  return encode_fn() != nullptr;
}

cudaError_t launch_fwd_sm100(const FwdArgs& a, cudaStream_t s) {
  if (a.dk == 128 && a.dv == 128) return launch_typed<128, 128>(a, s);
  if (a.dk == 128 && a.dv == 64) return launch_typed<128, 64>(a, s);
  if (a.dk == 64 && a.dv == 64) return launch_typed<64, 64>(a, s);
  if (a.dk == 64 && a.dv == 128) return launch_typed<64, 128>(a, s);
  return cudaErrorInvalidValue;
}

}  // namespace attn_sink
