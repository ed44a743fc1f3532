// Sink-attention forward on the sm_100a tensor cores (bf16 in, fp32 accumulation).
//
// What it computes (Huawei CANN ops-transformer flash_attn doc, "Function", the formula
// after "After adding sink"; softmax_lse formula of the same section):
//   S = scale * Q K^T,  m = max(sink, max S),
//   out = sum e^{S-m} V / (sum e^{S-m} + e^{sink-m}),   lse = log sum e^{S}  (no sink).
//
// One CTA owns a 128-row query tile of one (sequence, q head) and streams the 128-key
// tiles its rows can see (bottom-right causal / sliding window, PyTorch issue #108108
// "Proposal"; slime wrapper docstring "window_size").  Warp roles:
//   warp 0      TMA producer: Q once, then K and V tiles into a 2-stage ring (mbarriers).
//   warp 1      TMEM allocation and the MMA issuer (one thread):
//                 S_j = Q K_j^T   (tcgen05.mma, A and B from shared memory, D in TMEM)
//                 O  += P_j V_j   (tcgen05.mma, A = P from TMEM, B = V from shared memory)
//               S is double-buffered so Q K_{j+1}^T runs while the softmax works on S_j.
//   warps 2-5   softmax warpgroup: thread t owns query row t (TMEM lane t), so the row max
//               and row sum need no shuffles.  The running max starts at the sink (log2
//               domain: sink * log2 e -- the sink is in post-scale units); the running sum
//               counts keys only and e^{sink-m} joins the denominator in the epilogue, so
//               the vanilla lse falls out as m + log sum.  O is rescaled lazily: only when
//               a row's max grows by more than 2^8, which is exact because O and the sum
//               share the stale reference.
// TMEM columns: S0 [0,128) S1 [128,256) O [256,256+dv) P0 [384,448) P1 [448,512).
// Every mbarrier wait is bounded; a timeout sets the status word and the CTA drains and
// frees its TMEM instead of hanging.
#include <cuda.h>

#include "sm100_ptx.cuh"

namespace attn_sink {
namespace {

using namespace sm100;

constexpr int kBM = 128;       // query rows per tile
constexpr int kBN = 128;       // keys per tile
constexpr int kStages = 2;     // K / V ring depth
constexpr int kThreads = 192;  // 6 warps
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256, kColP0 = 384, kColP1 = 448;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

template <int DK, int DV>
struct Layout {
  static constexpr int KH = DK / 64, VH = DV / 64;           // 64-element (128-byte) column halves
  static constexpr int kHalfBytes = kBM * 128;               // one 128-row x 64-column box
  static constexpr int kQBytes = KH * kHalfBytes;
  static constexpr int kKBytes = KH * kHalfBytes;
  static constexpr int kVBytes = VH * kHalfBytes;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBytes;
  static constexpr int kOffV = kOffK + kStages * kKBytes;
  static constexpr int kOffBar = kOffV + kStages * kVBytes;
  // barriers: q_full, k_full[S], k_empty[S], v_full[S], v_empty[S], s_full[2], s_free[2],
  //           p_full[2], pv_done[2], drain
  static constexpr int kNumBars = 1 + 4 * kStages + 8 + 1;
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
  __device__ __forceinline__ uint32_t s_full(int i) const { return base + 8u * (1 + 4 * kStages + i); }
  __device__ __forceinline__ uint32_t s_free(int i) const { return base + 8u * (3 + 4 * kStages + i); }
  __device__ __forceinline__ uint32_t p_full(int i) const { return base + 8u * (5 + 4 * kStages + i); }
  __device__ __forceinline__ uint32_t pv_done(int i) const { return base + 8u * (7 + 4 * kStages + i); }
  __device__ __forceinline__ uint32_t drain() const { return base + 8u * (9 + 4 * kStages); }
};

template <int DK, int DV>
__global__ void __launch_bounds__(kThreads, 1)
fwd_sm100_kernel(const FwdArgs a, const __grid_constant__ CUtensorMap tm_q,
                 const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v) {
  using L = Layout<DK, DV>;
  extern __shared__ unsigned char smem_raw[];

  // ---- work unit: heaviest (largest) m-tiles launch first --------------------------------
  const int h = blockIdx.x, b = blockIdx.y;
  const int mt = (int)gridDim.z - 1 - (int)blockIdx.z;
  const long long q0 = a.cu_q[b], sq = a.cu_q[b + 1] - q0;
  const long long k0 = a.cu_k[b], sk = a.cu_k[b + 1] - k0;
  const long long m0 = (long long)mt * kBM;
  if (m0 >= sq) return;
  const int g = h / (a.hq / a.hkv);
  const long long nrows = (sq - m0 < kBM) ? sq - m0 : kBM;
  long long lo, hi, lo1, hi1;
  row_key_range(m0, sq, sk, a.left, a.right, lo, hi);
  row_key_range(m0 + nrows - 1, sq, sk, a.left, a.right, lo1, hi1);
  hi = hi1;  // visible ranges move right with the row, so the union is [lo(first), hi(last))
  const int n_tiles = hi > lo ? (int)((hi - lo + kBN - 1) / kBN) : 0;

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
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar.s_full(s), 1);
      mbar_init(bar.s_free(s), 4);   // one arrival per softmax warp
      mbar_init(bar.p_full(s), 4);
      mbar_init(bar.pv_done(s), 1);
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
    if (lane == 0 && n_tiles > 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      mbar_arrive_expect_tx(bar.q_full(), L::kQBytes);
      for (int hf = 0; hf < L::KH; ++hf)
        tma_load_3d(sQ + hf * L::kHalfBytes, &tm_q, bar.q_full(), hf * 64, h, (int)(q0 + m0));
      int issued = 0;
      bool ok = true;
      for (int j = 0; j < n_tiles && ok; ++j) {
        const int st = j % kStages;
        const uint32_t par = ((j / kStages) & 1) ^ 1;
        const int row = (int)(k0 + lo + (long long)j * kBN);
        ok = mbar_wait(bar.k_empty(st), par, a.status);
        if (!ok) break;
        mbar_arrive_expect_tx(bar.k_full(st), L::kKBytes);
        for (int hf = 0; hf < L::KH; ++hf)
          tma_load_3d(sK + st * L::kKBytes + hf * L::kHalfBytes, &tm_k, bar.k_full(st), hf * 64, g, row);
        ok = mbar_wait(bar.v_empty(st), par, a.status);
        if (!ok) { issued = j + 1; break; }
        mbar_arrive_expect_tx(bar.v_full(st), L::kVBytes);
        for (int hf = 0; hf < L::VH; ++hf)
          tma_load_3d(sV + st * L::kVBytes + hf * L::kHalfBytes, &tm_v, bar.v_full(st), hf * 64, g, row);
        issued = j + 1;
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
    if (lane == 0 && n_tiles > 0) {
      constexpr uint32_t idesc_qk = idesc_bf16(kBM, kBN, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16(kBM, DV, 0, 1);
      bool ok = mbar_wait(bar.q_full(), 0, a.status);
      auto issue_qk = [&](int j) -> bool {
        const int st = j % kStages, sb = j & 1;
        if (!mbar_wait(bar.k_full(st), (j / kStages) & 1, a.status)) return false;
        if (!mbar_wait(bar.s_free(sb), ((j >> 1) & 1) ^ 1, a.status)) return false;
        tc_fence_after();
        const uint32_t d = tmem + (sb ? kColS1 : kColS0);
#pragma unroll
        for (int ks = 0; ks < DK / 16; ++ks) {
          const uint32_t off = (ks >> 2) * L::kHalfBytes + (ks & 3) * 32;
          mma_ss(d, smem_desc(sQ + off, 16, 1024, kLayoutSwizzle128B),
                 smem_desc(sK + st * L::kKBytes + off, 16, 1024, kLayoutSwizzle128B), idesc_qk, ks > 0);
        }
        mma_commit(bar.s_full(sb));
        mma_commit(bar.k_empty(st));
        return true;
      };
      if (ok) ok = issue_qk(0);
      for (int j = 0; j < n_tiles && ok; ++j) {
        if (j + 1 < n_tiles) ok = issue_qk(j + 1);
        if (!ok) break;
        const int st = j % kStages, pb = j & 1;
        ok = mbar_wait(bar.p_full(pb), (j >> 1) & 1, a.status) &&
             mbar_wait(bar.v_full(st), (j / kStages) & 1, a.status);
        if (!ok) break;
        tc_fence_after();
        const uint32_t p_col = tmem + (pb ? kColP1 : kColP0);
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          // V tile: key rows of 128 bytes, 8-row swizzle atoms (1 KB apart), the two
          // 64-column halves 16 KB apart; 16 keys per MMA step.
          mma_ts(tmem + kColO, p_col + kk * 8,
                 smem_desc(sV + st * L::kVBytes + kk * 2048, L::kHalfBytes, 1024, kLayoutSwizzle128B),
                 idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(bar.pv_done(pb));
        mma_commit(bar.v_empty(st));
      }
      // every MMA must be complete before the TMEM is freed
      mma_commit(bar.drain());
      mbar_wait(bar.drain(), 0, a.status);
    }
  } else {
    // ================================ softmax warpgroup ==================================
    const int lg = warp & 3;                      // TMEM lane quarter this warp may access
    const int r = lg * 32 + lane;                 // row within the tile
    const uint32_t lane_off = (uint32_t)(lg * 32) << 16;
    const long long i = m0 + r;
    const bool row_ok = i < sq;
    long long rlo = 0, rhi = 0;
    if (row_ok) row_key_range(i, sq, sk, a.left, a.right, rlo, rhi);
    const float sink2 = a.sink ? a.sink[h] * kLog2e : kNegInf;
    const float scale2 = a.scale * kLog2e;
    float m = sink2, l = 0.f;
    bool ok = true;

    for (int j = 0; j < n_tiles; ++j) {
      const int sb = j & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(bar.s_full(sb), (j >> 1) & 1, a.status))) { ok = false; break; }
      tc_fence_after();
      uint32_t sr[kBN];
#pragma unroll
      for (int c = 0; c < kBN / 32; ++c) {
        uint32_t (&chunk)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]);
        tmem_ld32(tmem + lane_off + (sb ? kColS1 : kColS0) + c * 32, chunk);
      }
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar.s_free(sb));

      float* s = reinterpret_cast<float*>(sr);
      const long long n0 = lo + (long long)j * kBN;   // key index of column 0
      float mx = kNegInf;
      if (row_ok && n0 >= rlo && n0 + kBN <= rhi) {
#pragma unroll
        for (int c = 0; c < kBN; ++c) mx = fmaxf(mx, s[c]);
      } else {
#pragma unroll
        for (int c = 0; c < kBN; ++c) {
          const long long key = n0 + c;
          if (!(row_ok && key >= rlo && key < rhi)) s[c] = kNegInf;
          mx = fmaxf(mx, s[c]);
        }
      }
      const float m_tile = mx * scale2;
      const bool need = m_tile > m + kRescaleThreshold;
      float alpha = 1.f;
      if (need) {
        alpha = (m == kNegInf) ? 0.f : ex2(m - m_tile);
        m = m_tile;
      }
      const bool any_rescale = __any_sync(0xffffffffu, need);
      float sum = 0.f;
#pragma unroll
      for (int c = 0; c < kBN; ++c) {
        const float p = (s[c] == kNegInf) ? 0.f : ex2(fmaf(s[c], scale2, -m));
        s[c] = p;
        sum += p;
      }
      l = l * alpha + sum;

      // P_j goes to buffer sb: the MMA of P_{j-2} must have finished reading it
      if (j >= 2 && !__all_sync(0xffffffffu, mbar_wait(bar.pv_done(sb), ((j - 2) >> 1) & 1, a.status))) {
        ok = false;
        break;
      }
      if (any_rescale && j >= 1) {
        // O holds sum_{t<j} P_t V_t: wait for the last of those MMAs, then scale rows
        if (!__all_sync(0xffffffffu, mbar_wait(bar.pv_done((j - 1) & 1), ((j - 1) >> 1) & 1, a.status))) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < DV / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tmem + lane_off + kColO + c * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(tmem + lane_off + kColO + c * 32, o);
        }
      }
      uint32_t pk[kBN / 2];
#pragma unroll
      for (int c = 0; c < kBN / 2; ++c) pk[c] = pack_bf16x2(s[2 * c], s[2 * c + 1]);
#pragma unroll
      for (int c = 0; c < kBN / 64; ++c) {
        const uint32_t (&chunk)[32] = *reinterpret_cast<const uint32_t(*)[32]>(&pk[c * 32]);
        tmem_st32(tmem + lane_off + (sb ? kColP1 : kColP0) + c * 32, chunk);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar.p_full(sb));
    }

    // ---- epilogue: out = O / (l + 2^{sink2 - m}),  lse = (m + log2 l) ln 2 -----------------
    const bool have_o = __all_sync(0xffffffffu, ok && n_tiles > 0 &&
                                   mbar_wait(bar.pv_done((n_tiles - 1) & 1), ((n_tiles - 1) >> 1) & 1, a.status));
    tc_fence_after();
    const float e_sink = (sink2 == kNegInf || m == kNegInf) ? 0.f : ex2(sink2 - m);
    const float den = l + e_sink;
    const float inv = (den > 0.f && have_o) ? 1.f / den : 0.f;
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(a.out);
    uint4* orow = reinterpret_cast<uint4*>(out + ((q0 + i) * a.hq + h) * DV);
#pragma unroll
    for (int c = 0; c < DV / 32; ++c) {
      uint32_t o[32];
      if (n_tiles > 0) {
        tmem_ld32(tmem + lane_off + kColO + c * 32, o);
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
      a.lse[(long long)h * a.total_q + q0 + i] = (l > 0.f && have_o) ? (m + __log2f(l)) * kLn2 : kNegInf;
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
  dim3 grid(a.hq, a.batch, mtiles);
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
