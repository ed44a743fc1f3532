// Split-KV decode for bf16 and fp16: one query per sequence, GQA heads of a kv head together.  K/V
// are either packed ([total_k, hkv, d] with cu_seqlens_k) or paged ([num_blocks, block_size,
// hkv, d] with a block table and per-sequence key counts; CANN flash_attn doc, "Paged
// Attention Parameter Group" and the PA_BBND layout of k in its parameter table).
//
// Work unit: (sequence b, kv head g, block of up to 16 q heads of g's group, key chunk c).
// The visible keys of a decode query form one contiguous range [vlo, vhi) (bottom-right
// alignment puts the query at key position sk - 1; PyTorch issue #108108, "Benefits").
// That range is cut into fixed-size chunks, so every CTA streams the same number of K/V
// bytes whatever the sequence length.  A chunk produces, per q head, its local max m_c,
// local sum l_c and unnormalised output o_c -- WITHOUT the sink.  The merge kernel then
// combines the chunks through their maxima and applies the sink once:
//   m = max(sink, max_c m_c),  den = sum_c l_c e^{m_c - m} + e^{sink - m},
//   out = sum_c o_c e^{m_c - m} / den,  lse = log sum_c l_c e^{m_c - M} + M (no sink),
// the combination of partial results the CANN flash_attn doc describes for softmax_lse
// (note under "Return Value") and the sink formula of its "Function" section.
//
// Each key is read from HBM once per 16 q heads; K/V go HBM -> shared memory through a
// 3-stage cp.async pipeline (16-byte copies, XOR-swizzled rows so ldmatrix is
// conflict-free).  The two contractions per 16 keys (S = Q K^T over the head dim and
// O += P V over the keys) use m16n8k16 MMAs (bf16 or f16 inputs) with fp32 accumulation; the query
// heads form the M dimension.  S is summed over the head dim in independent partial sums (short
// dependency chains), and at head dim 256 two warps share each 16-key group, each computing the
// scores and half of the output columns.  Scores are kept in the log2 domain (scale * log2 e folded
// into one multiply) and exponentiated with ex2.approx.
#include <type_traits>

#include "common.cuh"

namespace attn_sink {
namespace {

constexpr int kKeyGroups = 4;      // 16-key groups of a stage
constexpr int kStageKeys = 64;     // keys per pipeline stage (16 per key group)
// pipeline depth: 3 stages (at head dim 256 64 KB a stage, 192 KB, one CTA per SM)
template <int DK, int DV>
__host__ __device__ constexpr int stages_of() { return 3; }
template <int DK, int DV>
__host__ __device__ constexpr int ctas_per_sm() { return DK + DV > 256 ? 1 : 2; }
// Warps of a CTA: one per key group, or at head dim 256 (one CTA per SM) two per key group,
// each computing the group's scores and half of its output columns, so that two warps per
// SM sub-partition hide each other's MMA and shared-memory latencies.
template <int DK, int DV>
__host__ __device__ constexpr int warps_of() { return DK + DV > 256 ? 8 : 4; }

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;   // 0 source bytes = zero-fill
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(n));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                            uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                                  uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// D += A B for one m16n8k16 tile with fp32 accumulation; A and B both bf16 or both f16.
template <typename T>
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  if constexpr (std::is_same<T, __half>::value)
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  else
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// physical 16-byte chunk of logical chunk c in a row of NCH chunks
template <int NCH>
__device__ __forceinline__ int swz(int row, int c) {
  constexpr int M = (NCH < 8 ? NCH : 8) - 1;
  return c ^ (row & M);
}

// Visible key range of the single decode query of sequence b.  Packed K/V: the sequence's
// keys start at row k0 = cu_k[b].  Paged K/V: k0 = 0 and the key count is seqused_k[b],
// clamped (with the status bit set) to what the sequence's block-table row can address.
__device__ __forceinline__ void decode_range(const DecodeArgs& a, int b, long long& k0,
                                             long long& vlo, long long& vhi) {
  long long sk;
  if (a.block_table) {
    k0 = 0;
    sk = a.seqused_k[b];
    const long long cap = (long long)a.max_blocks * a.block_size;
    if (sk < 0 || sk > cap) {
      set_status(a.status, kStatusBadIndex);
      sk = sk < 0 ? 0 : cap;
    }
  } else {
    k0 = a.cu_k[b];
    sk = a.cu_k[b + 1] - k0;
  }
  row_key_range(0, 1, sk, a.left, a.right, vlo, vhi);
}

// K/V addressing of the split kernel: packed rows, or a block table read from shared memory
// (the chunk's block ids staged once per CTA) or, when they do not fit, from global memory.
enum KvMode { kPacked = 0, kPagedSmemTable = 1, kPagedGlobalTable = 2 };

template <typename T, int DK, int DV, int MODE>
__global__ void __launch_bounds__(warps_of<DK, DV>() * 32, ctas_per_sm<DK, DV>()) decode_split_kernel(const DecodeArgs a,
                                                                                        int chunk, int extra_off) {
  constexpr int kStages = stages_of<DK, DV>();
  constexpr bool PAGED = MODE != kPacked;
  constexpr int KCH = DK / 8, VCH = DV / 8;        // 16-byte chunks per row
  constexpr int kThr = warps_of<DK, DV>() * 32;
  constexpr int DVW = DV * kKeyGroups / warps_of<DK, DV>();   // output columns per warp
  constexpr int KSTEPS = DK / 16, VTILES = DVW / 8;
  constexpr int STAGE_BYTES = kStageKeys * (DK + DV) * 2;
  extern __shared__ __align__(128) unsigned char smem[];

  const int c = blockIdx.x;
  const int group = a.hq / a.hkv;
  const int hblocks = (group + 15) / 16;
  const int g = blockIdx.y / hblocks, hb = blockIdx.y % hblocks;
  const int b = blockIdx.z;
  long long k0, vlo, vhi;
  decode_range(a, b, k0, vlo, vhi);
  const long long c_lo = vlo + (long long)c * chunk;
  if (c_lo >= vhi) return;
  const long long c_hi = (c_lo + chunk < vhi) ? c_lo + chunk : vhi;
  const int nkeys = (int)(c_hi - c_lo);
  const int nstages = (nkeys + kStageKeys - 1) / kStageKeys;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int kg = warp % kKeyGroups, dh = warp / kKeyGroups;   // key group, output-column half
  const int h_base = g * group + hb * 16;
  const int nh = (group - hb * 16) < 16 ? (group - hb * 16) : 16;
  const T* kp = static_cast<const T*>(a.k);
  const T* vp = static_cast<const T*>(a.v);
  const T* qp = static_cast<const T*>(a.q);
  // Paged K/V: the cache row of every key of a stage is computed once, by one thread per key,
  // into s_row (kStages stage slots of 64 rows, -1 = no key or a block id outside the cache)
  // one iteration before the stage's copies are issued; the copies then read it like the
  // packed path reads k0 + t.  With the shared-memory table, the chunk's block ids
  // [first block, last block] are staged once per CTA in s_blk.
  const unsigned bs = PAGED ? (unsigned)a.block_size : 1u;
  const bool bs_pow2 = (bs & (bs - 1)) == 0;
  const int bs_log2 = __ffs((int)bs) - 1;
  const long long blk_first = PAGED ? c_lo / bs : 0;
  long long* s_row = reinterpret_cast<long long*>(smem + extra_off);
  int* s_blk = reinterpret_cast<int*>(smem + extra_off + kStages * kStageKeys * 8);
  const int* trow = PAGED ? a.block_table + (long long)b * a.max_blocks : nullptr;
  if constexpr (MODE == kPagedSmemTable) {
    const int n_blk = (int)((c_hi - 1) / bs - blk_first + 1);
    for (int i = tid; i < n_blk; i += kThr) s_blk[i] = trow[blk_first + i];
    __syncthreads();
  }
  auto compute_rows = [&](int st) {
    if (tid < kStageKeys) {
      const long long t = c_lo + (long long)st * kStageKeys + tid;
      long long row = -1;
      if (t < c_hi) {
        const unsigned tu = (unsigned)t;   // keys are below 2^31
        const unsigned q = bs_pow2 ? tu >> bs_log2 : tu / bs;
        const int blk = (MODE == kPagedSmemTable) ? s_blk[q - (unsigned)blk_first] : trow[q];
        if ((unsigned)blk < (unsigned)a.num_blocks)
          row = (long long)blk * bs + (bs_pow2 ? (tu & (bs - 1)) : tu % bs);
        else
          set_status(a.status, kStatusBadIndex);
      }
      s_row[(st % kStages) * kStageKeys + tid] = row;
    }
  };
  if constexpr (PAGED) {
#pragma unroll
    for (int st = 0; st < kStages; ++st) compute_rows(st);
    __syncthreads();
  }

  auto issue_stage = [&](int st) {
    unsigned char* base = smem + (st % kStages) * STAGE_BYTES;
    const uint32_t k_s = smem_u32(base), v_s = smem_u32(base + kStageKeys * DK * 2);
    const long long t0 = c_lo + (long long)st * kStageKeys;
    if constexpr (!PAGED && KCH == VCH) {
      // K and V rows of a key coincide: one address per copy pair
      constexpr int NR = kStageKeys * KCH / kThr;
#pragma unroll
      for (int k = 0; k < NR; ++k) {
        const int idx = tid + k * kThr, r = idx / KCH, ch = idx % KCH;
        const bool ok = t0 + r < c_hi;
        const long long base = ((k0 + t0 + r) * a.hkv + g) * DK + ch * 8;
        cp_async16(k_s + (r * KCH + swz<KCH>(r, ch)) * 16, ok ? kp + base : kp, ok);
        cp_async16(v_s + (r * VCH + swz<VCH>(r, ch)) * 16, ok ? vp + base : vp, ok);
      }
    } else if constexpr (!PAGED) {
      for (int idx = tid; idx < kStageKeys * KCH; idx += kThr) {
        const int r = idx / KCH, ch = idx % KCH;
        const bool ok = t0 + r < c_hi;
        const T* src = ok ? kp + ((k0 + t0 + r) * a.hkv + g) * DK + ch * 8 : kp;
        cp_async16(k_s + (r * KCH + swz<KCH>(r, ch)) * 16, src, ok);
      }
      for (int idx = tid; idx < kStageKeys * VCH; idx += kThr) {
        const int r = idx / VCH, ch = idx % VCH;
        const bool ok = t0 + r < c_hi;
        const T* src = ok ? vp + ((k0 + t0 + r) * a.hkv + g) * DV + ch * 8 : vp;
        cp_async16(v_s + (r * VCH + swz<VCH>(r, ch)) * 16, src, ok);
      }
    } else if constexpr (KCH == VCH && DK <= 128) {
      // K and V rows of a key coincide: every row this thread copies is read from shared
      // memory first, all loads before the first copy, then K and V are issued from them
      constexpr int NR = kStageKeys * KCH / kThr;
      const long long* rows = s_row + (st % kStages) * kStageKeys;
      long long rw[NR];
#pragma unroll
      for (int k = 0; k < NR; ++k) rw[k] = rows[(tid + k * kThr) / KCH];
#pragma unroll
      for (int k = 0; k < NR; ++k) {
        const int idx = tid + k * kThr, r = idx / KCH, ch = idx % KCH;
        const bool ok = rw[k] >= 0;
        const long long base = (rw[k] * a.hkv + g) * DK + ch * 8;
        cp_async16(k_s + (r * KCH + swz<KCH>(r, ch)) * 16, ok ? kp + base : kp, ok);
        cp_async16(v_s + (r * VCH + swz<VCH>(r, ch)) * 16, ok ? vp + base : vp, ok);
      }
    } else {
      const long long* rows = s_row + (st % kStages) * kStageKeys;
      for (int idx = tid; idx < kStageKeys * KCH; idx += kThr) {
        const int r = idx / KCH, ch = idx % KCH;
        const long long row = rows[r];
        const bool ok = row >= 0;
        const T* src = ok ? kp + (row * a.hkv + g) * DK + ch * 8 : kp;
        cp_async16(k_s + (r * KCH + swz<KCH>(r, ch)) * 16, src, ok);
      }
      for (int idx = tid; idx < kStageKeys * VCH; idx += kThr) {
        const int r = idx / VCH, ch = idx % VCH;
        const long long row = rows[r];
        const bool ok = row >= 0;
        const T* src = ok ? vp + (row * a.hkv + g) * DV + ch * 8 : vp;
        cp_async16(v_s + (r * VCH + swz<VCH>(r, ch)) * 16, src, ok);
      }
    }
  };

#pragma unroll
  for (int st = 0; st < kStages - 1; ++st) {
    if (st < nstages) issue_stage(st);
    cp_async_commit();
  }

  // Q as A fragments (rows = q heads of this block; rows >= nh are zero)
  uint32_t qa[KSTEPS][4];
  {
    const int r0 = lane >> 2, r1 = r0 + 8, cc = (lane & 3) * 2;
#pragma unroll
    for (int ks = 0; ks < KSTEPS; ++ks) {
      auto ld = [&](int r, int col) -> uint32_t {
        if (r >= nh) return 0u;
        return *reinterpret_cast<const uint32_t*>(qp + ((long long)b * a.hq + h_base + r) * DK + col);
      };
      qa[ks][0] = ld(r0, ks * 16 + cc);
      qa[ks][1] = ld(r1, ks * 16 + cc);
      qa[ks][2] = ld(r0, ks * 16 + cc + 8);
      qa[ks][3] = ld(r1, ks * 16 + cc + 8);
    }
  }

  const float scale_log2 = a.scale * kLog2e;
  float m_run[2] = {kNegInf, kNegInf};   // rows lane/4 and lane/4 + 8, log2 domain
  float l_run[2] = {0.f, 0.f};           // per-thread partial sums
  float o_acc[VTILES][4];
#pragma unroll
  for (int nt = 0; nt < VTILES; ++nt) o_acc[nt][0] = o_acc[nt][1] = o_acc[nt][2] = o_acc[nt][3] = 0.f;

  for (int st = 0; st < nstages; ++st) {
    cp_async_wait<kStages - 2>();
    __syncthreads();
    if (st + kStages - 1 < nstages) issue_stage(st + kStages - 1);
    cp_async_commit();
    // the slot of stage st (issued two iterations ago) now takes stage st + kStages's rows;
    // the barrier at the top of the next iteration orders these writes before their reads
    if constexpr (PAGED)
      if (st + kStages < nstages) compute_rows(st + kStages);

    const unsigned char* base = smem + (st % kStages) * STAGE_BYTES;
    const uint32_t k_s = smem_u32(base), v_s = smem_u32(base + kStageKeys * DK * 2);
    const int key0 = kg * 16;                         // this warp's 16 keys of the stage
    const long long t_abs = c_lo + (long long)st * kStageKeys + key0;
    if (t_abs >= c_hi) continue;                      // warp-uniform: nothing left for this warp

    // S = Q K^T  (two n8 tiles of 8 keys)
    constexpr int NP = KSTEPS >= 8 ? 4 : 2;   // independent partial sums over the head dim
    float sp[NP][2][4];
#pragma unroll
    for (int q_ = 0; q_ < NP; ++q_)
#pragma unroll
      for (int e = 0; e < 4; ++e) sp[q_][0][e] = sp[q_][1][e] = 0.f;
#pragma unroll
    for (int ks = 0; ks < KSTEPS; ++ks) {
      const int mi = lane >> 3, rr = lane & 7;
      const int row = key0 + (mi >> 1) * 8 + rr;
      const int ch = ks * 2 + (mi & 1);
      uint32_t b0, b1, b2, b3;
      ldmatrix_x4(k_s + (row * KCH + swz<KCH>(row, ch)) * 16, b0, b1, b2, b3);
      mma16816<T>(sp[ks % NP][0], qa[ks], b0, b1);
      mma16816<T>(sp[ks % NP][1], qa[ks], b2, b3);
    }
    float s[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float acc = sp[0][nt][e];
#pragma unroll
        for (int q_ = 1; q_ < NP; ++q_) acc += sp[q_][nt][e];
        s[nt][e] = acc;
      }
    // mask keys past the chunk end, online softmax in the log2 domain
    const int kc = (lane & 3) * 2;
    float mx[2] = {kNegInf, kNegInf};
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const long long t = t_abs + nt * 8 + kc + (e & 1);
        s[nt][e] = (t < c_hi) ? s[nt][e] * scale_log2 : kNegInf;
        mx[e >> 1] = fmaxf(mx[e >> 1], s[nt][e]);
      }
    float alpha[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
      const float m_new = fmaxf(m_run[r], mx[r]);
      alpha[r] = (m_run[r] == kNegInf) ? 0.f : ex2(m_run[r] - m_new);
      if (m_new == kNegInf) alpha[r] = 1.f;
      m_run[r] = m_new;
    }
    float p[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float m = m_run[e >> 1];
        p[nt][e] = (s[nt][e] == kNegInf) ? 0.f : ex2(s[nt][e] - m);
      }
#pragma unroll
    for (int r = 0; r < 2; ++r)
      l_run[r] = l_run[r] * alpha[r] + p[0][2 * r] + p[0][2 * r + 1] + p[1][2 * r] + p[1][2 * r + 1];
#pragma unroll
    for (int nt = 0; nt < VTILES; ++nt) {
      o_acc[nt][0] *= alpha[0];
      o_acc[nt][1] *= alpha[0];
      o_acc[nt][2] *= alpha[1];
      o_acc[nt][3] *= alpha[1];
    }
    uint32_t pa[4];
    pa[0] = pack2<T>(p[0][0], p[0][1]);
    pa[1] = pack2<T>(p[0][2], p[0][3]);
    pa[2] = pack2<T>(p[1][0], p[1][1]);
    pa[3] = pack2<T>(p[1][2], p[1][3]);
    // O += P V
#pragma unroll
    for (int ntp = 0; ntp < VTILES / 2; ++ntp) {
      const int mi = lane >> 3, rr = lane & 7;
      const int row = key0 + (mi & 1) * 8 + rr;
      const int ch = dh * (DVW / 8) + ntp * 2 + (mi >> 1);
      uint32_t b0, b1, b2, b3;
      ldmatrix_x4_trans(v_s + (row * VCH + swz<VCH>(row, ch)) * 16, b0, b1, b2, b3);
      mma16816<T>(o_acc[2 * ntp], pa, b0, b1);
      mma16816<T>(o_acc[2 * ntp + 1], pa, b2, b3);
    }
  }
  cp_async_wait<0>();
  __syncthreads();

  // combine the key groups' states through shared memory (the stage buffers are free now);
  // the two warps of a key group at head dim 256 hold the same max and sum
  float* s_o = reinterpret_cast<float*>(smem);                 // [kKeyGroups][16][DV]
  float* s_m = s_o + kKeyGroups * 16 * DV;                      // [kKeyGroups][16]
  float* s_l = s_m + kKeyGroups * 16;                           // [kKeyGroups][16]
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    float l = l_run[r];
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    const int row = (lane >> 2) + r * 8;
    if ((lane & 3) == 0 && dh == 0) {
      s_m[kg * 16 + row] = m_run[r];
      s_l[kg * 16 + row] = l;
    }
  }
#pragma unroll
  for (int nt = 0; nt < VTILES; ++nt) {
    const int col = dh * DVW + nt * 8 + (lane & 3) * 2, row = lane >> 2;
    s_o[(kg * 16 + row) * DV + col] = o_acc[nt][0];
    s_o[(kg * 16 + row) * DV + col + 1] = o_acc[nt][1];
    s_o[(kg * 16 + row + 8) * DV + col] = o_acc[nt][2];
    s_o[(kg * 16 + row + 8) * DV + col + 1] = o_acc[nt][3];
  }
  __syncthreads();
  for (int idx = tid; idx < nh * DV; idx += kThr) {
    const int row = idx / DV, col = idx % DV;
    float m = kNegInf;
#pragma unroll
    for (int w = 0; w < kKeyGroups; ++w) m = fmaxf(m, s_m[w * 16 + row]);
    float o = 0.f, l = 0.f;
    if (m != kNegInf) {
#pragma unroll
      for (int w = 0; w < kKeyGroups; ++w) {
        const float mw = s_m[w * 16 + row];
        const float f = (mw == kNegInf) ? 0.f : ex2(mw - m);
        o += f * s_o[(w * 16 + row) * DV + col];
        l += f * s_l[w * 16 + row];
      }
    }
    const long long pidx = ((long long)b * a.hq + h_base + row) * a.splits + c;
    const long long nrows = (long long)a.batch * a.hq * a.splits;
    if (!store_ok(pidx, pidx, nrows, a.status)) continue;
    a.part_o[pidx * DV + col] = o;
    if (col == 0) {
      a.part_ml[pidx * 2 + 0] = m;
      a.part_ml[pidx * 2 + 1] = l;
    }
  }
}

// One warp per (sequence, q head): merge the chunks of that row, apply the sink once.
template <typename T, int DV>
__global__ void __launch_bounds__(128) decode_merge_kernel(const DecodeArgs a, int chunk) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * 4 + warp;   // b * hq + h
  if (row >= (long long)a.batch * a.hq) return;
  const int b = (int)(row / a.hq), h = (int)(row % a.hq);
  long long k0, vlo, vhi;
  decode_range(a, b, k0, vlo, vhi);
  int n = vhi > vlo ? (int)((vhi - vlo + chunk - 1) / chunk) : 0;
  if (n > a.splits) {  // more keys than max_seqlen_k announced: only a.splits chunks exist
    set_status(a.status, kStatusBadIndex);
    n = a.splits;
  }
  const float* ml = a.part_ml + row * a.splits * 2;
  float M = kNegInf;
  for (int c = lane; c < n; c += 32) M = fmaxf(M, ml[2 * c]);
  M = warp_max(M);
  const float sink2 = a.sink ? a.sink[h] * kLog2e : kNegInf;
  const float m = fmaxf(M, sink2);
  constexpr int VPL = DV / 32;
  float o[VPL];
#pragma unroll
  for (int j = 0; j < VPL; ++j) o[j] = 0.f;
  float lM = 0.f, lm = 0.f;
  for (int c = 0; c < n; ++c) {
    const float mc = ml[2 * c], lc = ml[2 * c + 1];
    if (mc == kNegInf) continue;
    const float w = ex2(mc - m);
    lm += lc * w;
    lM += lc * ex2(mc - M);
    const float* oc = a.part_o + (row * a.splits + c) * DV;
#pragma unroll
    for (int j = 0; j < VPL; ++j) o[j] = fmaf(w, oc[lane + 32 * j], o[j]);
  }
  const float den = lm + ((sink2 == kNegInf || m == kNegInf) ? 0.f : ex2(sink2 - m));
  const float inv = den > 0.f ? 1.f / den : 0.f;
  T* out = static_cast<T*>(a.out);
  if (!store_ok(row * DV, row * DV + DV - 1, (long long)a.batch * a.hq * DV, a.status)) return;
#pragma unroll
  for (int j = 0; j < VPL; ++j) out[row * DV + lane + 32 * j] = from_float<T>(o[j] * inv);
  if (a.lse && lane == 0)
    a.lse[(long long)h * a.batch + b] = (M == kNegInf || lM <= 0.f) ? kNegInf : (M + __log2f(lM)) * kLn2;
}

template <typename T, int DK, int DV, int MODE>
cudaError_t launch_split(const DecodeArgs& a, int chunk, int smem, int extra_off, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(decode_split_kernel<T, DK, DV, MODE>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int group = a.hq / a.hkv;
  dim3 grid(a.splits, a.hkv * ((group + 15) / 16), a.batch);
  decode_split_kernel<T, DK, DV, MODE><<<grid, warps_of<DK, DV>() * 32, smem, s>>>(a, chunk, extra_off);
  return cudaGetLastError();
}

template <typename T, int DK, int DV>
cudaError_t launch_typed(const DecodeArgs& a, cudaStream_t s) {
  const int group = a.hq / a.hkv;
  const int hblocks = (group + 15) / 16;
  // chunk length so that `splits` chunks cover the longest visible range
  const int chunk = (a.max_sk + a.splits - 1) / a.splits;
  constexpr int STAGE_BYTES = kStageKeys * (DK + DV) * 2;
  constexpr int kStages = stages_of<DK, DV>();
  constexpr int PIPE = kStages * STAGE_BYTES;
  constexpr int COMBINE = kKeyGroups * 16 * (DV + 2) * 4;
  constexpr int SMEM = PIPE > COMBINE ? PIPE : COMBINE;
  (void)hblocks;
  const int ch = chunk > 0 ? chunk : 1;
  cudaError_t e;
  if (!a.block_table) {
    e = launch_split<T, DK, DV, kPacked>(a, ch, SMEM, 0, s);
  } else {
    // a chunk spans at most ch / block_size + 2 blocks; stage their ids in shared memory
    // when that keeps the CTAs per SM (two of 113 KB, or one of 227 KB at head dim 256),
    // else read the table from global memory
    const long long rows = kStages * kStageKeys * 8;
    const long long ids = (long long)ch / a.block_size + 2;
    const long long smem_t = (long long)SMEM + rows + 4 * ((ids + 31) / 32 * 32);
    const long long cap = ctas_per_sm<DK, DV>() == 2 ? 113 * 1024 : 227 * 1024;
    e = smem_t <= cap ? launch_split<T, DK, DV, kPagedSmemTable>(a, ch, (int)smem_t, SMEM, s)
                             : launch_split<T, DK, DV, kPagedGlobalTable>(a, ch, SMEM + (int)rows, SMEM, s);
  }
  if (e != cudaSuccess) return e;
  const long long rows = (long long)a.batch * a.hq;
  decode_merge_kernel<T, DV><<<(unsigned)((rows + 3) / 4), 128, 0, s>>>(a, chunk > 0 ? chunk : 1);
  return cudaGetLastError();
}

}  // namespace

bool decode_split_supported(int dk, int dv, int dtype) {
  return (dtype == 0 || dtype == 2) &&
         (((dk == 64 || dk == 128) && (dv == 32 || dv == 64 || dv == 128)) || (dk == 256 && dv == 256));
}

namespace {
template <typename T>
cudaError_t launch_dims(const DecodeArgs& a, cudaStream_t s) {
#define ATTN_SINK_DEC_CASE(DK_, DV_) \
  if (a.dk == DK_ && a.dv == DV_) return launch_typed<T, DK_, DV_>(a, s);
  ATTN_SINK_DEC_CASE(64, 32)
  ATTN_SINK_DEC_CASE(64, 64)
  ATTN_SINK_DEC_CASE(64, 128)
  ATTN_SINK_DEC_CASE(128, 32)
  ATTN_SINK_DEC_CASE(128, 64)
  ATTN_SINK_DEC_CASE(128, 128)
  ATTN_SINK_DEC_CASE(256, 256)
#undef ATTN_SINK_DEC_CASE
  return cudaErrorInvalidValue;
}
}  // namespace

cudaError_t launch_decode_split(const DecodeArgs& a, int dtype, cudaStream_t s) {
  return dtype == 2 ? launch_dims<__half>(a, s) : launch_dims<__nv_bfloat16>(a, s);
}

}  // namespace attn_sink
