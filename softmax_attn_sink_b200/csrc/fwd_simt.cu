// Sink-attention forward on the CUDA cores (no tensor cores).
//
// Used for fp32 problems, where the tolerance needs true fp32 products, and for head
// dims the tensor-core kernel does not cover.  One warp owns a query row at a time;
// lanes take one key each for S = scale * q.k, then one output dimension each for
// O += P V.  The online softmax starts its running max at the sink, so the sink is
// "folded into the running max at init"; the running sum counts only the keys and the
// sink's e^{sink - m} joins the denominator in the epilogue (CANN flash_attn doc,
// "Function" formula: m = max(sink, max S), den = sum e^{S-m} + e^{sink-m}).  The
// returned lse is m + log(sum) -- the keys only, no sink (CANN doc, softmax_lse).
#include "common.cuh"

namespace attn_sink {
namespace {

constexpr int kRowsPerWarp = 4;
constexpr int kWarps = 4;
constexpr int kRows = kRowsPerWarp * kWarps;   // query rows per block
constexpr int kKeys = 32;                      // keys per tile (one per lane)

// Shared-memory bytes (dynamic: at head dim 256 they exceed 48 KB).
template <int DK, int DV>
constexpr int fwd_smem_bytes() {
  return 4 * (kRows * DK + kKeys * (DK + 1) + kKeys * DV);
}

template <typename T, int DK, int DV>
__global__ void __launch_bounds__(kWarps * 32)
fwd_simt_kernel(const FwdArgs a) {
  constexpr int VPL = DV / 32;  // output dims per lane
  extern __shared__ float smem_f[];
  float(*s_q)[DK] = reinterpret_cast<float(*)[DK]>(smem_f);
  float(*s_k)[DK + 1] = reinterpret_cast<float(*)[DK + 1]>(smem_f + kRows * DK);
  float(*s_v)[DV] = reinterpret_cast<float(*)[DV]>(smem_f + kRows * DK + kKeys * (DK + 1));

  const int b = blockIdx.z, h = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  long long q0, sq;
  if (a.cu_q) {
    q0 = a.cu_q[b];
    sq = a.cu_q[b + 1] - q0;
  } else {
    q0 = b;
    sq = 1;
  }
  const long long k0 = a.cu_k[b], sk = a.cu_k[b + 1] - k0;
  const long long r0 = (long long)blockIdx.x * kRows;
  if (r0 >= sq) return;
  const int g = h / (a.hq / a.hkv);
  const T* q = static_cast<const T*>(a.q);
  const T* kp = static_cast<const T*>(a.k);
  const T* vp = static_cast<const T*>(a.v);

  for (int idx = threadIdx.x; idx < kRows * DK; idx += blockDim.x) {
    const int r = idx / DK, c = idx % DK;
    s_q[r][c] = (r0 + r < sq) ? to_float(q[((q0 + r0 + r) * a.hq + h) * DK + c]) : 0.f;
  }

  // union of the visible key ranges of the block's rows
  const long long r_last = (r0 + kRows < sq ? r0 + kRows : sq) - 1;
  long long lo0, hi0, lo1, hi1;
  row_key_range(r0, sq, sk, a.left, a.right, lo0, hi0);
  row_key_range(r_last, sq, sk, a.left, a.right, lo1, hi1);
  const long long lo = lo0 < lo1 ? lo0 : lo1;
  const long long hi = hi0 > hi1 ? hi0 : hi1;

  const float sink = a.sink ? a.sink[h] : kNegInf;
  float m[kRowsPerWarp], l[kRowsPerWarp], o[kRowsPerWarp][VPL];
#pragma unroll
  for (int rr = 0; rr < kRowsPerWarp; ++rr) {
    m[rr] = sink;
    l[rr] = 0.f;
#pragma unroll
    for (int c = 0; c < VPL; ++c) o[rr][c] = 0.f;
  }

  for (long long t0 = lo; t0 < hi; t0 += kKeys) {
    __syncthreads();
    for (int idx = threadIdx.x; idx < kKeys * DK; idx += blockDim.x) {
      const int j = idx / DK, c = idx % DK;
      s_k[j][c] = (t0 + j < hi) ? to_float(kp[((k0 + t0 + j) * a.hkv + g) * DK + c]) : 0.f;
    }
    for (int idx = threadIdx.x; idx < kKeys * DV; idx += blockDim.x) {
      const int j = idx / DV, c = idx % DV;
      s_v[j][c] = (t0 + j < hi) ? to_float(vp[((k0 + t0 + j) * a.hkv + g) * DV + c]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int rr = 0; rr < kRowsPerWarp; ++rr) {
      const int r = warp * kRowsPerWarp + rr;
      const long long i = r0 + r;
      if (i >= sq) continue;  // warp-uniform
      const long long j = t0 + lane;
      const bool vis = (j < hi) && visible(i, j, sq, sk, a.left, a.right);
      float s = kNegInf;
      if (vis) {
        float acc = 0.f;
#pragma unroll 8
        for (int c = 0; c < DK; ++c) acc = fmaf(s_q[r][c], s_k[lane][c], acc);
        s = acc * a.scale;
      }
      const float m_new = fmaxf(m[rr], warp_max(s));
      if (m_new == kNegInf) continue;  // nothing visible yet and no sink (warp-uniform)
      const float alpha = (m[rr] == kNegInf) ? 0.f : __expf(m[rr] - m_new);
      const float p = vis ? __expf(s - m_new) : 0.f;
      l[rr] = l[rr] * alpha + warp_sum(p);
#pragma unroll
      for (int c = 0; c < VPL; ++c) o[rr][c] *= alpha;
#pragma unroll 4
      for (int jj = 0; jj < kKeys; ++jj) {
        const float pj = __shfl_sync(0xffffffffu, p, jj);
#pragma unroll
        for (int c = 0; c < VPL; ++c) o[rr][c] = fmaf(pj, s_v[jj][lane + 32 * c], o[rr][c]);
      }
      m[rr] = m_new;
    }
  }

  T* out = static_cast<T*>(a.out);
#pragma unroll
  for (int rr = 0; rr < kRowsPerWarp; ++rr) {
    const long long i = r0 + warp * kRowsPerWarp + rr;
    if (i >= sq) continue;
    const float e_sink = (sink == kNegInf) ? 0.f : __expf(sink - m[rr]);
    const float den = l[rr] + e_sink;
    const float inv = den > 0.f ? 1.f / den : 0.f;
#pragma unroll
    for (int c = 0; c < VPL; ++c)
      out[((q0 + i) * a.hq + h) * DV + lane + 32 * c] = from_float<T>(o[rr][c] * inv);
    if (a.lse && lane == 0)
      a.lse[(long long)h * a.total_q + q0 + i] = l[rr] > 0.f ? m[rr] + __logf(l[rr]) : kNegInf;
  }
}

template <typename T, int DK, int DV>
cudaError_t launch_typed(const FwdArgs& a, cudaStream_t s) {
  const int max_sq = a.cu_q ? a.max_sq : 1;
  constexpr int smem = fwd_smem_bytes<DK, DV>();
  cudaError_t e = cudaFuncSetAttribute(fwd_simt_kernel<T, DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid((max_sq + kRows - 1) / kRows, a.hq, a.batch);
  fwd_simt_kernel<T, DK, DV><<<grid, kWarps * 32, smem, s>>>(a);
  return cudaGetLastError();
}

template <typename T>
cudaError_t dispatch_dims(const FwdArgs& a, cudaStream_t s) {
#define ATTN_SINK_FWD_CASE(DK_, DV_) \
  if (a.dk == DK_ && a.dv == DV_) return launch_typed<T, DK_, DV_>(a, s);
  ATTN_SINK_FWD_CASE(64, 32)
  ATTN_SINK_FWD_CASE(64, 64)
  ATTN_SINK_FWD_CASE(64, 128)
  ATTN_SINK_FWD_CASE(128, 32)
  ATTN_SINK_FWD_CASE(128, 64)
  ATTN_SINK_FWD_CASE(128, 128)
  ATTN_SINK_FWD_CASE(256, 256)
#undef ATTN_SINK_FWD_CASE
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_fwd_simt(const FwdArgs& a, int dtype, cudaStream_t s) {
  if (dtype == 1) return dispatch_dims<float>(a, s);
  return dtype == 2 ? dispatch_dims<__half>(a, s) : dispatch_dims<__nv_bfloat16>(a, s);
}

}  // namespace attn_sink
