// Sink-attention backward on the CUDA cores (fp32 problems and uncovered head dims),
// plus the preprocess pass every backward uses.
//
// Gradient of the sink forward for the loss sum(dout * out).  With the forward's vanilla
// lse and lse_tot = logaddexp(lse, sink), the sink-normalised probabilities are
// P_ij = e^{S_ij - lse_tot_i} and the sink's share is p_sink_i = e^{sink - lse_tot_i}.
// Then D_i = dout_i . out_i, dS = P * (dout V^T - D), dq = scale dS K, dk = scale dS^T Q,
// dv = P^T dout and dsink = -sum_i p_sink_i D_i.  slime's learnable_softmax_attention.py
// states the same gradient as dS = P_van * s * (D - s * di) with s = sigmoid(lse - offset)
// (class docstring) and d_offset = -sum (dout . out_van) s (1 - s) (``backward``);
// P = s P_van and D = s di make the two forms equal.
#include "common.cuh"

namespace attn_sink {
namespace {

__device__ __forceinline__ float logaddexp(float a, float b) {
  if (a == kNegInf) return b;
  if (b == kNegInf) return a;
  const float mx = fmaxf(a, b);
  return mx + log1pf(__expf(-fabsf(a - b)));
}

// --- preprocess: D, lse_tot and dsink ------------------------------------------------
// grid (ceil(total_q / 64), hq), 256 threads: each warp handles 8 rows of one head.
template <typename T>
__global__ void __launch_bounds__(256) bwd_preprocess_kernel(const BwdArgs a) {
  const int h = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const T* out = static_cast<const T*>(a.out);
  const T* dout = static_cast<const T*>(a.dout);
  const float sink = a.sink ? a.sink[h] : kNegInf;
  float ds_acc = 0.f;
  for (int rr = 0; rr < 8; ++rr) {
    const long long i = ((long long)blockIdx.x * 8 + warp) * 8 + rr;
    if (i >= a.total_q) break;
    const long long base = (i * a.hq + h) * a.dv;
    float d = 0.f;
    for (int c = lane; c < a.dv; c += 32) d = fmaf(to_float(out[base + c]), to_float(dout[base + c]), d);
    d = warp_sum(d);
    const float lse = a.lse[(long long)h * a.total_q + i];
    const float lt = logaddexp(lse, sink);
    if (lane == 0) {
      a.D[(long long)h * a.total_q + i] = d;
      a.lse_tot[(long long)h * a.total_q + i] = lt;
    }
    if (sink != kNegInf && lt != kNegInf) ds_acc -= __expf(sink - lt) * d;
  }
  __shared__ float red[8];
  if (lane == 0) red[warp] = ds_acc;
  __syncthreads();
  if (threadIdx.x == 0 && a.dsink) {
    float s = 0.f;
    for (int w = 0; w < 8; ++w) s += red[w];
    a.dsink_part[(long long)h * gridDim.x + blockIdx.x] = s;   // summed in a fixed order later
  }
}

// The same pass with 16-byte loads, for head dims that are a multiple of one load: a row of
// out / dout is split over L lanes (L = DV / elements per load, at most 32), each warp covers
// its 8 rows in 8 L / 32 passes whose loads are all issued before any product is summed, and
// the L lanes of a row reduce with xor shuffles.  Same grid, rows and partial layout as above.
__device__ __forceinline__ float dot16(uint4 x, uint4 y, const __nv_bfloat16*) {
  const uint32_t xs[4] = {x.x, x.y, x.z, x.w}, ys[4] = {y.x, y.y, y.z, y.w};
  float d = 0.f;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float2 u = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xs[k]));
    const float2 v = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ys[k]));
    d = fmaf(u.x, v.x, d);
    d = fmaf(u.y, v.y, d);
  }
  return d;
}
__device__ __forceinline__ float dot16(uint4 x, uint4 y, const __half*) {
  const uint32_t xs[4] = {x.x, x.y, x.z, x.w}, ys[4] = {y.x, y.y, y.z, y.w};
  float d = 0.f;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float2 u = __half22float2(*reinterpret_cast<const __half2*>(&xs[k]));
    const float2 v = __half22float2(*reinterpret_cast<const __half2*>(&ys[k]));
    d = fmaf(u.x, v.x, d);
    d = fmaf(u.y, v.y, d);
  }
  return d;
}
__device__ __forceinline__ float dot16(uint4 x, uint4 y, const float*) {
  float d = __uint_as_float(x.x) * __uint_as_float(y.x);
  d = fmaf(__uint_as_float(x.y), __uint_as_float(y.y), d);
  d = fmaf(__uint_as_float(x.z), __uint_as_float(y.z), d);
  return fmaf(__uint_as_float(x.w), __uint_as_float(y.w), d);
}

template <typename T, int DV>
__global__ void __launch_bounds__(256) bwd_preprocess_vec_kernel(const BwdArgs a) {
  constexpr int kEpv = 16 / (int)sizeof(T);      // elements per 16-byte load
  constexpr int kNv = DV / kEpv;                 // loads per row
  constexpr int kL = kNv < 32 ? kNv : 32;        // lanes per row
  constexpr int kVpl = kNv / kL;                 // loads per lane and row
  constexpr int kR = 32 / kL;                    // rows per pass
  constexpr int kP = 8 / kR;                     // passes over the warp's 8 rows
  static_assert(kNv * kEpv == DV && kL * kVpl == kNv && kR * kP == 8, "row split");
  const int h = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = lane % kL, rsub = lane / kL;
  const float sink = a.sink ? a.sink[h] : kNegInf;
  const uint4* out = static_cast<const uint4*>(a.out);
  const uint4* dout = static_cast<const uint4*>(a.dout);
  const long long r0 = ((long long)blockIdx.x * 8 + warp) * 8;
  uint4 xo[kP][kVpl], xd[kP][kVpl];
#pragma unroll
  for (int p = 0; p < kP; ++p) {
    const long long i = r0 + p * kR + rsub;
    const long long base = (i * a.hq + h) * kNv;   // in 16-byte loads
#pragma unroll
    for (int v = 0; v < kVpl; ++v) {
      if (i < a.total_q) {
        xo[p][v] = __ldg(out + base + sub + v * kL);
        xd[p][v] = __ldg(dout + base + sub + v * kL);
      } else {
        xo[p][v] = make_uint4(0u, 0u, 0u, 0u);
        xd[p][v] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
  }
  float ds_acc = 0.f;
#pragma unroll
  for (int p = 0; p < kP; ++p) {
    float d = 0.f;
#pragma unroll
    for (int v = 0; v < kVpl; ++v) d += dot16(xo[p][v], xd[p][v], static_cast<const T*>(nullptr));
#pragma unroll
    for (int o = kL / 2; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
    const long long i = r0 + p * kR + rsub;
    if (sub == 0 && i < a.total_q) {
      const long long k = (long long)h * a.total_q + i;
      const float lt = logaddexp(a.lse[k], sink);
      a.D[k] = d;
      a.lse_tot[k] = lt;
      if (sink != kNegInf && lt != kNegInf) ds_acc -= __expf(sink - lt) * d;
    }
  }
  ds_acc = warp_sum(ds_acc);
  __shared__ float red[8];
  if (lane == 0) red[warp] = ds_acc;
  __syncthreads();
  if (threadIdx.x == 0 && a.dsink) {
    float s = 0.f;
    for (int w = 0; w < 8; ++w) s += red[w];
    a.dsink_part[(long long)h * gridDim.x + blockIdx.x] = s;   // summed in a fixed order later
  }
}

template <typename T>
void launch_preprocess_typed(const BwdArgs& a, dim3 grid, cudaStream_t s) {
  switch (a.dv) {
    case 32: bwd_preprocess_vec_kernel<T, 32><<<grid, 256, 0, s>>>(a); return;
    case 64: bwd_preprocess_vec_kernel<T, 64><<<grid, 256, 0, s>>>(a); return;
    case 128: bwd_preprocess_vec_kernel<T, 128><<<grid, 256, 0, s>>>(a); return;
    case 256: bwd_preprocess_vec_kernel<T, 256><<<grid, 256, 0, s>>>(a); return;
    default: bwd_preprocess_kernel<T><<<grid, 256, 0, s>>>(a); return;
  }
}

// d_sink[h] = sum over the preprocess blocks of their partials, one warp per head: lane l
// adds blocks l, l + 32, ... in order, then a fixed butterfly combines the lanes, so the
// result does not depend on the order in which blocks ran.
__global__ void __launch_bounds__(32) dsink_reduce_kernel(const BwdArgs a, int nblocks) {
  const int h = blockIdx.x, lane = threadIdx.x;
  const float* part = a.dsink_part + (long long)h * nblocks;
  float s = 0.f;
  for (int i = lane; i < nblocks; i += 32) s += part[i];
  s = warp_sum(s);
  if (lane == 0) a.dsink[h] = s;
}

// --- dK / dV: key-stationary -----------------------------------------------------------
// grid (ceil(max_sk / 8), hkv, batch), 4 warps x 2 keys.  Each block owns its keys for
// one kv head and loops over every q head of the group, so no atomics are needed.
constexpr int kKeysPerWarp = 2;
constexpr int kWarps = 4;
constexpr int kBlockKeys = kKeysPerWarp * kWarps;
constexpr int kTile = 32;

// Shared-memory bytes of the dK/dV kernel (dynamic: at head dim 256 it exceeds 48 KB).
template <int DK, int DV>
constexpr int dkdv_smem_bytes() {
  return 4 * (kBlockKeys * DK + kBlockKeys * DV + kTile * (DK + 1) + kTile * (DV + 1) + 2 * kTile);
}

template <typename T, int DK, int DV>
__global__ void __launch_bounds__(kWarps * 32) bwd_dkdv_simt_kernel(const BwdArgs a) {
  constexpr int KPL = DK / 32, VPL = DV / 32;
  extern __shared__ float smem_f[];
  float(*s_k)[DK] = reinterpret_cast<float(*)[DK]>(smem_f);
  float(*s_v)[DV] = reinterpret_cast<float(*)[DV]>(smem_f + kBlockKeys * DK);
  float(*s_q)[DK + 1] = reinterpret_cast<float(*)[DK + 1]>(smem_f + kBlockKeys * (DK + DV));
  float(*s_do)[DV + 1] = reinterpret_cast<float(*)[DV + 1]>(smem_f + kBlockKeys * (DK + DV) + kTile * (DK + 1));
  float* s_lt = smem_f + kBlockKeys * (DK + DV) + kTile * (DK + 1) + kTile * (DV + 1);
  float* s_D = s_lt + kTile;

  const int b = blockIdx.z, g = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long q0 = a.cu_q[b], sq = a.cu_q[b + 1] - q0;
  const long long k0 = a.cu_k[b], sk = a.cu_k[b + 1] - k0;
  const long long j0 = (long long)blockIdx.x * kBlockKeys;
  if (j0 >= sk) return;
  const int group = a.hq / a.hkv;
  const T* q = static_cast<const T*>(a.q);
  const T* kp = static_cast<const T*>(a.k);
  const T* vp = static_cast<const T*>(a.v);
  const T* dout = static_cast<const T*>(a.dout);

  for (int idx = threadIdx.x; idx < kBlockKeys * DK; idx += blockDim.x) {
    const int j = idx / DK, c = idx % DK;
    s_k[j][c] = (j0 + j < sk) ? to_float(kp[((k0 + j0 + j) * a.hkv + g) * DK + c]) : 0.f;
  }
  for (int idx = threadIdx.x; idx < kBlockKeys * DV; idx += blockDim.x) {
    const int j = idx / DV, c = idx % DV;
    s_v[j][c] = (j0 + j < sk) ? to_float(vp[((k0 + j0 + j) * a.hkv + g) * DV + c]) : 0.f;
  }
  const long long j_last = (j0 + kBlockKeys < sk ? j0 + kBlockKeys : sk) - 1;
  long long lo0, hi0, lo1, hi1;
  key_query_range(j0, sq, sk, a.left, a.right, lo0, hi0);
  key_query_range(j_last, sq, sk, a.left, a.right, lo1, hi1);
  const long long lo = lo0 < lo1 ? lo0 : lo1;
  const long long hi = hi0 > hi1 ? hi0 : hi1;

  float dk_acc[kKeysPerWarp][KPL], dv_acc[kKeysPerWarp][VPL];
#pragma unroll
  for (int kk = 0; kk < kKeysPerWarp; ++kk) {
#pragma unroll
    for (int c = 0; c < KPL; ++c) dk_acc[kk][c] = 0.f;
#pragma unroll
    for (int c = 0; c < VPL; ++c) dv_acc[kk][c] = 0.f;
  }

  for (int hh = 0; hh < group; ++hh) {
    const int h = g * group + hh;
    for (long long t0 = lo; t0 < hi; t0 += kTile) {
      __syncthreads();
      for (int idx = threadIdx.x; idx < kTile * DK; idx += blockDim.x) {
        const int i = idx / DK, c = idx % DK;
        s_q[i][c] = (t0 + i < hi) ? to_float(q[((q0 + t0 + i) * a.hq + h) * DK + c]) : 0.f;
      }
      for (int idx = threadIdx.x; idx < kTile * DV; idx += blockDim.x) {
        const int i = idx / DV, c = idx % DV;
        s_do[i][c] = (t0 + i < hi) ? to_float(dout[((q0 + t0 + i) * a.hq + h) * DV + c]) : 0.f;
      }
      if (threadIdx.x < kTile) {
        const long long i = t0 + threadIdx.x;
        s_lt[threadIdx.x] = (i < hi) ? a.lse_tot[(long long)h * a.total_q + q0 + i] : 0.f;
        s_D[threadIdx.x] = (i < hi) ? a.D[(long long)h * a.total_q + q0 + i] : 0.f;
      }
      __syncthreads();
      const long long i = t0 + lane;
#pragma unroll
      for (int kk = 0; kk < kKeysPerWarp; ++kk) {
        const int jl = warp * kKeysPerWarp + kk;
        const long long j = j0 + jl;
        if (j >= sk) continue;  // warp-uniform
        const bool vis = (i < hi) && visible(i, j, sq, sk, a.left, a.right);
        float p = 0.f, ds = 0.f;
        if (vis) {
          float s = 0.f, dp = 0.f;
#pragma unroll 8
          for (int c = 0; c < DK; ++c) s = fmaf(s_q[lane][c], s_k[jl][c], s);
#pragma unroll 8
          for (int c = 0; c < DV; ++c) dp = fmaf(s_do[lane][c], s_v[jl][c], dp);
          p = __expf(s * a.scale - s_lt[lane]);
          ds = p * (dp - s_D[lane]);
        }
#pragma unroll 4
        for (int ii = 0; ii < kTile; ++ii) {
          const float pi = __shfl_sync(0xffffffffu, p, ii);
          const float dsi = __shfl_sync(0xffffffffu, ds, ii);
#pragma unroll
          for (int c = 0; c < VPL; ++c) dv_acc[kk][c] = fmaf(pi, s_do[ii][lane + 32 * c], dv_acc[kk][c]);
#pragma unroll
          for (int c = 0; c < KPL; ++c) dk_acc[kk][c] = fmaf(dsi, s_q[ii][lane + 32 * c], dk_acc[kk][c]);
        }
      }
    }
  }

  T* dk = static_cast<T*>(a.grad_k);
  T* dv = static_cast<T*>(a.grad_v);
#pragma unroll
  for (int kk = 0; kk < kKeysPerWarp; ++kk) {
    const long long j = j0 + warp * kKeysPerWarp + kk;
    if (j >= sk) continue;
#pragma unroll
    for (int c = 0; c < KPL; ++c)
      dk[((k0 + j) * a.hkv + g) * DK + lane + 32 * c] = from_float<T>(dk_acc[kk][c] * a.scale);
#pragma unroll
    for (int c = 0; c < VPL; ++c)
      dv[((k0 + j) * a.hkv + g) * DV + lane + 32 * c] = from_float<T>(dv_acc[kk][c]);
  }
}

// --- dQ: query-stationary ------------------------------------------------------------------
constexpr int kRowsPerWarp = 2;
constexpr int kBlockRows = kRowsPerWarp * kWarps;

template <int DK, int DV>
constexpr int dq_smem_bytes() {
  return 4 * (kBlockRows * DK + kBlockRows * DV + kTile * (DK + 1) + kTile * (DV + 1));
}

template <typename T, int DK, int DV>
__global__ void __launch_bounds__(kWarps * 32) bwd_dq_simt_kernel(const BwdArgs a) {
  constexpr int KPL = DK / 32;
  extern __shared__ float smem_f[];
  float(*s_q)[DK] = reinterpret_cast<float(*)[DK]>(smem_f);
  float(*s_do)[DV] = reinterpret_cast<float(*)[DV]>(smem_f + kBlockRows * DK);
  float(*s_k)[DK + 1] = reinterpret_cast<float(*)[DK + 1]>(smem_f + kBlockRows * (DK + DV));
  float(*s_v)[DV + 1] = reinterpret_cast<float(*)[DV + 1]>(smem_f + kBlockRows * (DK + DV) + kTile * (DK + 1));

  const int b = blockIdx.z, h = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long q0 = a.cu_q[b], sq = a.cu_q[b + 1] - q0;
  const long long k0 = a.cu_k[b], sk = a.cu_k[b + 1] - k0;
  const long long r0 = (long long)blockIdx.x * kBlockRows;
  if (r0 >= sq) return;
  const int g = h / (a.hq / a.hkv);
  const T* q = static_cast<const T*>(a.q);
  const T* kp = static_cast<const T*>(a.k);
  const T* vp = static_cast<const T*>(a.v);
  const T* dout = static_cast<const T*>(a.dout);

  for (int idx = threadIdx.x; idx < kBlockRows * DK; idx += blockDim.x) {
    const int r = idx / DK, c = idx % DK;
    s_q[r][c] = (r0 + r < sq) ? to_float(q[((q0 + r0 + r) * a.hq + h) * DK + c]) : 0.f;
  }
  for (int idx = threadIdx.x; idx < kBlockRows * DV; idx += blockDim.x) {
    const int r = idx / DV, c = idx % DV;
    s_do[r][c] = (r0 + r < sq) ? to_float(dout[((q0 + r0 + r) * a.hq + h) * DV + c]) : 0.f;
  }
  float lt[kRowsPerWarp], Dr[kRowsPerWarp], acc[kRowsPerWarp][KPL];
#pragma unroll
  for (int rr = 0; rr < kRowsPerWarp; ++rr) {
    const long long i = r0 + warp * kRowsPerWarp + rr;
    lt[rr] = (i < sq) ? a.lse_tot[(long long)h * a.total_q + q0 + i] : 0.f;
    Dr[rr] = (i < sq) ? a.D[(long long)h * a.total_q + q0 + i] : 0.f;
#pragma unroll
    for (int c = 0; c < KPL; ++c) acc[rr][c] = 0.f;
  }
  const long long r_last = (r0 + kBlockRows < sq ? r0 + kBlockRows : sq) - 1;
  long long lo0, hi0, lo1, hi1;
  row_key_range(r0, sq, sk, a.left, a.right, lo0, hi0);
  row_key_range(r_last, sq, sk, a.left, a.right, lo1, hi1);
  const long long lo = lo0 < lo1 ? lo0 : lo1;
  const long long hi = hi0 > hi1 ? hi0 : hi1;

  for (long long t0 = lo; t0 < hi; t0 += kTile) {
    __syncthreads();
    for (int idx = threadIdx.x; idx < kTile * DK; idx += blockDim.x) {
      const int j = idx / DK, c = idx % DK;
      s_k[j][c] = (t0 + j < hi) ? to_float(kp[((k0 + t0 + j) * a.hkv + g) * DK + c]) : 0.f;
    }
    for (int idx = threadIdx.x; idx < kTile * DV; idx += blockDim.x) {
      const int j = idx / DV, c = idx % DV;
      s_v[j][c] = (t0 + j < hi) ? to_float(vp[((k0 + t0 + j) * a.hkv + g) * DV + c]) : 0.f;
    }
    __syncthreads();
    const long long j = t0 + lane;
#pragma unroll
    for (int rr = 0; rr < kRowsPerWarp; ++rr) {
      const int r = warp * kRowsPerWarp + rr;
      const long long i = r0 + r;
      if (i >= sq) continue;
      const bool vis = (j < hi) && visible(i, j, sq, sk, a.left, a.right);
      float ds = 0.f;
      if (vis) {
        float s = 0.f, dp = 0.f;
#pragma unroll 8
        for (int c = 0; c < DK; ++c) s = fmaf(s_q[r][c], s_k[lane][c], s);
#pragma unroll 8
        for (int c = 0; c < DV; ++c) dp = fmaf(s_do[r][c], s_v[lane][c], dp);
        const float p = __expf(s * a.scale - lt[rr]);
        ds = p * (dp - Dr[rr]);
      }
#pragma unroll 4
      for (int jj = 0; jj < kTile; ++jj) {
        const float dsj = __shfl_sync(0xffffffffu, ds, jj);
#pragma unroll
        for (int c = 0; c < KPL; ++c) acc[rr][c] = fmaf(dsj, s_k[jj][lane + 32 * c], acc[rr][c]);
      }
    }
  }
  T* dq = static_cast<T*>(a.grad_q);
#pragma unroll
  for (int rr = 0; rr < kRowsPerWarp; ++rr) {
    const long long i = r0 + warp * kRowsPerWarp + rr;
    if (i >= sq) continue;
#pragma unroll
    for (int c = 0; c < KPL; ++c)
      dq[((q0 + i) * a.hq + h) * DK + lane + 32 * c] = from_float<T>(acc[rr][c] * a.scale);
  }
}

// Every key row of every sequence is written by the dk/dv pass (zeros where no query sees
// it) and every query row by the dq pass, so no output needs clearing first.
template <typename T, int DK, int DV>
cudaError_t launch_typed(const BwdArgs& a, cudaStream_t s) {
  constexpr int smem1 = dkdv_smem_bytes<DK, DV>(), smem2 = dq_smem_bytes<DK, DV>();
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(bwd_dkdv_simt_kernel<T, DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                smem1)) != cudaSuccess)
    return e;
  if ((e = cudaFuncSetAttribute(bwd_dq_simt_kernel<T, DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                smem2)) != cudaSuccess)
    return e;
  dim3 g1((a.max_sk + kBlockKeys - 1) / kBlockKeys, a.hkv, a.batch);
  bwd_dkdv_simt_kernel<T, DK, DV><<<g1, kWarps * 32, smem1, s>>>(a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  dim3 g2((a.max_sq + kBlockRows - 1) / kBlockRows, a.hq, a.batch);
  bwd_dq_simt_kernel<T, DK, DV><<<g2, kWarps * 32, smem2, s>>>(a);
  return cudaGetLastError();
}

template <typename T>
cudaError_t dispatch_dims(const BwdArgs& a, cudaStream_t s) {
#define ATTN_SINK_BWD_CASE(DK_, DV_) \
  if (a.dk == DK_ && a.dv == DV_) return launch_typed<T, DK_, DV_>(a, s);
  ATTN_SINK_BWD_CASE(64, 32)
  ATTN_SINK_BWD_CASE(64, 64)
  ATTN_SINK_BWD_CASE(64, 128)
  ATTN_SINK_BWD_CASE(128, 32)
  ATTN_SINK_BWD_CASE(128, 64)
  ATTN_SINK_BWD_CASE(128, 128)
  ATTN_SINK_BWD_CASE(256, 256)
#undef ATTN_SINK_BWD_CASE
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_bwd_preprocess(const BwdArgs& a, int dtype, cudaStream_t s) {
  dim3 grid((a.total_q + 63) / 64, a.hq);
  if (dtype == 1)
    launch_preprocess_typed<float>(a, grid, s);
  else if (dtype == 2)
    launch_preprocess_typed<__half>(a, grid, s);
  else
    launch_preprocess_typed<__nv_bfloat16>(a, grid, s);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || !a.dsink) return e;
  dsink_reduce_kernel<<<a.hq, 32, 0, s>>>(a, (int)grid.x);
  return cudaGetLastError();
}

cudaError_t launch_bwd_simt(const BwdArgs& a, int dtype, cudaStream_t s) {
  cudaError_t e = launch_bwd_preprocess(a, dtype, s);
  if (e != cudaSuccess) return e;
  if (dtype == 1) return dispatch_dims<float>(a, s);
  return dtype == 2 ? dispatch_dims<__half>(a, s) : dispatch_dims<__nv_bfloat16>(a, s);
}

}  // namespace attn_sink
