// Chunk-reset selective scan producing the keys and the values (KV-SSM).
//
// Method: pith.science review of Attamba, "Core claim" -- K = SSM_K(X),
// V = SSM_V(X), one SSM each in place of W_K and W_V; "Assumptions & free
// parameters" -- the SSM is Mamba's selective SSM (Section 3.2, Eq. 3);
// "What carries the argument" -- each chunk of P tokens is compressed
// independently, so the state restarts at every chunk start.  Per token t,
// channel d:  delta = softplus(dt[t,d] + bias[d]);
//             h[d,:] = exp(delta A[d,:]) h[d,:] + delta x[t,d] B[t,:];
//             y[t,d] = C[t,:] . h[d,:].
//
// Mapping (B200): chunks are independent, so the grid runs over
// (channel pairs, groups of chunks, SSM) and every thread walks the tokens of
// its chunk group for two channels, holding the 2 x N state and the 2 x N
// decay rates (A * log2 e) in registers.  B and C, shared by all channels of a
// token, are staged once per block in shared memory as fp32 and read as
// broadcasts.  x and dt are read as packed pairs, coalesced across the warp.
// The only global writes are the outputs (and the compact chunk-end rows).
// The cost is set by the N exponentials per (token, channel, SSM), not by HBM.
#include "common.cuh"
#include "launch.h"

namespace attamba {

namespace {
constexpr int kScanThreads = 128;
constexpr int kStageTokens = 32;
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ float softplus_f(float z) {
  return z > 20.f ? z : log1pf(__expf(z));
}

template <typename T, int NS>
__global__ void __launch_bounds__(kScanThreads) kv_ssm_scan_kernel(ScanArgs p, int32_t chunks_per_block) {
  __shared__ __align__(16) float sB[kStageTokens][NS];
  __shared__ __align__(16) float sC[kStageTokens][NS];

  const int s = blockIdx.z;
  const int D = p.D;
  const int d0 = (blockIdx.x * kScanThreads + threadIdx.x) * 2;
  const bool active = d0 < D;
  const int32_t c_begin = blockIdx.y * chunks_per_block;
  if (c_begin >= p.n_chunks) return;
  const int32_t c_end = min(c_begin + chunks_per_block, p.n_chunks);

  const T* __restrict__ x = static_cast<const T*>(p.x);
  const T* __restrict__ dt = static_cast<const T*>(p.dt[s]);
  const T* __restrict__ Bm = static_cast<const T*>(p.Bm[s]);
  const T* __restrict__ Cm = static_cast<const T*>(p.Cm[s]);
  T* __restrict__ out = static_cast<T*>(p.out[s]);
  T* __restrict__ outc = static_cast<T*>(p.outc[s]);
  const int32_t* __restrict__ cu = p.cu;

  float a2[2][NS];
  float bias[2] = {0.f, 0.f};
  float h[2][NS];
#pragma unroll
  for (int j = 0; j < 2; ++j) {
#pragma unroll
    for (int n = 0; n < NS; ++n) {
      a2[j][n] = active ? p.A[s][(size_t)(d0 + j) * NS + n] * kLog2e : 0.f;
      h[j][n] = 0.f;
    }
    if (active) bias[j] = p.bias[s][d0 + j];
  }

  const int64_t t_begin = cu[c_begin];
  const int64_t t_end = cu[c_end];
  int32_t c = c_begin;
  int64_t next_start = cu[c + 1];

  for (int64_t tb = t_begin; tb < t_end; tb += kStageTokens) {
    const int nt = (int)((t_end - tb) < kStageTokens ? (t_end - tb) : kStageTokens);
    __syncthreads();
    for (int e = threadIdx.x; e < nt * NS; e += kScanThreads) {
      const int k = e / NS, n = e - k * NS;
      sB[k][n] = Elem<T>::to_f(Bm[(tb + k) * NS + n]);
      sC[k][n] = Elem<T>::to_f(Cm[(tb + k) * NS + n]);
    }
    __syncthreads();
    if (!active) continue;
    for (int k = 0; k < nt; ++k) {
      const int64_t t = tb + k;
      if (t == next_start) {  // a new chunk: restart the state
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
          for (int n = 0; n < NS; ++n) h[j][n] = 0.f;
        ++c;
        next_start = cu[c + 1];
      }
      const float2 xv = load2(x + t * D + d0);
      const float2 zv = load2(dt + t * D + d0);
      const float dl0 = softplus_f(zv.x + bias[0]);
      const float dl1 = softplus_f(zv.y + bias[1]);
      const float dx0 = dl0 * xv.x, dx1 = dl1 * xv.y;
      float y0 = 0.f, y1 = 0.f;
#pragma unroll
      for (int n = 0; n < NS; ++n) {
        const float bn = sB[k][n], cn = sC[k][n];
        h[0][n] = fmaf(ex2(dl0 * a2[0][n]), h[0][n], dx0 * bn);
        h[1][n] = fmaf(ex2(dl1 * a2[1][n]), h[1][n], dx1 * bn);
        y0 = fmaf(cn, h[0][n], y0);
        y1 = fmaf(cn, h[1][n], y1);
      }
      store2(out + t * D + d0, y0, y1);
      if (outc != nullptr && t + 1 == next_start) store2(outc + (int64_t)c * D + d0, y0, y1);
    }
  }
}
}  // namespace

cudaError_t launch_kv_ssm_scan(attamba_dtype_t dtype, const ScanArgs& a, cudaStream_t s) {
  // about 64 tokens of chunks per block
  int64_t cpb = (64 * (int64_t)a.n_chunks) / (a.T > 0 ? a.T : 1);
  if (cpb < 1) cpb = 1;
  while ((a.n_chunks + cpb - 1) / cpb > 65535) cpb *= 2;
  dim3 grid((a.D / 2 + kScanThreads - 1) / kScanThreads, (unsigned)((a.n_chunks + cpb - 1) / cpb), 2);
  if (dtype == ATTAMBA_BF16)
    kv_ssm_scan_kernel<__nv_bfloat16, 16><<<grid, kScanThreads, 0, s>>>(a, (int32_t)cpb);
  else
    kv_ssm_scan_kernel<float, 16><<<grid, kScanThreads, 0, s>>>(a, (int32_t)cpb);
  return cudaGetLastError();
}

}  // namespace attamba
