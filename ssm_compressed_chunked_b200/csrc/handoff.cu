// Prefill -> decode cache handoff.
//
// Method: pith.science review of Attamba, "Core claim" -- at inference only the
// boundary states are cached; "If this is right" -- the final SSM state of each
// chunk is what the cache keeps (P = 8 with 64 leading tokens gives about 8x);
// "What carries the argument" -- the L most recent tokens stay uncompressed
// (Eq. 8).  A prefill of positions [0, n0) therefore leaves: the keys/values at
// the positions p < n0 that end a chunk (the uniform chunk rule of the decode,
// so a last chunk the prefill cut at n0 - 1 is not one of them), the keys/values
// of the L most recent positions in the ring, and the SSM states after n0 - 1.
//
// The states are not kept by the prefill scan: they depend only on the tokens
// of the chunk holding n0 - 1 (the state restarts at every chunk start), so one
// thread per (SSM, sequence, channel) reruns the recurrence over those at most P
// tokens.  Two launches: the row copies, then the state rerun.
#include "common.cuh"
#include "launch.h"

namespace attamba {

namespace {
constexpr int kDH = 64;
constexpr float kLog2e = 1.4426950408889634f;

// one past the first chunk end of a uniform chunking: the offset mod P, or P when that is 0
__host__ __device__ __forceinline__ int32_t first_boundary_end(int32_t P, int32_t offset) {
  const int32_t o = ((offset % P) + P) % P;
  return o == 0 ? P : o;
}

// block (item, b): item < nb copies boundary item (position f - 1 + item P) into
// Kb / Vb row item, otherwise ring position n0 - nring + (item - nb) into slot p mod L
__global__ void __launch_bounds__(128) handoff_copy_kernel(HandoffArgs a) {
  const attamba_cache_t& c = a.c;
  const int b = blockIdx.y, item = blockIdx.x;
  const int nring = min(c.L, a.n0);
  const bool bnd = item < a.nb;
  const int p = bnd ? first_boundary_end(c.P, c.offset) - 1 + item * c.P : a.n0 - nring + (item - a.nb);
  const int D = c.H * kDH;
  const size_t row = ((size_t)b * a.n0 + p) * D;
  const uint4* k = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.K) + row);
  const uint4* v = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.V) + row);
  for (int u = threadIdx.x; u < D / 8; u += blockDim.x) {
    const int h = u / (kDH / 8), e = (u - h * (kDH / 8)) * 8;
    size_t dst;
    if (bnd) dst = (((size_t)b * c.H + h) * c.cap + item) * kDH + e;
    else dst = (((size_t)b * c.H + h) * c.L + (p % c.L)) * kDH + e;
    __nv_bfloat16* dk = static_cast<__nv_bfloat16*>(bnd ? c.Kb : c.Kr) + dst;
    __nv_bfloat16* dv = static_cast<__nv_bfloat16*>(bnd ? c.Vb : c.Vr) + dst;
    *reinterpret_cast<uint4*>(dk) = k[u];
    *reinterpret_cast<uint4*>(dv) = v[u];
  }
  if (threadIdx.x == 0) {
    if (bnd) c.bpos[(size_t)b * c.cap + item] = p;
    if (item == 0) {
      c.nb[b] = a.nb;
      c.pos[b] = a.n0;
    }
  }
}

// thread (s, b, d): the SSM state after position n0 - 1, rerun from the start of its chunk
template <int kNS>
__global__ void __launch_bounds__(128) handoff_state_kernel(HandoffArgs a) {
  const attamba_cache_t& c = a.c;
  const int D = c.H * c.dh;
  const int s = blockIdx.z, b = blockIdx.y;
  const int d = blockIdx.x * blockDim.x + threadIdx.x;
  if (d >= D) return;
  const int f = first_boundary_end(c.P, c.offset);
  const int last = a.n0 - 1;
  const int s0 = last < f ? 0 : f + ((last - f) / c.P) * c.P;   // start of the chunk holding n0 - 1
  const __nv_bfloat16* x = static_cast<const __nv_bfloat16*>(a.x);
  const __nv_bfloat16* dt = static_cast<const __nv_bfloat16*>(a.dt[s]);
  const __nv_bfloat16* Bm = static_cast<const __nv_bfloat16*>(a.Bm[s]);
  const float* A = a.A[s] + (size_t)d * kNS;
  float Al[kNS], h[kNS];
#pragma unroll
  for (int n = 0; n < kNS; ++n) {
    Al[n] = A[n] * kLog2e;
    h[n] = 0.f;
  }
  for (int t = s0; t < a.n0; ++t) {
    const size_t r = (size_t)b * a.n0 + t;
    const float z = __bfloat162float(dt[r * D + d]) + a.bias[s][d];
    const float delta = z > 20.f ? z : log1pf(__expf(z));
    const float dx = delta * __bfloat162float(x[r * D + d]);
#pragma unroll
    for (int n = 0; n < kNS; ++n)
      h[n] = fmaf(ex2(delta * Al[n]), h[n], dx * __bfloat162float(Bm[r * kNS + n]));
  }
  float* st = c.state + ((size_t)(s * c.B + b) * kNS) * D + d;
#pragma unroll
  for (int n = 0; n < kNS; ++n) st[(size_t)n * D] = h[n];
}
}  // namespace

int32_t handoff_boundaries(int32_t n0, int32_t P, int32_t offset) {
  const int32_t f = first_boundary_end(P, offset);
  return n0 >= f ? (n0 - f) / P + 1 : 0;
}

cudaError_t launch_cache_from_prefill(const HandoffArgs& a, cudaStream_t s) {
  const int nring = a.c.L < a.n0 ? a.c.L : a.n0;
  handoff_copy_kernel<<<dim3(a.nb + nring, a.c.B), 128, 0, s>>>(a);
  const int D = a.c.H * a.c.dh;
  if (a.c.N == 32)
    handoff_state_kernel<32><<<dim3((D + 127) / 128, a.c.B, 2), 128, 0, s>>>(a);
  else
    handoff_state_kernel<16><<<dim3((D + 127) / 128, a.c.B, 2), 128, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace attamba
