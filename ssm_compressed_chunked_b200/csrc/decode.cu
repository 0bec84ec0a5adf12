// One decode step over the boundary-state cache.
//
// Method: pith.science review of Attamba, "Core claim" -- at inference only the
// chunk-boundary states are cached, so the cache and the attention map shrink by
// about P; "If this is right" -- P = 8 with 64 leading tokens gives about 8x
// compression; "What carries the argument" -- M_test (Eq. 7) plus the L leading
// tokens (Eq. 8); Referee Report, comment on Eq. (7) -- the current chunk is
// reached only through the leading tokens.
//
// Two stream-ordered launches, no inter-CTA waiting:
//   decode_attn_kernel    per (split, head, sequence): the last split first runs the
//                         SSM step of the head's channels (reset at a chunk start,
//                         state [2,B,N,D] read and written coalesced, k_t / v_t into
//                         ring slot t mod L and, at a chunk end, into the boundary
//                         list); every split then streams its share of the
//                         (boundaries below the window) + (window) keys with
//                         16-byte loads, 8 lanes per key row, fp32 online softmax,
//                         and writes (max, sum, unnormalised output) to the workspace
//   decode_combine_kernel per (sequence, head): merges the splits, writes o_t,
//                         and advances pos / nb
// The step is bound by streaming the cached K/V from HBM.
#include <mutex>

#include "common.cuh"
#include "launch.h"

namespace attamba {

// Split-K scratch of attamba_decode_step_noalloc: a fixed array in the
// library's own device memory, so that entry point never allocates.  It holds
// B * H * splits * (head_dim + 2) floats of partial results; every (sequence,
// head, split) slot is written by decode_attn_kernel before decode_combine_kernel
// reads it, so nothing in it has to start at zero.  All calls on a device share
// it: two no-alloc calls whose kernels overlap on the GPU (different streams,
// no ordering between them) corrupt each other's partials.
constexpr size_t kNoAllocScratchFloats = (size_t)1 << 20;  // 4 MiB
static __device__ __align__(256) float g_decode_scratch[kNoAllocScratchFloats];

namespace {
constexpr int kDH = 64;
constexpr int kAttnThreads = 128;
constexpr int kUnroll = 4;
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ bool chunk_starts_at(int t, int P, int o) {
  return t == 0 || (t >= o && (t - o) % P == 0);
}
__device__ __forceinline__ bool chunk_ends_at(int t, int P, int o) {
  return (t + 1 >= o) && ((t + 1 - o) % P == 0);
}

// One SSM step of channel d of sequence b for SSM s: reset at a chunk start, state
// [2,B,N,D] read and written coalesced, k_t / v_t into ring slot t mod L and, at a
// chunk end, into the boundary list.
template <int kNS>
__device__ __forceinline__ void ssm_step(const DecodeArgs& a, int s, int b, int d) {
  const attamba_cache_t& c = a.c;
  const int D = c.H * c.dh;
  const int o = ((c.offset % c.P) + c.P) % c.P;
  const int t = a.c.pos[b];
  const bool start = chunk_starts_at(t, c.P, o);
  const bool end = chunk_ends_at(t, c.P, o);
  const __nv_bfloat16* x = static_cast<const __nv_bfloat16*>(a.x);
  const __nv_bfloat16* dt = static_cast<const __nv_bfloat16*>(a.dt[s]);
  const __nv_bfloat16* Bm = static_cast<const __nv_bfloat16*>(a.Bm[s]) + (size_t)b * kNS;
  const __nv_bfloat16* Cm = static_cast<const __nv_bfloat16*>(a.Cm[s]) + (size_t)b * kNS;
  const float z = __bfloat162float(dt[(size_t)b * D + d]) + a.bias[s][d];
  const float delta = z > 20.f ? z : log1pf(__expf(z));
  const float dx = delta * __bfloat162float(x[(size_t)b * D + d]);
  float* st = c.state + ((size_t)(s * c.B + b) * kNS) * D + d;
  const float* A = a.A[s] + (size_t)d * kNS;
  // all 16 state loads are issued before any use (one memory latency, not sixteen)
  float h[kNS];
#pragma unroll
  for (int n = 0; n < kNS; ++n) h[n] = start ? 0.f : st[(size_t)n * D];
  float y = 0.f;
#pragma unroll
  for (int n = 0; n < kNS; ++n) {
    h[n] = fmaf(ex2(delta * A[n] * kLog2e), h[n], dx * __bfloat162float(Bm[n]));
    y = fmaf(__bfloat162float(Cm[n]), h[n], y);
  }
#pragma unroll
  for (int n = 0; n < kNS; ++n) st[(size_t)n * D] = h[n];
  const int head = d / c.dh, e = d - head * c.dh;
  const __nv_bfloat16 yb = __float2bfloat16_rn(y);
  __nv_bfloat16* ring = static_cast<__nv_bfloat16*>(s == 0 ? c.Kr : c.Vr);
  ring[(((size_t)b * c.H + head) * c.L + (t % c.L)) * c.dh + e] = yb;
  if (end) {
    const int nbv = c.nb[b];
    if (nbv < c.cap) {
      __nv_bfloat16* bl = static_cast<__nv_bfloat16*>(s == 0 ? c.Kb : c.Vb);
      bl[(((size_t)b * c.H + head) * c.cap + nbv) * c.dh + e] = yb;
      if (s == 0 && d == 0) c.bpos[(size_t)b * c.cap + nbv] = t;
    } else if (s == 0 && d == 0) {
      raise_status(a.status, ATTAMBA_DEV_CACHE_FULL);
    }
  }
}

__device__ __forceinline__ void bf16x8_to_f(const uint4& u, float (&f)[8]) {
  const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 v = __bfloat1622float2(p[i]);
    f[2 * i] = v.x;
    f[2 * i + 1] = v.y;
  }
}

template <int kNS>
__global__ void __launch_bounds__(kAttnThreads) decode_attn_kernel(DecodeArgs a) {
  const attamba_cache_t& c = a.c;
  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // The last split of (b, h) holds the newest key (position t): it first runs the SSM step of
  // the head's 64 channels for both SSMs (one per thread), which writes k_t, v_t into the ring.
  // No other block reads that slot (it held position t - L, now outside the window), and the
  // boundary appended at a chunk end lies inside the window, so no other split reads it either.
  if (split == a.splits - 1) {
    ssm_step<kNS>(a, threadIdx.x >> 6, b, h * kDH + (threadIdx.x & 63));
    __syncthreads();
  }
  const int g = lane >> 3;          // key group within the warp
  const int e8 = (lane & 7) * 8;    // head-dim slice of this lane
  const int L = c.L, cap = c.cap;
  const int t = c.pos[b];
  const int lo = max(0, t - L + 1);
  const int nw = t + 1 - lo;
  // boundaries strictly below the window
  const int32_t* bp = c.bpos + (size_t)b * cap;
  int l0 = 0, h0 = min(max(c.nb[b], 0), cap);
  while (l0 < h0) {
    const int mid = (l0 + h0) >> 1;
    if (bp[mid] < lo) l0 = mid + 1; else h0 = mid;
  }
  const int nbb = l0;
  const int nkeys = nbb + nw;
  const int per = (nkeys + a.splits - 1) / a.splits;
  const int kb = split * per;
  const int ke = min(nkeys, kb + per);

  const size_t bh = (size_t)b * c.H + h;
  const __nv_bfloat16* Kb = static_cast<const __nv_bfloat16*>(c.Kb) + bh * cap * kDH + e8;
  const __nv_bfloat16* Vb = static_cast<const __nv_bfloat16*>(c.Vb) + bh * cap * kDH + e8;
  const __nv_bfloat16* Kr = static_cast<const __nv_bfloat16*>(c.Kr) + bh * L * kDH + e8;
  const __nv_bfloat16* Vr = static_cast<const __nv_bfloat16*>(c.Vr) + bh * L * kDH + e8;

  float qf[8];
  {
    const uint4 qu = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.q) + bh * kDH + e8);
    bf16x8_to_f(qu, qf);
    const float sc = a.scale * kLog2e;
#pragma unroll
    for (int i = 0; i < 8; ++i) qf[i] *= sc;
  }
  float m = -INFINITY, l = 0.f, acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;

  // Keys are processed in sweeps of 16 (4 warps x 4 key groups) x kUnroll; two register
  // buffers alternate so one sweep's loads are in flight while the other is computed.
  auto load_sweep = [&](int kk, uint4 (&kr)[kUnroll], uint4 (&vr)[kUnroll]) {
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int k = kk + u * 16 + g;
      if (k < ke) {
        if (k < nbb) {
          kr[u] = __ldg(reinterpret_cast<const uint4*>(Kb + (size_t)k * kDH));
          vr[u] = __ldg(reinterpret_cast<const uint4*>(Vb + (size_t)k * kDH));
        } else {
          // the ring is written during the step (slot of t): read it through L2, not the
          // read-only path
          const int slot = (lo + (k - nbb)) % L;
          kr[u] = __ldcg(reinterpret_cast<const uint4*>(Kr + (size_t)slot * kDH));
          vr[u] = __ldcg(reinterpret_cast<const uint4*>(Vr + (size_t)slot * kDH));
        }
      } else {
        kr[u] = make_uint4(0, 0, 0, 0);
        vr[u] = make_uint4(0, 0, 0, 0);
      }
    }
  };
  auto compute_sweep = [&](int kk, const uint4 (&kr)[kUnroll], const uint4 (&vr)[kUnroll]) {
    float sc[kUnroll];
    float mt = -INFINITY;
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      float kf[8];
      bf16x8_to_f(kr[u], kf);
      float dot = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) dot = fmaf(qf[i], kf[i], dot);
      dot += __shfl_xor_sync(0xffffffffu, dot, 1);
      dot += __shfl_xor_sync(0xffffffffu, dot, 2);
      dot += __shfl_xor_sync(0xffffffffu, dot, 4);
      sc[u] = (kk + u * 16 + g < ke) ? dot : -INFINITY;
      mt = fmaxf(mt, sc[u]);
    }
    const float m_new = fmaxf(m, mt);
    if (m_new != -INFINITY) {
      const float alpha = ex2(m - m_new);
      l *= alpha;
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] *= alpha;
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const float p = ex2(sc[u] - m_new);
        l += p;
        float vf[8];
        bf16x8_to_f(vr[u], vf);
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = fmaf(p, vf[i], acc[i]);
      }
      m = m_new;
    }
  };
  constexpr int kSweep = 16 * kUnroll;
  uint4 kA[kUnroll], vA[kUnroll], kB[kUnroll], vB[kUnroll];
  int kk = kb + warp * 4;
  if (kk < ke) load_sweep(kk, kA, vA);
  while (kk < ke) {
    const bool more = kk + kSweep < ke;
    if (more) load_sweep(kk + kSweep, kB, vB);
    compute_sweep(kk, kA, vA);
    if (!more) break;
    kk += kSweep;
    const bool more2 = kk + kSweep < ke;
    if (more2) load_sweep(kk + kSweep, kA, vA);
    compute_sweep(kk, kB, vB);
    if (!more2) break;
    kk += kSweep;
  }

  // merge the four key groups of the warp (lanes with the same slice: xor 8, 16)
#pragma unroll
  for (int off = 8; off <= 16; off <<= 1) {
    const float mo = __shfl_xor_sync(0xffffffffu, m, off);
    const float lo_ = __shfl_xor_sync(0xffffffffu, l, off);
    const float mn = fmaxf(m, mo);
    const float fa = (m == -INFINITY) ? 0.f : ex2(m - mn);
    const float fb = (mo == -INFINITY) ? 0.f : ex2(mo - mn);
    l = l * fa + lo_ * fb;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float ao = __shfl_xor_sync(0xffffffffu, acc[i], off);
      acc[i] = acc[i] * fa + ao * fb;
    }
    m = mn;
  }
  // merge the four warps through shared memory
  __shared__ float s_m[4], s_l[4], s_acc[4][kDH];
  if (lane < 8) {
#pragma unroll
    for (int i = 0; i < 8; ++i) s_acc[warp][e8 + i] = acc[i];
    if (lane == 0) { s_m[warp] = m; s_l[warp] = l; }
  }
  __syncthreads();
  if (threadIdx.x < kDH) {
    const int e = threadIdx.x;
    float M = -INFINITY;
    for (int w = 0; w < 4; ++w) M = fmaxf(M, s_m[w]);
    float lsum = 0.f, o = 0.f;
    for (int w = 0; w < 4; ++w) {
      if (s_m[w] == -INFINITY) continue;
      const float f = ex2(s_m[w] - M);
      lsum += s_l[w] * f;
      o += s_acc[w][e] * f;
    }
    float* wk = a.work + (bh * a.splits + split) * (kDH + 2);
    wk[e] = o;
    if (e == 0) { wk[kDH] = M; wk[kDH + 1] = lsum; }
  }
}

__global__ void __launch_bounds__(kDH) decode_combine_kernel(DecodeArgs a) {
  const attamba_cache_t& c = a.c;
  const int bh = blockIdx.x;
  const int e = threadIdx.x;
  const float* wk = a.work + (size_t)bh * a.splits * (kDH + 2);
  float M = -INFINITY;
  for (int sp = 0; sp < a.splits; ++sp) M = fmaxf(M, wk[sp * (kDH + 2) + kDH]);
  float lsum = 0.f, o = 0.f;
  for (int sp = 0; sp < a.splits; ++sp) {
    const float ms = wk[sp * (kDH + 2) + kDH];
    if (ms == -INFINITY) continue;
    const float f = ex2(ms - M);
    lsum += wk[sp * (kDH + 2) + kDH + 1] * f;
    o += wk[sp * (kDH + 2) + e] * f;
  }
  static_cast<__nv_bfloat16*>(a.o)[(size_t)bh * kDH + e] = __float2bfloat16_rn(lsum > 0.f ? o / lsum : 0.f);
  if (e == 0 && bh % c.H == 0) {
    const int b = bh / c.H;
    const int o_ = ((c.offset % c.P) + c.P) % c.P;
    const int t = c.pos[b];
    if (chunk_ends_at(t, c.P, o_) && c.nb[b] < c.cap) c.nb[b] += 1;
    c.pos[b] = t + 1;
  }
}
}  // namespace

int32_t decode_splits(const attamba_cache_t& c) {
  const int64_t bh = (int64_t)c.B * c.H;
  const int64_t target = 8 * 148;
  int64_t sp = (target + bh - 1) / bh;
  const int64_t max_sp = ((int64_t)c.cap + c.L) / 128;
  if (sp > max_sp) sp = max_sp;
  if (sp < 1) sp = 1;
  return (int32_t)sp;
}

size_t decode_noalloc_scratch_bytes() { return kNoAllocScratchFloats * sizeof(float); }

// Device address of g_decode_scratch on the current device.  The name is a host
// stand-in, not a device pointer, so the address is asked of the runtime once
// per device (with that device current) and cached.
cudaError_t decode_noalloc_scratch(float** out) {
  static std::mutex mu;
  static float* cached[128] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 128) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (cached[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return e;
    cached[dev] = static_cast<float*>(p);
  }
  *out = cached[dev];
  return cudaSuccess;
}

size_t decode_workspace_bytes(const attamba_cache_t& c) {
  return (size_t)c.B * c.H * decode_splits(c) * (kDH + 2) * sizeof(float);
}

cudaError_t launch_decode_step(const DecodeArgs& a, cudaStream_t s) {
  if (a.c.N == 32)
    decode_attn_kernel<32><<<dim3(a.splits, a.c.H, a.c.B), kAttnThreads, 0, s>>>(a);
  else
    decode_attn_kernel<16><<<dim3(a.splits, a.c.H, a.c.B), kAttnThreads, 0, s>>>(a);
  decode_combine_kernel<<<a.c.B * a.c.H, kDH, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace attamba
