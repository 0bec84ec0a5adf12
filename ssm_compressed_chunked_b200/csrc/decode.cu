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
//   decode_attn_kernel    per (split, head, sequence), warps 0-3 compute and warp 4
//                         copies.  The last split first runs the SSM step of the
//                         head's channels (reset at a chunk start, state [2,B,N,D]
//                         read and written coalesced, k_t / v_t into ring slot
//                         t mod L and, at a chunk end, into the boundary list) while
//                         warp 4 finds, with a 32-way search of the sorted boundary
//                         positions, how many boundaries lie below the window.  The
//                         split's keys -- (boundaries below the window) then
//                         (window) -- are contiguous row runs of the cache (at most
//                         three per 64-key stage: boundary rows, then the ring
//                         before and after its wrap), so one thread streams them
//                         into a ring of shared-memory stages with bulk async
//                         copies (cp.async.bulk, completion on an mbarrier) and
//                         keeps several stages in flight per CTA; the compute warps
//                         read each key row as 8 lanes x 16 bytes, keep an fp32
//                         online softmax, and write (max, sum, unnormalised output)
//                         to the workspace
//   decode_combine_kernel per (sequence, head): merges the splits, writes o_t,
//                         and advances pos / nb; launched as a programmatic
//                         dependent of the attention kernel (its launch overlaps
//                         that kernel's tail; it waits for the grid's completion
//                         before reading the workspace)
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
constexpr int kComputeThreads = 128;                      // warps 0-3
constexpr int kAttnThreads = kComputeThreads + 32;        // + warp 4, the copy warp
constexpr int kUnroll = 4;                                // keys per lane group and stage
constexpr int kStageKeys = 16 * kUnroll;                  // 4 warps x 4 lane groups x kUnroll
#ifndef ATTAMBA_DECODE_STAGES
#define ATTAMBA_DECODE_STAGES 4
#endif
constexpr int kStages = ATTAMBA_DECODE_STAGES;
constexpr uint32_t kRowBytes = kDH * 2;                   // one bf16 key or value row
constexpr uint32_t kStageBytes = kStageKeys * kRowBytes;  // per tensor
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint64_t kWaitNs = 2000000000ull;

struct DecodeBars {
  uint64_t full[kStages];    // the stage's K and V rows have landed (transaction count)
  uint64_t empty[kStages];   // the four compute warps have read the stage
  int nbb;                   // boundaries below the window
  int abort;
};
constexpr uint32_t kSmemBytes = 2 * kStages * kStageBytes + sizeof(DecodeBars);
// CTAs per SM that the stages allow (about 227 KB of shared memory per SM), for the register budget
constexpr int kMinBlocks = (int)((220u * 1024u) / (kSmemBytes + 2048u)) < 8 ? (int)((220u * 1024u) / (kSmemBytes + 2048u)) : 8;

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// Number of entries of the ascending row p[0, n) that are below v, by all 32 lanes:
// each round probes 32 evenly spaced entries and keeps the gap where the answer lies.
__device__ __forceinline__ int count_below_warp(const int32_t* p, int n, int v, int lane) {
  int l = 0, h = n;   // the answer lies in [l, h]
  while (l < h) {
    const int step = (h - l + 31) >> 5;
    const int idx = l + lane * step;
    const bool below = idx < h && p[idx] < v;
    const int c = __popc(__ballot_sync(0xffffffffu, below));
    if (c == 0) break;                       // p[l] >= v: the answer is l
    const int nl = l + (c - 1) * step + 1;   // p[l + (c - 1) step] < v
    h = min(h, l + c * step);                // p[l + c step] >= v, or the end
    l = nl;
  }
  return l;
}

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
  if (!in_bounds(t >= 0, a.status)) return;   // a position below 0 has no ring slot
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
__global__ void __launch_bounds__(kAttnThreads, kMinBlocks) decode_attn_kernel(DecodeArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  __nv_bfloat16* Ks = reinterpret_cast<__nv_bfloat16*>(smem);
  __nv_bfloat16* Vs = reinterpret_cast<__nv_bfloat16*>(smem + kStages * kStageBytes);
  DecodeBars* bars = reinterpret_cast<DecodeBars*>(smem + 2 * kStages * kStageBytes);
  const attamba_cache_t& c = a.c;
  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int L = c.L, cap = c.cap;
  const int t = c.pos[b];
  const int lo = max(0, t - L + 1);
  if (warp == 4) {
    if (lane == 0) {
      for (int i = 0; i < kStages; ++i) {
        mbar_init(&bars->full[i], 1);
        mbar_init(&bars->empty[i], 4);
      }
      bars->abort = 0;
      fence_mbar_init();
    }
    // boundaries strictly below the window (the entry the SSM step may append lies past nb)
    const int nbb = count_below_warp(c.bpos + (size_t)b * cap, min(max(c.nb[b], 0), cap), lo, lane);
    if (lane == 0) bars->nbb = nbb;
  } else if (split == a.splits - 1) {
    // The last split of (b, h) holds the newest key (position t): it first runs the SSM step of
    // the head's 64 channels for both SSMs (one per thread), which writes k_t, v_t into the ring.
    // No other block reads that slot (it held position t - L, now outside the window), and the
    // boundary appended at a chunk end lies inside the window, so no other split reads it either.
    ssm_step<kNS>(a, threadIdx.x >> 6, b, h * kDH + (threadIdx.x & 63));
    // the copy warp reads the ring through the async proxy
    asm volatile("fence.proxy.async.global;" ::: "memory");
  }
  __syncthreads();
  const int nbb = bars->nbb;
  const int nkeys = nbb + (t + 1 - lo);   // >= 1: the window holds t itself
  // Splits are dealt from the end of the key list: split s covers
  // [nkeys - (splits - s) per, nkeys - (splits - 1 - s) per) cut at 0, so the last split always
  // holds key nkeys - 1 (position t, the ring slot its own SSM step wrote above) and any split
  // left without keys is a leading one.  No CTA reads a slot another CTA writes in this launch.
  const int per = (nkeys + a.splits - 1) / a.splits;
  const int ke = max(0, nkeys - (a.splits - 1 - split) * per);
  const int kb = max(0, ke - per);
  // the boundary rows read lie below the stored count and the capacity, the window starts at 0 or later
  const bool rows_ok = in_bounds(t >= 0 && nbb <= min(max(c.nb[b], 0), cap) && kb >= 0 && ke <= nkeys, a.status);
  const int nst = (rows_ok && ke > kb) ? (ke - kb + kStageKeys - 1) / kStageKeys : 0;
  const size_t bh = (size_t)b * c.H + h;
  volatile int* abort_flag = &bars->abort;

  if (warp == 4) {
    // ------------------------------------------------------------ copy warp
    if (lane == 0) {
      const uint8_t* Kb = static_cast<const uint8_t*>(c.Kb) + bh * cap * kRowBytes;
      const uint8_t* Vb = static_cast<const uint8_t*>(c.Vb) + bh * cap * kRowBytes;
      const uint8_t* Kr = static_cast<const uint8_t*>(c.Kr) + bh * L * kRowBytes;
      const uint8_t* Vr = static_cast<const uint8_t*>(c.Vr) + bh * L * kRowBytes;
      bool ok = true;
      int s = 0;
      for (; s < nst; ++s) {
        const int st = s % kStages;
        if (s >= kStages && !mbar_wait_bounded(&bars->empty[st], ((s / kStages) - 1) & 1, abort_flag, kWaitNs)) {
          ok = false;
          break;
        }
        const int k0 = kb + s * kStageKeys, k1 = min(ke, k0 + kStageKeys);
        uint64_t* bar = &bars->full[st];
        mbar_arrive_expect_tx(bar, (uint32_t)(k1 - k0) * 2 * kRowBytes);
        uint8_t* dK = reinterpret_cast<uint8_t*>(Ks) + st * kStageBytes;
        uint8_t* dV = reinterpret_cast<uint8_t*>(Vs) + st * kStageBytes;
        // boundary rows k0 .. min(k1, nbb) - 1
        const int b1 = min(k1, nbb);
        if (b1 > k0) {
          bulk_g2s(dK, Kb + (size_t)k0 * kRowBytes, (uint32_t)(b1 - k0) * kRowBytes, bar);
          bulk_g2s(dV, Vb + (size_t)k0 * kRowBytes, (uint32_t)(b1 - k0) * kRowBytes, bar);
        }
        // window keys: key k >= nbb is position lo + (k - nbb), in ring slot (lo + k - nbb) mod L
        for (int k = max(k0, nbb); k < k1;) {
          const int slot = (lo + (k - nbb)) % L;
          const int cnt = min(k1 - k, L - slot);
          bulk_g2s(dK + (k - k0) * kRowBytes, Kr + (size_t)slot * kRowBytes, (uint32_t)cnt * kRowBytes, bar);
          bulk_g2s(dV + (k - k0) * kRowBytes, Vr + (size_t)slot * kRowBytes, (uint32_t)cnt * kRowBytes, bar);
          k += cnt;
        }
      }
      if (!ok) {
        *abort_flag = 1;
        // copies may still be in flight into the stages: they must land before the CTA exits
        for (int j = max(0, s - kStages); j < s; ++j)
          mbar_wait_timeout(&bars->full[j % kStages], (j / kStages) & 1, kWaitNs);
      }
    }
    return;
  }

  // -------------------------------------------------------------- compute warps 0-3
  const int g = lane >> 3;          // key group within the warp
  const int e8 = (lane & 7) * 8;    // head-dim slice of this lane
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

  bool ok = true;
  for (int s = 0; s < nst; ++s) {
    const int st = s % kStages;
    if (!__all_sync(0xffffffffu, mbar_wait_bounded(&bars->full[st], (s / kStages) & 1, abort_flag, kWaitNs))) {
      ok = false;
      break;
    }
    const int cnt = min(ke - kb - s * kStageKeys, kStageKeys);
    const __nv_bfloat16* ks = Ks + st * (kStageKeys * kDH) + e8;
    const __nv_bfloat16* vs = Vs + st * (kStageKeys * kDH) + e8;
    uint4 kr[kUnroll], vr[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int row = u * 16 + warp * 4 + g;
      if (row < cnt) {
        kr[u] = *reinterpret_cast<const uint4*>(ks + row * kDH);
        vr[u] = *reinterpret_cast<const uint4*>(vs + row * kDH);
      } else {
        kr[u] = make_uint4(0, 0, 0, 0);
        vr[u] = make_uint4(0, 0, 0, 0);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars->empty[st]);   // this warp's rows of the stage are in registers
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
      sc[u] = (u * 16 + warp * 4 + g < cnt) ? dot : -INFINITY;
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
  }
  if (!ok) {
    *abort_flag = 1;
    if (lane == 0) raise_status(a.status, ATTAMBA_DEV_TIMEOUT);
  }
  // the combine may be scheduled once every CTA is past its key loop (it still waits for this
  // grid to complete before it reads the workspace)
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

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
  // merge the four warps through shared memory (a barrier of the compute warps only: every one
  // of them gets here, a timed-out wait included)
  __shared__ float s_m[4], s_l[4], s_acc[4][kDH];
  if (lane < 8) {
#pragma unroll
    for (int i = 0; i < 8; ++i) s_acc[warp][e8 + i] = acc[i];
    if (lane == 0) { s_m[warp] = m; s_l[warp] = l; }
  }
  asm volatile("bar.sync 1, %0;" ::"n"(kComputeThreads) : "memory");
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
  // launched as a programmatic dependent of decode_attn_kernel: wait for that grid's completion
  // and memory before reading what it wrote
  asm volatile("griddepcontrol.wait;" ::: "memory");
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
#ifndef ATTAMBA_DECODE_TARGET
#define ATTAMBA_DECODE_TARGET (8 * 148)
#endif
  const int64_t target = ATTAMBA_DECODE_TARGET;
  int64_t sp = (target + bh - 1) / bh;
  const int64_t max_sp = ((int64_t)c.cap + c.L) / 128;
  if (sp > max_sp) sp = max_sp;
  if (sp < 1) sp = 1;
  return (int32_t)sp;
}

size_t decode_noalloc_scratch_bytes() { return kNoAllocScratchFloats * sizeof(float); }

// Device address of g_decode_scratch on the current device.  The name is a host
// stand-in, not a device pointer, so the address is asked of the runtime (with
// the device current) and cached.  The address belongs to the copy of this
// library's device code loaded into the device's current context; a context
// torn down and created again (cudaDeviceReset) loads it again, perhaps
// elsewhere, so the cache is keyed on the context's process-unique id as well
// as the device.  Where the driver cannot report that id, the address is asked
// for on every call (a lookup, no allocation).
namespace {
bool current_context_id(unsigned long long* id) {
  static PFN_cuCtxGetCurrent_v4000 get_current = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    return cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 4000, cudaEnableDefault, &q) == cudaSuccess &&
                   q == cudaDriverEntryPointSuccess
               ? reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p)
               : nullptr;
  }();
  static PFN_cuCtxGetId_v12000 get_id = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    return cudaGetDriverEntryPointByVersion("cuCtxGetId", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
                   q == cudaDriverEntryPointSuccess
               ? reinterpret_cast<PFN_cuCtxGetId_v12000>(p)
               : nullptr;
  }();
  CUcontext ctx = nullptr;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}
}  // namespace

cudaError_t decode_noalloc_scratch(float** out) {
  struct Entry {
    unsigned long long ctx_id;
    float* ptr;
  };
  static std::mutex mu;
  static Entry cached[128] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 128) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  unsigned long long id = 0;
  bool have_id = current_context_id(&id);
  if (have_id && cached[dev].ptr != nullptr && cached[dev].ctx_id == id) {
    *out = cached[dev].ptr;
    return cudaSuccess;
  }
  void* p = nullptr;
  e = cudaGetSymbolAddress(&p, g_decode_scratch);   // makes the device's primary context current
  if (e != cudaSuccess) return e;
  if (!have_id) have_id = current_context_id(&id);
  cached[dev] = have_id ? Entry{id, static_cast<float*>(p)} : Entry{0, nullptr};
  *out = static_cast<float*>(p);
  return cudaSuccess;
}

size_t decode_workspace_bytes(const attamba_cache_t& c) {
  return (size_t)c.B * c.H * decode_splits(c) * (kDH + 2) * sizeof(float);
}

cudaError_t launch_decode_step(const DecodeArgs& a, cudaStream_t s) {
  const void* k = a.c.N == 32 ? reinterpret_cast<const void*>(decode_attn_kernel<32>)
                              : reinterpret_cast<const void*>(decode_attn_kernel<16>);
  cudaError_t e = raise_smem_limit(k, (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  if (a.c.N == 32)
    decode_attn_kernel<32><<<dim3(a.splits, a.c.H, a.c.B), kAttnThreads, kSmemBytes, s>>>(a);
  else
    decode_attn_kernel<16><<<dim3(a.splits, a.c.H, a.c.B), kAttnThreads, kSmemBytes, s>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // the combine's launch overlaps the attention kernel's tail (programmatic dependent launch)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(a.c.B * a.c.H));
  cfg.blockDim = dim3(kDH);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_combine_kernel, a);
}

}  // namespace attamba
