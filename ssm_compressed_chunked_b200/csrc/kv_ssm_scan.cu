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
// Mapping (B200).  Chunks are independent, so the work splits into units of
// (channel group, run of chunks, SSM), one block each, and each thread walks the
// tokens of its chunk run for CPT channels, holding the CPT x N state and the decay rates
// (A * log2 e) in registers as f32x2 pairs over the state index, so the four
// multiply-adds per element issue as two-wide instructions.  B and C, shared
// by all channels of a token, are staged per block in shared memory as fp32 and
// read as broadcast 16-byte loads.  x and dt of the next token are loaded while
// the current one is computed.  The only global writes are the outputs.  Units
// are ~128 tokens for the first 60% of the chunks, then halves and quarters for
// the rest, numbered in that order, so the blocks that start last, while the
// grid drains and SMs fall below three blocks, are short (2-3% faster than equal
// units on the bench workloads, outputs bit-identical).
//
// The work is one exponential per (token, channel, state, SSM): 2 T D N of them
// against 10 D bytes per token, so the multi-function unit (16 ex2 per clock
// per SM), not HBM, sets the pace; on the bench workload it is about 80% busy.
// An FMA-pipe alternative is compiled in for bf16 outputs but off by default
// (ATTAMBA_SCAN_POLY_PAIRS = 0): kPolyPairs of the N/2 state pairs would take
// 2^x = 2^j * 2^f with j = round(x) (added to the exponent field) and 2^f from a
// degree-3 polynomial fitted here by the Remez exchange algorithm to the
// minimax relative error on [-1/2, 1/2] (max relative error 7.5e-5, far below
// bf16's 2^-8), valid for x >= -125 (a token where any lane could go below uses
// the hardware exponential for every pair).  Measured on B200 every share of
// it, like an FMA-pipe softplus or skipping the decay at chunk starts behind a
// branch, was slower: the unit is busy, but the FMA pipe and the instruction
// schedule (one basic block per token pair) are close behind.
#include <type_traits>

#include "common.cuh"
#include "launch.h"

#ifndef ATTAMBA_SCAN_POLY_PAIRS
#define ATTAMBA_SCAN_POLY_PAIRS 0
#endif
#ifndef ATTAMBA_SCAN_CPT
#define ATTAMBA_SCAN_CPT 2
#endif
#ifndef ATTAMBA_SCAN_MINB
#define ATTAMBA_SCAN_MINB 3
#endif

namespace attamba {

namespace {
constexpr int kScanThreads = 128;
#ifndef ATTAMBA_SCAN_F1
#define ATTAMBA_SCAN_F1 60   // percent of the chunks in full units
#endif
#ifndef ATTAMBA_SCAN_F2
#define ATTAMBA_SCAN_F2 80   // percent of the remaining chunks in half units (the rest in quarters)
#endif
#ifndef ATTAMBA_SCAN_TOKENS
#define ATTAMBA_SCAN_TOKENS 128
#endif
constexpr int kStageTokens = 64;       // B/C staging window (even, so token pairs never straddle one)
constexpr int kMaxChunksPerBlock = 256;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kPolyMinExp = -125.f;
// 2^f on [-1/2, 1/2], minimax relative error (own Remez fit), f32 coefficients
constexpr float kP0 = 0.9999280571937561f;
constexpr float kP1 = 0.6932609677314758f;
constexpr float kP2 = 0.2426111251115799f;
constexpr float kP3 = 0.0551716685295105f;

__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;"
      : "=l"(reinterpret_cast<uint64_t&>(d))
      : "l"(reinterpret_cast<const uint64_t&>(a)), "l"(reinterpret_cast<const uint64_t&>(b)),
        "l"(reinterpret_cast<const uint64_t&>(c)));
  return d;
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  float2 d;
  asm("mul.rn.f32x2 %0, %1, %2;"
      : "=l"(reinterpret_cast<uint64_t&>(d))
      : "l"(reinterpret_cast<const uint64_t&>(a)), "l"(reinterpret_cast<const uint64_t&>(b)));
  return d;
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  float2 d;
  asm("add.rn.f32x2 %0, %1, %2;"
      : "=l"(reinterpret_cast<uint64_t&>(d))
      : "l"(reinterpret_cast<const uint64_t&>(a)), "l"(reinterpret_cast<const uint64_t&>(b)));
  return d;
}

__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
  float2 d;
  asm("sub.rn.f32x2 %0, %1, %2;"
      : "=l"(reinterpret_cast<uint64_t&>(d))
      : "l"(reinterpret_cast<const uint64_t&>(a)), "l"(reinterpret_cast<const uint64_t&>(b)));
  return d;
}

// 2^x for x in [-125, 0] on the FMA pipe (see the file comment)
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  const float2 magic = make_float2(12582912.f, 12582912.f);  // 1.5 * 2^23: x + magic rounds x to an integer
  const float2 t = add2(x, magic);
  const float2 j = add2(t, make_float2(-12582912.f, -12582912.f));
  const float2 f = sub2(x, j);
  float2 p = fma2(f, make_float2(kP3, kP3), make_float2(kP2, kP2));
  p = fma2(p, f, make_float2(kP1, kP1));
  p = fma2(p, f, make_float2(kP0, kP0));
  // the low mantissa bits of t hold j; shifted into the exponent field they scale p by 2^j
  return make_float2(__uint_as_float(__float_as_uint(t.x) * 8388608u + __float_as_uint(p.x)),
                     __uint_as_float(__float_as_uint(t.y) * 8388608u + __float_as_uint(p.y)));
}

// softplus(z) = log(1 + e^z) with u = e^z:  log2(1 + u) on the multi-function unit
// when u >= 1/16 (its absolute error, about 2^-22, is then below 3e-6 of the
// result), the series u - u^2/2 + u^3/3 - u^4/4 + u^5/5 below (truncation under
// u^5/6 relative), and z itself above 20.
__device__ __forceinline__ float softplus_f(float z) {
  const float u = ex2(z * kLog2e);
  float lg;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(lg) : "f"(1.f + u));
  const float ser = u * fmaf(u, fmaf(u, fmaf(u, fmaf(u, 0.2f, -0.25f), 1.f / 3.f), -0.5f), 1.f);
  const float v = u < 0.0625f ? ser : lg * 0.6931471805599453f;
  return z > 20.f ? z : v;
}

template <typename T, int CPT> struct Vec;
template <> struct Vec<__nv_bfloat16, 2> {
  using raw = uint32_t;
  static __device__ __forceinline__ raw load(const __nv_bfloat16* p) { return __ldg(reinterpret_cast<const uint32_t*>(p)); }
  static __device__ __forceinline__ void unpack(raw r, float (&v)[2]) {
    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&r));
    v[0] = f.x; v[1] = f.y;
  }
  static __device__ __forceinline__ void store(__nv_bfloat16* p, const float (&v)[2]) {
    *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(v[0], v[1]);
  }
};
template <> struct Vec<__nv_bfloat16, 1> {
  using raw = unsigned short;
  static __device__ __forceinline__ raw load(const __nv_bfloat16* p) { return __ldg(reinterpret_cast<const unsigned short*>(p)); }
  static __device__ __forceinline__ void unpack(raw r, float (&v)[1]) { v[0] = __uint_as_float((uint32_t)r << 16); }
  static __device__ __forceinline__ void store(__nv_bfloat16* p, const float (&v)[1]) { *p = __float2bfloat16_rn(v[0]); }
};
template <> struct Vec<float, 1> {
  using raw = float;
  static __device__ __forceinline__ raw load(const float* p) { return __ldg(p); }
  static __device__ __forceinline__ void unpack(raw r, float (&v)[1]) { v[0] = r; }
  static __device__ __forceinline__ void store(float* p, const float (&v)[1]) { *p = v[0]; }
};
template <> struct Vec<float, 2> {
  using raw = float2;
  static __device__ __forceinline__ raw load(const float* p) { return __ldg(reinterpret_cast<const float2*>(p)); }
  static __device__ __forceinline__ void unpack(raw r, float (&v)[2]) { v[0] = r.x; v[1] = r.y; }
  static __device__ __forceinline__ void store(float* p, const float (&v)[2]) {
    *reinterpret_cast<float2*>(p) = make_float2(v[0], v[1]);
  }
};

// Per-thread state of the scan: CPT channels x NS/2 state pairs.
template <int CPT, int NS> struct ScanState {
  static constexpr int kNP = NS / 2;
  float2 a2[CPT][kNP];  // A * log2 e
  float2 h[CPT][kNP];
  float bias[CPT];
  float amax;           // largest |A| log2 e of the thread's channels
};

// One token: decay, input, readout.  `reset` marks a chunk start: its delta in
// the exponent is replaced by a huge value so exp(delta A) = 0 (A < 0) and the
// state restarts from the token's own input, with no branch.
template <typename T, int CPT, int NS, int POLY_PAIRS>
__device__ __forceinline__ void scan_token(ScanState<CPT, NS>& st, const float* __restrict__ bc, const float (&dl)[CPT],
                                           const float (&dx)[CPT], bool reset, bool poly_ok, float (&y)[CPT]) {
  constexpr int kNP = NS / 2;
  const float4* bc4 = reinterpret_cast<const float4*>(bc);
  float2 Bp[kNP], Cp[kNP];
#pragma unroll
  for (int q = 0; q < kNP / 2; ++q) {
    const float4 b4 = bc4[q], c4 = bc4[kNP / 2 + q];
    Bp[2 * q] = make_float2(b4.x, b4.y);
    Bp[2 * q + 1] = make_float2(b4.z, b4.w);
    Cp[2 * q] = make_float2(c4.x, c4.y);
    Cp[2 * q + 1] = make_float2(c4.z, c4.w);
  }
#pragma unroll
  for (int cc = 0; cc < CPT; ++cc) {
    const float de = reset ? 1e30f : dl[cc];
    const float2 dl2 = make_float2(de, de);
    const float2 dx2 = make_float2(dx[cc], dx[cc]);
    float2 ya = make_float2(0.f, 0.f), yb = make_float2(0.f, 0.f);
#pragma unroll
    for (int q = 0; q < kNP; ++q) {
      const float2 e = mul2(dl2, st.a2[cc][q]);
      float2 a;
      if (q < POLY_PAIRS && poly_ok) a = exp2_poly2(e);
      else a = make_float2(ex2(e.x), ex2(e.y));
      st.h[cc][q] = fma2(a, st.h[cc][q], mul2(dx2, Bp[q]));
      if (q & 1) yb = fma2(Cp[q], st.h[cc][q], yb);
      else ya = fma2(Cp[q], st.h[cc][q], ya);
    }
    y[cc] = (ya.x + ya.y) + (yb.x + yb.y);
  }
}

// Work units: (chunk range, channel group, SSM).  Blocks are numbered big units first, then halves,
// then quarters, and within a size all channel groups and both SSMs of one chunk range are adjacent,
// so the units that start last, as the grid drains, are the short ones.
struct ScanGrid {
  int32_t groups;        // channel groups (grid lanes = 2 * groups)
  int32_t size[3];       // chunks per unit in each phase
  int32_t start[3];      // first chunk of each phase
  int32_t blocks[3];     // blocks of each phase
};
__device__ __forceinline__ void scan_unit(const ScanGrid& gr, int32_t n_chunks, int& xg, int& ssm, int32_t& c_begin,
                                          int32_t& c_end) {
  int i = blockIdx.x;
  int ph = 0;
  while (ph < 2 && i >= gr.blocks[ph]) { i -= gr.blocks[ph]; ++ph; }
  const int lanes = 2 * gr.groups;
  const int lane = i % lanes;
  xg = lane % gr.groups;
  ssm = lane / gr.groups;
  c_begin = gr.start[ph] + (i / lanes) * gr.size[ph];
  c_end = min(c_begin + gr.size[ph], ph < 2 ? gr.start[ph + 1] : n_chunks);
}

// WIDE: element offsets into the [T, D] and [T, N] arrays in 64 bits (T * D or T * N >= 2^31);
// otherwise in 32 bits, which the token loop issues fewer instructions for.
template <typename T, int CPT, int NS, int POLY_PAIRS, int MINB, bool SPLIT_X, bool WIDE>
__global__ void __launch_bounds__(kScanThreads, MINB) kv_ssm_scan_kernel(ScanArgs p, ScanGrid gr) {
  using Off = typename std::conditional<WIDE, int64_t, int32_t>::type;
  using V = Vec<T, CPT>;
  constexpr int kNS = NS;
  constexpr int kNP = NS / 2;
  __shared__ __align__(16) float sBC[kStageTokens][2 * kNS];  // B then C of each staged token
  __shared__ int sCu[kMaxChunksPerBlock + 1];                 // chunk starts of this block
  // launched as a programmatic dependent of the previous kernel in the stream: its outputs may be
  // this kernel's inputs, so nothing is read before that grid has completed
  asm volatile("griddepcontrol.wait;" ::: "memory");

  int xg, s;
  int32_t c_begin, c_end;
  scan_unit(gr, p.n_chunks, xg, s, c_begin, c_end);
  const Off D = p.D;  // element offsets t * D in 32 bits unless WIDE
  const int d0 = (xg * kScanThreads + threadIdx.x) * CPT;
  const bool active = d0 < D;
  if (c_begin >= c_end) return;
  for (int i = threadIdx.x; i <= c_end - c_begin; i += kScanThreads) sCu[i] = p.cu[c_begin + i];

  // one input for both SSMs unless SPLIT_X (kept projections): a base chosen per grid z
  // measured 7% slower on the shared-input workload, so the shared case reads x[0] directly
  const T* __restrict__ x = static_cast<const T*>(SPLIT_X ? p.x[s] : p.x[0]) + d0;
  const T* __restrict__ dt = static_cast<const T*>(p.dt[s]) + d0;
  const T* __restrict__ Bm = static_cast<const T*>(p.Bm[s]);
  const T* __restrict__ Cm = static_cast<const T*>(p.Cm[s]);
  T* __restrict__ out = static_cast<T*>(p.out[s]) + d0;
  T* __restrict__ outc = static_cast<T*>(p.outc[s]);

  ScanState<CPT, NS> st;
  st.amax = 0.f;
#pragma unroll
  for (int c = 0; c < CPT; ++c) {
    st.bias[c] = active ? p.bias[s][d0 + c] : 0.f;
#pragma unroll
    for (int q = 0; q < kNP; ++q) {
      float2 v = make_float2(0.f, 0.f);
      if (active) v = *reinterpret_cast<const float2*>(p.A[s] + (size_t)(d0 + c) * kNS + 2 * q);
      st.a2[c][q] = make_float2(v.x * kLog2e, v.y * kLog2e);
      st.amax = fmaxf(st.amax, fmaxf(-st.a2[c][q].x, -st.a2[c][q].y));
      st.h[c][q] = make_float2(0.f, 0.f);
    }
  }
  __syncthreads();
  const int t_begin = sCu[0];
  const int t_end = sCu[c_end - c_begin];
  // every thread reads the same offsets, so a failed check returns the whole block before its barriers
  if (!in_bounds(t_begin >= 0 && t_begin < t_end && (int64_t)t_end <= p.T && c_end <= p.n_chunks, p.status)) return;
  int ci = 0;                 // chunk of the current token, relative to c_begin
  int next_start = sCu[1];

  // Software pipeline over token pairs: the deltas of the pair being computed
  // come from loads issued one pair earlier, and the loads for the pair after
  // next are issued once the registers they land in have been consumed.
  // With one input per SSM (SPLIT_X) neither SSM's x is in L2 from the other's read, and the loads
  // go a second pair further ahead (184-185 against 189 us on the bench shapes; with the shared
  // input the deeper pipeline measured 2-3 us slower, so it stays one pair ahead there).
  constexpr bool kAhead2 = SPLIT_X;
  float dlA[CPT], dxA[CPT], dlB[CPT], dxB[CPT];
  typename V::raw xA, zA, xB, zB;
  typename V::raw xC = {}, zC = {}, xD = {}, zD = {};   // the pair after that (kAhead2)
  auto delta_of = [&](typename V::raw xr, typename V::raw zr, float (&dl)[CPT], float (&dx)[CPT]) {
    float xv[CPT], zv[CPT];
    V::unpack(xr, xv);
    V::unpack(zr, zv);
#pragma unroll
    for (int cc = 0; cc < CPT; ++cc) {
      dl[cc] = softplus_f(zv[cc] + st.bias[cc]);
      dx[cc] = dl[cc] * xv[cc];
    }
  };
  auto tok = [&](int t) { return min(t, t_end - 1); };  // clamped: harmless reloads past the end
  if (active) {
    delta_of(V::load(x + tok(t_begin) * D), V::load(dt + tok(t_begin) * D), dlA, dxA);
    delta_of(V::load(x + tok(t_begin + 1) * D), V::load(dt + tok(t_begin + 1) * D), dlB, dxB);
    xA = V::load(x + tok(t_begin + 2) * D); zA = V::load(dt + tok(t_begin + 2) * D);
    xB = V::load(x + tok(t_begin + 3) * D); zB = V::load(dt + tok(t_begin + 3) * D);
    if (kAhead2) {
      xC = V::load(x + tok(t_begin + 4) * D); zC = V::load(dt + tok(t_begin + 4) * D);
      xD = V::load(x + tok(t_begin + 5) * D); zD = V::load(dt + tok(t_begin + 5) * D);
    }
  }

  auto step = [&](int t, const float* bc, const float (&dl)[CPT], const float (&dx)[CPT]) {
    float dmax = 0.f;
#pragma unroll
    for (int cc = 0; cc < CPT; ++cc) dmax = fmaxf(dmax, dl[cc]);
    const bool reset = (t == next_start);
    ci += reset ? 1 : 0;
    next_start = sCu[ci + 1];
    bool poly_ok = false;
    if (POLY_PAIRS > 0) poly_ok = !reset && !__any_sync(__activemask(), dmax * st.amax > -kPolyMinExp);
    float y[CPT];
    scan_token<T, CPT, NS, POLY_PAIRS>(st, bc, dl, dx, reset, poly_ok, y);
    V::store(out + t * D, y);
    if (outc != nullptr && t + 1 == next_start && in_bounds(c_begin + ci < p.n_chunks, p.status))
      V::store(outc + (c_begin + ci) * D + d0, y);
  };

  for (int tb = t_begin; tb < t_end; tb += kStageTokens) {
    const int nt = min(kStageTokens, t_end - tb);
    if (tb != t_begin) __syncthreads();
    for (int e = threadIdx.x; e < nt * kNS; e += kScanThreads) {
      const int k = e / kNS, n = e - k * kNS;
      sBC[k][n] = Elem<T>::to_f(Bm[(Off)(tb + k) * kNS + n]);
      sBC[k][kNS + n] = Elem<T>::to_f(Cm[(Off)(tb + k) * kNS + n]);
    }
    __syncthreads();
    if (!active) continue;
    // token pairs are counted from t_begin, so the pipeline stays aligned across windows
    for (int k = 0; k < nt; k += 2) {
      const int t = tb + k;
      step(t, &sBC[k][0], dlA, dxA);
      if (k + 1 < nt) step(t + 1, &sBC[k + 1][0], dlB, dxB);
      delta_of(xA, zA, dlA, dxA);
      delta_of(xB, zB, dlB, dxB);
      if (kAhead2) {
        xA = xC; zA = zC; xB = xD; zB = zD;
        xC = V::load(x + tok(t + 6) * D); zC = V::load(dt + tok(t + 6) * D);
        xD = V::load(x + tok(t + 7) * D); zD = V::load(dt + tok(t + 7) * D);
      } else {
        xA = V::load(x + tok(t + 4) * D); zA = V::load(dt + tok(t + 4) * D);
        xB = V::load(x + tok(t + 5) * D); zB = V::load(dt + tok(t + 5) * D);
      }
    }
  }
}
}  // namespace

namespace {
// N = 16: two channels per thread; N = 32: one (the state and A of two channels would not fit)
template <int NS, int CPT, int MINB, bool SPLIT_X, bool WIDE>
cudaError_t launch_scan(attamba_dtype_t dtype, const ScanArgs& a, cudaStream_t s) {
  // about ATTAMBA_SCAN_TOKENS tokens of chunks per full unit; the chunks after the first
  // ATTAMBA_SCAN_F1 percent in half and quarter units
  int64_t cpb = ((int64_t)ATTAMBA_SCAN_TOKENS * a.n_chunks) / (a.T > 0 ? a.T : 1);
  if (cpb < 1) cpb = 1;
  if (cpb > kMaxChunksPerBlock) cpb = kMaxChunksPerBlock;
  ScanGrid gr;
  gr.groups = (a.D / CPT + kScanThreads - 1) / kScanThreads;
  gr.size[0] = (int32_t)cpb;
  gr.size[1] = (int32_t)(cpb >= 2 ? cpb / 2 : 1);
  gr.size[2] = (int32_t)(cpb >= 4 ? cpb / 4 : 1);
  const int64_t C = a.n_chunks;
  const int64_t c1 = (C * ATTAMBA_SCAN_F1 / 100 / gr.size[0]) * gr.size[0];
  const int64_t c2 = c1 + ((C - c1) * ATTAMBA_SCAN_F2 / 100 / gr.size[1]) * gr.size[1];
  gr.start[0] = 0;
  gr.start[1] = (int32_t)c1;
  gr.start[2] = (int32_t)c2;
  const int lanes = 2 * gr.groups;
  gr.blocks[0] = (int32_t)(c1 / gr.size[0]) * lanes;
  gr.blocks[1] = (int32_t)((c2 - c1) / gr.size[1]) * lanes;
  gr.blocks[2] = (int32_t)((C - c2 + gr.size[2] - 1) / gr.size[2]) * lanes;
  const int64_t nblocks = (int64_t)gr.blocks[0] + gr.blocks[1] + gr.blocks[2];
  if (nblocks < 1 || nblocks > 0x7fffffff) return cudaErrorInvalidValue;
  dim3 grid((unsigned)nblocks);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kScanThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (dtype == ATTAMBA_BF16)
    return cudaLaunchKernelEx(
        &cfg, kv_ssm_scan_kernel<__nv_bfloat16, CPT, NS, NS == 16 ? ATTAMBA_SCAN_POLY_PAIRS : 0, MINB, SPLIT_X, WIDE>, a,
        gr);
  return cudaLaunchKernelEx(&cfg, kv_ssm_scan_kernel<float, CPT, NS, 0, MINB, SPLIT_X, WIDE>, a, gr);
}

template <bool WIDE>
cudaError_t launch_scan_offsets(attamba_dtype_t dtype, const ScanArgs& a, cudaStream_t s) {
  const bool split = a.x[0] != a.x[1];
  if (a.N == 32)
    return split ? launch_scan<32, 1, 3, true, WIDE>(dtype, a, s) : launch_scan<32, 1, 3, false, WIDE>(dtype, a, s);
  return split ? launch_scan<16, ATTAMBA_SCAN_CPT, ATTAMBA_SCAN_MINB, true, WIDE>(dtype, a, s)
               : launch_scan<16, ATTAMBA_SCAN_CPT, ATTAMBA_SCAN_MINB, false, WIDE>(dtype, a, s);
}
}  // namespace

cudaError_t launch_kv_ssm_scan(attamba_dtype_t dtype, const ScanArgs& a, cudaStream_t s) {
  // 32-bit element offsets while they can address every element, 64-bit beyond
  const bool wide = a.T * a.D >= ((int64_t)1 << 31) || a.T * a.N >= ((int64_t)1 << 31);
  return wide ? launch_scan_offsets<true>(dtype, a, s) : launch_scan_offsets<false>(dtype, a, s);
}

}  // namespace attamba
