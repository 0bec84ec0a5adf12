// extern "C" entry points: host-side validation, then the stream-ordered launches.
// The passages each entry point follows are cited in include/attamba.h.
#include <stdio.h>
#include <string.h>

#include "attamba.h"
#include "launch.h"

namespace {
thread_local char g_err[256] = "";

attamba_status_t cuda_fail(cudaError_t e, const char* where) {
  snprintf(g_err, sizeof(g_err), "%s: %s", where, cudaGetErrorString(e));
  return ATTAMBA_ERR_CUDA;
}
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool ok_dtype(attamba_dtype_t d) { return d == ATTAMBA_F32 || d == ATTAMBA_BF16; }
constexpr int64_t kMaxTokens = (int64_t)1 << 31;
}  // namespace

extern "C" {

const char* attamba_version(void) {
#if defined(ATTAMBA_CHECKED)
  return "attamba-b200 0.1 (sm_100a) checked";
#else
  return "attamba-b200 0.1 (sm_100a)";
#endif
}

const char* attamba_status_string(attamba_status_t s) {
  switch (s) {
    case ATTAMBA_OK: return "ok";
    case ATTAMBA_ERR_INVALID_ARG: return "invalid argument";
    case ATTAMBA_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case ATTAMBA_ERR_CUDA: return "CUDA error";
  }
  return "unknown status";
}

const char* attamba_last_error(void) { return g_err; }

int32_t attamba_uniform_chunk_count(int32_t n, int32_t P, int32_t offset) {
  if (n < 1 || P < 1) return -1;
  const int32_t o = ((offset % P) + P) % P;
  // starts: 0, then o + kP in (0, n)
  int32_t cnt = 1;
  const int32_t first = (o == 0) ? P : o;
  if (first < n) cnt += 1 + (n - 1 - first) / P;
  return cnt;
}

attamba_status_t attamba_chunk_index(const int32_t* cu_in, int32_t n_chunks, int32_t B, int32_t n,
                                     int32_t P, int32_t offset, int32_t L, attamba_mask_t mode,
                                     const attamba_index_t* out, int32_t* d_status,
                                     attamba_stream_t stream) {
  if (!out || B < 1 || n < 1 || (int64_t)B * n >= kMaxTokens || L < 0 || n_chunks < B)
    return ATTAMBA_ERR_INVALID_ARG;
  if (mode != ATTAMBA_MASK_TRAIN && mode != ATTAMBA_MASK_TEST) return ATTAMBA_ERR_INVALID_ARG;
  if (!out->cu || !out->bpos || !out->bptr || !out->ls || !out->nbb) return ATTAMBA_ERR_INVALID_ARG;
  if (out->n_chunks != n_chunks || out->B != B || out->n != n) return ATTAMBA_ERR_INVALID_ARG;
  if (n_chunks > (int64_t)B * n) return ATTAMBA_ERR_INVALID_ARG;
  if (cu_in == nullptr) {
    if (P < 1) return ATTAMBA_ERR_INVALID_ARG;
    if ((int64_t)attamba_uniform_chunk_count(n, P, offset) * B != n_chunks) return ATTAMBA_ERR_INVALID_ARG;
  }
  cudaError_t e = attamba::launch_chunk_index(cu_in, n_chunks, B, n, P, offset, L, (int)mode, *out, d_status,
                                              reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ATTAMBA_OK : cuda_fail(e, "attamba_chunk_index");
}

namespace {
attamba_status_t scan_entry(attamba_dtype_t dtype, const void* u_k, const void* u_v, const void* dt_k,
                            const void* dt_v, const float* bias_k, const float* bias_v, const float* A_k,
                            const float* A_v, const void* B_k, const void* C_k, const void* B_v, const void* C_v,
                            const int32_t* cu, int32_t n_chunks, int64_t T, int32_t D, int32_t N, void* K,
                            void* V, void* Kc, void* Vc, int32_t* d_status, cudaStream_t stream, const char* name) {
  if (!ok_dtype(dtype)) return ATTAMBA_ERR_UNSUPPORTED;
  if (N != 16 && N != 32) return ATTAMBA_ERR_UNSUPPORTED;
  if (T < 1 || T >= kMaxTokens || D < 8 || D % 8 != 0 || n_chunks < 1 || n_chunks > T)
    return ATTAMBA_ERR_INVALID_ARG;
  const void* req[] = {u_k, u_v, dt_k, dt_v, bias_k, bias_v, A_k, A_v, B_k, C_k, B_v, C_v, cu, K, V};
  for (const void* p : req)
    if (!p || !aligned16(p)) return ATTAMBA_ERR_INVALID_ARG;
  if ((Kc == nullptr) != (Vc == nullptr)) return ATTAMBA_ERR_INVALID_ARG;
  if (Kc && (!aligned16(Kc) || !aligned16(Vc))) return ATTAMBA_ERR_INVALID_ARG;
  attamba::ScanArgs a{};
  a.x[0] = u_k; a.x[1] = u_v;
  a.dt[0] = dt_k; a.dt[1] = dt_v;
  a.bias[0] = bias_k; a.bias[1] = bias_v;
  a.A[0] = A_k; a.A[1] = A_v;
  a.Bm[0] = B_k; a.Bm[1] = B_v;
  a.Cm[0] = C_k; a.Cm[1] = C_v;
  a.cu = cu;
  a.n_chunks = n_chunks;
  a.T = T;
  a.D = D;
  a.N = N;
  a.out[0] = K; a.out[1] = V;
  a.outc[0] = Kc; a.outc[1] = Vc;
  a.status = d_status;
  cudaError_t e = attamba::launch_kv_ssm_scan(dtype, a, stream);
  return e == cudaSuccess ? ATTAMBA_OK : cuda_fail(e, name);
}
}  // namespace

attamba_status_t attamba_kv_ssm_scan(attamba_dtype_t dtype, const void* x, const void* dt_k,
                                     const void* dt_v, const float* bias_k, const float* bias_v,
                                     const float* A_k, const float* A_v, const void* B_k,
                                     const void* C_k, const void* B_v, const void* C_v,
                                     const int32_t* cu, int32_t n_chunks, int64_t T, int32_t D,
                                     int32_t N, void* K, void* V, void* Kc, void* Vc,
                                     int32_t* d_status, attamba_stream_t stream) {
  return scan_entry(dtype, x, x, dt_k, dt_v, bias_k, bias_v, A_k, A_v, B_k, C_k, B_v, C_v, cu, n_chunks, T, D, N,
                    K, V, Kc, Vc, d_status, reinterpret_cast<cudaStream_t>(stream), "attamba_kv_ssm_scan");
}

attamba_status_t attamba_kv_ssm_scan_u(attamba_dtype_t dtype, const void* u_k, const void* u_v,
                                       const void* dt_k, const void* dt_v, const float* bias_k,
                                       const float* bias_v, const float* A_k, const float* A_v,
                                       const void* B_k, const void* C_k, const void* B_v, const void* C_v,
                                       const int32_t* cu, int32_t n_chunks, int64_t T, int32_t D, int32_t N,
                                       void* K, void* V, void* Kc, void* Vc, int32_t* d_status,
                                       attamba_stream_t stream) {
  return scan_entry(dtype, u_k, u_v, dt_k, dt_v, bias_k, bias_v, A_k, A_v, B_k, C_k, B_v, C_v, cu, n_chunks, T, D,
                    N, K, V, Kc, Vc, d_status, reinterpret_cast<cudaStream_t>(stream), "attamba_kv_ssm_scan_u");
}

attamba_status_t attamba_proj_gemm(attamba_dtype_t dtype, const void* X, const void* W, int64_t M, int32_t Nout,
                                   int32_t K, const attamba_proj_seg_t* segs, int32_t nseg, int32_t* d_status,
                                   attamba_stream_t stream) {
  if (dtype != ATTAMBA_BF16) return ATTAMBA_ERR_UNSUPPORTED;
  if (M < 1 || Nout < 1 || K < 64 || K % 64 != 0 || !segs || nseg < 1 || nseg > attamba::kMaxProjSegs)
    return ATTAMBA_ERR_INVALID_ARG;
  if (M >= ((int64_t)1 << 31) || M * (int64_t)K >= ((int64_t)1 << 40) || M * (int64_t)Nout >= ((int64_t)1 << 40))
    return ATTAMBA_ERR_INVALID_ARG;
  if (!X || !W || !aligned16(X) || !aligned16(W)) return ATTAMBA_ERR_INVALID_ARG;
  attamba::ProjArgs a{};
  a.X = X; a.W = W; a.M = M; a.Nout = Nout; a.K = K; a.nseg = nseg; a.status = d_status;
  int32_t end = 0;
  for (int s = 0; s < nseg; ++s) {
    const attamba_proj_seg_t& g = segs[s];
    if (!g.ptr || !aligned16(g.ptr) || g.col0 < end || g.width < 8 || g.col0 % 8 != 0 || g.width % 8 != 0 ||
        (int64_t)g.col0 + g.width > Nout)
      return ATTAMBA_ERR_INVALID_ARG;
    a.seg_ptr[s] = g.ptr;
    a.seg_col0[s] = g.col0;
    a.seg_width[s] = g.width;
    end = g.col0 + g.width;
  }
  cudaError_t e = attamba::launch_proj_gemm(a, reinterpret_cast<cudaStream_t>(stream));
  if (e == cudaErrorNotSupported) return ATTAMBA_ERR_UNSUPPORTED;
  return e == cudaSuccess ? ATTAMBA_OK : cuda_fail(e, "attamba_proj_gemm");
}

attamba_status_t attamba_chunk_attn_fwd(attamba_dtype_t dtype, const void* q, const void* K,
                                        const void* V, const void* Kc, const void* Vc,
                                        const attamba_index_t* idx, int32_t H, int32_t dh,
                                        float scale, void* O, float* lse, int32_t* d_status,
                                        attamba_stream_t stream) {
  if (!ok_dtype(dtype)) return ATTAMBA_ERR_UNSUPPORTED;
  if (dh != 64) return ATTAMBA_ERR_UNSUPPORTED;
  if (!idx || H < 1 || idx->B < 1 || idx->n < 1 || idx->n_chunks < idx->B) return ATTAMBA_ERR_INVALID_ARG;
  const int64_t T = (int64_t)idx->B * idx->n;
  if (T >= kMaxTokens || T * H >= kMaxTokens) return ATTAMBA_ERR_INVALID_ARG;
  const void* req[] = {q, K, V, Kc, Vc, O};
  for (const void* p : req)
    if (!p || !aligned16(p)) return ATTAMBA_ERR_INVALID_ARG;
  if (!idx->bpos || !idx->bptr || !idx->ls || !idx->nbb) return ATTAMBA_ERR_INVALID_ARG;
  if (!(scale > 0.f)) return ATTAMBA_ERR_INVALID_ARG;
  attamba::AttnArgs a{};
  a.q = q; a.K = K; a.V = V; a.Kc = Kc; a.Vc = Vc;
  a.bpos = idx->bpos; a.bptr = idx->bptr; a.ls = idx->ls; a.nbb = idx->nbb;
  a.B = idx->B; a.n = idx->n; a.H = H; a.dh = dh; a.n_chunks = idx->n_chunks;
  a.scale = scale; a.O = O; a.lse = lse; a.status = d_status;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = (dtype == ATTAMBA_BF16) ? attamba::launch_chunk_attn_bf16(a, s) : attamba::launch_chunk_attn_f32(a, s);
  if (e == cudaErrorNotSupported) {
    snprintf(g_err, sizeof(g_err), "attamba_chunk_attn_fwd: cuTensorMapEncodeTiled unavailable or rejected");
    return ATTAMBA_ERR_CUDA;
  }
  return e == cudaSuccess ? ATTAMBA_OK : cuda_fail(e, "attamba_chunk_attn_fwd");
}

attamba_status_t attamba_selftest_wait_timeout(uint64_t limit_ns, int32_t* d_status, attamba_stream_t stream) {
  if (!d_status || limit_ns < 1000 || limit_ns > 1000000000ull) return ATTAMBA_ERR_INVALID_ARG;
  const cudaError_t e = attamba::launch_wait_selftest(limit_ns, d_status, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ATTAMBA_OK : cuda_fail(e, "attamba_selftest_wait_timeout");
}

size_t attamba_cache_bytes(const attamba_cache_t* cache) {
  if (!cache || cache->B < 1 || cache->H < 1 || cache->N < 1 || cache->L < 1 || cache->cap < 1 || cache->dh != 64)
    return 0;
  const uint64_t B = (uint64_t)cache->B, H = (uint64_t)cache->H, dh = (uint64_t)cache->dh;
  const uint64_t N = (uint64_t)cache->N, L = (uint64_t)cache->L, cap = (uint64_t)cache->cap;
  auto up = [](uint64_t bytes) { return (bytes + 255) & ~uint64_t(255); };
  const uint64_t bytes = up(2 * B * N * H * dh * 4)          // state [2, B, N, D] fp32
                         + 2 * up(B * H * cap * dh * 2)     // Kb, Vb [B, H, cap, dh] bf16
                         + up(B * cap * 4)                  // bpos [B, cap] int32
                         + 2 * up(B * H * L * dh * 2)       // Kr, Vr [B, H, L, dh] bf16
                         + 2 * up(B * 4);                   // nb, pos [B] int32
  return (size_t)bytes;
}

size_t attamba_decode_workspace_size(const attamba_cache_t* cache) {
  if (!cache || cache->B < 1 || cache->H < 1 || cache->cap < 1 || cache->L < 1) return 0;
  return attamba::decode_workspace_bytes(*cache);
}

attamba_status_t attamba_decode_step(attamba_dtype_t dtype, const attamba_cache_t* cache,
                                     const void* q_t, const void* x_t, const void* dt_k,
                                     const void* dt_v, const float* bias_k, const float* bias_v,
                                     const float* A_k, const float* A_v, const void* B_k,
                                     const void* C_k, const void* B_v, const void* C_v,
                                     float scale, void* o_t, void* workspace,
                                     size_t workspace_bytes, int32_t* d_status,
                                     attamba_stream_t stream) {
  if (dtype != ATTAMBA_BF16) return ATTAMBA_ERR_UNSUPPORTED;
  if (!cache) return ATTAMBA_ERR_INVALID_ARG;
  const attamba_cache_t& c = *cache;
  if (c.dh != 64 || (c.N != 16 && c.N != 32)) return ATTAMBA_ERR_UNSUPPORTED;
  if (c.B < 1 || c.H < 1 || c.P < 1 || c.L < 1 || c.cap < 1) return ATTAMBA_ERR_INVALID_ARG;
  if ((int64_t)c.B * c.H * c.cap * c.dh >= ((int64_t)1 << 40)) return ATTAMBA_ERR_INVALID_ARG;
  const void* req[] = {c.state, c.Kb, c.Vb, c.bpos, c.Kr, c.Vr, c.nb, c.pos, q_t, x_t, dt_k, dt_v,
                       bias_k, bias_v, A_k, A_v, B_k, C_k, B_v, C_v, o_t, workspace};
  for (const void* p : req)
    if (!p) return ATTAMBA_ERR_INVALID_ARG;
  const void* al[] = {c.Kb, c.Vb, c.Kr, c.Vr, q_t, workspace};
  for (const void* p : al)
    if (!aligned16(p)) return ATTAMBA_ERR_INVALID_ARG;
  if (workspace_bytes < attamba::decode_workspace_bytes(c)) return ATTAMBA_ERR_INVALID_ARG;
  if (!(scale > 0.f)) return ATTAMBA_ERR_INVALID_ARG;
  attamba::DecodeArgs a{};
  a.c = c;
  a.q = q_t; a.x = x_t;
  a.dt[0] = dt_k; a.dt[1] = dt_v;
  a.bias[0] = bias_k; a.bias[1] = bias_v;
  a.A[0] = A_k; a.A[1] = A_v;
  a.Bm[0] = B_k; a.Bm[1] = B_v;
  a.Cm[0] = C_k; a.Cm[1] = C_v;
  a.scale = scale; a.o = o_t;
  a.work = static_cast<float*>(workspace);
  a.splits = attamba::decode_splits(c);
  a.status = d_status;
  cudaError_t e = attamba::launch_decode_step(a, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ATTAMBA_OK : cuda_fail(e, "attamba_decode_step");
}

attamba_status_t attamba_cache_from_prefill(attamba_dtype_t dtype, const attamba_cache_t* cache,
                                            const void* K, const void* V, const void* x,
                                            const void* dt_k, const void* dt_v, const float* bias_k,
                                            const float* bias_v, const float* A_k, const float* A_v,
                                            const void* B_k, const void* C_k, const void* B_v,
                                            const void* C_v, int32_t n0, int32_t* d_status,
                                            attamba_stream_t stream) {
  (void)d_status;  // nothing is detected on the device: every limit is checked here
  if (dtype != ATTAMBA_BF16) return ATTAMBA_ERR_UNSUPPORTED;
  if (!cache) return ATTAMBA_ERR_INVALID_ARG;
  const attamba_cache_t& c = *cache;
  if (c.dh != 64 || (c.N != 16 && c.N != 32)) return ATTAMBA_ERR_UNSUPPORTED;
  if (c.B < 1 || c.H < 1 || c.P < 1 || c.L < 1 || c.cap < 1 || n0 < 1) return ATTAMBA_ERR_INVALID_ARG;
  if ((int64_t)c.B * c.H * c.cap * c.dh >= ((int64_t)1 << 40)) return ATTAMBA_ERR_INVALID_ARG;
  if ((int64_t)c.B * n0 * c.H * c.dh >= ((int64_t)1 << 40)) return ATTAMBA_ERR_INVALID_ARG;
  const void* req[] = {c.state, c.Kb, c.Vb, c.bpos, c.Kr, c.Vr, c.nb, c.pos, K, V, x, dt_k, dt_v,
                       bias_k, bias_v, A_k, A_v, B_k, C_k, B_v, C_v};
  for (const void* p : req)
    if (!p) return ATTAMBA_ERR_INVALID_ARG;
  const void* al[] = {c.Kb, c.Vb, c.Kr, c.Vr, K, V};
  for (const void* p : al)
    if (!aligned16(p)) return ATTAMBA_ERR_INVALID_ARG;
  const int32_t nb = attamba::handoff_boundaries(n0, c.P, c.offset);
  if (nb > c.cap) {
    snprintf(g_err, sizeof(g_err), "attamba_cache_from_prefill: %d boundaries in [0, %d) exceed cap %d", nb, n0,
             c.cap);
    return ATTAMBA_ERR_INVALID_ARG;
  }
  attamba::HandoffArgs a{};
  a.c = c;
  a.K = K; a.V = V; a.x = x;
  a.dt[0] = dt_k; a.dt[1] = dt_v;
  a.bias[0] = bias_k; a.bias[1] = bias_v;
  a.A[0] = A_k; a.A[1] = A_v;
  a.Bm[0] = B_k; a.Bm[1] = B_v;
  a.Cm[0] = C_k; a.Cm[1] = C_v;
  a.n0 = n0;
  a.nb = nb;
  cudaError_t e = attamba::launch_cache_from_prefill(a, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ATTAMBA_OK : cuda_fail(e, "attamba_cache_from_prefill");
}

attamba_status_t attamba_decode_step_noalloc(attamba_dtype_t dtype, const attamba_cache_t* cache,
                                             const void* q_t, const void* x_t, const void* dt_k,
                                             const void* dt_v, const float* bias_k, const float* bias_v,
                                             const float* A_k, const float* A_v, const void* B_k,
                                             const void* C_k, const void* B_v, const void* C_v,
                                             float scale, void* o_t, int32_t* d_status,
                                             attamba_stream_t stream) {
  if (dtype != ATTAMBA_BF16) return ATTAMBA_ERR_UNSUPPORTED;
  if (!cache) return ATTAMBA_ERR_INVALID_ARG;
  const attamba_cache_t& c = *cache;
  if (c.dh != 64 || (c.N != 16 && c.N != 32)) return ATTAMBA_ERR_UNSUPPORTED;
  if (c.B < 1 || c.H < 1 || c.P < 1 || c.L < 1 || c.cap < 1) return ATTAMBA_ERR_INVALID_ARG;
  if ((int64_t)c.B * c.H * c.cap * c.dh >= ((int64_t)1 << 40)) return ATTAMBA_ERR_INVALID_ARG;
  const void* req[] = {c.state, c.Kb, c.Vb, c.bpos, c.Kr, c.Vr, c.nb, c.pos, q_t, x_t, dt_k, dt_v,
                       bias_k, bias_v, A_k, A_v, B_k, C_k, B_v, C_v, o_t};
  for (const void* p : req)
    if (!p) return ATTAMBA_ERR_INVALID_ARG;
  const void* al[] = {c.Kb, c.Vb, c.Kr, c.Vr, q_t};
  for (const void* p : al)
    if (!aligned16(p)) return ATTAMBA_ERR_INVALID_ARG;
  if (!(scale > 0.f)) return ATTAMBA_ERR_INVALID_ARG;
  const size_t need = attamba::decode_workspace_bytes(c);
  if (need > attamba::decode_noalloc_scratch_bytes()) {
    snprintf(g_err, sizeof(g_err),
             "attamba_decode_step_noalloc: this cache needs %zu bytes of split-K scratch, the built-in "
             "scratch holds %zu; use attamba_decode_step with a workspace",
             need, attamba::decode_noalloc_scratch_bytes());
    return ATTAMBA_ERR_UNSUPPORTED;
  }
  float* scratch = nullptr;
  cudaError_t e = attamba::decode_noalloc_scratch(&scratch);
  if (e != cudaSuccess) return cuda_fail(e, "attamba_decode_step_noalloc (scratch address)");
  attamba::DecodeArgs a{};
  a.c = c;
  a.q = q_t; a.x = x_t;
  a.dt[0] = dt_k; a.dt[1] = dt_v;
  a.bias[0] = bias_k; a.bias[1] = bias_v;
  a.A[0] = A_k; a.A[1] = A_v;
  a.Bm[0] = B_k; a.Bm[1] = B_v;
  a.Cm[0] = C_k; a.Cm[1] = C_v;
  a.scale = scale; a.o = o_t;
  a.work = scratch;
  a.splits = attamba::decode_splits(c);
  a.status = d_status;
  e = attamba::launch_decode_step(a, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ATTAMBA_OK : cuda_fail(e, "attamba_decode_step_noalloc");
}

}  // extern "C"
