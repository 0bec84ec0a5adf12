/*
 * attamba.h -- C ABI of the Attamba attention layer's forward hot path on B200 (sm_100a).
 *
 * The method (arXiv 2411.17685, "Attamba: Attending To Multi-Token States"):
 * two selective state-space scans (KV-SSM) produce the keys and values in place
 * of W_K and W_V, their state restarting at every chunk start; softmax
 * attention then reads, for each query, the last token of every completed
 * chunk plus either its own partial chunk (M_train) or a window of L leading
 * tokens (M_test).  Passages are cited as page + section:
 *   [pith, carries]  pith.science review, "What carries the argument"
 *                    (M_train Eq. 5, M_test Eq. 7, leading tokens Eq. 8, cyclic chunking)
 *   [pith, core]     pith.science review, "Core claim" (K = SSM_K(X), V = SSM_V(X);
 *                    only boundary states are cached at inference)
 *   [pith, if]       pith.science review, "If this is right" (cu_seqlens chunks,
 *                    8x cache compression at P = 8, L = 64)
 *   [pith, ref-eq7]  pith.science review, Referee Report, major comment on Eq. (7)
 *                    (only completed chunks are attended at test time)
 *   [pith, params]   pith.science review, "Assumptions & free parameters"
 *                    (Mamba selective SSM, Section 3.2 Eq. 3; P, L, offset = layer index)
 *
 * Conventions for every call
 *   - Every tensor pointer is caller-owned DEVICE memory, row-major, contiguous,
 *     16-byte aligned.  The library allocates nothing and keeps no state
 *     between calls; it is thread-safe.
 *   - Every call is asynchronous on the given stream (a cudaStream_t; NULL is
 *     the legacy default stream) and never synchronizes.  The scans and the
 *     bf16 attention are programmatic dependent launches: they may start while
 *     the previous kernel in the stream is finishing, but read no input before
 *     that kernel has completed, so stream order holds as for any launch.
 *   - Arguments the host can check are checked before any launch; a bad one
 *     returns ATTAMBA_ERR_INVALID_ARG (or ATTAMBA_ERR_UNSUPPORTED for a shape
 *     or dtype outside the supported set) and launches nothing.
 *   - Errors only the device can see (malformed chunk offsets, a full decode
 *     cache, a wait that ran out of time) are OR-ed as ATTAMBA_DEV_* bits into
 *     the caller's int32 status word `d_status` (device memory, nullable), which
 *     the caller reads whenever it chooses.  No kernel traps.
 *   - A launch failure returns ATTAMBA_ERR_CUDA; attamba_last_error() gives the
 *     CUDA error text of the calling thread's last failure.
 *   - Layout names: T = B*n tokens of B sequences of length n laid end to end;
 *     D = d_model = H*dh; N = SSM state size; head h owns channels [h*dh, (h+1)*dh).
 */
#ifndef ATTAMBA_H
#define ATTAMBA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* attamba_stream_t; /* same object as cudaStream_t */

typedef enum {
  ATTAMBA_OK = 0,
  ATTAMBA_ERR_INVALID_ARG = 1,
  ATTAMBA_ERR_UNSUPPORTED = 2,
  ATTAMBA_ERR_CUDA = 3
} attamba_status_t;

typedef enum { ATTAMBA_F32 = 0, ATTAMBA_BF16 = 1 } attamba_dtype_t;

/* M_train (Eq. 5): completed-chunk ends + own partial chunk + L leading tokens.
 * M_test  (Eq. 7 read causally, [pith, ref-eq7]): completed-chunk ends + L leading tokens. */
typedef enum { ATTAMBA_MASK_TRAIN = 0, ATTAMBA_MASK_TEST = 1 } attamba_mask_t;

/* Bits OR-ed into *d_status by the device. */
#define ATTAMBA_DEV_BAD_CHUNKS 0x1 /* cu not increasing, not 0..T, or a chunk crosses a sequence start */
#define ATTAMBA_DEV_CACHE_FULL 0x2 /* decode: boundary list at capacity, the new boundary was dropped */
#define ATTAMBA_DEV_TIMEOUT 0x4    /* a pipeline wait gave up; outputs of that tile are not written */
#define ATTAMBA_DEV_BOUNDS 0x8     /* checked builds only (libattamba_checked.so, compiled with
                                      ATTAMBA_CHECKED): an index fell outside the array it addresses;
                                      the access was skipped (a TMA load, which reads the fill value
                                      out of range, is reported and still made) */

/* Compact per-query key index built by attamba_chunk_index [pith, carries]:
 * query i (sequence-relative position) of sequence b reads
 *     S(i) = { bpos[bptr[b] + k] : k < nbb(i) }  united with  [ls(i), i].
 * All arrays are caller-owned device memory. */
typedef struct {
  int32_t* cu;   /* [n_chunks + 1] chunk starts over the T flattened tokens; cu[n_chunks] = T */
  int32_t* bpos; /* [n_chunks] last position of chunk c, relative to its sequence start */
  int32_t* bptr; /* [B + 1] first chunk of each sequence; bptr[B] = n_chunks */
  int32_t* ls;   /* [T] first position of the local segment of each query (sequence-relative) */
  int32_t* nbb;  /* [T] number of its sequence's chunk ends strictly below ls */
  int32_t n_chunks;
  int32_t B;
  int32_t n;
} attamba_index_t;

/* Library version string. */
const char* attamba_version(void);
/* Static text of a status code. */
const char* attamba_status_string(attamba_status_t s);
/* CUDA error text of this thread's last ATTAMBA_ERR_CUDA ("" if none). */
const char* attamba_last_error(void);

/* Chunks per sequence for uniform chunking of size P with cyclic offset
 * (offset mod P) [pith, carries], [pith, params]: starts are {0} and
 * {o + kP : 0 < o + kP < n}.  Returns -1 for n < 1 or P < 1. Host only. */
int32_t attamba_uniform_chunk_count(int32_t n, int32_t P, int32_t offset);

/* attamba_chunk_index -- chunk boundaries and the compact key index of every query.
 * [pith, carries] (M_train Eq. 5, M_test Eq. 7, leading tokens Eq. 8), [pith, if]
 * (cu_seqlens-style variable chunks), [pith, ref-eq7].
 *   cu_in    nullable [n_chunks+1] device: variable chunks (P, offset ignored);
 *            NULL: uniform chunks of size P with offset (offset mod P), and
 *            n_chunks must equal B * attamba_uniform_chunk_count(n, P, offset).
 *   B, n     sequences and tokens per sequence; B * n < 2^31 (positions are int32).
 *   L        leading tokens, >= 0;  mode  ATTAMBA_MASK_TRAIN / _TEST.
 *   out      host struct of device arrays; out->n_chunks, ->B, ->n must match.
 *            out->cu receives the chunk starts (it may alias cu_in).
 * Local start: M_train ls = max(0, min(start(i), i-L+1)); M_test ls = max(0, i-L+1).
 * Device errors: ATTAMBA_DEV_BAD_CHUNKS for a malformed cu_in (outputs then undefined). */
attamba_status_t attamba_chunk_index(const int32_t* cu_in, int32_t n_chunks, int32_t B, int32_t n,
                                     int32_t P, int32_t offset, int32_t L, attamba_mask_t mode,
                                     const attamba_index_t* out, int32_t* d_status,
                                     attamba_stream_t stream);

/* One output segment of attamba_proj_gemm: columns [col0, col0 + width) of Y,
 * written to ptr as a row-major [M, width] bf16 array. */
typedef struct {
  void* ptr;
  int32_t col0;
  int32_t width;
} attamba_proj_seg_t;

/* attamba_proj_gemm -- the layer's projections as one tensor-core GEMM, Y = X W^T.
 * [pith, core] the SSMs replace W_K and W_V, the query and output projections stay;
 * [pith, params] the selective SSM's step and B, C are projections of the input.
 * The seven input projections (W_Q, W_dK, W_dV, W_BK, W_CK, W_BV, W_CV stacked along
 * their output features) are one call whose segments are q, dt_k, dt_v, B_k, C_k,
 * B_v, C_v; the output projection W_O is another with one segment.
 *   X      [M, K] bf16 row-major;  W  [Nout, K] bf16 row-major (output x input features).
 *   segs   nseg (1..8) segments, sorted by col0, not overlapping, col0 and width
 *          multiples of 8, col0 + width <= Nout; columns no segment names are not written.
 *   K      a multiple of 64.  fp32 accumulation, bf16 rounding of Y.
 * X, W and every segment pointer 16-byte aligned.  bf16 only. */
attamba_status_t attamba_proj_gemm(attamba_dtype_t dtype, const void* X, const void* W, int64_t M, int32_t Nout,
                                   int32_t K, const attamba_proj_seg_t* segs, int32_t nseg, int32_t* d_status,
                                   attamba_stream_t stream);

/* attamba_kv_ssm_scan -- both KV-SSMs over the layer input, state reset at chunk starts.
 * [pith, core] K = SSM_K(X), V = SSM_V(X); [pith, params] Mamba selective SSM (Eq. 3);
 * [pith, carries] one state per chunk of P tokens.  Per token t, channel d, SSM s:
 *     delta = softplus(dt_s[t,d] + bias_s[d])
 *     h[d,:] = exp(delta * A_s[d,:]) * h[d,:] + delta * x[t,d] * B_s[t,:]   (h = 0 at chunk starts)
 *     out_s[t,d] = sum_n C_s[t,n] * h[d,n]
 *   dtype     ATTAMBA_F32 or ATTAMBA_BF16: type of x, dt_*, B_*, C_*, K, V, Kc, Vc.
 *   x         [T, D];  dt_k, dt_v [T, D]  pre-softplus steps.
 *   bias_k/v  [D] f32;  A_k/v [D, N] f32 (negative).
 *   B_k, C_k, B_v, C_v   [T, N].
 *   cu        [n_chunks+1] chunk starts (as written by attamba_chunk_index).
 *   N         16 or 32 (the supported state sizes; 32 is the pages' default Ds)  D a multiple of 8.
 *   K, V      [T, D] outputs (viewed as [T, H, dh] by the attention).
 *   Kc, Vc    nullable [n_chunks, D]: K, V at the last token of each chunk (the
 *             boundary states), the compact copy the attention reads.
 * State is fp32 in registers; nothing but the outputs is written. */
attamba_status_t attamba_kv_ssm_scan(attamba_dtype_t dtype, const void* x, const void* dt_k,
                                     const void* dt_v, const float* bias_k, const float* bias_v,
                                     const float* A_k, const float* A_v, const void* B_k,
                                     const void* C_k, const void* B_v, const void* C_v,
                                     const int32_t* cu, int32_t n_chunks, int64_t T, int32_t D,
                                     int32_t N, void* K, void* V, void* Kc, void* Vc,
                                     int32_t* d_status, attamba_stream_t stream);

/* attamba_kv_ssm_scan_u -- attamba_kv_ssm_scan with a separate input per SSM: the
 * keys SSM reads u_k, the values SSM u_v.  This is the kept-projection variant
 * [pith, if] (removing the explicit K and V projections costs about 1%, so with
 * them kept the SSM input is u = x W_K for the keys and u = x W_V for the values);
 * the projections are the caller's, as for q.  Same arguments, layouts, limits and
 * errors as attamba_kv_ssm_scan otherwise; u_k == u_v is the shared-input case. */
attamba_status_t attamba_kv_ssm_scan_u(attamba_dtype_t dtype, const void* u_k, const void* u_v,
                                       const void* dt_k, const void* dt_v, const float* bias_k,
                                       const float* bias_v, const float* A_k, const float* A_v,
                                       const void* B_k, const void* C_k, const void* B_v, const void* C_v,
                                       const int32_t* cu, int32_t n_chunks, int64_t T, int32_t D, int32_t N,
                                       void* K, void* V, void* Kc, void* Vc, int32_t* d_status,
                                       attamba_stream_t stream);

/* attamba_chunk_attn_fwd -- softmax attention of every query over its key set S(i).
 * [pith, carries] (attention map (n/P + L) x (n/P + L)), [pith, core].
 *   q, K, V   [T, H, dh] (T = idx->B * idx->n);  Kc, Vc [idx->n_chunks, H, dh].
 *   idx       the index from attamba_chunk_index.
 *   dh        64 (supported);  scale  usually 1/sqrt(dh).
 *   O         [T, H, dh] output;  lse  nullable [B, H, n] f32 natural-log sum-exp.
 * A query with an empty key set gets O = 0 and lse = -inf.
 * bf16: tcgen05 tensor-core tiles fed by TMA, fp32 online softmax.
 * f32 : CUDA-core fp32 arithmetic. */
attamba_status_t attamba_chunk_attn_fwd(attamba_dtype_t dtype, const void* q, const void* K,
                                        const void* V, const void* Kc, const void* Vc,
                                        const attamba_index_t* idx, int32_t H, int32_t dh,
                                        float scale, void* O, float* lse, int32_t* d_status,
                                        attamba_stream_t stream);

/* Decode cache of B sequences [pith, core], [pith, if]: the boundary states of
 * completed chunks and the L most recent tokens, plus the SSM states. */
typedef struct {
  float* state;   /* [2, B, N, D] fp32 SSM state (keys SSM, values SSM) */
  void* Kb;       /* [B, H, cap, dh] boundary keys */
  void* Vb;       /* [B, H, cap, dh] boundary values */
  int32_t* bpos;  /* [B, cap] position of each stored boundary, increasing */
  void* Kr;       /* [B, H, L, dh] keys of the L most recent positions, slot = position mod L */
  void* Vr;       /* [B, H, L, dh] values, same slots */
  int32_t* nb;    /* [B] number of stored boundaries */
  int32_t* pos;   /* [B] position of the next token */
  int32_t B, H, dh, N, P, offset, L, cap;
} attamba_cache_t;

/* attamba_cache_from_prefill -- the decode cache a prefill of positions [0, n0) leaves.
 * [pith, core] at inference only the boundary states are cached; [pith, if] the
 * final SSM state of each chunk, P = 8 with 64 leading tokens; [pith, carries] the
 * leading-token window (Eq. 8).  Uniform chunks of the cache's P and offset.
 *   cache     the cache to fill (its B, H, dh, N, P, offset, L, cap; device arrays).
 *             Written: Kb, Vb, bpos rows 0..nb-1 (the positions p < n0 that end a
 *             chunk, in order), the ring slots p mod L for p in [max(0, n0 - L), n0),
 *             state (both SSMs after position n0 - 1: the recurrence rerun over the
 *             tokens of the chunk holding n0 - 1), nb[b] = nb, pos[b] = n0.
 *   K, V      [B, n0, H, dh] keys / values of the prefill (attamba_kv_ssm_scan).
 *   x .. C_v  the prefill's scan inputs, token rows b * n0 + t, as in attamba_kv_ssm_scan.
 *   n0        prefill length, >= 1.
 * dtype ATTAMBA_BF16, dh 64, N 16 or 32, L >= 1.  ATTAMBA_ERR_INVALID_ARG when the
 * boundaries of [0, n0) exceed cap (checked on the host: chunks are uniform). */
attamba_status_t attamba_cache_from_prefill(attamba_dtype_t dtype, const attamba_cache_t* cache,
                                            const void* K, const void* V, const void* x,
                                            const void* dt_k, const void* dt_v, const float* bias_k,
                                            const float* bias_v, const float* A_k, const float* A_v,
                                            const void* B_k, const void* C_k, const void* B_v,
                                            const void* C_v, int32_t n0, int32_t* d_status,
                                            attamba_stream_t stream);

/* Self-test of the device failure path (no counterpart in the method): one thread waits, with the
 * same bounded wait every pipeline kernel uses, on a shared-memory barrier that nothing completes;
 * after limit_ns nanoseconds (1e3 .. 1e9) it gives up, ORs ATTAMBA_DEV_TIMEOUT into *d_status
 * (device memory, required) and returns, leaving the context usable.  No trap, no fault.
 * ATTAMBA_ERR_INVALID_ARG for a null d_status or a limit out of range. */
attamba_status_t attamba_selftest_wait_timeout(uint64_t limit_ns, int32_t* d_status, attamba_stream_t stream);

/* Bytes of device memory a bf16 decode cache with the dimensions in `cache` takes (its
 * pointers are not read): the arrays state, Kb, Vb, bpos, Kr, Vr, nb, pos in that order,
 * each rounded up to 256 bytes, so one allocation of this size holds them all at
 * 256-byte aligned offsets.  0 for a dimension out of range (B, H, N, L, cap < 1, dh != 64). */
size_t attamba_cache_bytes(const attamba_cache_t* cache);

/* Bytes of device workspace attamba_decode_step needs for this cache. */
size_t attamba_decode_workspace_size(const attamba_cache_t* cache);

/* attamba_decode_step -- one new token per sequence over the boundary-state cache.
 * [pith, core] (only boundary states cached), [pith, carries] (M_test + window),
 * [pith, ref-eq7] (current chunk reached through the window only).
 * At position t = pos[b]: reset both SSM states if t starts a uniform chunk
 * (t == 0 or (t >= o and (t-o) mod P == 0), o = offset mod P); update them with
 * the step inputs; write k_t, v_t to ring slot t mod L; if t ends a chunk, append
 * them to the boundary list (ATTAMBA_DEV_CACHE_FULL if nb == cap); then attend
 * q_t over { boundaries at positions < t-L+1 } united with [t-L+1, t].  Finally
 * pos[b] += 1 and nb[b] grows by the append.
 *   dtype      ATTAMBA_BF16 (the cache and the step tensors);  L >= 1, dh = 64, N = 16 or 32.
 *   q_t        [B, H, dh];  x_t, dt_k, dt_v [B, D];  B_k, C_k, B_v, C_v [B, N].
 *   bias_*, A_* as in attamba_kv_ssm_scan.
 *   o_t        [B, H, dh] output.
 *   workspace  device scratch of at least attamba_decode_workspace_size(cache) bytes. */
attamba_status_t attamba_decode_step(attamba_dtype_t dtype, const attamba_cache_t* cache,
                                     const void* q_t, const void* x_t, const void* dt_k,
                                     const void* dt_v, const float* bias_k, const float* bias_v,
                                     const float* A_k, const float* A_v, const void* B_k,
                                     const void* C_k, const void* B_v, const void* C_v,
                                     float scale, void* o_t, void* workspace,
                                     size_t workspace_bytes, int32_t* d_status,
                                     attamba_stream_t stream);

/* attamba_decode_step_noalloc -- attamba_decode_step without a caller workspace.
 * The paper has no counterpart to this entry point; it exists for callers that
 * cannot allocate device memory when they step the decoder: hosts that hand out
 * all device memory up front from their own pool and forbid cudaMalloc later
 * (it may synchronize the device and can fail mid-stream), or callers that have
 * no channel for passing this library a scratch buffer.
 *   Same arguments and behaviour as attamba_decode_step, minus workspace and
 *   workspace_bytes.  The split-K scratch is a fixed 4 MiB array inside the
 *   library, allocated with the library's device code on each GPU that loads it
 *   and kept until the process exits.  A cache needing more than that
 *   (attamba_decode_workspace_size(cache) > 4 MiB) is rejected with
 *   ATTAMBA_ERR_UNSUPPORTED before any launch; attamba_last_error() says so.
 *   The first call on a device looks up the array's device address (no
 *   allocation), and so does the first call after the device's context was
 *   destroyed and created again (cudaDeviceReset); make that first call
 *   before capturing a stream.
 *   All calls on a device share the array and it keeps the last call's
 *   contents (nothing in it needs to start at zero).  Calls whose kernels can
 *   overlap on the GPU (unordered streams) race on it; order them on one stream. */
attamba_status_t attamba_decode_step_noalloc(attamba_dtype_t dtype, const attamba_cache_t* cache,
                                             const void* q_t, const void* x_t, const void* dt_k,
                                             const void* dt_v, const float* bias_k, const float* bias_v,
                                             const float* A_k, const float* A_v, const void* B_k,
                                             const void* C_k, const void* B_v, const void* C_v,
                                             float scale, void* o_t, int32_t* d_status,
                                             attamba_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* ATTAMBA_H */
