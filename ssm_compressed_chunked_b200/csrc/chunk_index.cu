// Chunk boundaries and the compact per-query key index.
//
// Method: pith.science review of Attamba, "What carries the argument" -- M_train
// (Eq. 5) reads the last token of every completed chunk plus the query's own
// partial chunk, M_test (Eq. 7) the completed-chunk ends, and the L leading
// tokens (Eq. 8) are added to either; "If this is right" -- variable chunks
// come as cu_seqlens-style prefix offsets; Referee Report, comment on Eq. (7) --
// at test time only completed chunks count.
//
// The key set of query i is kept compact: the chunk ends below a local start
// ls(i) (a prefix of the sequence's sorted chunk ends, length nbb(i)) plus the
// contiguous local segment [ls(i), i].  Two launch-bound kernels: one thread
// per chunk (offsets, chunk-end positions, per-sequence chunk ranges,
// validation), then one thread per token (ls, nbb by binary search).
#include "common.cuh"
#include "launch.h"

namespace attamba {

// start of chunk k (sequence-relative) for uniform chunks of size P, offset o in [0, P)
__device__ __forceinline__ int32_t uniform_start(int32_t k, int32_t P, int32_t o) {
  if (k == 0) return 0;
  return o == 0 ? k * P : o + (k - 1) * P;
}

__global__ void chunk_table_kernel(const int32_t* __restrict__ cu_in, int32_t n_chunks, int32_t B,
                                   int32_t n, int32_t P, int32_t o, int32_t cps, int32_t* cu,
                                   int32_t* bpos, int32_t* bptr, int32_t* status) {
  const int32_t c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= n_chunks) return;
  const int64_t T = (int64_t)B * n;
  int32_t s0, s1;  // flattened [start, next start)
  if (cu_in == nullptr) {
    const int32_t b = c / cps, k = c % cps;
    s0 = b * n + uniform_start(k, P, o);
    s1 = (k + 1 < cps) ? b * n + uniform_start(k + 1, P, o) : (b + 1) * n;
    cu[c] = s0;
    if (c == n_chunks - 1) cu[n_chunks] = (int32_t)T;
  } else {
    s0 = cu_in[c];
    s1 = cu_in[c + 1];
    bool bad = (s0 >= s1) || s0 < 0 || (int64_t)s1 > T;
    if (c == 0 && s0 != 0) bad = true;
    if (c == n_chunks - 1 && (int64_t)s1 != T) bad = true;
    if (!bad && (s0 / n) != ((s1 - 1) / n)) bad = true;  // crosses a sequence start
    if (bad) {
      raise_status(status, ATTAMBA_DEV_BAD_CHUNKS);
      s1 = s0 + 1;
    }
    if (cu != cu_in) {
      cu[c] = s0;
      if (c == n_chunks - 1) cu[n_chunks] = cu_in[n_chunks];
    }
  }
  const int32_t b = min(max(s0, 0) / n, B - 1);
  bpos[c] = s1 - 1 - b * n;
  if (s0 == b * n) bptr[b] = c;
  if (c == n_chunks - 1) bptr[B] = n_chunks;
}

// first index in [lo, hi) with a[idx] > v  (a increasing)
__device__ __forceinline__ int32_t upper_bound(const int32_t* a, int32_t lo, int32_t hi, int32_t v) {
  while (lo < hi) {
    const int32_t mid = (lo + hi) >> 1;
    if (a[mid] <= v) lo = mid + 1; else hi = mid;
  }
  return lo;
}
// first index in [lo, hi) with a[idx] >= v
__device__ __forceinline__ int32_t lower_bound(const int32_t* a, int32_t lo, int32_t hi, int32_t v) {
  while (lo < hi) {
    const int32_t mid = (lo + hi) >> 1;
    if (a[mid] < v) lo = mid + 1; else hi = mid;
  }
  return lo;
}

__global__ void query_index_kernel(const int32_t* __restrict__ cu, const int32_t* __restrict__ bpos,
                                   const int32_t* __restrict__ bptr, int32_t n_chunks, int32_t B,
                                   int32_t n, int32_t L, int mode, int32_t* ls_out, int32_t* nbb_out) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (int64_t)B * n) return;
  const int32_t b = (int32_t)(i / n);
  const int32_t r = (int32_t)(i - (int64_t)b * n);
  // chunk holding i: last c with cu[c] <= i
  int32_t c = upper_bound(cu, 0, n_chunks, (int32_t)i) - 1;
  c = max(0, min(c, n_chunks - 1));
  const int32_t start = cu[c] - b * n;
  int32_t ls = r - L + 1;
  if (mode == ATTAMBA_MASK_TRAIN) ls = min(start, ls);
  ls = max(0, ls);
  const int32_t lo = max(0, min(bptr[b], n_chunks));
  const int32_t hi = max(lo, min(bptr[b + 1], n_chunks));
  ls_out[i] = ls;
  nbb_out[i] = lower_bound(bpos, lo, hi, ls) - lo;
}

cudaError_t launch_chunk_index(const int32_t* cu_in, int32_t n_chunks, int32_t B, int32_t n,
                               int32_t P, int32_t offset, int32_t L, int mode,
                               const attamba_index_t& out, int32_t* d_status, cudaStream_t s) {
  const int32_t o = (cu_in == nullptr) ? ((offset % P) + P) % P : 0;
  const int32_t cps = (cu_in == nullptr) ? n_chunks / B : 0;
  chunk_table_kernel<<<(n_chunks + 255) / 256, 256, 0, s>>>(cu_in, n_chunks, B, n, P, o, cps, out.cu,
                                                            out.bpos, out.bptr, d_status);
  const int64_t T = (int64_t)B * n;
  query_index_kernel<<<(unsigned)((T + 255) / 256), 256, 0, s>>>(out.cu, out.bpos, out.bptr, n_chunks,
                                                                  B, n, L, mode, out.ls, out.nbb);
  return cudaGetLastError();
}

}  // namespace attamba
