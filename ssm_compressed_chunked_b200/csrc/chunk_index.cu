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
// contiguous local segment [ls(i), i].  One launch: thread c < n_chunks writes
// chunk c's row of the table (offset, chunk-end position, the sequence's first
// chunk; validation of caller chunks), thread i < T writes token i's (ls, nbb).
// No thread reads what another writes: with uniform chunks both follow from
// closed forms, with caller chunks (cu_seqlens-style offsets) from binary
// searches of the caller's offsets.
#include "common.cuh"
#include "launch.h"

namespace attamba {

namespace {
// start of chunk k (sequence-relative) for uniform chunks of size P, offset o in [0, P)
__device__ __forceinline__ int32_t uniform_start(int32_t k, int32_t P, int32_t o) {
  if (k == 0) return 0;
  return o == 0 ? k * P : o + (k - 1) * P;
}
// the uniform chunk holding sequence position r (< cps chunks)
__device__ __forceinline__ int32_t uniform_chunk(int32_t r, int32_t P, int32_t o, int32_t cps) {
  const int32_t k = o == 0 ? r / P : (r < o ? 0 : 1 + (r - o) / P);
  return min(k, cps - 1);
}

// first index in [lo, hi) with a[idx] > v  (a increasing)
__device__ __forceinline__ int32_t upper_bound(const int32_t* a, int32_t lo, int32_t hi, int32_t v) {
  while (lo < hi) {
    const int32_t mid = (lo + hi) >> 1;
    if (__ldg(a + mid) <= v) lo = mid + 1; else hi = mid;
  }
  return lo;
}
// first index in [lo, hi) with a[idx] >= v
__device__ __forceinline__ int32_t lower_bound(const int32_t* a, int32_t lo, int32_t hi, int32_t v) {
  while (lo < hi) {
    const int32_t mid = (lo + hi) >> 1;
    if (__ldg(a + mid) < v) lo = mid + 1; else hi = mid;
  }
  return lo;
}

__global__ void chunk_index_kernel(const int32_t* __restrict__ cu_in, int32_t n_chunks, int32_t B, int32_t n,
                                   int32_t P, int32_t o, int32_t cps, int32_t L, int mode,
                                   attamba_index_t out, int32_t* status) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t T = (int64_t)B * n;
  if (i < n_chunks) {
    // ------------------------------------------------ chunk table row c
    const int32_t c = (int32_t)i;
    int32_t s0, s1;  // flattened [start, next start)
    if (cu_in == nullptr) {
      const int32_t b = c / cps, k = c % cps;
      s0 = b * n + uniform_start(k, P, o);
      s1 = (k + 1 < cps) ? b * n + uniform_start(k + 1, P, o) : (b + 1) * n;
      out.cu[c] = s0;
      if (c == n_chunks - 1) out.cu[n_chunks] = (int32_t)T;
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
      if (out.cu != cu_in) {
        out.cu[c] = s0;
        if (c == n_chunks - 1) out.cu[n_chunks] = cu_in[n_chunks];
      }
    }
    const int32_t b = min(max(s0, 0) / n, B - 1);
    out.bpos[c] = s1 - 1 - b * n;
    if (s0 == b * n) out.bptr[b] = c;
    if (c == n_chunks - 1) out.bptr[B] = n_chunks;
  }
  if (i < T) {
    // ------------------------------------------------ key index of token i
    const int32_t b = (int32_t)(i / n);
    const int32_t r = (int32_t)(i - (int64_t)b * n);
    int32_t start, ls, nbb;
    if (cu_in == nullptr) {
      start = uniform_start(uniform_chunk(r, P, o, cps), P, o);
      ls = r - L + 1;
      if (mode == ATTAMBA_MASK_TRAIN) ls = min(start, ls);
      ls = max(0, ls);
      // completed chunks ending before ls = chunks starting at or before ls, minus the first;
      // ls = n (M_test, L = 0, last token) is past every chunk end, the cut last one included
      nbb = ls >= n ? cps : uniform_chunk(ls, P, o, cps);
    } else {
      // chunk holding i: last c with cu[c] <= i; the sequence's chunks: [first c with cu[c] >= b n, ...)
      int32_t c = upper_bound(cu_in, 0, n_chunks, (int32_t)i) - 1;
      c = max(0, min(c, n_chunks - 1));
      start = __ldg(cu_in + c) - b * n;
      ls = r - L + 1;
      if (mode == ATTAMBA_MASK_TRAIN) ls = min(start, ls);
      ls = max(0, ls);
      const int32_t c_lo = lower_bound(cu_in, 0, n_chunks, b * n);
      // chunk ends (cu[c + 1] - 1) below b n + ls: chunks c >= c_lo with cu[c + 1] <= b n + ls
      nbb = max(0, upper_bound(cu_in, c_lo + 1, n_chunks + 1, b * n + ls) - (c_lo + 1));
    }
    out.ls[i] = ls;
    out.nbb[i] = nbb;
  }
}
}  // namespace

cudaError_t launch_chunk_index(const int32_t* cu_in, int32_t n_chunks, int32_t B, int32_t n,
                               int32_t P, int32_t offset, int32_t L, int mode,
                               const attamba_index_t& out, int32_t* d_status, cudaStream_t s) {
  const int32_t o = (cu_in == nullptr) ? ((offset % P) + P) % P : 0;
  const int32_t cps = (cu_in == nullptr) ? n_chunks / B : 0;
  const int64_t T = (int64_t)B * n;
  const int64_t work = T > n_chunks ? T : n_chunks;
  chunk_index_kernel<<<(unsigned)((work + 255) / 256), 256, 0, s>>>(cu_in, n_chunks, B, n, P, o, cps, L, mode, out,
                                                                     d_status);
  return cudaGetLastError();
}

}  // namespace attamba
