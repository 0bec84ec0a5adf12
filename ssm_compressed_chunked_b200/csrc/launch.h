// Internal launchers behind the C ABI (abi.cu validates, these launch).
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "attamba.h"

namespace attamba {

// cuTensorMapEncodeTiled from the driver (null when unavailable)
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();
// SM count of the current device (cached per device)
int device_sm_count();
// raise `kernel`'s dynamic shared-memory limit on the current device, once per device
cudaError_t raise_smem_limit(const void* kernel, int bytes);

cudaError_t launch_chunk_index(const int32_t* cu_in, int32_t n_chunks, int32_t B, int32_t n,
                               int32_t P, int32_t offset, int32_t L, int mode,
                               const attamba_index_t& out, int32_t* d_status, cudaStream_t s);

struct ScanArgs {
  const void* x[2];   // SSM input of the keys SSM and of the values SSM (the same array unless kept projections)
  const void* dt[2];
  const float* bias[2];
  const float* A[2];
  const void* Bm[2];
  const void* Cm[2];
  const int32_t* cu;
  int32_t n_chunks;
  int64_t T;
  int32_t D;
  int32_t N;
  void* out[2];
  void* outc[2];
  int32_t* status;
};
cudaError_t launch_kv_ssm_scan(attamba_dtype_t dtype, const ScanArgs& a, cudaStream_t s);

struct AttnArgs {
  const void* q;
  const void* K;
  const void* V;
  const void* Kc;
  const void* Vc;
  const int32_t* bpos;
  const int32_t* bptr;
  const int32_t* ls;
  const int32_t* nbb;
  int32_t B, n, H, dh, n_chunks;
  float scale;
  void* O;
  float* lse;
  int32_t* status;
};
// returns cudaErrorNotSupported when the tensor-map encoder is unavailable
cudaError_t launch_chunk_attn_bf16(const AttnArgs& a, cudaStream_t s);
cudaError_t launch_chunk_attn_f32(const AttnArgs& a, cudaStream_t s);

struct DecodeArgs {
  attamba_cache_t c;
  const void* q;
  const void* x;
  const void* dt[2];
  const float* bias[2];
  const float* A[2];
  const void* Bm[2];
  const void* Cm[2];
  float scale;
  void* o;
  float* work;
  int32_t splits;
  int32_t* status;
};
int32_t decode_splits(const attamba_cache_t& c);
size_t decode_workspace_bytes(const attamba_cache_t& c);
size_t decode_noalloc_scratch_bytes();
cudaError_t decode_noalloc_scratch(float** out);
cudaError_t launch_decode_step(const DecodeArgs& a, cudaStream_t s);

constexpr int kMaxProjSegs = 8;
struct ProjArgs {
  const void* X;   // [M, K]
  const void* W;   // [Nout, K]
  int64_t M;
  int32_t Nout;
  int32_t K;
  int32_t nseg;
  void* seg_ptr[kMaxProjSegs];     // segment s: columns [col0, col0 + width) -> [M, width]
  int32_t seg_col0[kMaxProjSegs];
  int32_t seg_width[kMaxProjSegs];
  int32_t* status;
};
cudaError_t launch_proj_gemm(const ProjArgs& a, cudaStream_t s);

struct HandoffArgs {
  attamba_cache_t c;
  const void* K;
  const void* V;
  const void* x;
  const void* dt[2];
  const float* bias[2];
  const float* A[2];
  const void* Bm[2];
  const void* Cm[2];
  int32_t n0;
  int32_t nb;   // boundaries in [0, n0)
};
// number of positions p < n0 that end a uniform chunk (size P, offset)
int32_t handoff_boundaries(int32_t n0, int32_t P, int32_t offset);
cudaError_t launch_cache_from_prefill(const HandoffArgs& a, cudaStream_t s);

// one CTA whose thread waits, with the pipelines' bounded wait, on a barrier that nothing completes
cudaError_t launch_wait_selftest(uint64_t limit_ns, int32_t* status, cudaStream_t s);

}  // namespace attamba
