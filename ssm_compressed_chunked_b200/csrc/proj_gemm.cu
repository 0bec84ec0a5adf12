// Projections of the layer as one tensor-core GEMM: Y = X W^T, bf16 in and out,
// fp32 accumulation, with the output columns split into segments that land in
// separate arrays.
//
// Method: pith.science review of Attamba, "Core claim" -- the SSMs replace W_K and
// W_V, while the query projection and the output projection stay; "Assumptions &
// free parameters" -- the SSM is Mamba's selective SSM, whose step Δ and matrices
// B, C are projections of the input.  So one layer needs x W_Q, x W_ΔK, x W_ΔV,
// x W_BK, x W_CK, x W_BV, x W_CV before the hot path and O W_O after it.  With the
// seven input weights concatenated along their output features they are one GEMM
// whose epilogue writes each column segment to the array the hot path reads
// (q [T, D], dt_k [T, D], ..., B_k [T, N], ...); W_O is the same kernel with one
// segment.
//
// Kernel (sm_100a), persistent, one CTA per SM walking 128 x 256 output tiles
// (all row tiles of one weight block before the next, so the block stays in L2):
//   warp 0     TMA producer: X tile (128 rows x 64 K) and W tile (256 rows x 64 K)
//              per K step into a 4-stage ring, 128-byte swizzle
//   warp 1     one thread issues tcgen05.mma M128 N256 K16 into a TMEM accumulator;
//              two accumulators (512 columns) so a tile's epilogue overlaps the next
//              tile's MMAs
//   warps 2-5  epilogue: each thread owns one accumulator row (TMEM lane), reads it
//              32 columns at a time, rounds to bf16 and stores 16-byte pieces into
//              the segment each 8-column group belongs to
// All waits are bounded; a give-up raises ATTAMBA_DEV_TIMEOUT.
#include "common.cuh"
#include "launch.h"

namespace attamba {

namespace {
constexpr int kBM = 128;
constexpr int kBN = 256;
constexpr int kBK = 64;
constexpr int kStages = 4;
constexpr int kThreads = 192;
constexpr uint32_t kABytes = kBM * kBK * 2;               // 16 KB
constexpr uint32_t kBBytes = kBN * kBK * 2;               // 32 KB
constexpr uint32_t kStageBytes = kABytes + kBBytes;
constexpr uint32_t kBarOff = kStages * kStageBytes;
constexpr uint32_t kSmemBytes = kBarOff + 256 + 1024;     // + barriers + alignment slack
constexpr uint32_t kTmemCols = 512;                       // two 256-column accumulators
constexpr uint64_t kWaitNs = 4000000000ull;

struct Bars {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t acc_full[2];    // accumulator a holds a finished tile (tcgen05.commit)
  uint64_t acc_empty[2];   // the epilogue has read accumulator a (128 arrivals)
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(Bars) <= 256, "barrier block overflows its shared-memory slot");

__global__ void __launch_bounds__(kThreads, 1)
    proj_gemm_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                     ProjArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + kBarOff);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_mt = (int)((a.M + kBM - 1) / kBM);
  const int n_nt = (a.Nout + kBN - 1) / kBN;
  const int n_tiles = n_mt * n_nt;
  const int n_k = a.K / kBK;

  if (warp == 0 && lane == 0) {
    for (int i = 0; i < kStages; ++i) { mbar_init(&bars->full[i], 1); mbar_init(&bars->empty[i], 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(&bars->acc_full[i], 1); mbar_init(&bars->acc_empty[i], kBM); }
    mbar_init(&bars->mma_done, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort_flag = &bars->abort;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_x);
      tma_prefetch_desc(&tm_w);
      int cnt = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x) {
        const int nt = t / n_mt, mt = t - nt * n_mt;
        for (int k = 0; k < n_k; ++k, ++cnt) {
          const int st = cnt % kStages;
          if (cnt >= kStages &&
              !mbar_wait_bounded(&bars->empty[st], ((cnt / kStages) - 1) & 1, abort_flag, kWaitNs)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + st * kStageBytes;
          mbar_arrive_expect_tx(&bars->full[st], kStageBytes);
          tma_load_2d(sa, &tm_x, k * kBK, mt * kBM, &bars->full[st]);
          tma_load_2d(sa + kABytes, &tm_w, k * kBK, nt * kBN, &bars->full[st]);
        }
      }
      if (!ok) *abort_flag = 1;
      for (int j = max(0, cnt - kStages); j < cnt; ++j)
        mbar_wait_timeout(&bars->full[j % kStages], (j / kStages) & 1, kWaitNs);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_bf16(kBM, kBN, 0, 0);
      int cnt = 0, i = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x, ++i) {
        const int acc = i & 1;
        // the epilogue has read this accumulator's previous tile (i - 2)
        if (i >= 2 && !mbar_wait_bounded(&bars->acc_empty[acc], ((i - 2) >> 1) & 1, abort_flag, kWaitNs)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + acc * kBN;
        for (int k = 0; k < n_k; ++k, ++cnt) {
          const int st = cnt % kStages;
          if (!mbar_wait_bounded(&bars->full[st], (cnt / kStages) & 1, abort_flag, kWaitNs)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + st * kStageBytes);
          const uint32_t sb = sa + kABytes;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            umma_bf16(d, umma_desc_sw128(sa + kk * 32, 16, 1024), umma_desc_sw128(sb + kk * 32, 16, 1024), idesc,
                      (k > 0 || kk > 0) ? 1u : 0u);
          umma_commit(&bars->empty[st]);
        }
        if (!ok) break;
        umma_commit(&bars->acc_full[acc]);
      }
      if (!ok) *abort_flag = 1;
      umma_commit(&bars->mma_done);
      mbar_wait_timeout(&bars->mma_done, 0, kWaitNs);
    }
  } else {
    // ------------------------------------------------------------ epilogue warps 2-5
    const int q = warp & 3;                   // TMEM lane quadrant this warp may access
    const int r = q * 32 + lane;              // accumulator row
    const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16);
    int i = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++i) {
      const int nt = t / n_mt, mt = t - nt * n_mt;
      const int acc = i & 1;
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(&bars->acc_full[acc], (i >> 1) & 1, abort_flag, kWaitNs))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int64_t row = (int64_t)mt * kBM + r;
      const bool row_ok = row < a.M;
#pragma unroll 1
      for (int c32 = 0; c32 < kBN / 32; ++c32) {
        uint32_t v[32];
        tmem_ld32_sync(lane_base + acc * kBN + c32 * 32, v);
        const int col0 = nt * kBN + c32 * 32;
        if (!row_ok) continue;
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const int col = col0 + g * 8;
          if (col >= a.Nout) break;
          // the segment holding columns [col, col + 8): segments are 8-column aligned
          int s = 0;
          while (s + 1 < a.nseg && col >= a.seg_col0[s] + a.seg_width[s]) ++s;
          const int c = col - a.seg_col0[s];
          if (c < 0 || c >= a.seg_width[s]) continue;   // a column no segment takes
          uint4 pk;
          pk.x = pack_bf16x2(__uint_as_float(v[g * 8 + 0]), __uint_as_float(v[g * 8 + 1]));
          pk.y = pack_bf16x2(__uint_as_float(v[g * 8 + 2]), __uint_as_float(v[g * 8 + 3]));
          pk.z = pack_bf16x2(__uint_as_float(v[g * 8 + 4]), __uint_as_float(v[g * 8 + 5]));
          pk.w = pack_bf16x2(__uint_as_float(v[g * 8 + 6]), __uint_as_float(v[g * 8 + 7]));
          __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(a.seg_ptr[s]) + row * a.seg_width[s] + c;
          *reinterpret_cast<uint4*>(dst) = pk;
        }
      }
      tc_fence_before();
      mbar_arrive(&bars->acc_empty[acc]);
    }
    if (!ok) {
      *abort_flag = 1;
      raise_status(a.status, ATTAMBA_DEV_TIMEOUT);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// [rows, cols] bf16 row-major as a 2-D tensor, box 64 columns x box_rows rows, 128-byte swizzle
bool encode_2d(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int box_rows) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}
}  // namespace

cudaError_t launch_proj_gemm(const ProjArgs& a, cudaStream_t s) {
  CUtensorMap tx, tw;
  if (!encode_2d(&tx, a.X, a.M, a.K, kBM) || !encode_2d(&tw, a.W, a.Nout, a.K, kBN)) return cudaErrorNotSupported;
  cudaError_t e = raise_smem_limit(reinterpret_cast<const void*>(proj_gemm_kernel), (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  const int sms = device_sm_count();
  const int64_t tiles = ((a.M + kBM - 1) / kBM) * ((a.Nout + kBN - 1) / kBN);
  const int grid = (int)(tiles < sms ? tiles : sms);
  proj_gemm_kernel<<<grid, kThreads, kSmemBytes, s>>>(tx, tw, a);
  return cudaGetLastError();
}

}  // namespace attamba
