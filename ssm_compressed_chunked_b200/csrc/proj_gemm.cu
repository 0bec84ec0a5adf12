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
// Kernel (sm_100a), persistent, CTA pairs (clusters of two, one CTA per SM)
// walking 256 x 256 output tiles (all row tiles of one weight block before the
// next, so the block stays in L2), each tile one two-SM MMA (tcgen05
// cta_group::2, M 256): CTA r of the pair holds rows [128 r, 128 r + 128) of the
// X tile and of the W tile, the MMA reads both CTAs' shared memory, and each CTA's
// TMEM receives its own 128 rows of the product.  Per SM and K step that is
// 32 KB of operands for a 128 x 256 x 64 product, a third less than one SM
// alone needs, so six stages fit.
//   warp 0     TMA producer (both CTAs): its X and W halves per K step into a
//              6-stage ring, 128-byte swizzle, completing on the first CTA's
//              barrier (which expects both CTAs' bytes)
//   warp 1     first CTA only: one thread issues tcgen05.mma.cta_group::2 M256 N256
//              K16 into a TMEM accumulator and commits to both CTAs' barriers; two
//              accumulators (512 columns) so a tile's epilogue overlaps the next
//              tile's MMAs
//   warps 2-5  epilogue (both CTAs): each thread owns one accumulator row (TMEM
//              lane), reads it 32 columns at a time, rounds to bf16 and stores
//              16-byte pieces into the segment each 8-column group belongs to,
//              then tells the first CTA the accumulator is free
// All waits are bounded; a give-up raises ATTAMBA_DEV_TIMEOUT.
#include <mutex>

#include "common.cuh"
#include "launch.h"

namespace attamba {

namespace {
constexpr int kBM = 128;                                  // rows per CTA (the pair: 256)
constexpr int kBN = 256;                                  // columns per tile (each CTA loads half of W's rows)
constexpr int kBK = 64;
constexpr int kStages = 6;
constexpr int kThreads = 192;
constexpr uint32_t kABytes = kBM * kBK * 2;               // 16 KB
constexpr uint32_t kBBytes = (kBN / 2) * kBK * 2;         // 16 KB
constexpr uint32_t kStageBytes = kABytes + kBBytes;
constexpr uint32_t kBarOff = kStages * kStageBytes;
constexpr uint32_t kSmemBytes = kBarOff + 256 + 1024;     // + barriers + alignment slack
constexpr uint32_t kTmemCols = 512;                       // two 256-column accumulators
constexpr uint64_t kWaitNs = 4000000000ull;
constexpr int kMaxDevices = 64;

struct Bars {
  uint64_t full[kStages];  // first CTA: both CTAs' operands of the stage have landed
  uint64_t empty[kStages]; // the MMAs reading the stage have finished (commit from the first CTA)
  uint64_t acc_full[2];    // accumulator a holds a finished tile (commit from the first CTA)
  uint64_t acc_empty[2];   // first CTA: both epilogues have read accumulator a (256 arrivals)
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(Bars) <= 256, "barrier block overflows its shared-memory slot");

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// the shared::cluster address of this CTA's variable at shared address a in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t peer_addr(uint32_t a, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
  return r;
}
// relaxed: the arrival orders this thread's TMEM reads (complete at tcgen05.wait::ld), not its global
// stores, so it need not wait for them to be visible across the cluster
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_bar) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar) : "memory");
}
// 2-D tiled load into this CTA's shared memory, completion counted on the first CTA's barrier
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const void* tmap, int x, int y, uint32_t cluster_bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
      "[%4];" ::"r"(smem_u32(dst)),
      "l"(tmap), "r"(x), "r"(y), "r"(cluster_bar)
      : "memory");
}
__device__ __forceinline__ void umma_bf16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                               uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// the barrier at cluster address `bar` (either CTA of the pair) tracks the completion of every
// two-SM MMA this thread has issued so far
__device__ __forceinline__ void umma_commit_pair(uint32_t cluster_bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(cluster_bar)
               : "memory");
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    proj_gemm_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                     ProjArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + kBarOff);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_rank();                 // 0: issues the MMAs; 1: its peer
  const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
  const int n_mt = (int)((a.M + 2 * kBM - 1) / (2 * kBM));   // 256-row tiles
  const int n_nt = (a.Nout + kBN - 1) / kBN;
  const int n_tiles = n_mt * n_nt;
  const int n_k = a.K / kBK;

  if (warp == 0 && lane == 0) {
    for (int i = 0; i < kStages; ++i) { mbar_init(&bars->full[i], 1); mbar_init(&bars->empty[i], 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(&bars->acc_full[i], 1); mbar_init(&bars->acc_empty[i], 2 * kBM); }
    mbar_init(&bars->mma_done, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    // both CTAs' warp 1: one allocation at the same TMEM address in each
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&bars->tmem_base)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();   // both CTAs' barriers are initialised before either CTA signals the other's
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
      for (int t = pair; ok && t < n_tiles; t += n_pairs) {
        const int nt = t / n_mt, mt = t - nt * n_mt;
        for (int k = 0; k < n_k; ++k, ++cnt) {
          const int st = cnt % kStages;
          if (cnt >= kStages &&
              !mbar_wait_bounded(&bars->empty[st], ((cnt / kStages) - 1) & 1, abort_flag, kWaitNs)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + st * kStageBytes;
          const uint32_t full0 = peer_addr(smem_u32(&bars->full[st]), 0);
          // the first CTA's barrier expects both CTAs' bytes; the other CTA's copies only complete on it
          if (rank == 0) mbar_arrive_expect_tx(&bars->full[st], 2 * kStageBytes);
          tma_load_2d_pair(sa, &tm_x, k * kBK, mt * 2 * kBM + rank * kBM, full0);
          tma_load_2d_pair(sa + kABytes, &tm_w, k * kBK, nt * kBN + rank * (kBN / 2), full0);
        }
      }
      if (!ok) *abort_flag = 1;
      // the first CTA drains: the last copies into every stage, both CTAs', have landed (short
      // limit: after an abort some of them were never issued)
      if (rank == 0)
        for (int j = max(0, cnt - kStages); j < cnt; ++j)
          mbar_wait_timeout(&bars->full[j % kStages], (j / kStages) & 1, ok ? kWaitNs : 10000000ull);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (first CTA of the pair)
    if (lane == 0 && rank == 0) {
      const uint32_t idesc = umma_idesc_bf16(2 * kBM, kBN, 0, 0);
      // every commit goes to this CTA's barrier and to the same barrier of the peer
      auto commit2 = [&](uint64_t* bar) {
        umma_commit_pair(smem_u32(bar));
        umma_commit_pair(peer_addr(smem_u32(bar), 1));
      };
      int cnt = 0, i = 0;
      bool ok = true;
      for (int t = pair; ok && t < n_tiles; t += n_pairs, ++i) {
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
            umma_bf16_pair(d, umma_desc_sw128(sa + kk * 32, 16, 1024), umma_desc_sw128(sb + kk * 32, 16, 1024), idesc,
                           (k > 0 || kk > 0) ? 1u : 0u);
          commit2(&bars->empty[st]);
        }
        if (!ok) break;
        commit2(&bars->acc_full[acc]);
      }
      if (!ok) *abort_flag = 1;
      umma_commit_pair(smem_u32(&bars->mma_done));
      mbar_wait_timeout(&bars->mma_done, 0, kWaitNs);
    }
  } else {
    // ------------------------------------------------------------ epilogue warps 2-5
    const int q = warp & 3;                   // TMEM lane quadrant this warp may access
    const int r = q * 32 + lane;              // accumulator row
    const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16);
    int i = 0;
    bool ok = true;
    const uint32_t acc_empty0_a = peer_addr(smem_u32(&bars->acc_empty[0]), 0);
    const uint32_t acc_empty0_b = peer_addr(smem_u32(&bars->acc_empty[1]), 0);
    for (int t = pair; t < n_tiles; t += n_pairs, ++i) {
      const int nt = t / n_mt, mt = t - nt * n_mt;
      const int acc = i & 1;
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(&bars->acc_full[acc], (i >> 1) & 1, abort_flag, kWaitNs))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int64_t row = (int64_t)mt * 2 * kBM + rank * kBM + r;
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
      mbar_arrive_cluster(acc ? acc_empty0_b : acc_empty0_a);   // the first CTA's barrier, from either CTA
    }
    if (!ok) {
      *abort_flag = 1;
      raise_status(a.status, ATTAMBA_DEV_TIMEOUT);
    }
  }

  tc_fence_before();
  __syncthreads();
  // neither CTA leaves while the pair's MMAs may still read its shared memory or its TMEM
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
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
  if (!encode_2d(&tx, a.X, a.M, a.K, kBM) || !encode_2d(&tw, a.W, a.Nout, a.K, kBN / 2)) return cudaErrorNotSupported;
  cudaError_t e = raise_smem_limit(reinterpret_cast<const void*>(proj_gemm_kernel), (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  // as many CTA pairs as can be resident at once (a GPC with an odd number of free SMs leaves one
  // out), asked of the runtime once per device
  static std::mutex mu;
  static int max_pairs[kMaxDevices] = {};
  int dev = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  int pairs_max;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (max_pairs[dev] == 0) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(2 * (unsigned)(device_sm_count() / 2));
      cfg.blockDim = dim3(kThreads);
      cfg.dynamicSmemBytes = kSmemBytes;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, proj_gemm_kernel, &cfg) != cudaSuccess || n < 1) {
        cudaGetLastError();   // a failed query is not an error of this call
        n = device_sm_count() / 2;
      }
      max_pairs[dev] = n;
    }
    pairs_max = max_pairs[dev];
  }
  const int64_t tiles = ((a.M + 2 * kBM - 1) / (2 * kBM)) * ((a.Nout + kBN - 1) / kBN);
  const int64_t pairs = tiles < pairs_max ? tiles : pairs_max;
  const int grid = (int)(2 * (pairs > 0 ? pairs : 1));
  proj_gemm_kernel<<<grid, kThreads, kSmemBytes, s>>>(tx, tw, a);
  return cudaGetLastError();
}

}  // namespace attamba
