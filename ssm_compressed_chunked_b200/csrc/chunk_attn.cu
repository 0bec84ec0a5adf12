// Softmax attention over the chunk-aware key sets.
//
// Method: pith.science review of Attamba, "What carries the argument" -- the
// attention runs over the compressed keys/values: for query i the ends of the
// completed chunks plus its own partial chunk (M_train, Eq. 5) or the L leading
// tokens (M_test, Eq. 7 with Eq. 8), so the map is about (n/P + L) wide instead
// of n.  The compact index gives, per query, a prefix of the sequence's chunk
// ends (nbb(i) of them, stored contiguously in Kc/Vc) and a contiguous local
// segment [ls(i), i] of the full K/V.
//
// bf16 kernel (tcgen05): one CTA per (128 queries, head, sequence).  Its key
// tiles (128 keys each) are first the chunk-end tiles 0..nbb(last query), then
// the local band [ls(first query), last query]; both are plain TMA boxes.
//   warp 4     TMA producer: Q once, then K/V tiles into a 2-stage ring
//   warp 5     one thread issues tcgen05.mma: S = Q K^T (M128 N128 K64) into
//              TMEM, then O_j = P_j V_j (M128 N64 K128) into TMEM
//   warps 0-3  softmax, one query row per thread: tcgen05.ld of its S row,
//              mask, online max/sum in fp32, P as bf16 into shared memory
//              (the A operand of the PV MMA), then accumulate O_j in registers
// TMEM: S double buffer (2 x 128 columns) + O_j double buffer (2 x 64).
// Every wait is bounded; on a give-up the CTA raises ATTAMBA_DEV_TIMEOUT,
// drains its own copies and MMAs, frees TMEM and leaves the tile unwritten.
//
// f32 kernel: one thread per (query, head) on the CUDA cores, same key sets,
// fp32 online softmax (the fp32 tensor-core kinds round to tf32).
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "launch.h"

namespace attamba {

namespace {
constexpr int kBM = 128;
constexpr int kBN = 128;
constexpr int kDH = 64;
constexpr int kStages = 2;
constexpr int kThreads = 192;
constexpr uint32_t kTileBytes = kBN * kDH * 2;    // 16 KB: 128 rows x 128 bytes
constexpr uint32_t kQOff = 0;
constexpr uint32_t kKOff = kQOff + kTileBytes;              // 2 stages
constexpr uint32_t kVOff = kKOff + kStages * kTileBytes;    // 2 stages
constexpr uint32_t kPOff = kVOff + kStages * kTileBytes;    // 2 buffers x 2 column blocks
constexpr uint32_t kPBytes = 2 * kTileBytes;                // 128 rows x 128 keys bf16
constexpr uint32_t kBarOff = kPOff + 2 * kPBytes;
constexpr uint32_t kSmemBytes = kBarOff + 256 + 1024;       // + barriers + alignment slack
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSCol = 0;     // S buffers at columns 0 and 128
constexpr uint32_t kOCol = 256;   // O buffers at columns 256 and 320
constexpr uint64_t kWaitNs = 4000000000ull;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

struct Bars {
  uint64_t q_full;
  uint64_t kv_full[kStages];
  uint64_t kv_empty[kStages];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t o_full[2];
  uint64_t o_empty[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
};

__global__ void __launch_bounds__(kThreads, 1)
    chunk_attn_bf16_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                           const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_kc,
                           const __grid_constant__ CUtensorMap tm_vc, AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + kBarOff);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qt = gridDim.x - 1 - blockIdx.x;  // longest key lists first
  const int h = blockIdx.y, b = blockIdx.z;
  const int n = a.n, H = a.H;
  const int q0 = qt * kBM;
  const int q_last = min(q0 + kBM, n) - 1;
  const int64_t tok0 = (int64_t)b * n;

  const int ls_first = a.ls[tok0 + q0];
  const int nbb_last = a.nbb[tok0 + q_last];
  const int nbt = (nbb_last + kBN - 1) / kBN;
  // every row's local segment [ls(i), i] is empty only when ls(i) = i + 1 (M_test, L = 0);
  // ls(i) - i does not grow with i, so the last row decides
  const bool band_empty = a.ls[tok0 + q_last] > q_last;
  const int band_len = band_empty ? 0 : max(0, q_last - ls_first + 1);
  const int nband = (band_len + kBN - 1) / kBN;
  const int NT = nbt + nband;
  const int32_t chunk0 = a.bptr[b];

  __nv_bfloat16* O = static_cast<__nv_bfloat16*>(a.O);
  if (NT == 0) {  // every row of the tile has an empty key set
    if (tid < kBM && q0 + tid <= q_last) {
      const int i = q0 + tid;
      uint4* dst = reinterpret_cast<uint4*>(O + ((tok0 + i) * H + h) * kDH);
#pragma unroll
      for (int c = 0; c < kDH / 8; ++c) dst[c] = make_uint4(0, 0, 0, 0);
      if (a.lse) a.lse[((int64_t)b * H + h) * n + i] = -INFINITY;
    }
    return;
  }

  if (warp == 4 && lane == 0) {
    mbar_init(&bars->q_full, 1);
    for (int i = 0; i < kStages; ++i) { mbar_init(&bars->kv_full[i], 1); mbar_init(&bars->kv_empty[i], 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->p_full[i], kBM);
      mbar_init(&bars->o_full[i], 1);
      mbar_init(&bars->o_empty[i], kBM);
    }
    mbar_init(&bars->mma_done, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&bars->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort_flag = &bars->abort;

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q); tma_prefetch_desc(&tm_k); tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_kc); tma_prefetch_desc(&tm_vc);
      mbar_arrive_expect_tx(&bars->q_full, kTileBytes);
      tma_load_3d(smem + kQOff, &tm_q, 0, h, (int)(tok0 + q0), &bars->q_full);
      int issued = 0;
      for (int j = 0; j < NT; ++j) {
        const int st = j % kStages;
        if (j >= kStages &&
            !mbar_wait_bounded(&bars->kv_empty[st], ((j / kStages) - 1) & 1, abort_flag, kWaitNs)) {
          *abort_flag = 1;
          break;
        }
        mbar_arrive_expect_tx(&bars->kv_full[st], 2 * kTileBytes);
        if (j < nbt) {
          const int row = chunk0 + j * kBN;
          tma_load_3d(smem + kKOff + st * kTileBytes, &tm_kc, 0, h, row, &bars->kv_full[st]);
          tma_load_3d(smem + kVOff + st * kTileBytes, &tm_vc, 0, h, row, &bars->kv_full[st]);
        } else {
          const int row = (int)(tok0 + ls_first + (j - nbt) * kBN);
          tma_load_3d(smem + kKOff + st * kTileBytes, &tm_k, 0, h, row, &bars->kv_full[st]);
          tma_load_3d(smem + kVOff + st * kTileBytes, &tm_v, 0, h, row, &bars->kv_full[st]);
        }
        issued = j + 1;
      }
      // drain: the last loads of each stage must land before the CTA may exit
      mbar_wait_timeout(&bars->q_full, 0, kWaitNs);
      for (int j = max(0, issued - kStages); j < issued; ++j)
        mbar_wait_timeout(&bars->kv_full[j % kStages], (j / kStages) & 1, kWaitNs);
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_qk = umma_idesc_bf16(kBM, kBN, 0, 0);
      const uint32_t idesc_pv = umma_idesc_bf16(kBM, kDH, 0, 1);
      const uint32_t sq = smem_u32(smem + kQOff);
      bool ok = mbar_wait_bounded(&bars->q_full, 0, abort_flag, kWaitNs);
      auto issue_pv = [&](int jj) -> bool {
        const int sb = jj & 1, st = jj % kStages;
        if (!mbar_wait_bounded(&bars->p_full[sb], (jj >> 1) & 1, abort_flag, kWaitNs)) return false;
        if (jj >= 2 && !mbar_wait_bounded(&bars->o_empty[sb], ((jj - 2) >> 1) & 1, abort_flag, kWaitNs))
          return false;
        tc_fence_after();
        const uint32_t sp = smem_u32(smem + kPOff + sb * kPBytes);
        const uint32_t sv = smem_u32(smem + kVOff + st * kTileBytes);
#pragma unroll
        for (int k = 0; k < kBN / 16; ++k) {
          // A = P (K-major: 64-key column blocks of 16 KB, 32 bytes per 16 keys)
          const uint64_t adesc = umma_desc_sw128(sp + (k >> 2) * kTileBytes + (k & 3) * 32, 16, 1024);
          // B = V (MN-major: 16 keys = two 8-row groups of 1024 bytes)
          const uint64_t bdesc = umma_desc_sw128(sv + k * 2048, 16, 1024);
          umma_bf16(tmem + kOCol + sb * kDH, adesc, bdesc, idesc_pv, k > 0 ? 1u : 0u);
        }
        umma_commit(&bars->o_full[sb]);
        umma_commit(&bars->kv_empty[st]);
        return true;
      };
      for (int j = 0; ok && j < NT; ++j) {
        const int st = j % kStages, sb = j & 1;
        if (!mbar_wait_bounded(&bars->kv_full[st], (j / kStages) & 1, abort_flag, kWaitNs)) { ok = false; break; }
        tc_fence_after();
        const uint32_t sk = smem_u32(smem + kKOff + st * kTileBytes);
#pragma unroll
        for (int k = 0; k < kDH / 16; ++k) {
          const uint64_t adesc = umma_desc_sw128(sq + k * 32, 16, 1024);
          const uint64_t bdesc = umma_desc_sw128(sk + k * 32, 16, 1024);
          umma_bf16(tmem + kSCol + sb * kBN, adesc, bdesc, idesc_qk, k > 0 ? 1u : 0u);
        }
        umma_commit(&bars->s_full[sb]);
        if (j >= 1 && !issue_pv(j - 1)) { ok = false; break; }
      }
      if (ok) ok = issue_pv(NT - 1);
      if (!ok) *abort_flag = 1;
      umma_commit(&bars->mma_done);  // every MMA issued above has finished when this arrives
      mbar_wait_timeout(&bars->mma_done, 0, kWaitNs);
    }
  } else {
    // ------------------------------------------------------------ softmax warps 0-3
    const int r = tid;  // query row within the tile == TMEM lane
    const int i = q0 + r;
    const bool row_ok = i <= q_last;
    const int my_ls = row_ok ? a.ls[tok0 + i] : 0;
    const int my_nbb = row_ok ? a.nbb[tok0 + i] : 0;
    const float sl2 = a.scale * kLog2e;
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
    uint8_t* p_row_base = smem + kPOff + r * 128;
    const int sw = r & 7;

    float m_run = -INFINITY, l_run = 0.f;
    float m_acc_use = 0.f;
    bool acc_empty = true;
    float acc[kDH];
#pragma unroll
    for (int c = 0; c < kDH; ++c) acc[c] = 0.f;
    float m_tile_use = 0.f;  // running-max reference used for the previous tile's P
    bool ok = true;

    auto accumulate = [&](int jj, float m_ref) -> bool {
      const int ob = jj & 1;
      if (!mbar_wait_bounded(&bars->o_full[ob], (jj >> 1) & 1, abort_flag, kWaitNs)) return false;
      tc_fence_after();
      uint32_t o0[32], o1[32];
      tmem_ld32_sync(lane_base + kOCol + ob * kDH, o0);
      tmem_ld32_sync(lane_base + kOCol + ob * kDH + 32, o1);
      tc_fence_before();
      mbar_arrive(&bars->o_empty[ob]);
      const float f = acc_empty ? 0.f : ex2(m_acc_use - m_ref);
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        acc[c] = fmaf(acc[c], f, __uint_as_float(o0[c]));
        acc[c + 32] = fmaf(acc[c + 32], f, __uint_as_float(o1[c]));
      }
      m_acc_use = m_ref;
      acc_empty = false;
      return true;
    };

    for (int j = 0; j < NT; ++j) {
      const int sb = j & 1;
      int lo, hi;
      if (j < nbt) {
        lo = 0;
        hi = min(max(my_nbb - j * kBN, 0), kBN);
      } else {
        const int j0 = ls_first + (j - nbt) * kBN;
        lo = min(max(my_ls - j0, 0), kBN);
        hi = min(max(i - j0 + 1, 0), kBN);
      }
      if (!row_ok) { lo = 0; hi = 0; }
      if (!mbar_wait_bounded(&bars->s_full[sb], (j >> 1) & 1, abort_flag, kWaitNs)) { ok = false; break; }
      tc_fence_after();
      float s[kBN];
#pragma unroll
      for (int q = 0; q < kBN / 32; ++q) {
        uint32_t v[32];
        tmem_ld32_sync(lane_base + kSCol + sb * kBN + q * 32, v);
#pragma unroll
        for (int c = 0; c < 32; ++c) s[q * 32 + c] = __uint_as_float(v[c]);
      }
      float mt = -INFINITY;
#pragma unroll
      for (int c = 0; c < kBN; ++c) {
        const float v = (c >= lo && c < hi) ? s[c] * sl2 : -INFINITY;
        s[c] = v;
        mt = fmaxf(mt, v);
      }
      const float m_new = fmaxf(m_run, mt);
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
      const float alpha = ex2(m_run - m_use);  // 0 while nothing was seen
      float sum = 0.f;
#pragma unroll
      for (int c = 0; c < kBN; ++c) {
        s[c] = ex2(s[c] - m_use);
        sum += s[c];
      }
      l_run = l_run * alpha + sum;
      m_run = m_new;
      // P row -> shared memory, 128-byte swizzled K-major layout (16-byte chunk c of row r at c ^ (r & 7))
      uint8_t* prow = p_row_base + sb * kPBytes;
#pragma unroll
      for (int cc = 0; cc < kBN / 8; ++cc) {
        uint4 pk;
        pk.x = pack_bf16x2(s[cc * 8 + 0], s[cc * 8 + 1]);
        pk.y = pack_bf16x2(s[cc * 8 + 2], s[cc * 8 + 3]);
        pk.z = pack_bf16x2(s[cc * 8 + 4], s[cc * 8 + 5]);
        pk.w = pack_bf16x2(s[cc * 8 + 6], s[cc * 8 + 7]);
        *reinterpret_cast<uint4*>(prow + (cc >> 3) * kTileBytes + (((cc & 7) ^ sw) << 4)) = pk;
      }
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(&bars->p_full[sb]);
      if (j >= 1 && !accumulate(j - 1, m_tile_use)) { ok = false; break; }
      m_tile_use = m_use;
    }
    if (ok) ok = accumulate(NT - 1, m_tile_use);
    if (!ok) {
      *abort_flag = 1;
      raise_status(a.status, ATTAMBA_DEV_TIMEOUT);
    } else if (row_ok) {
      const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
      uint4* dst = reinterpret_cast<uint4*>(O + ((tok0 + i) * H + h) * kDH);
#pragma unroll
      for (int c = 0; c < kDH / 8; ++c) {
        uint4 pk;
        pk.x = pack_bf16x2(acc[c * 8 + 0] * inv, acc[c * 8 + 1] * inv);
        pk.y = pack_bf16x2(acc[c * 8 + 2] * inv, acc[c * 8 + 3] * inv);
        pk.z = pack_bf16x2(acc[c * 8 + 4] * inv, acc[c * 8 + 5] * inv);
        pk.w = pack_bf16x2(acc[c * 8 + 6] * inv, acc[c * 8 + 7] * inv);
        dst[c] = pk;
      }
      if (a.lse)
        a.lse[((int64_t)b * H + h) * n + i] = l_run > 0.f ? (m_run + __log2f(l_run)) * kLn2 : -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------- fp32, CUDA cores
__global__ void __launch_bounds__(128) chunk_attn_f32_kernel(AttnArgs a) {
  const int64_t T = (int64_t)a.B * a.n;
  const int64_t tok = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int h = blockIdx.y;
  if (tok >= T) return;
  const int H = a.H;
  const int b = (int)(tok / a.n);
  const int i = (int)(tok - (int64_t)b * a.n);
  const float* q = static_cast<const float*>(a.q) + (tok * H + h) * kDH;
  const float* K = static_cast<const float*>(a.K);
  const float* V = static_cast<const float*>(a.V);
  const float* Kc = static_cast<const float*>(a.Kc);
  const float* Vc = static_cast<const float*>(a.Vc);
  float qr[kDH], acc[kDH];
#pragma unroll
  for (int c = 0; c < kDH; ++c) { qr[c] = q[c] * a.scale; acc[c] = 0.f; }
  float m = -INFINITY, l = 0.f;
  const int nbb = a.nbb[tok], ls = a.ls[tok];
  const int64_t chunk0 = a.bptr[b];
  auto visit = [&](const float* kr, const float* vr) {
    float s = 0.f;
#pragma unroll
    for (int c = 0; c < kDH; ++c) s = fmaf(qr[c], kr[c], s);
    const float m_new = fmaxf(m, s);
    const float alpha = expf(m - m_new);
    const float p = expf(s - m_new);
    l = l * alpha + p;
#pragma unroll
    for (int c = 0; c < kDH; ++c) acc[c] = fmaf(acc[c], alpha, p * vr[c]);
    m = m_new;
  };
  for (int k = 0; k < nbb; ++k) {
    const int64_t row = chunk0 + k;
    visit(Kc + (row * H + h) * kDH, Vc + (row * H + h) * kDH);
  }
  for (int j = ls; j <= i; ++j) {
    const int64_t row = (int64_t)b * a.n + j;
    visit(K + (row * H + h) * kDH, V + (row * H + h) * kDH);
  }
  float* O = static_cast<float*>(a.O) + (tok * H + h) * kDH;
  const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
  for (int c = 0; c < kDH; ++c) O[c] = acc[c] * inv;
  if (a.lse) a.lse[((int64_t)b * H + h) * a.n + i] = l > 0.f ? m + logf(l) : -INFINITY;
}

// ---------------------------------------------------------------- tensor maps
PFN_cuTensorMapEncodeTiled_v12000 get_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// [rows, H, 64] bf16 viewed as a 3-D tensor; box = 64 x 1 x 128 with the 128-byte swizzle
bool encode_rows_map(CUtensorMap* m, const void* base, int64_t rows, int H) {
  auto enc = get_encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)kDH, (cuuint64_t)H, (cuuint64_t)rows};
  cuuint64_t strides[2] = {(cuuint64_t)kDH * 2, (cuuint64_t)H * kDH * 2};
  cuuint32_t box[3] = {(cuuint32_t)kDH, 1, (cuuint32_t)kBN};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}
}  // namespace

cudaError_t launch_chunk_attn_bf16(const AttnArgs& a, cudaStream_t s) {
  const int64_t T = (int64_t)a.B * a.n;
  CUtensorMap tq, tk, tv, tkc, tvc;
  if (!encode_rows_map(&tq, a.q, T, a.H) || !encode_rows_map(&tk, a.K, T, a.H) ||
      !encode_rows_map(&tv, a.V, T, a.H) || !encode_rows_map(&tkc, a.Kc, a.n_chunks, a.H) ||
      !encode_rows_map(&tvc, a.Vc, a.n_chunks, a.H))
    return cudaErrorNotSupported;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(chunk_attn_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  dim3 grid((a.n + kBM - 1) / kBM, a.H, a.B);
  chunk_attn_bf16_kernel<<<grid, kThreads, kSmemBytes, s>>>(tq, tk, tv, tkc, tvc, a);
  return cudaGetLastError();
}

cudaError_t launch_chunk_attn_f32(const AttnArgs& a, cudaStream_t s) {
  const int64_t T = (int64_t)a.B * a.n;
  dim3 grid((unsigned)((T + 127) / 128), a.H);
  chunk_attn_f32_kernel<<<grid, 128, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace attamba
