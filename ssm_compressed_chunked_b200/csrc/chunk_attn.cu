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
// bf16 kernel (tcgen05), persistent: two CTAs per SM walk work items of 128
// queries of one (sequence, head), longest key lists first.  An item's key
// tiles (64 keys each) are first the chunk-end tiles 0..nbb(last query), then
// the local band [ls(first query), last query]; both are plain TMA boxes.
//   warp 4     TMA producer: Q of each item (two buffers), then K/V tiles into
//              a 4-stage ring; it also stores each finished O tile
//   warp 5     one thread issues tcgen05.mma: S = Q K^T (M128 N64 K64, both
//              operands in shared memory) into TMEM, then O += P V (M128 N64
//              K64, P read from TMEM, V from shared memory)
//   warps 0-3  softmax, one query row per thread: one tcgen05.ld for its S row,
//              masking (a 64-bit column mask, one bit test and one select per
//              column) only where the row's key range cuts the tile, 32-column
//              chunks outside every row's range skipped, fp32 sums, P as bf16
//              pairs back into TMEM with one tcgen05.st
// TMEM per CTA (256 columns): S in two buffers of 64, P in two of 32, O 64.
// With S and P double-buffered the QK of tile g + 1 and the PV of tile g - 1
// run while the softmax works on tile g.  The one issuing thread orders the
// MMAs PV(g - 2) before QK(g), and a tcgen05.commit arrives only once every
// MMA that thread issued before it has completed, so two waits are implied
// and not made: the softmax, having seen S(g), may refill P buffer g & 1 (its
// last reader PV(g - 2) is done), and the issuer, having seen the P of tile
// g - 2 arrive (each softmax thread arrives after its load of S(g - 2) has
// completed), may overwrite S buffer g & 1 with QK(g).  Because the four
// softmax warps can drift up to two tiles apart, every barrier they arrive on
// exists per buffer.  O accumulates in TMEM across an item's tiles;
// P = exp2(s - m_ref) against a per-row reference that only has to keep P
// finite: it is the row max of the first tile where the row has keys, and it
// moves to the current row max (P recomputed, O and l rescaled in TMEM) only
// when a tile's row sum exceeds 2^16 or overflows, so the row max is computed
// on few tiles; the final O / l is exact whatever reference was used.  A full 128-row tile of O
// is staged (128-byte swizzle) in its item's own Q buffer, whose last reader,
// the item's last QK, has finished by then, and leaves with one TMA store; the
// producer issues the store and refills the buffer with the Q of the item two
// ahead only after the store has read it.  A partial tile (the end of a
// sequence) is written row by row.  At an item boundary the previous item's
// last PV is issued before the next item's first QK, so the epilogue does not
// wait for the next item's loads.
//
// Measured limits (B200, bench workload): the exponentials of a 64-column
// tile cost 512 cycles of the multi-function unit per warp; with two softmax
// warps per SM sub-partition the tile's other instructions (about half of them
// on the integer/logic pipe) and the barrier and TMEM latencies set the pace,
// so each instruction taken out of the tile loop shows: the column mask and
// the on-demand row max took 78.5 us to 70.6 us, and dropping the two implied
// waits to 66.5 us.  One thread issues a tcgen05.mma every ~90 cycles
// (measured, N = 64 or 128 alike), so the eight MMAs of a tile keep the issuing
// thread busy for ~720 of the ~1500 cycles a tile takes.  A third CTA does not fit (TMEM, shared memory); eight softmax
// warps with the 16-lane TMEM shapes, 128-key tiles, and moving a share of the
// exponentials to an FMA-pipe polynomial all measured slower.
//
// f32 kernel: one thread per (query, head) on the CUDA cores, same key sets,
// fp32 online softmax (the fp32 tensor-core kinds round to tf32).
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "launch.h"

namespace attamba {

// the driver's tensor-map encoder, resolved once at run time (the library links no driver API)
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  // resolved once (thread-safe static initialisation)
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    return static_cast<PFN_cuTensorMapEncodeTiled_v12000>(nullptr);
  }();
  return fn;
}

namespace {
constexpr int kBM = 128;                                    // queries per work item (TMEM lanes)
constexpr int kBN = 64;                                     // keys per tile
constexpr int kDH = 64;
#ifndef ATTAMBA_ATTN_STAGES
#define ATTAMBA_ATTN_STAGES 4
#endif
#ifndef ATTAMBA_ATTN_CTAS_PER_SM
#define ATTAMBA_ATTN_CTAS_PER_SM 2
#endif
constexpr int kStages = ATTAMBA_ATTN_STAGES;                // K/V ring depth
constexpr int kThreads = 192;
constexpr int kCtasPerSm = ATTAMBA_ATTN_CTAS_PER_SM;
constexpr int kMaxItems = 64;                               // work items per CTA (the host sizes the grid)
constexpr uint32_t kQBytes = kBM * kDH * 2;                 // 16 KB: 128 rows x 128 bytes
constexpr uint32_t kKVBytes = kBN * kDH * 2;                // 8 KB: 64 rows x 128 bytes
constexpr uint32_t kQOff = 0;                               // two Q tiles
constexpr uint32_t kKOff = kQOff + 2 * kQBytes;             // kStages K tiles
constexpr uint32_t kVOff = kKOff + kStages * kKVBytes;      // kStages V tiles
constexpr uint32_t kBarOff = kVOff + kStages * kKVBytes;
constexpr uint32_t kItemOff = kBarOff + 256;
constexpr uint32_t kSmemBytes = kItemOff + kMaxItems * 32 + 1024;   // + item table + alignment slack
constexpr uint32_t kTmemCols = 256;                         // power of two, >= 32
constexpr uint32_t kSCol = 0;                               // S, two buffers: columns 0..63, 64..127 (fp32)
constexpr uint32_t kPCol = 2 * kBN;                         // P, two buffers: columns 128..159, 160..191 (bf16 pairs)
constexpr uint32_t kOCol = 3 * kBN;                         // O: columns 192..255 (fp32)
constexpr uint64_t kWaitNs = 4000000000ull;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
static_assert(kOCol + kDH <= kTmemCols, "TMEM columns");

// Double-buffered resources (Q, S, P) use barrier pairs: use u of the resource is
// buffer u & 1, phase u >> 1 of that buffer's barrier; the K/V ring completes once
// per use of a stage.  The softmax warps may drift up to two key tiles apart, so
// every barrier they arrive on is per buffer: an arrival for tile g + 1 must not
// count towards tile g.
struct Bars {
  uint64_t q_full[2];
  uint64_t q_empty[2];
  uint64_t kv_full[kStages];
  uint64_t kv_empty[kStages];
  uint64_t s_full[2];    // QK of tile g done (tcgen05.commit)
  uint64_t p_full[2];    // every softmax thread has written P of tile g (128 arrivals)
  uint64_t pv_done[2];   // PV of tile g done (tcgen05.commit)
  uint64_t mma_done;
  uint64_t o_ready;      // every softmax thread has written its row of O into the item's Q buffer (128 arrivals)
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(Bars) <= 256, "barrier block overflows its shared-memory slot");

// One work item: 128 queries of one (sequence, head).  Items are numbered so
// that the longest key lists (last query tiles) come first.
struct Item {
  int b, h, q0, q_last, ls_first, nbt, NT, chunk0;
};

__device__ __forceinline__ Item decode_item(const AttnArgs& a, int item, int n_qt) {
  const int BH = a.B * a.H;
  const int qt = n_qt - 1 - item / BH;
  const int bh = item - (item / BH) * BH;
  Item it;
  it.b = bh / a.H;
  it.h = bh - it.b * a.H;
  it.q0 = qt * kBM;
  it.q_last = min(it.q0 + kBM, a.n) - 1;
  const int64_t tok0 = (int64_t)it.b * a.n;
  it.ls_first = a.ls[tok0 + it.q0];
  it.nbt = (a.nbb[tok0 + it.q_last] + kBN - 1) / kBN;
  // the local segment [ls(i), i] is empty only when ls(i) = i + 1 (M_test, L = 0);
  // ls(i) - i does not grow with i, so the last row decides
  const bool band_empty = a.ls[tok0 + it.q_last] > it.q_last;
  const int band_len = band_empty ? 0 : max(0, it.q_last - it.ls_first + 1);
  it.NT = it.nbt + (band_len + kBN - 1) / kBN;
  it.chunk0 = a.bptr[it.b];
  // the item's chunk-end tiles read the sequence's own chunk ends, its band starts inside the sequence
  if (!in_bounds(a.nbb[tok0 + it.q_last] <= a.bptr[it.b + 1] - it.chunk0 && it.ls_first >= 0 &&
                     it.ls_first <= it.q0 + 1 && it.q_last < a.n,
                 a.status))
    it.NT = 0;
  return it;
}

// 64 consecutive 32-bit TMEM columns of this thread's lane, one wait
__device__ __forceinline__ void tmem_ld64_sync(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,"
      "%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
      "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]),
        "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]),
        "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]),
        "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]),
        "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
      : "r"(taddr)
      : "memory");
}

// 32 consecutive 32-bit columns from registers into this thread's TMEM lane (not waited)
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;"
      : "=l"(reinterpret_cast<uint64_t&>(d))
      : "l"(reinterpret_cast<const uint64_t&>(a)), "l"(reinterpret_cast<const uint64_t&>(b)),
        "l"(reinterpret_cast<const uint64_t&>(c)));
  return d;
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  float2 d;
  asm("add.rn.f32x2 %0, %1, %2;"
      : "=l"(reinterpret_cast<uint64_t&>(d))
      : "l"(reinterpret_cast<const uint64_t&>(a)), "l"(reinterpret_cast<const uint64_t&>(b)));
  return d;
}

// 3-D tiled tensor store from this CTA's shared memory (bulk async group)
__device__ __forceinline__ void tma_store_3d(const void* tmap, const void* src, int x, int y, int z) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(tmap),
               "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z)
               : "memory");
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// the previous stores have finished reading shared memory
__device__ __forceinline__ void tma_store_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// the previous stores are complete
__device__ __forceinline__ void tma_store_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    chunk_attn_bf16_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                           const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_kc,
                           const __grid_constant__ CUtensorMap tm_vc, const __grid_constant__ CUtensorMap tm_o,
                           AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + kBarOff);
  Item* items = reinterpret_cast<Item*>(smem + kItemOff);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_qt = (a.n + kBM - 1) / kBM;
  const int n_items_all = n_qt * a.B * a.H;
  // this CTA's items: blockIdx.x, blockIdx.x + gridDim.x, ...
  const int my_items = (n_items_all - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;
  const int H = a.H, n = a.n;
  __nv_bfloat16* O = static_cast<__nv_bfloat16*>(a.O);

  if (my_items > kMaxItems) {  // the host sizes the grid so that this cannot happen
    if (tid == 0) raise_status(a.status, ATTAMBA_DEV_TIMEOUT);
    return;
  }
  if (warp == 4 && lane == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->q_full[b], 1);
      mbar_init(&bars->q_empty[b], 1);
      mbar_init(&bars->s_full[b], 1);
      mbar_init(&bars->pv_done[b], 1);
      mbar_init(&bars->p_full[b], kBM);
    }
    for (int i = 0; i < kStages; ++i) { mbar_init(&bars->kv_full[i], 1); mbar_init(&bars->kv_empty[i], 1); }
    mbar_init(&bars->mma_done, 1);
    mbar_init(&bars->o_ready, kBM);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&bars->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  // launched as a programmatic dependent of the previous kernel in the stream, whose outputs may be
  // this kernel's inputs: the set-up above reads none, everything below waits for that grid
  asm volatile("griddepcontrol.wait;" ::: "memory");
  for (int k = tid; k < my_items; k += kThreads) items[k] = decode_item(a, blockIdx.x + k * gridDim.x, n_qt);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort_flag = &bars->abort;

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q); tma_prefetch_desc(&tm_k); tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_kc); tma_prefetch_desc(&tm_vc); tma_prefetch_desc(&tm_o);
      int g = 0, wi = 0;
      int n_st = 0;              // O tiles stored so far (phases of o_ready)
      int q_item0 = -1, q_item1 = -1;  // the item whose Q (then O) each buffer holds
      // a whole 128-row O tile is staged by the softmax warps in its item's Q buffer; it leaves
      // with one TMA store, and the buffer takes new Q only once the store has read it
      auto store_o = [&](int u) -> bool {
        const Item& it = items[u ? q_item1 : q_item0];
        if (it.q_last != it.q0 + kBM - 1) return true;   // a partial tile was written row by row
        if (!mbar_wait_bounded(&bars->o_ready, n_st & 1, abort_flag, kWaitNs)) return false;
        tma_store_3d(&tm_o, smem + kQOff + u * kQBytes, 0, it.h, (int)((int64_t)it.b * n + it.q0));
        tma_store_wait_read();
        ++n_st;
        return true;
      };
      bool ok = true;
      for (int k = 0; ok && k < my_items; ++k) {
        const Item it = items[k];
        if (it.NT == 0) continue;
        const int64_t tok0 = (int64_t)it.b * n;
        const int qb = wi & 1;
        if (wi >= 2 && (!mbar_wait_bounded(&bars->q_empty[qb], ((wi - 2) >> 1) & 1, abort_flag, kWaitNs) ||
                        !store_o(qb))) {
          ok = false;
          break;
        }
        if (qb) q_item1 = k; else q_item0 = k;
        mbar_arrive_expect_tx(&bars->q_full[qb], kQBytes);
        tma_load_3d(smem + kQOff + qb * kQBytes, &tm_q, 0, it.h, (int)(tok0 + it.q0), &bars->q_full[qb]);
        ++wi;
        for (int j = 0; j < it.NT; ++j, ++g) {
          const int st = g % kStages;
          if (g >= kStages &&
              !mbar_wait_bounded(&bars->kv_empty[st], ((g / kStages) - 1) & 1, abort_flag, kWaitNs)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bars->kv_full[st], 2 * kKVBytes);
          const bool bnd = j < it.nbt;
          const int row = bnd ? it.chunk0 + j * kBN : (int)(tok0 + it.ls_first + (j - it.nbt) * kBN);
          tma_load_3d(smem + kKOff + st * kKVBytes, bnd ? &tm_kc : &tm_k, 0, it.h, row, &bars->kv_full[st]);
          tma_load_3d(smem + kVOff + st * kKVBytes, bnd ? &tm_vc : &tm_v, 0, it.h, row, &bars->kv_full[st]);
        }
      }
      // the last two items' O tiles
      for (int u = max(0, wi - 2); ok && u < wi; ++u) ok = store_o(u & 1);
      if (!ok) *abort_flag = 1;
      // drain: the last copies into each buffer must land, and the stores complete, before the CTA may exit
      for (int u = max(0, wi - 2); u < wi; ++u) mbar_wait_timeout(&bars->q_full[u & 1], (u >> 1) & 1, kWaitNs);
      for (int j = max(0, g - kStages); j < g; ++j)
        mbar_wait_timeout(&bars->kv_full[j % kStages], (j / kStages) & 1, kWaitNs);
      tma_store_wait_all();
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_qk = umma_idesc_bf16(kBM, kBN, 0, 0);
      const uint32_t idesc_pv = umma_idesc_bf16(kBM, kDH, 0, 1);
      // PV of tile gg: O (+)= P V with P from TMEM buffer gg & 1 (8 columns per 16 keys) and V
      // from shared memory (MN-major, 2048 bytes per 16 keys); the first tile of an item overwrites O
      auto issue_pv = [&](int gg, bool first) -> bool {
        const int st = gg % kStages;
        if (!mbar_wait_bounded(&bars->p_full[gg & 1], (gg >> 1) & 1, abort_flag, kWaitNs)) return false;
        tc_fence_after();
        const uint32_t sv = smem_u32(smem + kVOff + st * kKVBytes);
#pragma unroll
        for (int k = 0; k < kBN / 16; ++k)
          umma_bf16_ts(tmem + kOCol, tmem + kPCol + (gg & 1) * (kBN / 2) + k * 8,
                       umma_desc_sw128(sv + k * 2048, 16, 1024), idesc_pv, (first && k == 0) ? 0u : 1u);
        umma_commit(&bars->pv_done[gg & 1]);
        umma_commit(&bars->kv_empty[st]);
        return true;
      };
      int g = 0, wi = 0;
      bool pend = false, pend_first = false;   // PV(g - 1) not issued yet; it is its item's first tile
      bool ok = true;
      for (int k = 0; ok && k < my_items; ++k) {
        const Item it = items[k];
        if (it.NT == 0) continue;
        // the previous item's last PV goes first: its epilogue must not wait for this item's loads
        if (pend) {
          if (!issue_pv(g - 1, pend_first)) { ok = false; break; }
          pend = false;
        }
        const int qb = wi & 1;
        if (!mbar_wait_bounded(&bars->q_full[qb], (wi >> 1) & 1, abort_flag, kWaitNs)) { ok = false; break; }
        const uint32_t sq = smem_u32(smem + kQOff + qb * kQBytes);
        for (int j = 0; j < it.NT; ++j, ++g) {
          const int st = g % kStages;
          if (!mbar_wait_bounded(&bars->kv_full[st], (g / kStages) & 1, abort_flag, kWaitNs)) { ok = false; break; }
          // S buffer g & 1 was last read by the softmax for tile g - 2, whose P arrival (each thread
          // makes it after its S load has completed) was waited for before PV(g - 2) was issued
          tc_fence_after();
          const uint32_t sk = smem_u32(smem + kKOff + st * kKVBytes);
#pragma unroll
          for (int kk = 0; kk < kDH / 16; ++kk)
            umma_bf16(tmem + kSCol + (g & 1) * kBN, umma_desc_sw128(sq + kk * 32, 16, 1024),
                      umma_desc_sw128(sk + kk * 32, 16, 1024), idesc_qk, kk > 0 ? 1u : 0u);
          umma_commit(&bars->s_full[g & 1]);
          if (j == it.NT - 1) umma_commit(&bars->q_empty[qb]);  // Q free once the item's last QK is done
          if (pend && !issue_pv(g - 1, pend_first)) { ok = false; break; }
          pend = true;
          pend_first = (j == 0);
        }
        ++wi;
      }
      if (ok && pend) ok = issue_pv(g - 1, pend_first);
      if (!ok) *abort_flag = 1;
      umma_commit(&bars->mma_done);  // every MMA issued above has finished when this arrives
      mbar_wait_timeout(&bars->mma_done, 0, kWaitNs);
    }
  } else {
    // ------------------------------------------------------------ softmax warps 0-3
    const int r = tid;  // query row within the tile == TMEM lane
    const float sl2 = a.scale * kLog2e;
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
    const uint32_t o_tmem = lane_base + kOCol;
    const int sw = r & 7;
    int g = 0, wi = 0;   // key tiles and non-empty items so far (item wi's Q is in buffer wi & 1)
    bool ok = true;
    // wait for the PV of tile gg (barrier gg & 1, its phase gg >> 1; verdict warp-uniform)
    auto wait_pv = [&](int gg) -> bool {
      return __all_sync(0xffffffffu,
                        mbar_wait_bounded(&bars->pv_done[gg & 1], (gg >> 1) & 1, abort_flag, kWaitNs));
    };
    for (int k = 0; ok && k < my_items; ++k) {
      const Item it = items[k];
      const int64_t tok0 = (int64_t)it.b * n;
      const int i = it.q0 + r;
      const bool row_ok = i <= it.q_last;
      int my_ls = 0, my_nbb = 0;
      if (row_ok) {
        my_ls = a.ls[tok0 + i];
        my_nbb = a.nbb[tok0 + i];
        // the row's keys lie inside the item's tiles (the chunk-end tiles cover nbb(q_last) >= nbb(i),
        // the band starts at ls(first query) <= ls(i))
        if (!in_bounds(my_nbb <= it.nbt * kBN && my_ls >= it.ls_first, a.status)) {
          my_nbb = 0;
          my_ls = i + 1;
        }
      }
      if (it.NT == 0) {  // every row of the item has an empty key set
        if (row_ok) {
          uint4* dst = reinterpret_cast<uint4*>(O + ((tok0 + i) * H + it.h) * kDH);
#pragma unroll
          for (int c = 0; c < kDH / 8; ++c) dst[c] = make_uint4(0, 0, 0, 0);
          if (a.lse) a.lse[((int64_t)it.b * H + it.h) * n + i] = -INFINITY;
        }
        continue;
      }
      float m_ref = -INFINITY, l_run = 0.f;  // P of this item is exp2(s * sl2 - m_ref)
      for (int j = 0; j < it.NT; ++j, ++g) {
        int lo, hi;
        if (j < it.nbt) {
          lo = 0;
          hi = min(max(my_nbb - j * kBN, 0), kBN);
        } else {
          const int j0 = it.ls_first + (j - it.nbt) * kBN;
          lo = min(max(my_ls - j0, 0), kBN);
          hi = min(max(i - j0 + 1, 0), kBN);
        }
        if (!row_ok) { lo = 0; hi = 0; }
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(&bars->s_full[g & 1], (g >> 1) & 1, abort_flag, kWaitNs))) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t sr[kBN];
        tmem_ld64_sync(lane_base + kSCol + (g & 1) * kBN, &sr[0]);
        // row max of the raw scores over the valid columns [lo, hi); masked columns become -inf in place
        if (lo != 0 || hi != kBN) {
          // the valid columns as two 32-bit masks; each column is then one bit test and one select
          const uint64_t below_hi = hi >= 64 ? ~0ull : ((1ull << hi) - 1);
          const uint64_t below_lo = lo >= 64 ? ~0ull : ((1ull << lo) - 1);
          const uint64_t valid = (hi > lo) ? (below_hi & ~below_lo) : 0ull;
          const uint32_t v0 = (uint32_t)valid, v1 = (uint32_t)(valid >> 32);
#pragma unroll
          for (int c = 0; c < 32; ++c)
            if (!(v0 & (1u << c))) sr[c] = 0xff800000u;
#pragma unroll
          for (int c = 0; c < 32; ++c)
            if (!(v1 & (1u << c))) sr[32 + c] = 0xff800000u;
        }
#define S_(c) __uint_as_float(sr[c])
        // The reference m_ref only has to keep every P finite and of useful size; the final O / l
        // is exact whatever it is.  So a tile is first exponentiated against the reference it
        // finds, and the row max is taken only for a row with no reference yet, or when the row
        // sum says some score rose more than 2^16 above it (or overflowed); then the row moves
        // its reference to the max, P is recomputed and O and l are rescaled.
        auto row_max = [&]() -> float {
          float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll
          for (int c = 0; c < kBN; c += 8) {
            mx0 = max3(mx0, S_(c), S_(c + 1));
            mx1 = max3(mx1, S_(c + 2), S_(c + 3));
            mx2 = max3(mx2, S_(c + 4), S_(c + 5));
            mx3 = max3(mx3, S_(c + 6), S_(c + 7));
          }
          return fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * sl2;
        };
        uint32_t pk[kBN / 2];
        float tsum = 0.f;
        auto exps = [&]() {
          const float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;
          const float2 sl2x2 = make_float2(sl2, sl2), negm = make_float2(-m_use, -m_use);
          float2 sum0 = make_float2(0.f, 0.f), sum1 = make_float2(0.f, 0.f);
#pragma unroll
          for (int q = 0; q < kBN / 32; ++q) {
            // a 32-column chunk outside every lane's [lo, hi) needs no exponentials
            const bool need = __any_sync(0xffffffffu, lo < q * 32 + 32 && hi > q * 32);
            if (need) {
#pragma unroll
              for (int c = 0; c < 32; c += 4) {
                float2 e0 = ffma2(make_float2(S_(q * 32 + c), S_(q * 32 + c + 1)), sl2x2, negm);
                float2 e1 = ffma2(make_float2(S_(q * 32 + c + 2), S_(q * 32 + c + 3)), sl2x2, negm);
                e0 = make_float2(ex2(e0.x), ex2(e0.y));
                e1 = make_float2(ex2(e1.x), ex2(e1.y));
                sum0 = fadd2(sum0, e0);
                sum1 = fadd2(sum1, e1);
                pk[q * 16 + c / 2] = pack_bf16x2(e0.x, e0.y);
                pk[q * 16 + c / 2 + 1] = pack_bf16x2(e1.x, e1.y);
              }
            } else {
#pragma unroll
              for (int c = 0; c < 16; ++c) pk[q * 16 + c] = 0u;
            }
          }
          const float2 s2 = fadd2(sum0, sum1);
          tsum = s2.x + s2.y;
        };
        // a row with keys in this tile but no reference yet takes its max first
        const bool no_ref = m_ref == -INFINITY && hi > lo;
        if (__any_sync(0xffffffffu, no_ref)) {
          const float mt = row_max();
          if (no_ref) m_ref = mt;
        }
        exps();
        float fscale = 1.f;
        bool grow = false;
        if (__any_sync(0xffffffffu, !(tsum <= 65536.f))) {
          const float mt = row_max();
          grow = mt > m_ref;   // only rows whose max rose past the reference (a row's new keys
                               // never lower it)
          if (grow) {
            fscale = ex2(m_ref - mt);   // brings this row's O and l to the new reference
            l_run *= fscale;
            m_ref = mt;
          }
          exps();
        }
        const bool rescale = j > 0 && __any_sync(0xffffffffu, grow);
#undef S_
        l_run += tsum;
        // P buffer g & 1 was last read by the PV of tile g - 2: issued before S(g), so complete
        // once the commit of S(g) arrived
        tc_fence_after();
        tmem_st32(lane_base + kPCol + (g & 1) * (kBN / 2), &pk[0]);
        if (rescale) {
          // scale O (the PV of the tiles before j, complete once PV(g - 1) is) for the rows whose
          // reference max rose
          if (g >= 1 && !wait_pv(g - 1)) { ok = false; break; }
          tc_fence_after();
#pragma unroll 1
          for (int half = 0; half < 2; ++half) {
            uint32_t o0[32];
            tmem_ld32_sync(o_tmem + half * 32, o0);
#pragma unroll
            for (int c = 0; c < 32; ++c) o0[c] = __float_as_uint(__uint_as_float(o0[c]) * fscale);
            tmem_st32(o_tmem + half * 32, o0);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars->p_full[g & 1]);
      }
      if (!ok) break;
      // epilogue: the item's last PV, then O / l from TMEM (the next item's first PV is
      // issued only after this thread's next p_full arrival, so O is not overwritten early)
      if (!wait_pv(g - 1)) { ok = false; break; }
      tc_fence_after();
      const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
      // a full tile is staged in the item's Q buffer (its last QK finished before this PV did)
      // and leaves through one TMA store issued by the producer
      const bool whole = it.q_last == it.q0 + kBM - 1;
      uint8_t* orow = smem + kQOff + (wi & 1) * kQBytes + r * 128;
      ++wi;
      uint4* dst = reinterpret_cast<uint4*>(O + ((tok0 + i) * H + it.h) * kDH);
#pragma unroll 1
      for (int half = 0; half < 2; ++half) {
        uint32_t o0[32];
        tmem_ld32_sync(o_tmem + half * 32, o0);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint4 pq;
          pq.x = pack_bf16x2(__uint_as_float(o0[c * 8 + 0]) * inv, __uint_as_float(o0[c * 8 + 1]) * inv);
          pq.y = pack_bf16x2(__uint_as_float(o0[c * 8 + 2]) * inv, __uint_as_float(o0[c * 8 + 3]) * inv);
          pq.z = pack_bf16x2(__uint_as_float(o0[c * 8 + 4]) * inv, __uint_as_float(o0[c * 8 + 5]) * inv);
          pq.w = pack_bf16x2(__uint_as_float(o0[c * 8 + 6]) * inv, __uint_as_float(o0[c * 8 + 7]) * inv);
          const int cc = half * 4 + c;
          // 128-byte swizzle of the staging tile (16-byte chunk cc of row r at cc ^ (r & 7))
          if (whole) *reinterpret_cast<uint4*>(orow + ((cc ^ sw) << 4)) = pq;
          else if (row_ok) dst[cc] = pq;
        }
      }
      tc_fence_before();
      if (whole) {
        fence_async_smem();
        mbar_arrive(&bars->o_ready);
      }
      if (row_ok && a.lse)
        a.lse[((int64_t)it.b * H + it.h) * n + i] = l_run > 0.f ? (m_ref + __log2f(l_run)) * kLn2 : -INFINITY;
    }
    if (!ok) {
      *abort_flag = 1;
      raise_status(a.status, ATTAMBA_DEV_TIMEOUT);
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
// [rows, H, 64] bf16 viewed as a 3-D tensor; box = 64 x 1 x box_rows with the 128-byte swizzle
bool encode_rows_map(CUtensorMap* m, const void* base, int64_t rows, int H, int box_rows) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)kDH, (cuuint64_t)H, (cuuint64_t)rows};
  cuuint64_t strides[2] = {(cuuint64_t)kDH * 2, (cuuint64_t)H * kDH * 2};
  cuuint32_t box[3] = {(cuuint32_t)kDH, 1, (cuuint32_t)box_rows};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}
}  // namespace

cudaError_t launch_chunk_attn_bf16(const AttnArgs& a, cudaStream_t s) {
  const int64_t T = (int64_t)a.B * a.n;
  CUtensorMap tq, tk, tv, tkc, tvc, to;
  if (!encode_rows_map(&tq, a.q, T, a.H, kBM) || !encode_rows_map(&to, a.O, T, a.H, kBM) ||
      !encode_rows_map(&tk, a.K, T, a.H, kBN) ||
      !encode_rows_map(&tv, a.V, T, a.H, kBN) || !encode_rows_map(&tkc, a.Kc, a.n_chunks, a.H, kBN) ||
      !encode_rows_map(&tvc, a.Vc, a.n_chunks, a.H, kBN))
    return cudaErrorNotSupported;
  cudaError_t e = raise_smem_limit(reinterpret_cast<const void*>(chunk_attn_bf16_kernel), (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  const int sms = device_sm_count();
  // persistent: two CTAs per SM, each walking the work items (sequence, head, 128 queries) round
  // robin; more CTAs only when a CTA would hold more items than its table
  const int64_t items = (int64_t)((a.n + kBM - 1) / kBM) * a.B * a.H;
  int64_t grid = items < (int64_t)kCtasPerSm * sms ? items : (int64_t)kCtasPerSm * sms;
  if ((items + grid - 1) / grid > kMaxItems) grid = (items + kMaxItems - 1) / kMaxItems;
  if (grid > 2147483647) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, chunk_attn_bf16_kernel, tq, tk, tv, tkc, tvc, to, a);
}

cudaError_t launch_chunk_attn_f32(const AttnArgs& a, cudaStream_t s) {
  const int64_t T = (int64_t)a.B * a.n;
  dim3 grid((unsigned)((T + 127) / 128), a.H);
  chunk_attn_f32_kernel<<<grid, 128, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace attamba
