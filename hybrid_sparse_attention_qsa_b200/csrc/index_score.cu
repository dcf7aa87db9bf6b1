// Indexer block scoring.
//
// "Qwen3.8-Flash-Next architecture" (flozi.net), "Der Weg eines Tokens durch das Modell", item 2:
// the micro-block keys are scored with four indexer query heads that share one key head; the
// page notes that the 4x pooling cuts the indexer's prefill work but leaves it dependent on the
// context length.  Score (reading fixed in qsa.h): s(t,b) = sum_h w_h * max(0, qi[t,h] . kp[b]).
//
// Prefill: a dense contraction, run on the 5th-generation tensor cores.
//   D[kp row m][qi row n] = sum_d kp[m][d] * qi[n][d]  with M = 128 pooled keys, N = 256 indexer
//   rows (256/Hi queries x Hi heads), K = Di = 64 (four K=16 steps of tcgen05.mma kind::f16).
//   The pooled keys sit in the M (TMEM lane) dimension, so one thread of the epilogue owns one
//   pooled key and finds the Hi heads of a query in Hi adjacent TMEM columns: the ReLU-sum over
//   heads needs no cross-thread traffic, and 32 lanes write 32 consecutive scores of a query row
//   (one 128-byte store).  Both operands are K-major 128-byte-swizzled TMA boxes.
//   Warp roles: warp 0 = TMA producer (qi tile once, then a 4-stage ring of kp tiles), warp 1 =
//   TMEM allocator + single-thread MMA issuer, warps 2..9 = epilogue (two per TMEM lane quadrant,
//   each taking half of the 256 columns).  Two 256-column fp32 accumulators in TMEM let the
//   epilogue of tile i overlap the MMAs of tile i+1.  The causal bound is per CTA (tiles up to the
//   last query row's visible blocks); the store mask is per query.
// Decode: one query per sequence, so the contraction degenerates to a GEMV over the pooled-key
//   cache; it is HBM-bound: TMA-fed mma.sync tiles with the query heads in the N dimension.
#include <mutex>
#include <type_traits>

#include "pool_math.cuh"

namespace qsa {
namespace {

constexpr int kM = 128;          // pooled keys per tile (UMMA M, TMEM lanes)
constexpr int kN = 256;          // indexer rows per tile (UMMA N)
constexpr int kDi = 64;          // contraction depth (one 128-byte swizzle row)
constexpr int kStages = 4;       // kp ring depth
constexpr int kTilesPerCta = 16; // kp tiles handled by one CTA (split of long rows)
constexpr int kScoreEpiWarps = 16;   // epilogue warps: four per TMEM lane quadrant
constexpr int kScoreThreads = 64 + kScoreEpiWarps * 32;
constexpr int kQiBytes = kN * kDi * 2;   // 32768
constexpr int kKpBytes = kM * kDi * 2;   // 16384
constexpr int kScoreSmem = 1024 + kQiBytes + kStages * kKpBytes + 256 + 16384;  // last term: keep 1 CTA/SM

struct ScoreArgs {
  const float* head_w;
  float* scores;
  long long ld, batch_stride, q_pos0;
  int NBk, blk, mode, b0, row0, rows;
  // Column c of the kp map is pooled block (c << kshift) + koff: 0/0 for the scores themselves, a
  // stride for the sampled scores that set the selection thresholds.
  int kshift, koff;
  KernelCtl ctl;
};

// Columns of a map with stride 1 << kshift and offset koff that lie below nb blocks.
__host__ __device__ __forceinline__ int visible_cols(int nb, int kshift, int koff) {
  return nb > koff ? ((nb - koff - 1) >> kshift) + 1 : 0;
}

// TMA producer (one thread): the qi tile once, then kp tiles t_begin .. t_begin + nt - 1 through the
// ring.  Returns only when no copy it issued is still in flight.
__device__ __forceinline__ void produce_kp_tiles(const CUtensorMap* qi_map, const CUtensorMap* kp_map, uint8_t* qi_s,
                                                 uint8_t* kp_s, uint64_t* qi_full, uint64_t* kp_full,
                                                 uint64_t* kp_empty, int qi_row, int b, int t_begin, int nt,
                                                 const KernelCtl& ctl) {
  prefetch_tensormap(qi_map);
  prefetch_tensormap(kp_map);
  mbar_arrive_expect_tx(qi_full, kQiBytes);
  tma_load_3d(qi_s, qi_map, qi_full, 0, qi_row, b);
  int issued = 0;
  for (int i = 0; i < nt; ++i) {
    const int s = i % kStages;
    const unsigned ph = (i / kStages) & 1u;
    if (!mbar_wait_suspend(&kp_empty[s], ph ^ 1u, ctl)) break;
    mbar_arrive_expect_tx(&kp_full[s], kKpBytes);
    tma_load_3d(kp_s + s * kKpBytes, kp_map, &kp_full[s], 0, (t_begin + i) * kM, b);
    issued = i + 1;
  }
  // Never leave with a copy in flight: wait for the last fill of every stage and the qi tile.
  mbar_wait_suspend(qi_full, 0, ctl);
  for (int s = 0; s < kStages && s < issued; ++s) {
    const int last = s + ((issued - 1 - s) / kStages) * kStages;
    mbar_wait_suspend(&kp_full[s], (last / kStages) & 1u, ctl);
  }
}

// MMA issuer (one thread): tile i accumulates D = kp_tile . qi_tile^T into TMEM columns
// (i & 1) * kN .. + kN, then frees its kp stage and signals the epilogue.
__device__ __forceinline__ void issue_tile_mmas(uint32_t tmem, uint8_t* qi_s, uint8_t* kp_s, uint64_t* qi_full,
                                                uint64_t* kp_full, uint64_t* kp_empty, uint64_t* tm_full,
                                                uint64_t* tm_empty, uint64_t* mma_done, int nt, const KernelCtl& ctl) {
  const uint32_t idesc = umma_idesc_bf16_f32(kM, kN);
  const uint64_t bdesc = sw128_kmajor_desc(smem_u32(qi_s));
  bool ok = mbar_wait_suspend(qi_full, 0, ctl);
  for (int i = 0; ok && i < nt; ++i) {
    const int s = i % kStages;
    const unsigned ph = (i / kStages) & 1u;
    const int acc = i & 1;
    const unsigned aph = (i >> 1) & 1u;
    if (!mbar_wait_suspend(&kp_full[s], ph, ctl)) break;
    if (!mbar_wait_suspend(&tm_empty[acc], aph ^ 1u, ctl)) break;
    tc_fence_after();
    const uint64_t adesc = sw128_kmajor_desc(smem_u32(kp_s + s * kKpBytes));
#pragma unroll
    for (int kk = 0; kk < kDi / 16; ++kk) {
      // +32 bytes of K per step: +2 in the (>> 4) start-address field
      umma_bf16(tmem + acc * kN, adesc + 2 * kk, bdesc + 2 * kk, idesc, kk > 0 ? 1u : 0u);
    }
    umma_commit(&kp_empty[s]);
    umma_commit(&tm_full[acc]);
  }
  umma_commit(mma_done);
  mbar_wait_suspend(mma_done, 0, ctl);
}

template <int HI, int MODE>
__global__ void __launch_bounds__(kScoreThreads, 1)
    score_prefill_kernel(const __grid_constant__ CUtensorMap qi_map, const __grid_constant__ CUtensorMap kp_map,
                         ScoreArgs a) {
  constexpr int QPT = kN / HI;   // queries per tile
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* qi_s = smem;
  uint8_t* kp_s = smem + kQiBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(kp_s + kStages * kKpBytes);
  uint64_t* qi_full = bars;
  uint64_t* kp_full = bars + 1;
  uint64_t* kp_empty = kp_full + kStages;
  uint64_t* tm_full = kp_empty + kStages;
  uint64_t* tm_empty = tm_full + 2;
  uint64_t* mma_done = tm_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bz = blockIdx.z;
  const int b = a.b0 + bz;
  const int r_first = a.row0 + static_cast<int>(blockIdx.x) * QPT;
  const int r_last = min(r_first + QPT, a.row0 + a.rows) - 1;
  const long long pos_last = a.q_pos0 + r_last;
  const int nb_last = visible_cols(static_cast<int>(min(static_cast<long long>(a.NBk), pos_last / a.blk)), a.kshift,
                                   a.koff);
  const int ntiles = (nb_last + kM - 1) / kM;
  const int t_begin = static_cast<int>(blockIdx.y) * kTilesPerCta;
  const int t_end = min(ntiles, t_begin + kTilesPerCta);
  if (t_begin >= t_end) return;   // uniform over the CTA, before any barrier or TMEM use
  const int nt = t_end - t_begin;

  if (threadIdx.x == 0) {
    mbar_init(qi_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&kp_full[s], 1);
      mbar_init(&kp_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tm_full[i], 1);
      mbar_init(&tm_empty[i], kScoreEpiWarps);
    }
    mbar_init(mma_done, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0)
      produce_kp_tiles(&qi_map, &kp_map, qi_s, kp_s, qi_full, kp_full, kp_empty, r_first * HI, b, t_begin, nt, a.ctl);
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0)
      issue_tile_mmas(tmem, qi_s, kp_s, qi_full, kp_full, kp_empty, tm_full, tm_empty, mma_done, nt, a.ctl);
    __syncwarp();
  } else {
    const int ew = warp - 2;                 // 0 .. kScoreEpiWarps - 1
    const int quad = warp & 3;               // TMEM lane quadrant this warp may read
    constexpr int CW = kN / (kScoreEpiWarps / 4);   // columns of this warp: one column group
    const int colbase = (ew >> 2) * CW;
    const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
    float w[HI];
#pragma unroll
    for (int h = 0; h < HI; ++h) w[h] = a.head_w ? a.head_w[h] : 1.0f;
    // Row tl of the tile sits at position pos_first + tl and has (pos_first + tl) >> 2 candidates
    // (blk = 4).  Rows past r_last belong to the next window and are not written.
    const long long pos_first = a.q_pos0 + r_first;
    const int tl_last = r_last - r_first;
    const int nbk = a.NBk;
    const int ksh = a.kshift, kof = a.koff;
    float* srow = a.scores + static_cast<long long>(bz) * a.batch_stride + static_cast<long long>(r_first - a.row0) * a.ld;
    const long long ld = a.ld;
    for (int i = 0; i < nt; ++i) {
      const int acc = i & 1;
      const unsigned aph = (i >> 1) & 1u;
      if (!mbar_wait_suspend(&tm_full[acc], aph, a.ctl)) break;
      tc_fence_after();
      const int kb = (t_begin + i) * kM + quad * 32 + lane;   // pooled key owned by this thread
      float* col = srow + kb;
#pragma unroll
      for (int c = 0; c < CW; c += 32) {
        uint32_t r[32];
        tmem_ld_32x32(tmem + lane_addr + acc * kN + colbase + c, r);
        tmem_ld_wait();
        const int q0 = (colbase + c) / HI;
        // Queries q0 .. q0 + 32/HI - 1 of the tile: when all of them exist and see every pooled key
        // of this warp, the stores need no mask (all tiles below the diagonal band).
        float* dst = col + static_cast<long long>(q0) * ld;
        const bool full =
            q0 + 32 / HI - 1 <= tl_last &&
            (t_begin + i) * kM + quad * 32 + 31 < visible_cols(min(nbk, static_cast<int>((pos_first + q0) >> 2)), ksh, kof);
#pragma unroll
        for (int qq = 0; qq < 32 / HI; ++qq) {
          float acc_s = 0.0f;
#pragma unroll
          for (int h = 0; h < HI; ++h) {
            float x = __uint_as_float(r[qq * HI + h]);
            if (MODE == 0) x = fmaxf(x, 0.0f);
            acc_s = fmaf(w[h], x, acc_s);
          }
          bool ok = full;
          if (!full) {   // warp-uniform
            const int tl = q0 + qq;
            ok = tl <= tl_last && kb < visible_cols(min(nbk, static_cast<int>((pos_first + tl) >> 2)), ksh, kof);
          }
          if (ok) *dst = acc_s;
          dst += ld;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_relaxed(&tm_empty[acc]);   // the tile's TMEM loads are complete
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------------------ score + filter
// Selection without materialised scores.  The same tile pipeline as score_prefill_kernel, one CTA
// per strip of kN/HI queries over ALL their visible pooled keys (strips taken longest first).  The
// epilogue compares each score with its query's threshold tau (set beforehand from sampled scores,
// -inf for rows short enough to keep everything) and appends the survivors (fp32 score bits, block
// index) to the query's candidate list IN INDEX ORDER: the four warps that read the four TMEM
// lane quadrants of a column half exchange their per-query counts of a tile through shared memory,
// so every position is known without atomics.  Only the first `cap` entries of a list are stored;
// the full count is written, so the selection can tell an overflowing list.
constexpr int kFiltEpiWarps = 16;                 // four per TMEM lane quadrant
constexpr int kFiltGroups = kFiltEpiWarps / 4;      // column groups of kN / kFiltGroups columns
constexpr int kFiltThreads = 64 + kFiltEpiWarps * 32;
constexpr int kFiltSmem = 1024 + kQiBytes + kStages * kKpBytes + 256 + 2 * kFiltGroups * 4 * 32 * 4 +
                          kFiltEpiWarps * 32 * 4;

struct FilterArgs {
  const float* head_w;
  const float* tau;     // [rows] threshold of row row0 + i
  uint2* cand;          // [rows][cap] (fp32 score bits, block index)
  int* cnt;             // [rows] number of scores >= tau (may exceed cap)
  long long q_pos0;
  int NBk, b0, row0, rows, cap;
  KernelCtl ctl;
};

// A predicated 8-byte store: no branch around it, so a warp's stores of a query issue as one
// instruction whatever the lanes' predicates.
__device__ __forceinline__ void st_global_v2_if(bool pred, uint2* addr, uint32_t x, uint32_t y) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %0, 0;\n\t"
      "@p st.global.v2.u32 [%1], {%2, %3};\n\t}" ::"r"(static_cast<uint32_t>(pred)),
      "l"(addr), "r"(x), "r"(y)
      : "memory");
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

template <int HI, int MODE>
__global__ void __launch_bounds__(kFiltThreads, 1)
    score_filter_kernel(const __grid_constant__ CUtensorMap qi_map, const __grid_constant__ CUtensorMap kp_map,
                        FilterArgs a) {
  constexpr int QPT = kN / HI;                 // queries per strip
  constexpr int CW = kN / kFiltGroups;         // TMEM columns per epilogue warp
  constexpr int QW = CW / HI;                  // queries per epilogue warp
  constexpr int QC = 32 / HI;                  // queries per 32-column TMEM load
  static_assert(QW <= 32, "one lane per query of a warp");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* qi_s = smem;
  uint8_t* kp_s = smem + kQiBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(kp_s + kStages * kKpBytes);
  uint64_t* qi_full = bars;
  uint64_t* kp_full = bars + 1;
  uint64_t* kp_empty = kp_full + kStages;
  uint64_t* tm_full = kp_empty + kStages;
  uint64_t* tm_empty = tm_full + 2;
  uint64_t* mma_done = tm_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  uint32_t* xcnt = reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(bars) + 256);  // [2][groups][4][32]
  uint32_t* xoff = xcnt + 2 * kFiltGroups * 4 * 32;                                       // [warp][32]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bz = blockIdx.z;
  const int b = a.b0 + bz;
  const int strip = static_cast<int>(gridDim.x - 1 - blockIdx.x);   // longest strips first
  const int r_first = a.row0 + strip * QPT;
  const int r_last = min(r_first + QPT, a.row0 + a.rows) - 1;
  const long long pos_first = a.q_pos0 + r_first;
  const int nb_last = static_cast<int>(min(static_cast<long long>(a.NBk), (a.q_pos0 + r_last) >> 2));
  const int nt = (nb_last + kM - 1) / kM;
  const int tl_last = r_last - r_first;
  const long long list0 = static_cast<long long>(bz) * a.rows + (r_first - a.row0);   // list of the strip's row 0
  if (nt == 0) {   // uniform over the CTA: no visible block, every count is 0
    if (threadIdx.x <= tl_last) a.cnt[list0 + threadIdx.x] = 0;
    return;
  }

  if (threadIdx.x == 0) {
    mbar_init(qi_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&kp_full[s], 1);
      mbar_init(&kp_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tm_full[i], 1);
      mbar_init(&tm_empty[i], kFiltEpiWarps);
    }
    mbar_init(mma_done, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0)
      produce_kp_tiles(&qi_map, &kp_map, qi_s, kp_s, qi_full, kp_full, kp_empty, r_first * HI, b, 0, nt, a.ctl);
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0)
      issue_tile_mmas(tmem, qi_s, kp_s, qi_full, kp_full, kp_empty, tm_full, tm_empty, mma_done, nt, a.ctl);
    __syncwarp();
  } else {
    const int ew = warp - 2;          // 0 .. kFiltEpiWarps - 1
    const int quad = warp & 3;        // TMEM lane quadrant this warp may read
    const int grp = ew >> 2;          // column group: queries grp*QW .. grp*QW + QW - 1
    const int qbase = grp * QW;
    const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t lt = [] {
      uint32_t m;
      asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
      return m;
    }();
    float w[HI];
#pragma unroll
    for (int h = 0; h < HI; ++h) w[h] = a.head_w ? a.head_w[h] : 1.0f;
    // Thresholds of this warp's queries; a query past the strip's last row never passes.
    float tq[QW];
#pragma unroll
    for (int q = 0; q < QW; ++q) tq[q] = qbase + q <= tl_last ? a.tau[list0 + qbase + q] : INFINITY;
    // Slices below the first query's visible blocks need no visibility test when every query exists.
    const int nb_min_full =
        qbase + QW - 1 <= tl_last ? static_cast<int>(min(static_cast<long long>(a.NBk), (pos_first + qbase) >> 2)) : 0;
    uint2* list_q0 = a.cand + (list0 + qbase) * a.cap;   // list of the warp's first query
    uint32_t* my_off = xoff + ew * 32;
    const uint32_t lane_bit = 1u << lane;
    uint32_t run = 0;   // lane q: entries of query qbase + q before the current tile
    bool dead = false;  // a wait timed out: keep meeting the barriers, touch nothing
    for (int i = 0; i < nt; ++i) {
      const int acc = i & 1;
      const unsigned aph = (i >> 1) & 1u;
      if (!dead && !mbar_wait_suspend(&tm_full[acc], aph, a.ctl)) dead = true;
      tc_fence_after();
      const int kb = i * kM + quad * 32 + lane;   // pooled block owned by this thread
      float sc[QW];      // this thread's scores of the warp's queries
      uint32_t m[QW];    // per query: the lanes (blocks) whose score passes (warp-uniform)
      // One pass over the warp's scores of the tile; FULL: every query of the warp exists and sees
      // every block of its slice (tiles below the diagonal band), so no visibility test.
      auto filter_tile = [&](auto full_c) {
        constexpr bool FULL = decltype(full_c)::value;
#pragma unroll
        for (int c = 0; c < CW / 32; ++c) {
          uint32_t r[32];
          tmem_ld_32x32(tmem + lane_addr + acc * kN + grp * CW + c * 32, r);
          tmem_ld_wait();
#pragma unroll
          for (int qq = 0; qq < QC; ++qq) {
            const int q = c * QC + qq;
            float x0 = 0.0f;
#pragma unroll
            for (int h = 0; h < HI; ++h) {
              float x = __uint_as_float(r[qq * HI + h]);
              if (MODE == 0) x = fmaxf(x, 0.0f);
              x0 = fmaf(w[h], x, x0);
            }
            bool pass = x0 >= tq[q];
            if (!FULL)
              pass = pass && qbase + q <= tl_last &&
                     kb < static_cast<int>(min(static_cast<long long>(a.NBk), (pos_first + qbase + q) >> 2));
            sc[q] = x0;
            m[q] = __ballot_sync(0xffffffffu, pass);
          }
        }
      };
      if (!dead) {
        if (i * kM + quad * 32 + 31 < nb_min_full)
          filter_tile(std::integral_constant<bool, true>());
        else
          filter_tile(std::integral_constant<bool, false>());
      } else {
#pragma unroll
        for (int q = 0; q < QW; ++q) {
          sc[q] = 0.0f;
          m[q] = 0u;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_relaxed(&tm_empty[acc]);   // the tile's TMEM loads are complete
      // counts of this tile per (quadrant, query) -> the offset of each query's entries
      uint32_t* xc = xcnt + ((i & 1) * kFiltGroups + grp) * 4 * 32;
      if (lane == 0) {   // this warp's count of each query (the masks are warp-uniform)
#pragma unroll
        for (int q = 0; q < QW; ++q) xc[quad * 32 + q] = static_cast<uint32_t>(__popc(m[q]));
      }
      __syncwarp();
      named_bar_sync(1 + grp, 128);
      if (lane < QW) {
        uint32_t pre = 0, tot = 0;
#pragma unroll
        for (int o = 0; o < 4; ++o) {
          const uint32_t c = xc[o * 32 + lane];
          pre += o < quad ? c : 0u;
          tot += c;
        }
        my_off[lane] = run + pre;   // position of this warp's first entry of query q = lane
        run += tot;
      }
      __syncwarp();
      uint32_t offs[QW];   // every lane: the positions of all the warp's queries (broadcast loads)
#pragma unroll
      for (int q = 0; q < QW; q += 4) {
        const uint4 o4 = *reinterpret_cast<const uint4*>(my_off + q);
        offs[q] = o4.x;
        offs[q + 1] = o4.y;
        offs[q + 2] = o4.z;
        offs[q + 3] = o4.w;
      }
      // each query's passing lanes store (raw score bits, block) to consecutive list positions;
      // branch-free: a store with no passing lane is fully predicated off
#pragma unroll
      for (int q = 0; q < QW; ++q) {
        const uint32_t p = offs[q] + static_cast<uint32_t>(__popc(m[q] & lt));
        const uint32_t e = static_cast<uint32_t>(q) * static_cast<uint32_t>(a.cap) + p;   // < QW * cap
        st_global_v2_if((m[q] & lane_bit) != 0u && p < static_cast<uint32_t>(a.cap), list_q0 + e,
                        __float_as_uint(sc[q]), static_cast<uint32_t>(kb));
      }
      __syncwarp();   // my_off is rewritten by the next tile
    }
    if (quad == 0 && lane < QW && qbase + lane <= tl_last) a.cnt[list0 + qbase + lane] = static_cast<int>(run);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------------------ decode
// One query per sequence: s(b) for the pooled keys of the cache, a GEMV bound by reading 128 bytes
// per block.  A producer warp streams tiles of 128 pooled keys (16 KB, 128-byte swizzle) into a
// 4-stage ring with TMA; four consumer warps take 32 keys each and run mma.m16n8k16 (16 keys x 8
// head columns; the Hi indexer heads fill N, zero past Hi) with the query's B fragments in
// registers and the keys' A fragments from ldmatrix on the swizzled tile (conflict-free).  The four
// lanes of a key row then add their heads with two shuffles.
#ifndef QSA_DEC_STAGES
#define QSA_DEC_STAGES 3
#endif
constexpr int kDecStages = QSA_DEC_STAGES;
constexpr int kDecThreads = 160;
constexpr int kDecSmem = 1024 + kDecStages * kKpBytes + 128;

// With np.ki set, the last warp of each sequence's first CTA first pools that sequence's newest
// block when the new token has just completed it (L a multiple of blk): kp[b][L/blk - 1] from the
// key cache rows (L/blk - 1) * blk .. L - 1, rotated at their first position.  That block is the
// query's own block, never scored here (candidates are the blocks below it), so the pooling needs
// no ordering with this kernel's reads of kp (a tile may read the row only inside its masked tail).
template <int HI>
__global__ void __launch_bounds__(kDecThreads) score_decode_kernel(const __grid_constant__ CUtensorMap kp_map,
                                                                   const uint16_t* __restrict__ qi,
                                                                   const float* __restrict__ head_w,
                                                                   const int32_t* __restrict__ seqlens, int NBk,
                                                                   int blk, int mode, float* __restrict__ scores,
                                                                   long long ld, int part_len, KernelCtl ctl,
                                                                   NewBlockPool np) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + kDecStages * kKpBytes);
  uint64_t* empty = full + kDecStages;
  const int b = blockIdx.y;
  const int L = seqlens[b];
  if (np.ki != nullptr && blockIdx.x == 0 && (threadIdx.x >> 5) == kDecThreads / 32 - 1 && L >= blk &&
      L % blk == 0 && L / blk <= NBk) {
    const long long j = L / blk - 1;
    pool_row_warp(np.ki + b * np.ki_bs + j * blk * kDi, np.kp + b * np.kp_bs + j * kDi, kDi, blk, np.rp,
                  static_cast<double>(j * blk));
  }
  int nb = L >= 1 ? (L - 1) / blk : 0;
  if (L < 1 || nb > NBk) {
    if (blockIdx.x == 0 && threadIdx.x == 0) record_status(ctl, kStBadArg);
    nb = min(max(nb, 0), NBk);
  }
  const int lo = static_cast<int>(blockIdx.x) * part_len;
  const int c = max(0, min(nb, lo + part_len) - lo);
  if (c == 0) return;   // uniform over the CTA
  const int ntiles = (c + kM - 1) / kM;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int st = 0; st < kDecStages; ++st) {
      mbar_init(&full[st], 1);
      mbar_init(&empty[st], 4);
    }
    fence_mbar_init();
  }
  __syncthreads();
  if (warp == 0) {
    if (lane == 0) {
      prefetch_tensormap(&kp_map);
      int issued = 0;
      for (int i = 0; i < ntiles; ++i) {
        const int st = i % kDecStages;
        if (!mbar_wait(&empty[st], ((i / kDecStages) & 1u) ^ 1u, ctl)) break;
        mbar_arrive_expect_tx(&full[st], kKpBytes);
        tma_load_3d(ring + st * kKpBytes, &kp_map, &full[st], 0, lo + i * kM, b);
        issued = i + 1;
      }
      for (int st = 0; st < kDecStages && st < issued; ++st) {   // no copy left in flight
        const int last = st + ((issued - 1 - st) / kDecStages) * kDecStages;
        mbar_wait(&full[st], (last / kDecStages) & 1u, ctl);
      }
    }
    return;
  }
  const int cw = warp - 1;   // consumer 0..3: rows 32 cw .. 32 cw + 31 of each tile
  uint32_t bq[4][2];
  {
    const int n = lane >> 2;
    const uint16_t* qrow = qi + (static_cast<long long>(b) * HI + (n < HI ? n : 0)) * kDi;
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const int d0 = 16 * kk + 2 * (lane & 3);
      bq[kk][0] = n < HI ? __ldg(reinterpret_cast<const uint32_t*>(qrow + d0)) : 0u;
      bq[kk][1] = n < HI ? __ldg(reinterpret_cast<const uint32_t*>(qrow + d0 + 8)) : 0u;
    }
  }
  const int h0 = 2 * (lane & 3);
  const float w0 = (h0 < HI) ? (head_w ? head_w[h0] : 1.f) : 0.f;
  const float w1 = (h0 + 1 < HI) ? (head_w ? head_w[h0 + 1] : 1.f) : 0.f;
  float* srow = scores + static_cast<long long>(b) * ld + lo;
  // ldmatrix.x4 addressing in a 128-byte-swizzled tile: lane l reads row (l & 7) + 8 ((l >> 3) & 1)
  // of a 16-row slab, 16-byte chunk 2 kk + (l >> 4), stored at chunk position (chunk ^ (row & 7)).
  const int lrow = (lane & 7) + 8 * ((lane >> 3) & 1);
  const int lchunk = lane >> 4;
  for (int i = 0; i < ntiles; ++i) {
    const int st = i % kDecStages;
    if (!mbar_wait(&full[st], (i / kDecStages) & 1u, ctl)) return;
    const uint32_t tile = smem_u32(ring + st * kKpBytes);
#pragma unroll
    for (int h = 0; h < 2; ++h) {   // two 16-row slabs per warp
      const int row = 32 * cw + 16 * h + lrow;
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const int chunk = 2 * kk + lchunk;
        uint32_t a0, a1, a2, a3;
        ldsm_x4(tile + row * 128 + ((chunk ^ (row & 7)) << 4), a0, a1, a2, a3);
        mma_bf16_16816(acc, a0, a1, a2, a3, bq[kk][0], bq[kk][1]);
      }
      float x0 = acc[0], x1 = acc[1], x2 = acc[2], x3 = acc[3];
      if (mode == 0) {
        x0 = fmaxf(x0, 0.f);
        x1 = fmaxf(x1, 0.f);
        x2 = fmaxf(x2, 0.f);
        x3 = fmaxf(x3, 0.f);
      }
      float v0 = fmaf(w1, x1, w0 * x0);   // key row lane/4 of the slab: this lane's two head columns
      float v1 = fmaf(w1, x3, w0 * x2);   // key row lane/4 + 8
      v0 += __shfl_xor_sync(0xffffffffu, v0, 1);
      v1 += __shfl_xor_sync(0xffffffffu, v1, 1);
      v0 += __shfl_xor_sync(0xffffffffu, v0, 2);
      v1 += __shfl_xor_sync(0xffffffffu, v1, 2);
      const int r0 = i * kM + 32 * cw + 16 * h + (lane >> 2), r1 = r0 + 8;
      if ((lane & 3) == 0) {
        if (r0 < c) srow[r0] = v0;
        if (r1 < c) srow[r1] = v1;
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);
  }
}

// ------------------------------------------------------------------------------ host helpers
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 3-D bf16 map over [d2][d1][64] rows of 128 bytes (row pitch and batch pitch in bytes) with a
// 128-byte-swizzled box of {64, box_rows, 1}.
bool make_map_pitched(CUtensorMap* m, const void* base, unsigned long long d1, unsigned long long row_pitch,
                      unsigned long long d2, unsigned long long batch_pitch, unsigned box_rows) {
  EncodeTiledFn fn = encode_tiled();
  if (!fn) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(kDi), d1, d2};
  cuuint64_t strides[2] = {row_pitch, batch_pitch};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(kDi), box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}
bool make_map(CUtensorMap* m, const void* base, unsigned long long d1, unsigned long long d2, unsigned box_rows) {
  return make_map_pitched(m, base, d1, kDi * 2ull, d2, d1 * kDi * 2ull, box_rows);
}

template <int HI>
cudaError_t launch_prefill_hi(const void* qi, const void* kp, const float* head_w, int Tq, int NBk, int blk,
                              long long q_pos0, int mode, int b0, int nb, int row0, int rows, float* scores,
                              long long ld, long long batch_stride, int kshift, int koff, const KernelCtl& ctl,
                              cudaStream_t s) {
  static std::once_flag attr_once[64];
  int dev = 0;
  cudaGetDevice(&dev);
  std::call_once(attr_once[dev & 63], [] {
    cudaFuncSetAttribute(score_prefill_kernel<HI, 0>, cudaFuncAttributeMaxDynamicSharedMemorySize, kScoreSmem);
    cudaFuncSetAttribute(score_prefill_kernel<HI, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, kScoreSmem);
  });
  CUtensorMap qmap, kmap;
  // Maps span all batches so the batch index is a TMA coordinate.  With kshift > 0 the kp map
  // walks every (1 << kshift)-th pooled key starting at koff.
  const int Btot = b0 + nb;
  const int ncols = visible_cols(NBk, kshift, koff);
  if (ncols == 0) return cudaSuccess;
  const uint8_t* kbase = static_cast<const uint8_t*>(kp) + static_cast<size_t>(koff) * kDi * 2;
  if (!make_map(&qmap, qi, static_cast<unsigned long long>(Tq) * HI, static_cast<unsigned long long>(Btot), kN) ||
      !make_map_pitched(&kmap, kbase, static_cast<unsigned long long>(ncols), (kDi * 2ull) << kshift,
                        static_cast<unsigned long long>(Btot),
                        Btot == 1 ? std::max<unsigned long long>(static_cast<unsigned long long>(NBk) * kDi * 2,
                                                                 ((kDi * 2ull) << kshift) * ncols)
                                  : static_cast<unsigned long long>(NBk) * kDi * 2,
                        kM))
    return cudaErrorInvalidValue;
  constexpr int QPT = kN / HI;
  const long long pos_last = q_pos0 + row0 + rows - 1;
  const int nb_last = static_cast<int>(std::min<long long>(NBk, pos_last / blk));
  const int ntiles = (visible_cols(nb_last, kshift, koff) + kM - 1) / kM;
  if (ntiles == 0) return cudaSuccess;
  dim3 grid((rows + QPT - 1) / QPT, (ntiles + kTilesPerCta - 1) / kTilesPerCta, nb);
  ScoreArgs a{head_w, scores, ld, batch_stride, q_pos0, NBk, blk, mode, b0, row0, rows, kshift, koff, ctl};
  if (mode == 0)
    score_prefill_kernel<HI, 0><<<grid, kScoreThreads, kScoreSmem, s>>>(qmap, kmap, a);
  else
    score_prefill_kernel<HI, 1><<<grid, kScoreThreads, kScoreSmem, s>>>(qmap, kmap, a);
  return cudaPeekAtLastError();
}

template <int HI>
cudaError_t launch_filter_hi(const void* qi, const void* kp, const float* head_w, int Tq, int NBk, long long q_pos0,
                             int mode, int b0, int nb, int row0, int rows, const float* tau, uint2* cand, int* cnt,
                             int cap, const KernelCtl& ctl, cudaStream_t s) {
  static std::once_flag attr_once[64];
  int dev = 0;
  cudaGetDevice(&dev);
  std::call_once(attr_once[dev & 63], [] {
    cudaFuncSetAttribute(score_filter_kernel<HI, 0>, cudaFuncAttributeMaxDynamicSharedMemorySize, kFiltSmem);
    cudaFuncSetAttribute(score_filter_kernel<HI, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, kFiltSmem);
  });
  CUtensorMap qmap, kmap;
  const int Btot = b0 + nb;
  if (!make_map(&qmap, qi, static_cast<unsigned long long>(Tq) * HI, static_cast<unsigned long long>(Btot), kN) ||
      !make_map(&kmap, kp, static_cast<unsigned long long>(NBk), static_cast<unsigned long long>(Btot), kM))
    return cudaErrorInvalidValue;
  constexpr int QPT = kN / HI;
  dim3 grid((rows + QPT - 1) / QPT, 1, nb);
  FilterArgs a{head_w, tau, cand, cnt, q_pos0, NBk, b0, row0, rows, cap, ctl};
  if (mode == 0)
    score_filter_kernel<HI, 0><<<grid, kFiltThreads, kFiltSmem, s>>>(qmap, kmap, a);
  else
    score_filter_kernel<HI, 1><<<grid, kFiltThreads, kFiltSmem, s>>>(qmap, kmap, a);
  return cudaPeekAtLastError();
}

}  // namespace

cudaError_t launch_score_prefill(const DeviceInfo* di, const void* qi, const void* kp, const float* head_w, int B,
                                 int Tq, int NBk, int Hi, int Di, int blk, long long q_pos0, int mode, int b0, int nb,
                                 int row0, int rows, float* scores, long long ld, long long batch_stride,
                                 cudaStream_t s, int kshift, int koff) {
  (void)B;
  (void)Di;
  if (rows <= 0 || nb <= 0) return cudaSuccess;
  const KernelCtl ctl = kernel_ctl(di);
  switch (Hi) {
    case 1: return launch_prefill_hi<1>(qi, kp, head_w, Tq, NBk, blk, q_pos0, mode, b0, nb, row0, rows, scores, ld, batch_stride, kshift, koff, ctl, s);
    case 2: return launch_prefill_hi<2>(qi, kp, head_w, Tq, NBk, blk, q_pos0, mode, b0, nb, row0, rows, scores, ld, batch_stride, kshift, koff, ctl, s);
    case 4: return launch_prefill_hi<4>(qi, kp, head_w, Tq, NBk, blk, q_pos0, mode, b0, nb, row0, rows, scores, ld, batch_stride, kshift, koff, ctl, s);
    case 8: return launch_prefill_hi<8>(qi, kp, head_w, Tq, NBk, blk, q_pos0, mode, b0, nb, row0, rows, scores, ld, batch_stride, kshift, koff, ctl, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_score_filter(const DeviceInfo* di, const void* qi, const void* kp, const float* head_w, int Tq,
                                int NBk, int Hi, long long q_pos0, int mode, int b0, int nb, int row0, int rows,
                                const float* tau, uint2* cand, int* cnt, int cap, cudaStream_t s) {
  if (rows <= 0 || nb <= 0) return cudaSuccess;
  const KernelCtl ctl = kernel_ctl(di);
  switch (Hi) {
    case 4: return launch_filter_hi<4>(qi, kp, head_w, Tq, NBk, q_pos0, mode, b0, nb, row0, rows, tau, cand, cnt, cap, ctl, s);
    case 8: return launch_filter_hi<8>(qi, kp, head_w, Tq, NBk, q_pos0, mode, b0, nb, row0, rows, tau, cand, cnt, cap, ctl, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_score_decode(const DeviceInfo* di, const void* qi, const void* kp, const float* head_w,
                                const int32_t* seqlens, int B, int NBk, int Hi, int Di, int blk, int mode,
                                float* scores, long long ld, cudaStream_t s, const NewBlockPool* np) {
  (void)Di;
  if (B <= 0 || NBk <= 0) return cudaSuccess;
  const KernelCtl ctl = kernel_ctl(di);
  CUtensorMap kmap;
  if (!make_map(&kmap, kp, static_cast<unsigned long long>(NBk), static_cast<unsigned long long>(B), kM))
    return cudaErrorInvalidValue;
  static std::once_flag once[64];
  std::call_once(once[di->device & 63], [] {
    cudaFuncSetAttribute(score_decode_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, kDecSmem);
    cudaFuncSetAttribute(score_decode_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, kDecSmem);
    cudaFuncSetAttribute(score_decode_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, kDecSmem);
    cudaFuncSetAttribute(score_decode_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, kDecSmem);
  });
  // One wave: as many CTAs as fit on the device at once (a few stragglers in a second wave cost
  // more than the whole wave's tail), split evenly over the sequences; parts are whole tiles.
  static int occ[64][4];
  static std::once_flag occ_once[64];
  std::call_once(occ_once[di->device & 63], [di] {
    auto* o = occ[di->device & 63];
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o[0], score_decode_kernel<1>, kDecThreads, kDecSmem);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o[1], score_decode_kernel<2>, kDecThreads, kDecSmem);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o[2], score_decode_kernel<4>, kDecThreads, kDecSmem);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o[3], score_decode_kernel<8>, kDecThreads, kDecSmem);
  });
  const int hslot = Hi == 1 ? 0 : Hi == 2 ? 1 : Hi == 4 ? 2 : 3;
  const int slots = std::max(1, occ[di->device & 63][hslot]) * di->num_sms;
  const int want = std::max(1, slots / B);
  const int tiles = (NBk + kM - 1) / kM;
  const int part_tiles = std::max(1, (tiles + want - 1) / want);
  const int part_len = part_tiles * kM;
  dim3 grid((NBk + part_len - 1) / part_len, B);
  const uint16_t* q = static_cast<const uint16_t*>(qi);
  const NewBlockPool pool = np ? *np : NewBlockPool{};
  switch (Hi) {
    case 1: score_decode_kernel<1><<<grid, kDecThreads, kDecSmem, s>>>(kmap, q, head_w, seqlens, NBk, blk, mode, scores, ld, part_len, ctl, pool); break;
    case 2: score_decode_kernel<2><<<grid, kDecThreads, kDecSmem, s>>>(kmap, q, head_w, seqlens, NBk, blk, mode, scores, ld, part_len, ctl, pool); break;
    case 4: score_decode_kernel<4><<<grid, kDecThreads, kDecSmem, s>>>(kmap, q, head_w, seqlens, NBk, blk, mode, scores, ld, part_len, ctl, pool); break;
    case 8: score_decode_kernel<8><<<grid, kDecThreads, kDecSmem, s>>>(kmap, q, head_w, seqlens, NBk, blk, mode, scores, ld, part_len, ctl, pool); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaPeekAtLastError();
}

}  // namespace qsa
