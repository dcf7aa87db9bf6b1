// Query-tile sparse attention on the 5th-generation tensor cores (prefill; D = 128, GQA groups of 8).
//
// "Qwen3.8-Flash-Next architecture" (flozi.net), "Der Weg eines Tokens durch das Modell", item 2:
// after the selection, exact attention runs over only the selected tokens of each query (its top-k
// micro-blocks plus its own block), with 16 query heads over 2 KV heads.
//
// Consecutive queries select overlapping block sets, so a tile of 16 consecutive query rows is
// processed together: the tile attends over the UNION of its rows' blocks, each union block is
// gathered once per tile instead of once per row, and every row masks out the union blocks it did
// not select.  16 rows x the 8 query heads of one KV head are the 128 rows (M) of one tcgen05 MMA.
// The union of 16 rows is 0.38 (32K workload) to 0.46 (128K) of the sum of their lists, so the
// gathered bytes shrink 2.2-2.6x, while the contraction grows to the whole union for every row
// (about 7x the selected pairs at 128K).  The result is the same exact attention: a masked entry
// contributes exp(-inf) = 0, and the softmax runs in fp32 over exactly the selected tokens.
//
// tile_union_kernel (one CTA per tile): every listed block of the 16 rows, and each row's own block,
// sets the row's bit in the block's 16-bit mask in a shared-memory bitmap (windows of 8192 blocks);
// the blocks with a non-zero mask, ascending, are the union, written as (block, row mask) entries
// and as one 128-byte record per chunk of 16 entries (block ids, per-row member bits, per-row own
// slot) for the attention kernel.  Entries outside a row's causal range are skipped and recorded in
// the device status (-1 and the own block are skipped silently); list order does not matter.
//
// sparse_attn_tc_kernel (persistent, one CTA per SM, 512 threads), per (tile, KV head):
//   warps 0-6 producers: warp 0 loads the Q tile (two 128-byte-swizzled TMA boxes of [16 rows]
//            [8 heads][64 d]) and brings each chunk's record into shared memory beside its K/V
//            (one bulk copy); all seven issue the chunk's 64 TMA boxes of [4 tokens][64 d]
//            (block x K/V x half) into a 5-stage ring, each warp a fixed share, with the block ids
//            of the next chunk fetched ahead.  Each box costs its issuing warp ~80 cycles, so one
//            warp caps these 512-byte gathers near 2 TB/s device-wide; seven to eight reach
//            ~10 TB/s (the gather probe);
//   warp 7   MMA issuer (one thread), event-driven: copies the pass's Q tile into TMEM, then
//            S = Q K^T (M 128, N 64 tokens, K 128; Q read from TMEM as the A operand) into one of
//            three S buffers as soon as a chunk and a buffer are ready, and O += P V (P read from
//            TMEM as the A operand, V as an MN-major B operand) as soon as a chunk's P is written;
//            chunks alternate between two O accumulators;
//   warps 8-15 softmax, two groups of four warps (one TMEM lane quadrant each, one thread per row):
//            group g takes every other chunk of a pass and owns O[g]: mask, fp32 online softmax in
//            exp2 form with a lazy rescale of its O (only when the running max grows by more than
//            2^8), P packed to bf16 into the S buffer's columns; the slots that none of a warp's
//            4 query rows attends are skipped (their P is 0).  The epilogue merges the two
//            groups' (m, l) through shared memory and their O accumulators from TMEM, then writes
//            the bf16 rows and the log-sum-exp.
// Register split (setmaxnreg): producers and MMA drop to 64 registers, softmax rises to 192.
// TMEM: S0..S2 at columns 0, 64, 128, the Q tile at 192 (bf16 pairs, copied from shared memory with
// tcgen05.cp at the start of a pass: S reads its A operand from TMEM, which the pipe executes in 32
// cycles per K step at N = 64 against 48 with A in shared memory, where the 6 KB of operands an MMA
// reads bound it), O[0] at 256, O[1] at 384 (fp32, lane = row).  Every wait is bounded; the producer
// and softmax warps suspend while they wait (spinning would take issue slots from the softmax warps
// on their schedulers), the MMA thread polls its barriers with test_wait; a role whose wait runs out
// stops, and every role reaches the final barrier and TMEM release.
#include <algorithm>
#include <mutex>

#include "launch.h"

namespace qsa {
namespace {

constexpr int kTQ = 16;          // query rows per tile
constexpr int kGrp = 8;          // query heads per KV head (the M of a tile is kTQ * kGrp = 128)
constexpr int kD = 128;
constexpr int kCB = 16;          // union blocks per chunk
constexpr int kCT = kCB * 4;     // tokens per chunk (the N of S; S columns per buffer)
constexpr int kQHalf = 128 * 128;         // one 64-column half of the Q tile (128 rows x 128 B)
constexpr int kQBytes = 2 * kQHalf;
constexpr int kKVHalf = kCT * 128;        // one 64-column half of a chunk's K (or V): kCT rows x 128 B
constexpr int kKVBytes = 2 * kKVHalf;     // K (or V) of one chunk
constexpr int kStages = 5;                // K/V ring depth (shared memory)
constexpr int kSBuf = 3;                  // S buffers in TMEM (kCT columns each), then Q and two O accumulators
constexpr int kProdWarps = 7;             // warps issuing the TMA boxes (each box costs its warp ~80 cycles)
constexpr int kMmaWarp = 7;
constexpr int kSoftWarp0 = 8;             // softmax warps 8..15: group (w - 8) / 4 takes every other chunk
constexpr int kSoftWarps = 8;             // of a pass; warp w reads TMEM lane quadrant w % 4
constexpr int kThreads = (kSoftWarp0 + kSoftWarps) * 32;
// Register split (setmaxnreg): the block launches with kLaunchRegs per thread; warpgroups 0-1
// (producers, MMA) drop to kLowRegs and warpgroups 2-3 (softmax) rise to kHighRegs.  The sum must
// not exceed the launch's total, or the increase would wait for ever; the host refuses the launch
// unless the compiled kernel has exactly kLaunchRegs registers per thread.
constexpr int kLaunchRegs = 65536 / kThreads;
constexpr int kLowRegs = 64;
constexpr int kHighRegs = 192;
static_assert(kThreads == 512 && kSoftWarp0 == 8, "two warpgroups per side of the split");
static_assert(256 * kLowRegs + 256 * kHighRegs <= kThreads * kLaunchRegs, "register split");
constexpr int kQCol = kSBuf * kCT;        // TMEM columns of the Q tile (kD / 2 columns of bf16 pairs)
constexpr int kOCol = kQCol + kD / 2;     // TMEM columns of the two O accumulators (128 columns each)
static_assert(kOCol + 2 * kD <= 512, "TMEM columns");
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleLog2 = 8.0f;  // O is rescaled only when the row max grows by more than this

// One chunk of a tile's union, as the union kernel writes it and one bulk copy brings it to shared
// memory beside the chunk's K/V.
struct ChunkInfo {
  int blocks[kCB];        // union block of each slot (past the end of the union: a repeat, masked)
  uint16_t words[kTQ];    // per row: bit j = the row attends slot j
  int8_t oslot[kTQ];      // per row: the slot holding its own block, or -1
  uint8_t pad[16];
};
static_assert(sizeof(ChunkInfo) == 128, "one 128-byte bulk copy per chunk");

constexpr int kInfoOff = kQBytes + kStages * 2 * kKVBytes;
constexpr int kBarOff = kInfoOff + kStages * static_cast<int>(sizeof(ChunkInfo));
constexpr int kXchgOff = kBarOff + 512;   // [4 quadrants][2 groups][2 values][32 lanes] floats
constexpr int kSmem = 1024 + kXchgOff + 4 * 2 * 2 * 32 * 4;
static_assert(kSmem <= 227 * 1024, "shared memory per CTA");

struct TcArgs {
  const ChunkInfo* recs; // [tiles][capc] chunk records per tile of this launch
  const int* cnt;        // [tiles]
  uint16_t* out;
  float* lse;
  long long q_pos0;
  int B, Tq, Hq, Hkv, capc, tile0, ntiles, tpb;
  float scale_log2;
  KernelCtl ctl;
};

__device__ __forceinline__ int tile_chunks(int nu) { return max(1, (nu + kCB - 1) / kCB); }
// The chunks of tile tl (the debug build checks them against the record capacity).
__device__ __forceinline__ int tile_chunks(const TcArgs& a, int tl) {
  const int n = tile_chunks(a.cnt[tl]);
  return QSA_DCHECK(a.ctl, n <= a.capc) ? n : a.capc;
}

// 2^x on the special-function unit (flushes subnormal results to zero; 2^-inf = 0).  The
// probabilities it produces are rounded to bf16 for the P.V product anyway.
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ---------------------------------------------------------------------------- tile unions
constexpr int kUnionThreads = 512;
constexpr int kWin = 8192;                  // blocks per window of the union bitmap (32 KB: two CTAs a SM)
constexpr int kMaxListPerThread = 32;       // 16 rows x k_blocks <= 16384 entries -> 32 per thread

// One CTA per tile.  Every listed block of the tile's rows (and each row's own block) ORs the row's
// bit into the block's 16-bit mask in a shared-memory bitmap; the blocks whose mask is non-zero,
// ascending, are the union.  The block range is walked in windows of kWin blocks.
__global__ void __launch_bounds__(kUnionThreads, 2) tile_union_kernel(const int32_t* __restrict__ idx, int Tq, int kb,
                                                                  long long q_pos0, int tile0, int tpb,
                                                                  uint2* __restrict__ ent, int* __restrict__ cnt,
                                                                  int cap, ChunkInfo* __restrict__ recs, int capc,
                                                                  KernelCtl ctl) {
  extern __shared__ uint32_t umask[];       // [kWin] row masks of the window's blocks
  __shared__ int s_scan[kUnionThreads / 32 + 1];
  __shared__ int s_bad;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int tl = blockIdx.x;
  const int tile = tile0 + tl;
  const int b = tile / tpb, t0 = (tile % tpb) * kTQ;
  const int nrows = min(kTQ, Tq - t0);
  const int nlist = kTQ * kb;
  if (tid == 0) s_bad = 0;
  // this thread's entries, as (block << 4 | row), or ~0 when skipped
  uint32_t key[kMaxListPerThread];
  bool bad = false;
#pragma unroll
  for (int i = 0; i < kMaxListPerThread; ++i) {
    const int e = tid + i * kUnionThreads;
    key[i] = 0xFFFFFFFFu;
    if (e < nlist) {
      const int r = e / kb;
      const int row = t0 + r;
      if (row < Tq) {
        const int x = idx[(static_cast<long long>(b) * Tq + row) * kb + (e - r * kb)];
        const long long own = (q_pos0 + row) >> 2;
        if (x >= 0 && x < own)
          key[i] = (static_cast<uint32_t>(x) << 4) | static_cast<uint32_t>(r);
        else if (x != -1 && x != own)
          bad = true;
      }
    }
  }
  const long long own_first = (q_pos0 + t0) >> 2;
  const long long own_last = (q_pos0 + t0 + nrows - 1) >> 2;
  const int nblk = static_cast<int>(own_last + 1);   // every attended block lies below this
  __syncthreads();
  if (bad) s_bad = 1;
  uint2* te = ent + static_cast<long long>(tl) * cap;
  int total = 0;
  for (int w0 = 0; w0 < nblk; w0 += kWin) {
    const int wn = min(kWin, nblk - w0);
    for (int i = tid; i < wn; i += kUnionThreads) umask[i] = 0u;
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kMaxListPerThread; ++i) {
      const uint32_t x = key[i] >> 4;
      if (key[i] != 0xFFFFFFFFu && x >= static_cast<uint32_t>(w0) && x < static_cast<uint32_t>(w0 + wn))
        atomicOr(&umask[x - w0], 1u << (key[i] & 15u));
    }
    if (tid < nrows) {   // the rows' own blocks
      const long long o = (q_pos0 + t0 + tid) >> 2;
      if (o >= w0 && o < w0 + wn) atomicOr(&umask[o - w0], 1u << tid);
    }
    __syncthreads();
    // ascending compaction: thread tid scans its contiguous slice of the window
    const int per = (wn + kUnionThreads - 1) / kUnionThreads;
    const int i0 = min(wn, tid * per), i1 = min(wn, i0 + per);
    int mine = 0;
    for (int i = i0; i < i1; ++i) mine += umask[i] != 0u;
    int incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) s_scan[w] = incl;
    __syncthreads();
    if (tid == 0) {
      int run = 0;
      for (int q = 0; q < kUnionThreads / 32; ++q) {
        const int v = s_scan[q];
        s_scan[q] = run;
        run += v;
      }
      s_scan[kUnionThreads / 32] = run;
    }
    __syncthreads();
    int u = total + s_scan[w] + incl - mine;
    for (int i = i0; i < i1; ++i) {
      const uint32_t m = umask[i];
      if (m) {
        const uint2 e = make_uint2(static_cast<uint32_t>(w0 + i), m);
        if (QSA_DCHECK(ctl, u < cap)) te[u] = e;
        ++u;
      }
    }
    total += s_scan[kUnionThreads / 32];
    __syncthreads();   // the window is reused
  }
  (void)own_first;
  if (tid == 0) {
    cnt[tl] = total;
    if (s_bad) record_status(ctl, kStBadArg);
  }
  // the chunk records: one warp per chunk of 16 entries, read back from the union this CTA has just
  // written (L2; visible to the CTA's threads after the barrier)
  __syncthreads();
  const int nu = total;
  const int nch = max(1, (nu + kCB - 1) / kCB);
  ChunkInfo* tr = recs + static_cast<long long>(tl) * capc;
  for (int c = w; c < nch; c += kUnionThreads >> 5) {
    const int uu = c * kCB + lane;
    const uint2 e = __ldcg(te + min(uu, max(min(nu, cap) - 1, 0)));
    const uint32_t mask = (lane < kCB && uu < nu) ? e.y : 0u;
    uint32_t myw = 0;
    int myo = -1;
#pragma unroll
    for (int q = 0; q < kTQ; ++q) {
      const uint32_t bq = __ballot_sync(0xffffffffu, (mask >> q) & 1u);
      const uint32_t oq = __ballot_sync(0xffffffffu, ((mask >> q) & 1u) &&
                                                         static_cast<long long>(e.x) == ((q_pos0 + t0 + q) >> 2));
      if (lane == q) {
        myw = bq;
        myo = oq ? __ffs(oq) - 1 : -1;
      }
    }
    ChunkInfo* r = tr + c;
    if (!QSA_DCHECK(ctl, c < capc)) continue;
    if (lane < kCB) r->blocks[lane] = static_cast<int>(e.x);
    if (lane < kTQ) {
      r->words[lane] = static_cast<uint16_t>(myw);
      r->oslot[lane] = static_cast<int8_t>(myo);
    }
  }
}

// ---------------------------------------------------------------------------- attention
struct Bars {
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t s_full[kSBuf], p_full[kSBuf], s_free[kSBuf];
  uint64_t q_full, q_empty, o_full, o_free;
  uint64_t pair[4];      // per TMEM lane quadrant: both groups have posted their (m, l) of the pass
  uint32_t tmem;
};
static_assert(sizeof(Bars) <= 512, "barrier area");

template <int HKV>
__global__ void __launch_bounds__(kThreads, 1)
    sparse_attn_tc_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                          const __grid_constant__ CUtensorMap vmap, TcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* qs = smem;                                   // [2 halves][128 rows][128 B]
  uint8_t* kvs = smem + kQBytes;                        // per stage: K [2 halves][kCT tokens][128 B], V likewise
  ChunkInfo* info = reinterpret_cast<ChunkInfo*>(smem + kInfoOff);
  Bars* bar = reinterpret_cast<Bars*>(smem + kBarOff);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bar->kv_full[s], kProdWarps);   // every producer warp registers its own bytes
      mbar_init(&bar->kv_empty[s], 1);
    }
    for (int i = 0; i < kSBuf; ++i) {
      mbar_init(&bar->s_full[i], 1);
      mbar_init(&bar->p_full[i], kSoftWarps / 2);   // one group writes a chunk's P
      mbar_init(&bar->s_free[i], 1);
    }
    mbar_init(&bar->q_full, 1);
    mbar_init(&bar->q_empty, 1);
    mbar_init(&bar->o_full, 1);
    mbar_init(&bar->o_free, kSoftWarps);
    for (int i = 0; i < 4; ++i) mbar_init(&bar->pair[i], 2);
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&bar->tmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar->tmem;
  const int ntl = a.ntiles;
  if (warp < kSoftWarp0) {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kLowRegs));
  if (warp < kProdWarps) {
    // ------------------------------------------------------------------ producers
    // Every producer warp takes a fixed share of a chunk's 4 * kCB boxes (block x K/V x half), with
    // the block ids fetched one chunk ahead from the chunk records; it registers its own bytes on
    // the stage's full barrier and issues its boxes.  Warp 0 also brings the chunk's record.
    const bool lead = warp == 0;
    if (lead) {
      prefetch_tensormap(&qmap);
      prefetch_tensormap(&kmap);
      prefetch_tensormap(&vmap);
    }
    const int bx = lane * kProdWarps + warp;      // this lane's box of a chunk (none past 4 * kCB)
    const bool has_box = bx < 4 * kCB;
    const int bj = bx >> 2, btv = (bx >> 1) & 1, bhalf = bx & 1;
    const uint32_t nbox = __popc(__ballot_sync(0xffffffffu, has_box));
    const uint32_t my_bytes = nbox * 512 + (lead ? static_cast<uint32_t>(sizeof(ChunkInfo)) : 0u);
    int n = 0, hp = 0;
    bool alive = true;
    for (int it = blockIdx.x; alive && it < ntl; it += gridDim.x) {
      const int tl = ntl - 1 - it;
      const int tile = a.tile0 + tl;
      const int b = tile / a.tpb, t0 = (tile % a.tpb) * kTQ;
      const int nch = tile_chunks(a, tl);
      const ChunkInfo* tr = a.recs + static_cast<long long>(tl) * a.capc;
      for (int g = 0; alive && g < HKV; ++g, ++hp) {
        bool ok = true;
        if (lead && lane == 0) {
          ok = mbar_wait_suspend(&bar->q_empty, (hp & 1) ^ 1u, a.ctl);
          if (ok) {
            mbar_arrive_expect_tx(&bar->q_full, kQBytes);
            tma_load_4d(qs, &qmap, &bar->q_full, 0, g * kGrp, t0, b);
            tma_load_4d(qs + kQHalf, &qmap, &bar->q_full, 64, g * kGrp, t0, b);
          }
        }
        alive = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        int blk_next = has_box ? tr[0].blocks[bj] : 0;   // the first chunk's block of this lane's box
        for (int c = 0; alive && c < nch; ++c, ++n) {
          const int s = n % kStages;
          const unsigned f = static_cast<unsigned>(n / kStages);
          const int blk = blk_next;
          if (c + 1 < nch && has_box) blk_next = tr[c + 1].blocks[bj];   // in flight while this chunk is issued
          ok = true;
          if (lane == 0) {
            ok = mbar_wait_suspend(&bar->kv_empty[s], (f & 1u) ^ 1u, a.ctl);
            if (ok) mbar_arrive_expect_tx(&bar->kv_full[s], my_bytes);   // before this warp's copies
          }
          alive = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
          if (!alive) break;
          if (lead && lane == 0)
            bulk_g2s(&info[s], tr + c, static_cast<unsigned>(sizeof(ChunkInfo)), &bar->kv_full[s]);
          if (has_box) {
            const int blk_ok = QSA_DCHECK(a.ctl, blk >= 0 && 4ll * blk < a.q_pos0 + a.Tq) ? blk : 0;
            uint8_t* dst = kvs + s * 2 * kKVBytes + btv * kKVBytes + bhalf * kKVHalf + bj * 512;
            tma_load_4d(dst, btv ? &vmap : &kmap, &bar->kv_full[s], bhalf * 64, g, blk_ok * 4, b);
          }
        }
      }
    }
    // never leave with a copy in flight: the last fill of each stage (all warps' copies) and the
    // last Q tile
    if (lane == 0) {
      for (int s = 0; s < kStages && s < n; ++s) {
        const int last = s + ((n - 1 - s) / kStages) * kStages;
        mbar_wait_suspend(&bar->kv_full[s], static_cast<unsigned>(last / kStages) & 1u, a.ctl);
      }
      if (lead && hp > 0) mbar_wait_suspend(&bar->q_full, static_cast<unsigned>(hp - 1) & 1u, a.ctl);
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer
    // Within a (tile, head) pass, S(i) and PV(j) are issued as soon as each is ready (S(i): the
    // chunk's K/V and a free S buffer; PV(j): the softmax's P and, for each accumulator's first PV
    // of the pass, both accumulators read out by the previous epilogue), so a PV whose P is ready
    // never waits behind the next chunk's data.  The barriers are polled with test_wait, which
    // never suspends the thread (try_wait may hold it on a barrier that is not about to complete),
    // PV before S: a PV frees an S buffer and its chunk's K/V stage.  Chunk j of a pass accumulates
    // into O[j & 1].
    if (lane == 0) {
      const uint32_t idesc_s = umma_idesc_bf16_f32(128, kCT);
      const uint32_t idesc_pv = umma_idesc_bf16_f32_bmn(128, kD);
      int n0 = 0, hp = 0;   // n0: global index of the pass's first chunk
      bool alive = true;
      for (int it = blockIdx.x; alive && it < ntl; it += gridDim.x) {
        const int tl = ntl - 1 - it;
        const int nch = tile_chunks(a, tl);
        for (int g = 0; alive && g < HKV; ++g, ++hp, n0 += nch) {
          if (!mbar_wait_suspend(&bar->q_full, static_cast<unsigned>(hp) & 1u, a.ctl)) {
            alive = false;
            break;
          }
          // Q into TMEM, one K step (32 bytes of each row) per copy.  The previous pass's S MMAs, the
          // only readers of these columns, are complete: the producer loaded this Q only after they
          // had released the shared-memory copy (q_empty).
          tc_fence_after();
          const uint32_t qbase = smem_u32(qs);
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk)
            tmem_cp_128x256b(tmem + kQCol + kk * 8, sw128_kmajor_desc(qbase + (kk >> 2) * kQHalf) + 2 * (kk & 3));
          int si = 0, pj = 0;   // next S and next PV of the pass
          unsigned long long t_last = globaltimer_ns();
          while (pj < nch) {
            bool progress = false;
            if (pj < si) {
              const int m = n0 + pj, s = m % kStages, sb = m % kSBuf;
              const bool first = pj < 2;   // the accumulator's first PV of the pass
              if (mbar_test_wait(&bar->p_full[sb], static_cast<unsigned>(m / kSBuf) & 1u) &&
                  (!first || hp == 0 || mbar_test_wait(&bar->o_free, static_cast<unsigned>(hp - 1) & 1u))) {
                tc_fence_after();
                const uint32_t vbase = smem_u32(kvs + s * 2 * kKVBytes + kKVBytes);
                const uint32_t o_col = tmem + kOCol + (pj & 1) * kD;
#pragma unroll
                for (int kk = 0; kk < kCT / 16; ++kk) {
                  const uint64_t bd = sw128_mnmajor_desc(vbase + kk * 2048, kKVHalf, 1024);
                  umma_bf16_ta(o_col, tmem + sb * kCT + kk * 8, bd, idesc_pv, (first && kk == 0) ? 0u : 1u);
                }
                umma_commit(&bar->kv_empty[s]);
                umma_commit(&bar->s_free[sb]);
                ++pj;
                progress = true;
              }
            }
            if (si < nch) {
              const int n = n0 + si, s = n % kStages, sb = n % kSBuf;
              if (mbar_test_wait(&bar->kv_full[s], static_cast<unsigned>(n / kStages) & 1u) &&
                  mbar_test_wait(&bar->s_free[sb], (static_cast<unsigned>(n / kSBuf) & 1u) ^ 1u)) {
                tc_fence_after();
                const uint32_t kbase = smem_u32(kvs + s * 2 * kKVBytes);
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk) {
                  const uint64_t bd = sw128_kmajor_desc(kbase + (kk >> 2) * kKVHalf) + 2 * (kk & 3);
                  umma_bf16_ta(tmem + sb * kCT, tmem + kQCol + kk * 8, bd, idesc_s, kk > 0 ? 1u : 0u);
                }
                umma_commit(&bar->s_full[sb]);
                // the Q tile (shared memory and its TMEM copy) is free once the pass's S are done
                if (si == nch - 1) umma_commit(&bar->q_empty);
                ++si;
                progress = true;
              }
            }
            if (progress) {
              t_last = globaltimer_ns();
            } else if (globaltimer_ns() - t_last > a.ctl.wait_ns) {
              record_status(a.ctl, kStTimeout);
              alive = false;
              break;
            }
          }
          // O of this (tile, head) is final once every MMA issued so far is complete.  (The epilogue
          // cannot wait on a per-chunk barrier: the last PVs of a pass may be pending then, and a
          // parity wait cannot tell two phases apart.)
          if (alive) umma_commit(&bar->o_full);
        }
      }
    }
    __syncwarp();
  }
  } else {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kHighRegs));
  {
    // ------------------------------------------------------------------ softmax + epilogue
    // Two groups of four warps (one per TMEM lane quadrant) take alternate chunks of a pass, each
    // with its own running (m, l) and its own O accumulator, so two chunks are in the softmax at
    // once.  At the end of the pass the two states merge by log-sum-exp: each warp of a quadrant
    // pair writes 64 of the 128 output columns.
    const int quad = warp & 3;
    const int grp = (warp - kSoftWarp0) >> 2;
    const int row = quad * 32 + lane;
    const int t = row >> 3, hh = row & 7;
    const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t o_mine = tmem + lane_addr + kOCol + grp * kD;
    float* xchg = reinterpret_cast<float*>(smem + kXchgOff) + quad * 2 * 2 * 32;   // [grp][m, l][lane]
    int n0 = 0, hp = 0;
    bool alive = true;
    for (int it = blockIdx.x; alive && it < ntl; it += gridDim.x) {
      const int tl = ntl - 1 - it;
      const int tile = a.tile0 + tl;
      const int b = tile / a.tpb, t0 = (tile % a.tpb) * kTQ;
      const int nch = tile_chunks(a, tl);
      const bool vrow = t0 + t < a.Tq;
      const long long pos = a.q_pos0 + t0 + t;
      const int lim = static_cast<int>(pos & 3);
      for (int g = 0; alive && g < HKV; ++g, ++hp, n0 += nch) {
        float m_ref = -INFINITY, l = 0.f;
        for (int c = grp; c < nch; c += 2) {
          const int n = n0 + c, s = n % kStages, sb = n % kSBuf;
          if (!mbar_wait_suspend(&bar->s_full[sb], static_cast<unsigned>(n / kSBuf) & 1u, a.ctl) ||
              !mbar_wait_suspend(&bar->kv_full[s], static_cast<unsigned>(n / kStages) & 1u, a.ctl)) {
            alive = false;
            break;
          }
          tc_fence_after();
          // the row's member slots of the chunk and the slot of its own block
          const uint32_t word = vrow ? info[s].words[t] : 0u;
          const int oslot = vrow ? info[s].oslot[t] : -1;
          const uint32_t wor = __reduce_or_sync(0xffffffffu, word);   // slots some row of the warp attends
          const uint32_t s_addr = tmem + lane_addr + sb * kCT;
          uint32_t r[2][32];
          if (wor & 0xFFu) tmem_ld_32x32(s_addr, r[0]);
          if (wor & 0xFF00u) tmem_ld_32x32(s_addr + 32, r[1]);
          tmem_ld_wait();
          // masked raw scores (-inf where the row does not attend) and their maximum.  A slot that no
          // row of the warp attends (its bit clear in wor, the same for all 32 lanes) is skipped here
          // and below: its probabilities are exactly 0.  Within an attended slot, straight-line selects.
          float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
          for (int j = 0; j < kCB; ++j) {
            if (!((wor >> j) & 1u)) continue;
            const bool mem = (word >> j) & 1u;
            const int lj = j == oslot ? lim : 3;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float v = (mem && i <= lj) ? __uint_as_float(r[j >> 3][(j & 7) * 4 + i]) : -INFINITY;
              r[j >> 3][(j & 7) * 4 + i] = __float_as_uint(v);
              m4[i] = fmaxf(m4[i], v);
            }
          }
          const float mraw = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
          const float mx = mraw * a.scale_log2;   // scale > 0: the max of the scaled logits
          bool resc = false;
          float factor = 1.f;
          if (mx > m_ref + kRescaleLog2) {
            if (c >= 2) {   // the group's accumulator holds earlier chunks
              factor = fast_exp2(m_ref - mx);
              l *= factor;
              resc = true;
            }
            m_ref = mx;
          }
          if (__any_sync(0xffffffffu, resc)) {
            // The group's O holds its chunks before c once PV(n-2), its previous chunk, is complete
            // (its commit covers every earlier MMA): s_free of that S buffer.  That barrier's
            // previous phase, PV(n-2-kSBuf), is complete (S(n-2) waited for it), so the parity of
            // PV(n-2)'s phase is unambiguous.
            const int pm = n - 2;
            if (!mbar_wait_suspend(&bar->s_free[pm % kSBuf], static_cast<unsigned>(pm / kSBuf) & 1u, a.ctl)) {
              alive = false;
              break;
            }
            tc_fence_after();
#pragma unroll
            for (int p4 = 0; p4 < 4; ++p4) {
              uint32_t o[32];
              tmem_ld_32x32(o_mine + p4 * 32, o);
              tmem_ld_wait();
#pragma unroll
              for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * factor);
              tmem_st_32x32(o_mine + p4 * 32, o);
            }
            tmem_st_wait();
          }
          const float nref = m_ref == -INFINITY ? 0.f : -m_ref;
          float sum4[4] = {0.f, 0.f, 0.f, 0.f};
          // P of the chunk's kCB slots = bf16 pairs in the S buffer's first kCT / 2 columns
#pragma unroll
          for (int q8 = 0; q8 < 2; ++q8) {
            uint32_t pk[16];
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
              pk[2 * jj] = 0u;
              pk[2 * jj + 1] = 0u;
              if (!((wor >> (q8 * 8 + jj)) & 1u)) continue;
              float p[4];
#pragma unroll
              for (int i = 0; i < 4; ++i) {   // masked entries hold -inf: 2^-inf = 0
                p[i] = fast_exp2(fmaf(__uint_as_float(r[q8][jj * 4 + i]), a.scale_log2, nref));
                sum4[i] += p[i];
              }
              pk[2 * jj] = pack_bf16x2(p[0], p[1]);
              pk[2 * jj + 1] = pack_bf16x2(p[2], p[3]);
            }
            tmem_st_32x16(s_addr + q8 * 16, pk);
          }
          l += (sum4[0] + sum4[1]) + (sum4[2] + sum4[3]);
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar->p_full[sb]);
        }
        if (!alive) break;
        // ---- epilogue of (tile, head): merge the two groups' (m, l, O), O / l -> bf16, lse.
        // The exchange buffer is written once per pass: a warp posts again only after its partner
        // has arrived on o_free below, which it does after reading.
        xchg[(grp * 2 + 0) * 32 + lane] = m_ref;
        xchg[(grp * 2 + 1) * 32 + lane] = l;
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar->pair[quad]);
        if (!mbar_wait_suspend(&bar->pair[quad], static_cast<unsigned>(hp) & 1u, a.ctl) ||
            !mbar_wait_suspend(&bar->o_full, static_cast<unsigned>(hp) & 1u, a.ctl)) {
          alive = false;
          break;
        }
        const float m0 = xchg[0 * 32 + lane], l0 = xchg[1 * 32 + lane];
        const float m1 = xchg[2 * 32 + lane], l1 = xchg[3 * 32 + lane];
        tc_fence_after();
        const float M = fmaxf(m0, m1);
        const float f0 = m0 == -INFINITY ? 0.f : fast_exp2(m0 - M);
        const float f1 = m1 == -INFINITY ? 0.f : fast_exp2(m1 - M);
        const float lt = l0 * f0 + l1 * f1;
        const float inv = lt > 0.f ? 1.f / lt : 0.f;
        const float w0 = f0 * inv, w1 = f1 * inv;
        // an accumulator with no chunk in this pass (nch == 1: group 1) holds stale values: not read
        const bool use1 = nch > 1;
        const long long orow = (static_cast<long long>(b) * a.Tq + t0 + t) * a.Hq + g * kGrp + hh;
        uint4* op = reinterpret_cast<uint4*>(a.out + orow * kD + grp * 64);
        const bool row_ok = vrow && QSA_DCHECK(a.ctl, orow < static_cast<long long>(a.B) * a.Tq * a.Hq);
        const uint32_t oc0 = tmem + lane_addr + kOCol + grp * 64;      // this warp's 64 columns of O[0]
        const uint32_t oc1 = oc0 + kD;                                 // ... and of O[1]
#pragma unroll
        for (int p2 = 0; p2 < 2; ++p2) {
          uint32_t x0[32], x1[32];
          tmem_ld_32x32(oc0 + p2 * 32, x0);
          if (use1) tmem_ld_32x32(oc1 + p2 * 32, x1);
          tmem_ld_wait();
          if (row_ok) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              float v[8];
#pragma unroll
              for (int e = 0; e < 8; ++e)
                v[e] = __uint_as_float(x0[8 * i + e]) * w0 + (use1 ? __uint_as_float(x1[8 * i + e]) * w1 : 0.f);
              op[p2 * 4 + i] = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                                          pack_bf16x2(v[6], v[7]));
            }
          }
        }
        if (grp == 0 && row_ok && a.lse) a.lse[orow] = lt > 0.f ? (M + __log2f(lt)) * kLn2 : -INFINITY;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar->o_free);
      }
    }
  }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------- host side
using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                              const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                              CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn encode_fn() {
  static EncodeFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeFn>(p);
  });
  return fn;
}

// 4-D bf16 map over [d3][d2][d1][128] (innermost 128 elements = one head's row of D) with a
// 128-byte-swizzled box of {64, box1, box2, 1}.  The batch stride spans d2_stride rows of d2 (the
// map may cover only the first d2 of them).
bool make_map4(CUtensorMap* m, const void* base, unsigned long long d1, unsigned long long d2,
               unsigned long long d3, unsigned box1, unsigned box2, unsigned long long d2_stride = 0) {
  EncodeFn fn = encode_fn();
  if (!fn) return false;
  if (d2_stride == 0) d2_stride = d2;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(kD), d1, d2, d3};
  cuuint64_t strides[3] = {kD * 2ull, d1 * kD * 2ull, d2_stride * d1 * kD * 2ull};
  cuuint32_t box[4] = {64, box1, box2, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool attn_tc_supported(int Hq, int Hkv, int D, int k_blocks) {
  return D == kD && (Hkv == 1 || Hkv == 2) && Hq == kGrp * Hkv && k_blocks >= 1 && k_blocks <= 1024;
}

// Per tile: the count, the union entries (16 k + 16 at most) and one record per chunk of 16 entries.
size_t attn_tc_tile_bytes(int k_blocks) {
  return static_cast<size_t>(kTQ * k_blocks + kTQ) * sizeof(uint2) + static_cast<size_t>(k_blocks + 1) * sizeof(ChunkInfo) +
         sizeof(int);
}

cudaError_t launch_attn_prefill_tc(const DeviceInfo* di, const void* q, const void* k, const void* v,
                                   const int32_t* idx, int B, int Tq, int Tk, int Hq, int Hkv, int k_blocks,
                                   long long q_pos0, float scale, void* out, float* lse, void* ws, size_t ws_bytes,
                                   cudaStream_t s) {
  const int tpb = (Tq + kTQ - 1) / kTQ;
  const long long ntiles = static_cast<long long>(B) * tpb;
  const int cap = kTQ * k_blocks + kTQ;
  const int capc = k_blocks + 1;   // chunks of 16 entries
  const size_t per_tile = attn_tc_tile_bytes(k_blocks);
  const long long fit = static_cast<long long>((ws_bytes > 512 ? ws_bytes - 512 : 0) / per_tile);
  if (fit < 1 || ntiles > 0x7fffffffLL) return cudaErrorInvalidValue;
  const int R = static_cast<int>(std::min<long long>(ntiles, fit));
  // layout: cnt[R] (256-byte aligned), ent[R][cap], rec[R][capc] (256-byte aligned)
  int* cnt = static_cast<int*>(ws);
  const size_t ent_off = (static_cast<size_t>(R) * 4 + 255) & ~size_t(255);
  uint2* ent = reinterpret_cast<uint2*>(static_cast<uint8_t*>(ws) + ent_off);
  const size_t rec_off = (ent_off + static_cast<size_t>(R) * cap * sizeof(uint2) + 255) & ~size_t(255);
  ChunkInfo* recs = reinterpret_cast<ChunkInfo*>(static_cast<uint8_t*>(ws) + rec_off);
  // K and V are mapped only up to the call's last query position: a tile's last own block can
  // reach past it, and those rows then read as zeros (masked for every row; a zero times a zero
  // probability keeps the product finite whatever the buffer holds there).
  CUtensorMap qm, km, vm;
  const unsigned long long tk_used = static_cast<unsigned long long>(q_pos0 + Tq);
  if (!make_map4(&qm, q, Hq, Tq, B, kGrp, kTQ) || !make_map4(&km, k, Hkv, tk_used, B, 1, 4, static_cast<unsigned long long>(Tk)) ||
      !make_map4(&vm, v, Hkv, tk_used, B, 1, 4, static_cast<unsigned long long>(Tk)))
    return cudaErrorInvalidValue;
  const size_t usmem = static_cast<size_t>(kWin) * 4;
  if (kTQ * k_blocks > kMaxListPerThread * kUnionThreads) return cudaErrorInvalidValue;
  static std::once_flag once[64];
  std::call_once(once[di->device & 63], [] {
    cudaFuncSetAttribute(tile_union_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kWin * 4);
    cudaFuncSetAttribute(sparse_attn_tc_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    cudaFuncSetAttribute(sparse_attn_tc_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  });

  // the register split inside the kernel needs exactly kLaunchRegs registers per thread at launch
  static int regs_ok[64][2];   // 0 unknown, 1 ok, -1 refused
  int& rk = regs_ok[di->device & 63][Hkv - 1];
  if (rk == 0) {
    cudaFuncAttributes fa{};
    const cudaError_t e = Hkv == 1 ? cudaFuncGetAttributes(&fa, sparse_attn_tc_kernel<1>)
                                   : cudaFuncGetAttributes(&fa, sparse_attn_tc_kernel<2>);
    rk = (e == cudaSuccess && fa.numRegs == kLaunchRegs && fa.maxThreadsPerBlock >= kThreads) ? 1 : -1;
  }
  if (rk != 1) return cudaErrorInvalidConfiguration;
  TcArgs ta{};
  ta.recs = recs;
  ta.cnt = cnt;
  ta.out = static_cast<uint16_t*>(out);
  ta.lse = lse;
  ta.q_pos0 = q_pos0;
  ta.B = B;
  ta.Tq = Tq;
  ta.Hq = Hq;
  ta.Hkv = Hkv;
  ta.capc = capc;
  ta.tpb = tpb;
  ta.scale_log2 = scale * 1.4426950408889634f;
  ta.ctl = kernel_ctl(di);
  for (long long t0 = 0; t0 < ntiles; t0 += R) {
    const int nt = static_cast<int>(std::min<long long>(R, ntiles - t0));
    tile_union_kernel<<<nt, kUnionThreads, usmem, s>>>(idx, Tq, k_blocks, q_pos0, static_cast<int>(t0), tpb, ent, cnt,
                                                       cap, recs, capc, ta.ctl);
    cudaError_t e = cudaPeekAtLastError();
    if (e != cudaSuccess) return e;
    ta.tile0 = static_cast<int>(t0);
    ta.ntiles = nt;
    const int grid = std::min(nt, di->num_sms);
    if (Hkv == 1)
      sparse_attn_tc_kernel<1><<<grid, kThreads, kSmem, s>>>(qm, km, vm, ta);
    else
      sparse_attn_tc_kernel<2><<<grid, kThreads, kSmem, s>>>(qm, km, vm, ta);
    e = cudaPeekAtLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace qsa
