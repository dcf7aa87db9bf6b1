// Gather-sparse attention over the selected micro-blocks (prefill and split-KV decode).
//
// "Qwen3.8-Flash-Next architecture" (flozi.net), "Der Weg eines Tokens durch das Modell", item 2:
// after the selection, exact attention runs over only the selected tokens, with grouped query
// heads sharing KV heads.  For query position p and head h (KV head g = h / (Hq/Hkv)):
//   o = sum_{j in S} softmax_j(scale * q . k_j) v_j,  S = tokens of the listed blocks plus the own
//   block's tokens blk*floor(p/blk) .. p.
//
// Design (B200, HBM/L2-bound: ~8 flop per gathered byte):
//   * One work item = one query row (prefill) or one range of a sequence's index list (decode
//     split).  Persistent CTAs walk the items; a producer warp streams the selected blocks of
//     successive items through a 3-stage shared-memory ring without draining between items.
//   * A block of 4 tokens is one contiguous 4*Hkv*D*2-byte run of K (and of V) in the [T][Hkv][D]
//     layout, so each block is one 1-D bulk copy (cp.async.bulk, TMA engine) for K and one for V.
//     With K and V interleaved by block (KVI: [B][ceil(T/4)][K, V][4][Hkv][D], written by
//     interleave_kv_kernel) a block's K and V are one copy of twice the size, which the TMA engine
//     delivers at a higher rate.  A stage holds 16 blocks.  The smem pitch of a block slot is its
//     size + 16 bytes, so the same token row of 8 consecutive slots falls in 8 different 16-byte
//     bank groups: ldmatrix on "token j of slots 0..7" is conflict-free.
//   * Eight warps issue the copies (a leader that walks the index lists and publishes each stage's
//     slot map, and seven helpers): the per-SM bulk-copy rate grows with the issuing warps.  With
//     two KV heads the block has 512 threads and a setmaxnreg split (issuers 64 registers,
//     consumers 192).
//   * Consumer warp (g, j) owns KV head g and token j of every block: its 16 rows per stage are
//     token j of the 16 slots.  Scores are computed transposed, S^T[token][head] = K_g Q_g^T, with
//     mma.m16n8k16 (M = 16 tokens, N = 8 query heads of the group, K = D), so the 8 heads of a GQA
//     group fill N exactly.  The fp32 online softmax runs per head column (exp2 form); P^T is
//     transposed in registers (movmatrix) into the B operand of O^T[d][head] += V^T P^T.
//   * The 4 warps of a KV head hold partial softmax states over disjoint token sets; they are
//     merged through shared memory at the end of an item (log-sum-exp merge), then the output row
//     is staged in shared memory and written with 16-byte stores.
//   * Decode: each (sequence, split) is an item writing an unnormalised partial (o, m, l); a
//     small kernel merges the splits.  With one split the item writes the final row directly.
// Entries -1 and the own block in an index list are skipped; other entries outside [0, own) are
// skipped and recorded in the device status word.  Every mbarrier wait is bounded.
#include <algorithm>
#include <atomic>
#include <cfloat>
#include <mutex>

#include "launch.h"

namespace qsa {
namespace {

constexpr int kSlots = 16;
constexpr int kStages = 3;
constexpr int kSeg = 512;          // index-list entries staged in shared memory per buffer
constexpr int kIssuers_ = 4;       // warps that issue a stage's bulk copies in the wide kernel (the D = 128 kernel: 8)
constexpr int kD = 128;
constexpr int kBlk = 4;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Published by the leading producer warp for every stage it fills (and read by the helper
// producer warps and the consumers).  nslots == -1 tells the helpers that no stage follows.
struct StageInfo {
  int nslots;
  int last;
  const uint16_t* kbase;
  const uint16_t* vbase;
  int tok0[kSlots];
  uint8_t ntok[kSlots];
};

// Shared-memory ring of the copy pipeline: per stage SLOTS block slots of K, then SLOTS of V.  A
// block of 4 tokens of all KV heads is one contiguous run of kBlockBytes in the [T][Hkv][D] layout.
// KVI: K and V interleaved by block in memory ([B][ceil(T/4)][K, V][4][Hkv][D]), so a block's K
// and V are one contiguous run of 2 * kBlockBytes, fetched by one copy into a slot that holds the
// block's K followed by its V.
template <int HKV, int D, int SLOTS, int ISS = kIssuers_, bool KVI = false>
struct Ring {
  static_assert(SLOTS % ISS == 0 && SLOTS <= 16, "slots per issuer warp");
  static constexpr bool kKVI = KVI;
  static constexpr int kSlots = SLOTS;
  static constexpr int kTokBytes = HKV * D * 2;               // one token of K (or V), all KV heads
  static constexpr int kBlockBytes = kBlk * kTokBytes;        // one block of K (or of V)
  // +16: the same token row of consecutive slots falls in different 16-byte bank groups
  static constexpr int kPitch = (KVI ? 2 * kBlockBytes : kBlockBytes) + 16;
  static constexpr int kVOff = KVI ? kBlockBytes : SLOTS * kPitch;   // from a slot's K to its V
  static constexpr int kStageBytes = KVI ? SLOTS * kPitch : 2 * SLOTS * kPitch;
  static constexpr int kInfoStride = (sizeof(StageInfo) + 15) / 16 * 16;
};

template <int HKV, bool KVI = false>
struct Cfg {
  static constexpr int kBlockBytes = kBlk * HKV * kD * 2;     // one block of K (or of V)
  static constexpr int kPitch = (KVI ? 2 * kBlockBytes : kBlockBytes) + 16;
  static constexpr int kVOff = KVI ? kBlockBytes : kSlots * kPitch;
  static constexpr int kStageBytes = KVI ? kSlots * kPitch : 2 * kSlots * kPitch;
  static constexpr int kConsumerWarps = kBlk * HKV;
  // 8 issuing warps: the per-SM rate of 1-D bulk copies grows with the warps issuing them (the
  // gather probe: 12.5 TB/s from L2 with 4 warps, 13.9 with 8, same ring)
  static constexpr int kIssuers = 8;
  static constexpr int kThreads = (kConsumerWarps + kIssuers) * 32;
  // With 512 threads a thread launches with 128 registers; the issuer warpgroups give registers to
  // the consumer warpgroups (setmaxnreg): 256 x kLowRegs + 256 x kHighRegs = 512 x 128.
  static constexpr bool kRegSplit = kThreads == 512;
  static constexpr int kLowRegs = 64, kHighRegs = 192;
  static_assert(!kRegSplit || kConsumerWarps * 32 * kHighRegs + kIssuers * 32 * kLowRegs <= 65536, "register split");
  static constexpr int kMergeSlot = 32 * 32 * 4 + 32 * 4 * 4; // o fragments + (m0, m1, l0, l1) per lane
  static constexpr int kMergeBytes = 3 * HKV * kMergeSlot;
  static constexpr int kInfoBytes = kStages * ((sizeof(StageInfo) + 15) / 16 * 16);
  static constexpr int kBarBytes = (3 * kStages + 2 * HKV) * 8;
  static constexpr int kPendBytes = 64 * 4;
  static constexpr int kIdxBytes = 2 * kSeg * 4;              // double-buffered index-list segments
  static constexpr int kSmem =
      128 + kStages * kStageBytes + kMergeBytes + kInfoBytes + kBarBytes + kPendBytes + kIdxBytes;
};


struct AttnArgs {
  const uint16_t* q;
  const uint16_t* k;
  const uint16_t* v;
  const int32_t* idx;
  const uint16_t* kv;       // K and V interleaved by block (KVI kernels), else unused
  const int32_t* seqlens;   // decode when non-null
  uint16_t* out;
  float* lse;
  float* part;              // decode partials [items][Hq][D + 2]
  long long q_pos0;
  int B, Tq, Tk, Hq, kblocks, splits, num_items;
  int cluster;              // decode: the splits of a sequence form a thread-block cluster (1 item per CTA)
  float scale_log2;
  KernelCtl ctl;
};

#ifdef QSA_DEBUG
// Rows of out / lse the launch writes (prefill: B * Tq; decode: B); the decode partials have one
// row per item.
__device__ __forceinline__ long long out_rows(const AttnArgs& a) {
  return a.seqlens ? static_cast<long long>(a.B) : static_cast<long long>(a.B) * a.Tq;
}
#endif

struct Item {
  const uint16_t* kbase;
  const uint16_t* vbase;
  const int32_t* idx_row;
  long long pos;
  long long qrow;      // row of q ([B*Tq] or [B])
  long long orow;      // row of out / lse / part
  int lo, hi;
  bool diag, ok, partial;
};

template <int HKV, int D = kD>
__device__ __forceinline__ Item make_item(const AttnArgs& a, int i) {
  Item it;
  if (a.seqlens == nullptr) {
    const int t = a.Tq - 1 - i / a.B;   // longest rows first
    const int b = i % a.B;
    it.qrow = static_cast<long long>(b) * a.Tq + t;
    it.orow = it.qrow;
    it.pos = a.q_pos0 + t;
    if (a.kv) {   // interleaved: blocks of [K 4 tokens][V 4 tokens]
      const long long nblk = (a.Tk + kBlk - 1) / kBlk;
      it.kbase = a.kv + static_cast<long long>(b) * nblk * 2 * kBlk * HKV * D;
      it.vbase = it.kbase + kBlk * HKV * D;
    } else {
      it.kbase = a.k + static_cast<long long>(b) * a.Tk * HKV * D;
      it.vbase = a.v + static_cast<long long>(b) * a.Tk * HKV * D;
    }
    it.idx_row = a.idx + it.qrow * a.kblocks;
    it.lo = 0;
    it.hi = a.kblocks;
    it.diag = true;
    it.ok = true;
    it.partial = false;
  } else {
    const int b = i / a.splits, sp = i % a.splits;
    const int L = a.seqlens[b];
    it.ok = L >= 1 && L <= a.Tk;
    it.pos = static_cast<long long>(L) - 1;
    it.qrow = b;
    it.orow = a.splits > 1 ? i : b;
    it.kbase = a.k + static_cast<long long>(b) * a.Tk * HKV * D;
    it.vbase = a.v + static_cast<long long>(b) * a.Tk * HKV * D;
    it.idx_row = a.idx + static_cast<long long>(b) * a.kblocks;
    const int chunk = (a.kblocks + a.splits - 1) / a.splits;
    it.lo = min(a.kblocks, sp * chunk);
    it.hi = min(a.kblocks, it.lo + chunk);
    it.diag = sp == 0;
    it.partial = a.splits > 1;
  }
  return it;
}

// Copies of one slot: the block's K and V rows [tok0, tok0 + ntok) into kd and vd.  KVI: kbase is the
// interleaved block array (vbase = kbase + one block of K); a whole block is one copy of its K and V.
template <class R, int HKV, int D>
__device__ __forceinline__ void copy_slot(uint8_t* kd, uint8_t* vd, const uint16_t* kbase, const uint16_t* vbase,
                                          long long tok0, int ntok, uint64_t* bar) {
  const uint32_t bytes = static_cast<uint32_t>(ntok) * R::kTokBytes;
  if constexpr (R::kKVI) {
    const uint16_t* src = kbase + (tok0 / kBlk) * (2 * kBlk * HKV * D);
    if (ntok == kBlk) {
      bulk_g2s(kd, src, 2 * bytes, bar);
    } else {
      bulk_g2s(kd, src, bytes, bar);
      bulk_g2s(vd, src + kBlk * HKV * D, bytes, bar);
    }
  } else {
    bulk_g2s(kd, kbase + tok0 * HKV * D, bytes, bar);
    bulk_g2s(vd, vbase + tok0 * HKV * D, bytes, bar);
  }
}

// Helper issuer warp h (1 .. ISS - 1): issues slots h, h + ISS, ... of every stage the
// leading producer publishes, until it publishes nslots == -1.
template <int HKV, int D, int SLOTS, int ISS = kIssuers_, bool KVI = false>
__device__ __forceinline__ void attn_helper(const AttnArgs& a, int h, uint8_t* ring, uint8_t* info, uint64_t* full,
                                            uint64_t* ready) {
  using R = Ring<HKV, D, SLOTS, ISS, KVI>;
  const int lane = threadIdx.x & 31;
  auto info_at = [&](int s) { return reinterpret_cast<const StageInfo*>(info + s * R::kInfoStride); };
  // ------------------------------------------------------------------ helper issuer warps
  // The per-SM rate of 1-D bulk copies grows with the number of warps issuing them, so the
  // copies of a stage are spread over kIssuers warps: helper h issues slots h, h + kIssuers, ...
  int st = 0;
  unsigned ph = 0;
  const uint32_t tok_bytes = R::kTokBytes;
  for (;;) {
    if (!mbar_wait(&ready[st], ph, a.ctl)) break;
    const StageInfo* inf = info_at(st);
    const int n = inf->nslots;
    if (n < 0) break;
    const int slot = h + ISS * lane;
    if (lane < R::kSlots / ISS && slot < n) {
      const int ntok = inf->ntok[slot];
      const long long tok0 = inf->tok0[slot];
      uint8_t* kd = ring + st * R::kStageBytes + slot * R::kPitch;
      uint8_t* vd = kd + R::kVOff;
      if (QSA_DCHECK(a.ctl, tok0 >= 0 && ntok <= kBlk && tok0 + ntok <= a.Tk)) {
        copy_slot<R, HKV, D>(kd, vd, inf->kbase, inf->vbase, tok0, ntok, &full[st]);
      } else {
        mbar_complete_tx(&full[st], 2u * ntok * tok_bytes);
      }
    }
    __syncwarp();
    if (++st == kStages) {
      st = 0;
      ph ^= 1u;
    }
  }
}

// Asynchronous copy of index-list segment `seg` of work item `item` into idxbuf[buf], one
// committed cp.async group (issued by one warp; an empty group past the last item).
template <int HKV, int D>
__device__ __forceinline__ void attn_fetch_list(const AttnArgs& a, int item, int seg, int* idxbuf, int buf) {
  const int lane = threadIdx.x & 31;
  if (item < a.num_items) {
    const Item f = make_item<HKV, D>(a, item);
    const int base = f.lo + seg * kSeg;
    const int len = max(0, min(kSeg, f.hi - base));
    for (int e = lane; e < len; e += 32) cp_async4(&idxbuf[buf * kSeg + e], f.idx_row + base + e);
  }
  cp_async_commit();
}

// Leading producer warp: walks the work items, turns each index list into block copies (the
// query's own block last), publishes each stage's slot list for the helpers and issues its own
// share of the copies.  Returns only when no copy it registered is still in flight.  With
// `prefetched` the first segment of the CTA's first item is already on its way (attn_fetch_list).
template <int HKV, int D, int SLOTS, int ISS = kIssuers_, bool KVI = false>
__device__ __forceinline__ void attn_producer(const AttnArgs& a, uint8_t* ring, uint8_t* info, uint64_t* full,
                                              uint64_t* empty, uint64_t* ready, int* pend, int* idxbuf,
                                              bool prefetched = false) {
  using R = Ring<HKV, D, SLOTS, ISS, KVI>;
  const int lane = threadIdx.x & 31;
  auto info_at = [&](int s) { return reinterpret_cast<StageInfo*>(info + s * R::kInfoStride); };
  // ------------------------------------------------------------------ leading producer warp
  int st = 0;
  unsigned ph = 0;
  int fills = 0;
  bool alive = true;
  const uint32_t tok_bytes = R::kTokBytes;
  auto flush = [&](int n, bool last, const Item& it) -> bool {
    if (!mbar_wait(&empty[st], ph ^ 1u, a.ctl)) return false;
    int packed = lane < n ? pend[lane] : 0;
    const int ntok = packed & 7;
    const long long tok0 = packed >> 3;
    StageInfo* inf = info_at(st);
    if (lane < R::kSlots) {
      inf->ntok[lane] = static_cast<uint8_t>(lane < n ? ntok : 0);
      inf->tok0[lane] = static_cast<int>(tok0);
    }
    if (lane == 0) {
      inf->nslots = n;
      inf->last = last ? 1 : 0;
      inf->kbase = it.kbase;
      inf->vbase = it.vbase;
    }
    const uint32_t mine = lane < n ? 2u * ntok * tok_bytes : 0u;
    const uint32_t total = __reduce_add_sync(0xffffffffu, mine);
    __syncwarp();
    if (lane == 0) {
      mbar_arrive_expect_tx(&full[st], total);   // registered before any helper can issue a copy
      mbar_arrive(&ready[st]);
    }
    __syncwarp();
    if (lane < n && lane % ISS == 0) {
      uint8_t* kd = ring + st * R::kStageBytes + lane * R::kPitch;
      uint8_t* vd = kd + R::kVOff;
      if (QSA_DCHECK(a.ctl, tok0 >= 0 && ntok <= kBlk && tok0 + ntok <= a.Tk)) {
        copy_slot<R, HKV, D>(kd, vd, it.kbase, it.vbase, tok0, ntok, &full[st]);
      } else {
        mbar_complete_tx(&full[st], 2u * ntok * tok_bytes);
      }
    }
    // drop the flushed entries from the pending list
    int rest0 = n + lane < 64 ? pend[n + lane] : 0;
    int rest1 = n + lane + 32 < 64 ? pend[n + lane + 32] : 0;
    __syncwarp();
    pend[lane] = rest0;
    if (lane + 32 < 64) pend[lane + 32] = rest1;
    __syncwarp();
    ++fills;
    if (++st == kStages) {
      st = 0;
      ph ^= 1u;
    }
    return true;
  };
  // The index list of an item is staged in shared memory by asynchronous copies one segment
  // ahead (the next segment of this item or the first of the next item), so the copy ring never
  // waits on a global load of the list.
  auto fetch = [&](int item, int seg, int buf) { attn_fetch_list<HKV, D>(a, item, seg, idxbuf, buf); };
  int buf = 0;
  if (!prefetched) fetch(blockIdx.x, 0, 0);
  for (int item = blockIdx.x; alive && item < a.num_items; item += gridDim.x) {
    const Item it = make_item<HKV, D>(a, item);
    const long long own = it.pos >= 0 ? it.pos / kBlk : 0;
    int npend = 0;
    const int nseg = max(1, (it.hi - it.lo + kSeg - 1) / kSeg);
    for (int seg = 0; seg < nseg; ++seg) {
      if (seg + 1 < nseg)
        fetch(item, seg + 1, buf ^ 1);
      else
        fetch(item + gridDim.x, 0, buf ^ 1);
      cp_async_wait<1>();
      __syncwarp();
      const int len = max(0, min(kSeg, it.hi - (it.lo + seg * kSeg)));
      if (it.ok) {
        for (int c = 0; alive && c < len; c += 32) {
          const int e = c + lane < len ? idxbuf[buf * kSeg + c + lane] : -1;
          const bool valid = e >= 0 && e < own;
          if (!valid && e != -1 && e != own) record_status(a.ctl, kStBadArg);
          const unsigned m = __ballot_sync(0xffffffffu, valid);
          if (valid) pend[npend + __popc(m & ((1u << lane) - 1u))] = (e * kBlk) << 3 | kBlk;
          npend += __popc(m);
          __syncwarp();
          while (alive && npend > R::kSlots) {
            alive = flush(R::kSlots, false, it);
            npend -= R::kSlots;
          }
        }
      }
      __syncwarp();
      buf ^= 1;
    }
    if (it.ok) {
      if (it.diag) {
        if (lane == 0) pend[npend] = static_cast<int>((own * kBlk) << 3) | static_cast<int>(it.pos - own * kBlk + 1);
        ++npend;
        __syncwarp();
      }
    } else if (lane == 0) {
      record_status(a.ctl, kStBadArg);
    }
    while (alive && npend > R::kSlots) {
      alive = flush(R::kSlots, false, it);
      npend -= R::kSlots;
    }
    if (alive) alive = flush(npend, true, it);
  }
  cp_async_wait<0>();
  // Tell the helpers that no stage follows (the stage is free once every consumer released it).
  if (alive && mbar_wait(&empty[st], ph ^ 1u, a.ctl)) {
    if (lane == 0) {
      info_at(st)->nslots = -1;
      mbar_arrive(&ready[st]);
    }
    __syncwarp();
  }
  // Never leave with a copy in flight: wait for the last fill of every stage.
  for (int s = 0; s < kStages && s < fills; ++s) {
    const int last = s + ((fills - 1 - s) / kStages) * kStages;
    mbar_wait(&full[s], (last / kStages) & 1u, a.ctl);
  }
}

// CL: decode with the splits of a sequence merged inside its thread-block cluster (a separate
// instantiation, so that the prefill and split-partials code is compiled without it; there the
// label of the cluster tail has no jump to it).
#pragma nv_diag_suppress 177
template <int HKV, bool CL = false, bool KVI = false>
__global__ void __launch_bounds__(Cfg<HKV, KVI>::kThreads, 1) sparse_attn_kernel(AttnArgs a) {
  using C = Cfg<HKV, KVI>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  uint8_t* ring = smem;
  uint8_t* merge = ring + kStages * C::kStageBytes;
  StageInfo* info = reinterpret_cast<StageInfo*>(merge + C::kMergeBytes);
  constexpr int kInfoStride = (sizeof(StageInfo) + 15) / 16 * 16;
  auto info_at = [&](int s) { return reinterpret_cast<StageInfo*>(reinterpret_cast<uint8_t*>(info) + s * kInfoStride); };
  uint64_t* full = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(info) + C::kInfoBytes);
  uint64_t* empty = full + kStages;
  uint64_t* ready = empty + kStages;    // per stage: slot list published for the helper issuers
  uint64_t* mfull = ready + kStages;    // per KV head: the 3 partner warps have written their state
  uint64_t* mempty = mfull + HKV;       // per KV head: warp j=0 has consumed the merge slots
  int* pend = reinterpret_cast<int*>(mempty + HKV);
  int* idxbuf = pend + 64;              // [2][kSeg]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int group = a.Hq / HKV;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], C::kConsumerWarps);
      mbar_init(&ready[s], 1);
    }
    for (int g = 0; g < HKV; ++g) {
      mbar_init(&mfull[g], kBlk - 1);
      mbar_init(&mempty[g], 1);
    }
    fence_mbar_init();
  }
  // The producer starts fetching its first index-list segment while the ring is zeroed.
  if (warp == C::kConsumerWarps) attn_fetch_list<HKV, kD>(a, blockIdx.x, 0, idxbuf, 0);
  // Zero the V slots once so that unused slot rows are finite (their probabilities are 0, but
  // 0 * NaN = NaN).  Unused K rows need no zeroing: their scores are replaced by -inf (a select,
  // no arithmetic on them).
  constexpr int kVChunks = C::kBlockBytes / 16;   // 16-byte chunks of one slot's V block
  for (int i = threadIdx.x; i < kStages * kSlots * kVChunks; i += blockDim.x) {
    const int s = i / (kSlots * kVChunks), r = i - s * (kSlots * kVChunks), slot = r / kVChunks;
    reinterpret_cast<uint4*>(ring + s * C::kStageBytes + slot * C::kPitch + C::kVOff)[r - slot * kVChunks] =
        make_uint4(0, 0, 0, 0);
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // order these writes before the bulk copies
  __syncthreads();

  // In cluster mode every warp of every CTA passes the two cluster barriers of the split merge
  // exactly once (the consumer warps that merge inside their epilogue, the others here).
  if (warp >= C::kConsumerWarps) {
    if constexpr (C::kRegSplit) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::kLowRegs));
    if (warp > C::kConsumerWarps)
      attn_helper<HKV, kD, kSlots, C::kIssuers, KVI>(a, warp - C::kConsumerWarps, ring,
                                                     reinterpret_cast<uint8_t*>(info), full, ready);
    else
      attn_producer<HKV, kD, kSlots, C::kIssuers, KVI>(a, ring, reinterpret_cast<uint8_t*>(info), full, empty, ready,
                                                       pend, idxbuf, true);
    if constexpr (CL) {
      cluster_sync_all();
      cluster_sync_all();
    }
  } else {
  if constexpr (C::kRegSplit) asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::kHighRegs));

  // -------------------------------------------------------------------- consumer warps
  const int g = warp / kBlk;       // KV head
  const int j = warp % kBlk;       // token within each block
  const int n_head = lane >> 2;    // head column this lane feeds in the B operand
  const int cpair = 2 * (lane & 3);   // head columns of this lane's accumulators
  const uint32_t ring_u32 = smem_u32(ring);
  const int mi = lane >> 3;
  const uint32_t k_off = static_cast<uint32_t>(((lane & 7) + (mi & 1) * 8) * C::kPitch + (j * HKV + g) * kD * 2 +
                                               (mi >> 1) * 16);
  const uint32_t v_off = static_cast<uint32_t>(((lane & 7) + (mi >> 1) * 8) * C::kPitch + (j * HKV + g) * kD * 2 +
                                               (mi & 1) * 16);
  float* mslot_base = reinterpret_cast<float*>(merge);
  int st = 0;
  unsigned ph = 0;
  unsigned mph = 0;   // parity of the merge barriers (one phase per item)

  // B-operand fragments of the query heads of this KV head; the next item's are loaded before the
  // merge of the current one so that their latency overlaps it.
  const int hq = g * group + n_head;
  const bool hv = n_head < group;
  auto load_q = [&](int item, uint32_t (&f)[8][2]) {
    if (item >= a.num_items) return;
    const long long qrow = a.seqlens == nullptr
                               ? static_cast<long long>(item % a.B) * a.Tq + (a.Tq - 1 - item / a.B)
                               : static_cast<long long>(item / a.splits);
    const uint16_t* qp = a.q + (qrow * a.Hq + (hv ? hq : 0)) * kD;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const int d0 = 16 * kk + cpair;
      f[kk][0] = hv ? *reinterpret_cast<const uint32_t*>(qp + d0) : 0u;
      f[kk][1] = hv ? *reinterpret_cast<const uint32_t*>(qp + d0 + 8) : 0u;
    }
  };
  uint32_t qf[8][2], qn[8][2];
  load_q(blockIdx.x, qf);
  bool merged = false;   // CL: this warp has passed the two cluster barriers

  for (int item = blockIdx.x; item < a.num_items; item += gridDim.x) {
    const Item it = make_item<HKV>(a, item);
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    float o[8][4];
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;

    for (;;) {
      if (!mbar_wait(&full[st], ph, a.ctl)) {
        if constexpr (CL) goto consumer_tail;
        return;
      }
      const int ns = info_at(st)->nslots;
      const bool last = info_at(st)->last != 0;
      if (ns > 0) {
        const uint32_t kst = ring_u32 + st * C::kStageBytes;
        const uint32_t vst = kst + C::kVOff;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          uint32_t a0, a1, a2, a3;
          ldsm_x4(kst + k_off + kk * 32, a0, a1, a2, a3);
          mma_bf16_16816(acc, a0, a1, a2, a3, qf[kk][0], qf[kk][1]);
        }
        const int r0 = lane >> 2, r1 = r0 + 8;
        const bool v0 = r0 < ns && j < info_at(st)->ntok[r0];
        const bool v1 = r1 < ns && j < info_at(st)->ntok[r1];
        const float x0 = v0 ? acc[0] * a.scale_log2 : -INFINITY;
        const float x1 = v0 ? acc[1] * a.scale_log2 : -INFINITY;
        const float x2 = v1 ? acc[2] * a.scale_log2 : -INFINITY;
        const float x3 = v1 ? acc[3] * a.scale_log2 : -INFINITY;
        float t0 = fmaxf(x0, x2), t1 = fmaxf(x1, x3);
#pragma unroll
        for (int o2 = 4; o2 < 32; o2 <<= 1) {
          t0 = fmaxf(t0, __shfl_xor_sync(0xffffffffu, t0, o2));
          t1 = fmaxf(t1, __shfl_xor_sync(0xffffffffu, t1, o2));
        }
        const float mn0 = fmaxf(m0, t0), mn1 = fmaxf(m1, t1);
        const float ref0 = mn0 == -INFINITY ? 0.f : mn0;
        const float ref1 = mn1 == -INFINITY ? 0.f : mn1;
        const float al0 = exp2f(m0 - ref0), al1 = exp2f(m1 - ref1);
        const float p0 = exp2f(x0 - ref0), p1 = exp2f(x1 - ref1);
        const float p2 = exp2f(x2 - ref0), p3 = exp2f(x3 - ref1);
        l0 = l0 * al0 + (p0 + p2);
        l1 = l1 * al1 + (p1 + p3);
        m0 = mn0;
        m1 = mn1;
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          o[mt][0] *= al0;
          o[mt][1] *= al1;
          o[mt][2] *= al0;
          o[mt][3] *= al1;
        }
        const uint32_t b0 = movmatrix_t(pack_bf16x2(p0, p1));
        const uint32_t b1 = movmatrix_t(pack_bf16x2(p2, p3));
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          uint32_t a0, a1, a2, a3;
          ldsm_x4_t(vst + v_off + mt * 32, a0, a1, a2, a3);
          mma_bf16_16816(o[mt], a0, a1, a2, a3, b0, b1);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
      if (++st == kStages) {
        st = 0;
        ph ^= 1u;
      }
      if (last) break;
    }

    load_q(item + gridDim.x, qn);
    // ---- item epilogue: full row sums, merge the 4 token-warps of this KV head, write
#pragma unroll
    for (int o2 = 4; o2 < 32; o2 <<= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, o2);
      l1 += __shfl_xor_sync(0xffffffffu, l1, o2);
    }
    float* my_slot = mslot_base + (g * 3 + (j > 0 ? j - 1 : 0)) * (C::kMergeSlot / 4);
    if (j > 0) {
      if (!mbar_wait(&mempty[g], mph ^ 1u, a.ctl)) {
        if constexpr (CL) goto consumer_tail;
        return;
      }
#pragma unroll
      for (int mt = 0; mt < 8; ++mt)
#pragma unroll
        for (int e = 0; e < 4; ++e) my_slot[(mt * 4 + e) * 32 + lane] = o[mt][e];
      float* ml = my_slot + 1024;
      ml[lane] = m0;
      ml[32 + lane] = m1;
      ml[64 + lane] = l0;
      ml[96 + lane] = l1;
      __syncwarp();
      if (lane == 0) mbar_arrive(&mfull[g]);
    } else {
      if (!mbar_wait(&mfull[g], mph, a.ctl)) {
        if constexpr (CL) goto consumer_tail;
        return;
      }
    }
    if (j == 0) {
#pragma unroll 1
      for (int jj = 0; jj < kBlk - 1; ++jj) {
        const float* sl = mslot_base + (g * 3 + jj) * (C::kMergeSlot / 4);
        const float* ml = sl + 1024;
        const float om0 = ml[lane], om1 = ml[32 + lane], ol0 = ml[64 + lane], ol1 = ml[96 + lane];
        const float M0 = fmaxf(m0, om0), M1 = fmaxf(m1, om1);
        const float R0 = M0 == -INFINITY ? 0.f : M0, R1 = M1 == -INFINITY ? 0.f : M1;
        const float fs0 = exp2f(m0 - R0), fo0 = exp2f(om0 - R0);
        const float fs1 = exp2f(m1 - R1), fo1 = exp2f(om1 - R1);
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          o[mt][0] = o[mt][0] * fs0 + sl[(mt * 4 + 0) * 32 + lane] * fo0;
          o[mt][1] = o[mt][1] * fs1 + sl[(mt * 4 + 1) * 32 + lane] * fo1;
          o[mt][2] = o[mt][2] * fs0 + sl[(mt * 4 + 2) * 32 + lane] * fo0;
          o[mt][3] = o[mt][3] * fs1 + sl[(mt * 4 + 3) * 32 + lane] * fo1;
        }
        l0 = l0 * fs0 + ol0 * fo0;
        l1 = l1 * fs1 + ol1 * fo1;
        m0 = M0;
        m1 = M1;
      }
      if (CL && it.partial) {
        // Split merge inside the cluster: this warp's unnormalised state (o, m, l) goes to merge
        // slot (g, 0), which it has finished reading, in its register layout (36 floats a lane);
        // after a cluster barrier, rank 0 folds the other ranks' states into its own (log-sum-exp
        // merge, ranks in order) and writes the final row below; a second barrier keeps the
        // other CTAs (and their shared memory) alive until rank 0 has read them.
        float* cs = mslot_base + (g * 3) * (C::kMergeSlot / 4) + lane * 36;
#pragma unroll
        for (int mt = 0; mt < 8; ++mt)
          *reinterpret_cast<float4*>(cs + 4 * mt) = make_float4(o[mt][0], o[mt][1], o[mt][2], o[mt][3]);
        *reinterpret_cast<float4*>(cs + 32) = make_float4(m0, m1, l0, l1);
        cluster_sync_all();
        const uint32_t rank = cluster_rank();
        if (rank == 0) {
          for (int r = 1; r < a.splits; ++r) {
            const uint32_t ra = cluster_addr(cs, static_cast<uint32_t>(r));
            const float4 ml4 = ld_cluster_f4(ra + 128);
            const float M0 = fmaxf(m0, ml4.x), M1 = fmaxf(m1, ml4.y);
            const float R0 = M0 == -INFINITY ? 0.f : M0, R1 = M1 == -INFINITY ? 0.f : M1;
            const float fs0 = exp2f(m0 - R0), fo0 = exp2f(ml4.x - R0);
            const float fs1 = exp2f(m1 - R1), fo1 = exp2f(ml4.y - R1);
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) {
              const float4 ro = ld_cluster_f4(ra + 16 * mt);
              o[mt][0] = o[mt][0] * fs0 + ro.x * fo0;
              o[mt][1] = o[mt][1] * fs1 + ro.y * fo1;
              o[mt][2] = o[mt][2] * fs0 + ro.z * fo0;
              o[mt][3] = o[mt][3] * fs1 + ro.w * fo1;
            }
            l0 = l0 * fs0 + ml4.z * fo0;
            l1 = l1 * fs1 + ml4.w * fo1;
            m0 = M0;
            m1 = M1;
          }
        }
        __syncwarp();
        cluster_sync_all();
        merged = true;
      }
      if (!it.partial || (CL && cluster_rank() == 0)) {
        // stage the normalised rows [head][d] as bf16, then 16-byte stores
        // staged in merge slot (g, 0), which this warp has finished reading
        uint16_t* stg = reinterpret_cast<uint16_t*>(mslot_base + (g * 3) * (C::kMergeSlot / 4));
        const float inv0 = l0 > 0.f ? 1.f / l0 : 0.f, inv1 = l1 > 0.f ? 1.f / l1 : 0.f;
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          const int d = 16 * mt + (lane >> 2);
          stg[(cpair)*kD + d] = __bfloat16_as_ushort(__float2bfloat16_rn(o[mt][0] * inv0));
          stg[(cpair + 1) * kD + d] = __bfloat16_as_ushort(__float2bfloat16_rn(o[mt][1] * inv1));
          stg[(cpair)*kD + d + 8] = __bfloat16_as_ushort(__float2bfloat16_rn(o[mt][2] * inv0));
          stg[(cpair + 1) * kD + d + 8] = __bfloat16_as_ushort(__float2bfloat16_rn(o[mt][3] * inv1));
        }
        __syncwarp();
        const long long frow = it.partial ? it.qrow : it.orow;   // cluster mode: the sequence's row
        uint16_t* orow = a.out + (frow * a.Hq + g * group) * kD;
        const int chunks = group * kD / 8;   // 16-byte chunks of this KV head's output heads
        const bool row_ok = QSA_DCHECK(a.ctl, frow >= 0 && frow < out_rows(a));
        for (int c = lane; row_ok && c < chunks; c += 32)
          reinterpret_cast<uint4*>(orow)[c] = reinterpret_cast<const uint4*>(stg)[c];
        if (row_ok && a.lse && lane < 4) {
          if (cpair < group)
            a.lse[frow * a.Hq + g * group + cpair] = l0 > 0.f ? (m0 + __log2f(l0)) * kLn2 : -INFINITY;
          if (cpair + 1 < group)
            a.lse[frow * a.Hq + g * group + cpair + 1] = l1 > 0.f ? (m1 + __log2f(l1)) * kLn2 : -INFINITY;
        }
        __syncwarp();
      } else if (!CL && QSA_DCHECK(a.ctl, it.orow >= 0 && it.orow < a.num_items)) {
        // unnormalised partial: part[item][h][0..D) = o, part[item][h][D] = m (log2 units), [D+1] = l
        float* prow = a.part + it.orow * a.Hq * (kD + 2);
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          const int d = 16 * mt + (lane >> 2);
          if (cpair < group) {
            prow[(g * group + cpair) * (kD + 2) + d] = o[mt][0];
            prow[(g * group + cpair) * (kD + 2) + d + 8] = o[mt][2];
          }
          if (cpair + 1 < group) {
            prow[(g * group + cpair + 1) * (kD + 2) + d] = o[mt][1];
            prow[(g * group + cpair + 1) * (kD + 2) + d + 8] = o[mt][3];
          }
        }
        if (lane < 4) {
          if (cpair < group) {
            prow[(g * group + cpair) * (kD + 2) + kD] = m0;
            prow[(g * group + cpair) * (kD + 2) + kD + 1] = l0;
          }
          if (cpair + 1 < group) {
            prow[(g * group + cpair + 1) * (kD + 2) + kD] = m1;
            prow[(g * group + cpair + 1) * (kD + 2) + kD + 1] = l1;
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&mempty[g]);
    }
    mph ^= 1u;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      qf[kk][0] = qn[kk][0];
      qf[kk][1] = qn[kk][1];
    }
  }
consumer_tail:
  if constexpr (CL) {
    if (!merged) {
      cluster_sync_all();
      cluster_sync_all();
    }
  }
  }   // consumer warps
}
#pragma nv_diag_default 177

// ======================================================================================
// Wide variant: head dimension D (128 or 256) and GQA groups of up to 16 query heads (the model
// shape of the pages: D = 256, 24 query heads over 2 KV heads, groups of 12).  A stage holds 8 block
// slots (the ring of 3 stages stays within shared memory at D = 256).  Consumer warp (g, hs) owns KV
// head g and the query heads hs*8 .. hs*8+7 of its group (N = 8 of mma.m16n8k16; heads past the group
// are zero columns), and covers all 32 tokens of a stage as two m16 tiles, so no merge between
// warps is needed: m-tile t holds tokens 2t and 2t+1 of the 8 slots (rows = slot + 8 * token
// parity), which keeps ldmatrix on 8 different slots (conflict-free with the padded pitch).
constexpr int kWideSlots = 8;

template <int HKV, int D, int NSUB>
struct WideCfg {
  using R = Ring<HKV, D, kWideSlots>;
  static constexpr int kConsumerWarps = HKV * NSUB;
  static constexpr int kThreads = (kConsumerWarps + kIssuers_) * 32;
  static constexpr int kStageBytes = R::kStageBytes;
  static constexpr int kStgBytes = kConsumerWarps * 8 * D * 2;   // per-warp output staging [8 heads][D]
  static constexpr int kInfoBytes = kStages * R::kInfoStride;
  static constexpr int kBarBytes = 3 * kStages * 8;
  static constexpr int kPendBytes = 64 * 4;
  static constexpr int kIdxBytes = 2 * kSeg * 4;
  static constexpr int kSmem = 128 + kStages * kStageBytes + kStgBytes + kInfoBytes + kBarBytes + kPendBytes + kIdxBytes;
  static_assert(kSmem <= 227 * 1024, "shared memory per CTA");
};

template <int HKV, int D, int NSUB>
__global__ void __launch_bounds__(WideCfg<HKV, D, NSUB>::kThreads, 1) sparse_attn_wide_kernel(AttnArgs a) {
  using C = WideCfg<HKV, D, NSUB>;
  using R = typename C::R;
  constexpr int KS = D / 16;   // k-steps of the score product, m-tiles of the output
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  uint8_t* ring = smem;
  uint8_t* stg_all = ring + kStages * C::kStageBytes;
  uint8_t* info = stg_all + C::kStgBytes;
  auto info_at = [&](int s) { return reinterpret_cast<StageInfo*>(info + s * R::kInfoStride); };
  uint64_t* full = reinterpret_cast<uint64_t*>(info + C::kInfoBytes);
  uint64_t* empty = full + kStages;
  uint64_t* ready = empty + kStages;
  int* pend = reinterpret_cast<int*>(ready + kStages);
  int* idxbuf = pend + 64;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int group = a.Hq / HKV;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], C::kConsumerWarps);
      mbar_init(&ready[s], 1);
    }
    fence_mbar_init();
  }
  // Zero the ring once so that unused slot rows are finite (they are masked, but 0 * NaN = NaN).
  for (int i = threadIdx.x; i < kStages * C::kStageBytes / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(ring)[i] = make_uint4(0, 0, 0, 0);
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // order these writes before the bulk copies
  __syncthreads();

  if (warp > C::kConsumerWarps) {
    attn_helper<HKV, D, kWideSlots>(a, warp - C::kConsumerWarps, ring, info, full, ready);
    return;
  }
  if (warp == C::kConsumerWarps) {
    attn_producer<HKV, D, kWideSlots>(a, ring, info, full, empty, ready, pend, idxbuf);
    return;
  }

  // -------------------------------------------------------------------- consumer warps
  const int g = warp / NSUB;            // KV head
  const int hs = warp % NSUB;           // head subgroup: heads hs*8 .. hs*8+7 of the group
  const int nvalid = min(8, group - hs * 8);
  const int hbase = g * group + hs * 8;
  const int n_head = lane >> 2;         // head column this lane feeds in the B operand
  const int cpair = 2 * (lane & 3);     // head columns of this lane's accumulators
  const uint32_t ring_u32 = smem_u32(ring);
  // ldmatrix rows: lane & 7 = slot; the other lane bits pick the token parity and the 8-column half
  const int slot_l = lane & 7;
  const uint32_t k_off = static_cast<uint32_t>(slot_l * R::kPitch + (((lane >> 3) & 1) * HKV + g) * D * 2 +
                                               ((lane >> 4) & 1) * 16);
  const uint32_t v_off = static_cast<uint32_t>(slot_l * R::kPitch + (((lane >> 4) & 1) * HKV + g) * D * 2 +
                                               ((lane >> 3) & 1) * 16);
  constexpr uint32_t kTokPair = 2 * HKV * D * 2;   // bytes from tokens {0,1} to tokens {2,3} of a slot
  uint16_t* stg = reinterpret_cast<uint16_t*>(stg_all) + warp * 8 * D;
  int st = 0;
  unsigned ph = 0;

  auto load_q = [&](int item, uint32_t (&f)[KS][2]) {
    if (item >= a.num_items) return;
    const long long qrow = a.seqlens == nullptr
                               ? static_cast<long long>(item % a.B) * a.Tq + (a.Tq - 1 - item / a.B)
                               : static_cast<long long>(item / a.splits);
    const bool hv = n_head < nvalid;
    const uint16_t* qp = a.q + (qrow * a.Hq + (hv ? hbase + n_head : 0)) * D;
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
      const int d0 = 16 * kk + cpair;
      f[kk][0] = hv ? *reinterpret_cast<const uint32_t*>(qp + d0) : 0u;
      f[kk][1] = hv ? *reinterpret_cast<const uint32_t*>(qp + d0 + 8) : 0u;
    }
  };
  uint32_t qf[KS][2];
  load_q(blockIdx.x, qf);

  for (int item = blockIdx.x; item < a.num_items; item += gridDim.x) {
    const Item it = make_item<HKV, D>(a, item);
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    float o[KS][4];
#pragma unroll
    for (int mt = 0; mt < KS; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;

    for (;;) {
      if (!mbar_wait(&full[st], ph, a.ctl)) return;
      const int ns = info_at(st)->nslots;
      const bool last = info_at(st)->last != 0;
      if (ns > 0) {
        const uint32_t kst = ring_u32 + st * C::kStageBytes;
        const uint32_t vst = kst + kWideSlots * R::kPitch;
        float acc[2][4];
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
#pragma unroll
          for (int kk = 0; kk < KS; ++kk) {
            uint32_t a0, a1, a2, a3;
            ldsm_x4(kst + k_off + t * kTokPair + kk * 32, a0, a1, a2, a3);
            mma_bf16_16816(acc[t], a0, a1, a2, a3, qf[kk][0], qf[kk][1]);
          }
        }
        // rows: r0 = slot lane>>2 at token 2t, r1 = the same slot at token 2t + 1
        const int sr = lane >> 2;
        const int ntk = sr < ns ? info_at(st)->ntok[sr] : 0;
        float x[2][4];
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          const bool v0 = 2 * t < ntk, v1 = 2 * t + 1 < ntk;
          x[t][0] = v0 ? acc[t][0] * a.scale_log2 : -INFINITY;
          x[t][1] = v0 ? acc[t][1] * a.scale_log2 : -INFINITY;
          x[t][2] = v1 ? acc[t][2] * a.scale_log2 : -INFINITY;
          x[t][3] = v1 ? acc[t][3] * a.scale_log2 : -INFINITY;
        }
        float t0 = fmaxf(fmaxf(x[0][0], x[0][2]), fmaxf(x[1][0], x[1][2]));
        float t1 = fmaxf(fmaxf(x[0][1], x[0][3]), fmaxf(x[1][1], x[1][3]));
#pragma unroll
        for (int o2 = 4; o2 < 32; o2 <<= 1) {
          t0 = fmaxf(t0, __shfl_xor_sync(0xffffffffu, t0, o2));
          t1 = fmaxf(t1, __shfl_xor_sync(0xffffffffu, t1, o2));
        }
        const float mn0 = fmaxf(m0, t0), mn1 = fmaxf(m1, t1);
        const float ref0 = mn0 == -INFINITY ? 0.f : mn0;
        const float ref1 = mn1 == -INFINITY ? 0.f : mn1;
        const float al0 = exp2f(m0 - ref0), al1 = exp2f(m1 - ref1);
        float p[2][4];
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          p[t][0] = exp2f(x[t][0] - ref0);
          p[t][1] = exp2f(x[t][1] - ref1);
          p[t][2] = exp2f(x[t][2] - ref0);
          p[t][3] = exp2f(x[t][3] - ref1);
        }
        l0 = l0 * al0 + (p[0][0] + p[0][2] + p[1][0] + p[1][2]);
        l1 = l1 * al1 + (p[0][1] + p[0][3] + p[1][1] + p[1][3]);
        m0 = mn0;
        m1 = mn1;
#pragma unroll
        for (int mt = 0; mt < KS; ++mt) {
          o[mt][0] *= al0;
          o[mt][1] *= al1;
          o[mt][2] *= al0;
          o[mt][3] *= al1;
        }
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          const uint32_t b0 = movmatrix_t(pack_bf16x2(p[t][0], p[t][1]));
          const uint32_t b1 = movmatrix_t(pack_bf16x2(p[t][2], p[t][3]));
#pragma unroll
          for (int mt = 0; mt < KS; ++mt) {
            uint32_t a0, a1, a2, a3;
            ldsm_x4_t(vst + v_off + t * kTokPair + mt * 32, a0, a1, a2, a3);
            mma_bf16_16816(o[mt], a0, a1, a2, a3, b0, b1);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
      if (++st == kStages) {
        st = 0;
        ph ^= 1u;
      }
      if (last) break;
    }

    load_q(item + gridDim.x, qf);   // the next item's query (its latency overlaps the epilogue)
    // ---- item epilogue: full row sums, then the output of this warp's heads
#pragma unroll
    for (int o2 = 4; o2 < 32; o2 <<= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, o2);
      l1 += __shfl_xor_sync(0xffffffffu, l1, o2);
    }
    if (!it.partial) {
      const float inv0 = l0 > 0.f ? 1.f / l0 : 0.f, inv1 = l1 > 0.f ? 1.f / l1 : 0.f;
#pragma unroll
      for (int mt = 0; mt < KS; ++mt) {
        const int d = 16 * mt + (lane >> 2);
        stg[cpair * D + d] = __bfloat16_as_ushort(__float2bfloat16_rn(o[mt][0] * inv0));
        stg[(cpair + 1) * D + d] = __bfloat16_as_ushort(__float2bfloat16_rn(o[mt][1] * inv1));
        stg[cpair * D + d + 8] = __bfloat16_as_ushort(__float2bfloat16_rn(o[mt][2] * inv0));
        stg[(cpair + 1) * D + d + 8] = __bfloat16_as_ushort(__float2bfloat16_rn(o[mt][3] * inv1));
      }
      __syncwarp();
      uint16_t* orow = a.out + (it.orow * a.Hq + hbase) * D;
      const int chunks = nvalid * D / 8;   // 16-byte chunks of this warp's output heads
      const bool row_ok = QSA_DCHECK(a.ctl, it.orow >= 0 && it.orow < out_rows(a));
      for (int c = lane; row_ok && c < chunks; c += 32)
        reinterpret_cast<uint4*>(orow)[c] = reinterpret_cast<const uint4*>(stg)[c];
      if (row_ok && a.lse && lane < 4) {
        if (cpair < nvalid) a.lse[it.orow * a.Hq + hbase + cpair] = l0 > 0.f ? (m0 + __log2f(l0)) * kLn2 : -INFINITY;
        if (cpair + 1 < nvalid)
          a.lse[it.orow * a.Hq + hbase + cpair + 1] = l1 > 0.f ? (m1 + __log2f(l1)) * kLn2 : -INFINITY;
      }
      __syncwarp();
    } else if (QSA_DCHECK(a.ctl, it.orow >= 0 && it.orow < a.num_items)) {
      // unnormalised partial: part[item][h][0..D) = o, part[item][h][D] = m (log2 units), [D+1] = l
      float* prow = a.part + it.orow * a.Hq * (D + 2);
#pragma unroll
      for (int mt = 0; mt < KS; ++mt) {
        const int d = 16 * mt + (lane >> 2);
        if (cpair < nvalid) {
          prow[(hbase + cpair) * (D + 2) + d] = o[mt][0];
          prow[(hbase + cpair) * (D + 2) + d + 8] = o[mt][2];
        }
        if (cpair + 1 < nvalid) {
          prow[(hbase + cpair + 1) * (D + 2) + d] = o[mt][1];
          prow[(hbase + cpair + 1) * (D + 2) + d + 8] = o[mt][3];
        }
      }
      if (lane < 4) {
        if (cpair < nvalid) {
          prow[(hbase + cpair) * (D + 2) + D] = m0;
          prow[(hbase + cpair) * (D + 2) + D + 1] = l0;
        }
        if (cpair + 1 < nvalid) {
          prow[(hbase + cpair + 1) * (D + 2) + D] = m1;
          prow[(hbase + cpair + 1) * (D + 2) + D + 1] = l1;
        }
      }
    }
  }
}

// Merge of decode splits: out[b][h] = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s.  One thread per
// element of the head dimension D (blockDim.x == D).
__global__ void __launch_bounds__(256) combine_kernel(const float* __restrict__ part, int splits, int Hq, int D,
                                                      uint16_t* __restrict__ out, float* __restrict__ lse) {
  const int b = blockIdx.x, h = blockIdx.y, d = threadIdx.x;
  const float* p = part + (static_cast<long long>(b) * splits * Hq + h) * (D + 2);
  const long long step = static_cast<long long>(Hq) * (D + 2);
  float M = -INFINITY;
  for (int s = 0; s < splits; ++s) M = fmaxf(M, p[s * step + D]);
  const float R = M == -INFINITY ? 0.f : M;
  float acc = 0.f, l = 0.f;
  for (int s = 0; s < splits; ++s) {
    const float f = exp2f(p[s * step + D] - R);
    acc += f * p[s * step + d];
    l += f * p[s * step + D + 1];
  }
  out[(static_cast<long long>(b) * Hq + h) * D + d] = __bfloat16_as_ushort(__float2bfloat16_rn(l > 0.f ? acc / l : 0.f));
  if (lse && d == 0) lse[static_cast<long long>(b) * Hq + h] = l > 0.f ? (M + __log2f(l)) * kLn2 : -INFINITY;
}

// With the register split the block must launch with exactly 128 registers a thread: the
// consumers' setmaxnreg.inc draws on what the launch reserved, and would wait for ever if the
// issuers' release could not cover it.  A build where ptxas chose fewer is refused, not launched.
template <int HKV, bool CL, bool KVI = false>
cudaError_t check_reg_split() {
  using C = Cfg<HKV, KVI>;
  if constexpr (C::kRegSplit) {
    cudaFuncAttributes fa{};
    const cudaError_t e = cudaFuncGetAttributes(&fa, sparse_attn_kernel<HKV, CL, KVI>);
    if (e != cudaSuccess) return e;
    if (fa.numRegs * C::kThreads != 65536) return cudaErrorInvalidConfiguration;
  }
  return cudaSuccess;
}

template <int HKV, bool KVI = false>
cudaError_t launch_attn(const DeviceInfo* di, AttnArgs a, cudaStream_t s) {
  using C = Cfg<HKV, KVI>;
  static std::once_flag once[64];
  std::call_once(once[di->device & 63], [] {
    cudaFuncSetAttribute(sparse_attn_kernel<HKV, false, KVI>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  });
  if (const cudaError_t e = check_reg_split<HKV, false, KVI>(); e != cudaSuccess) return e;
  const int grid = std::min(a.num_items, di->num_sms);
  if (grid <= 0) return cudaSuccess;
  sparse_attn_kernel<HKV, false, KVI><<<grid, C::kThreads, C::kSmem, s>>>(a);
  return cudaPeekAtLastError();
}

// K and V interleaved by block: kv[b][j][0] = k[b][4j .. 4j+3], kv[b][j][1] = v[b][4j .. 4j+3]
// ([4][Hkv][D] each), positions >= Tk zero.  One CTA per (block, sequence), one 16-byte chunk per
// thread: thread w copies chunk w of the block, i.e. part w >> (2 + lg) (K or V), token
// (w >> lg) & 3, chunk w & (2^lg - 1) of the token (2^lg chunks per token of all KV heads).
__global__ void __launch_bounds__(256) interleave_kv_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v,
                                                            uint4* __restrict__ kv, int Tk, int lg, long long j0) {
  const long long j = j0 + blockIdx.x;
  const long long b = blockIdx.y;
  const long long nblk = (Tk + kBlk - 1) / kBlk;
  const int w = threadIdx.x;
  const int which = w >> (2 + lg);
  const long long t = j * kBlk + ((w >> lg) & 3);
  const int c = w & ((1 << lg) - 1);
  uint4 val = make_uint4(0u, 0u, 0u, 0u);
  if (t < Tk) val = (which ? v : k)[((b * Tk + t) << lg) + c];
  kv[((b * nblk + j) << (3 + lg)) + w] = val;
}

template <int HKV, int D, int NSUB>
cudaError_t launch_attn_wide_cfg(const DeviceInfo* di, AttnArgs a, cudaStream_t s) {
  using C = WideCfg<HKV, D, NSUB>;
  static std::once_flag once[64];
  std::call_once(once[di->device & 63], [] {
    cudaFuncSetAttribute(sparse_attn_wide_kernel<HKV, D, NSUB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         C::kSmem);
  });
  const int grid = std::min(a.num_items, di->num_sms);
  if (grid <= 0) return cudaSuccess;
  sparse_attn_wide_kernel<HKV, D, NSUB><<<grid, C::kThreads, C::kSmem, s>>>(a);
  return cudaPeekAtLastError();
}

// D = 128 with groups of up to 8 heads takes the 16-slot kernel; D = 256, or groups of 9 .. 16,
// the wide one.
cudaError_t launch_attn_any(const DeviceInfo* di, AttnArgs a, int Hkv, int D, cudaStream_t s) {
  const int group = a.Hq / Hkv;
  if (a.kv) return Hkv == 1 ? launch_attn<1, true>(di, a, s) : launch_attn<2, true>(di, a, s);
  if (D == kD && group <= 8) return Hkv == 1 ? launch_attn<1>(di, a, s) : launch_attn<2>(di, a, s);
  const int nsub = group <= 8 ? 1 : 2;
  if (D == 128) {
    if (Hkv == 1) return nsub == 1 ? launch_attn_wide_cfg<1, 128, 1>(di, a, s) : launch_attn_wide_cfg<1, 128, 2>(di, a, s);
    return nsub == 1 ? launch_attn_wide_cfg<2, 128, 1>(di, a, s) : launch_attn_wide_cfg<2, 128, 2>(di, a, s);
  }
  if (Hkv == 1) return nsub == 1 ? launch_attn_wide_cfg<1, 256, 1>(di, a, s) : launch_attn_wide_cfg<1, 256, 2>(di, a, s);
  return nsub == 1 ? launch_attn_wide_cfg<2, 256, 1>(di, a, s) : launch_attn_wide_cfg<2, 256, 2>(di, a, s);
}

}  // namespace

cudaError_t launch_attn_prefill(const DeviceInfo* di, const void* q, const void* k, const void* v, const int32_t* idx,
                                int B, int Tq, int Tk, int Hq, int Hkv, int D, int k_blocks, long long q_pos0,
                                float scale, void* out, float* lse, cudaStream_t s) {
  AttnArgs a{};
  a.q = static_cast<const uint16_t*>(q);
  a.k = static_cast<const uint16_t*>(k);
  a.v = static_cast<const uint16_t*>(v);
  a.idx = idx;
  a.seqlens = nullptr;
  a.out = static_cast<uint16_t*>(out);
  a.lse = lse;
  a.part = nullptr;
  a.q_pos0 = q_pos0;
  a.B = B;
  a.Tq = Tq;
  a.Tk = Tk;
  a.Hq = Hq;
  a.kblocks = k_blocks;
  a.splits = 1;
  a.num_items = B * Tq;
  a.scale_log2 = scale * kLog2e;
  a.ctl = kernel_ctl(di);
  return launch_attn_any(di, a, Hkv, D, s);
}

bool attn_kv_supported(int Hq, int Hkv, int D) { return D == kD && (Hkv == 1 || Hkv == 2) && Hq / Hkv <= 8; }

size_t attn_kv_bytes(int B, int Tk, int Hkv, int D) {
  return static_cast<size_t>(B) * ((Tk + kBlk - 1) / kBlk) * 2 * kBlk * Hkv * D * 2;
}

cudaError_t launch_interleave_kv(const DeviceInfo* di, const void* k, const void* v, void* kv, int B, int Tk, int Hkv,
                                 int D, long long j0, long long j1, cudaStream_t s) {
  (void)di;
  if (j1 <= j0 || B <= 0) return cudaSuccess;
  const int tok16 = Hkv * D * 2 / 16;   // 16-byte chunks of one token of all KV heads: 16 or 32
  const int lg = tok16 == 32 ? 5 : 4;
  if ((1 << lg) != tok16 || j1 - j0 > 0x7fffffffLL || B > 65535) return cudaErrorInvalidValue;
  interleave_kv_kernel<<<dim3(static_cast<unsigned>(j1 - j0), static_cast<unsigned>(B)), 8 * tok16, 0, s>>>(
      static_cast<const uint4*>(k), static_cast<const uint4*>(v), static_cast<uint4*>(kv), Tk, lg, j0);
  return cudaPeekAtLastError();
}

cudaError_t launch_attn_prefill_kv(const DeviceInfo* di, const void* q, const void* kv, const int32_t* idx, int B,
                                   int Tq, int Tk, int Hq, int Hkv, int k_blocks, long long q_pos0, float scale,
                                   void* out, float* lse, cudaStream_t s) {
  AttnArgs a{};
  a.q = static_cast<const uint16_t*>(q);
  a.kv = static_cast<const uint16_t*>(kv);
  a.idx = idx;
  a.seqlens = nullptr;
  a.out = static_cast<uint16_t*>(out);
  a.lse = lse;
  a.part = nullptr;
  a.q_pos0 = q_pos0;
  a.B = B;
  a.Tq = Tq;
  a.Tk = Tk;
  a.Hq = Hq;
  a.kblocks = k_blocks;
  a.splits = 1;
  a.num_items = B * Tq;
  a.scale_log2 = scale * kLog2e;
  a.ctl = kernel_ctl(di);
  return launch_attn_any(di, a, Hkv, kD, s);
}

// Split-KV decode as clusters: one CTA per item (B * splits <= SMs), a cluster of `splits` CTAs per
// sequence, the D = 128 kernel (groups of up to 8 heads), and all clusters resident at once.
bool decode_cluster_ok(const DeviceInfo* di, int B, int Hq, int Hkv, int D, int splits) {
  if (splits < 2 || splits > 8 || D != kD || Hq / Hkv > 8 || (Hkv != 1 && Hkv != 2)) return false;
  if (static_cast<long long>(B) * splits > di->num_sms) return false;
  static std::atomic<int> max_clusters[64][2][9];   // 0: not asked yet; -1: the query failed
  static std::once_flag once[64];
  std::call_once(once[di->device & 63], [] {
    cudaFuncSetAttribute(sparse_attn_kernel<1, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg<1>::kSmem);
    cudaFuncSetAttribute(sparse_attn_kernel<2, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg<2>::kSmem);
  });
  std::atomic<int>& slot = max_clusters[di->device & 63][Hkv - 1][splits];
  int mc = slot.load(std::memory_order_relaxed);
  if (mc == 0) {   // cached per device, KV head count and cluster size (two first callers may both ask)
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(splits * B));
    cfg.blockDim = dim3(Hkv == 1 ? Cfg<1>::kThreads : Cfg<2>::kThreads);
    cfg.dynamicSmemBytes = Hkv == 1 ? Cfg<1>::kSmem : Cfg<2>::kSmem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(splits);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    const cudaError_t e = Hkv == 1 ? cudaOccupancyMaxActiveClusters(&n, sparse_attn_kernel<1, true>, &cfg)
                                   : cudaOccupancyMaxActiveClusters(&n, sparse_attn_kernel<2, true>, &cfg);
    mc = (e == cudaSuccess && n > 0) ? n : -1;
    if (e != cudaSuccess) cudaGetLastError();
    slot.store(mc, std::memory_order_relaxed);
  }
  return mc >= B;
}

template <int HKV>
cudaError_t launch_attn_cluster(const DeviceInfo* di, AttnArgs a, cudaStream_t s) {
  using C = Cfg<HKV>;
  (void)di;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(a.num_items));   // one item per CTA
  cfg.blockDim = dim3(C::kThreads);
  cfg.dynamicSmemBytes = C::kSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(a.splits);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (const cudaError_t e = check_reg_split<HKV, true>(); e != cudaSuccess) return e;
  return cudaLaunchKernelEx(&cfg, sparse_attn_kernel<HKV, true>, a);
}

int decode_default_splits(const DeviceInfo* di, int B, int k_blocks) {
  // One wave: at most one item per SM (a second, partial wave of items costs more than the longer
  // items it saves), at most 8 splits per sequence, and at least ~32 blocks per split.
  const int want = std::max(1, std::min(8, di->num_sms / std::max(B, 1)));
  const int cap = std::max(1, (k_blocks + 31) / 32);
  return std::min(want, cap);
}

cudaError_t launch_attn_decode(const DeviceInfo* di, const void* q, const void* kc, const void* vc,
                               const int32_t* seqlens, const int32_t* idx, int B, int Lmax, int Hq, int Hkv, int D,
                               int k_blocks, float scale, int num_splits, void* out, float* lse, float* part,
                               cudaStream_t s) {
  AttnArgs a{};
  a.q = static_cast<const uint16_t*>(q);
  a.k = static_cast<const uint16_t*>(kc);
  a.v = static_cast<const uint16_t*>(vc);
  a.idx = idx;
  a.seqlens = seqlens;
  a.out = static_cast<uint16_t*>(out);
  a.lse = lse;
  a.part = part;
  a.q_pos0 = 0;
  a.B = B;
  a.Tq = 1;
  a.Tk = Lmax;
  a.Hq = Hq;
  a.kblocks = k_blocks;
  a.splits = num_splits;
  a.num_items = B * num_splits;
  a.scale_log2 = scale * kLog2e;
  a.ctl = kernel_ctl(di);
  if (num_splits > 1 && decode_cluster_ok(di, B, Hq, Hkv, D, num_splits)) {
    a.cluster = 1;   // the splits of a sequence merge inside their cluster: no partials, no merge kernel
    return Hkv == 1 ? launch_attn_cluster<1>(di, a, s) : launch_attn_cluster<2>(di, a, s);
  }
  cudaError_t e = launch_attn_any(di, a, Hkv, D, s);
  if (e != cudaSuccess || num_splits <= 1) return e;
  combine_kernel<<<dim3(B, Hq), D, 0, s>>>(part, num_splits, Hq, D, static_cast<uint16_t*>(out), lse);
  return cudaPeekAtLastError();
}

}  // namespace qsa
