// Per-query top-k block selection.
//
// "Qwen3.8-Flash-Next architecture" (flozi.net), "Der Weg eines Tokens durch das Modell", item 2:
// each query keeps a budget of 512 fully selected micro-blocks (2048 tokens) plus its own,
// possibly incomplete, block.  Reading fixed in qsa.h: the top-k of the fp32 scores over the
// candidates b < floor(p/blk), equal scores to the lower index, ascending output, -1 padded.
//
// One CTA per score row; the row is read from memory once on the fast path:
//   1. a 2048-point sample of the row gives a threshold tau a little below the k-th largest
//      score (its rank among the samples is chosen so that ~2.5k scores are expected above it);
//   2. one coalesced pass collects every (key, index) with key >= tau into shared memory;
//   3. an exact radix select on the candidates' order-preserving 32-bit keys gives the k-th key K*
//      and how many keys equal to K* are taken; if equal keys must be split, a second radix select
//      on their indices finds the largest index I* that is kept (lower index wins);
//   4. the kept set {key > K*} U {key == K*, index <= I*} is marked in a shared bitmap of the row
//      and emitted in ascending order by a block-wide scan of the bitmap's word counts.
// Rows with at most `kCap` candidates skip steps 1-2.  If the threshold leaves fewer than k or more
// than kCap candidates (heavy ties), it is moved and the pass retried; after that, or when the row
// is too long for the bitmap, an exact three-pass radix select over the row in memory is used.
// Lanes of a warp that hit the same histogram bin are merged with match.any (one atomic per bin).
//
// Also in this file: a warp-per-row variant for launches with many short rows, the decode kernel
// that spreads each of a few long rows over a thread-block cluster (slices merged through
// distributed shared memory), and the exact redo of rows the filtered prefill selection could not
// settle.
#include <algorithm>
#include <mutex>

#include "launch.h"

namespace qsa {
namespace {

// Tuning knobs (compile time): threads per row, samples for the threshold, loads in flight per
// thread in the filter pass, and how a warp appends its candidates (0: warp scan + one shared
// atomic per warp; 1: one shared atomic per thread that has candidates).
#ifndef QSA_TOPK_THREADS
#define QSA_TOPK_THREADS 512
#endif
#ifndef QSA_TOPK_SAMPLES
#define QSA_TOPK_SAMPLES 2048
#endif
#ifndef QSA_TOPK_LOADS
#define QSA_TOPK_LOADS 4
#endif
#ifndef QSA_TOPK_APPEND
#define QSA_TOPK_APPEND 1
#endif
constexpr int kTopkThreads = QSA_TOPK_THREADS;
constexpr int kWarps = kTopkThreads / 32;
constexpr int kBins = 2048;
constexpr int kCap = 6144;          // candidate capacity of the fast path
constexpr int kSamples = QSA_TOPK_SAMPLES;
constexpr int kMaxBitmapWords = 24576;   // rows up to 786432 candidates use the fast path
constexpr int kFixedSmem = kCap * 8 + kBins * 4 + kSamples * 4 + (kWarps + 8) * 4;

__device__ __forceinline__ uint32_t key_of(float s) {
  return score_key(s + 0.0f);   // -0 -> +0, so the two zeros compare equal as in fp32
}

// Exclusive scan of one value per thread over the block; returns the exclusive prefix and the
// block total.  Uses `ws` (kWarps + 1 words); ends with the block synchronised.
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* ws, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) ws[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = lane < kWarps ? ws[lane] : 0u;
    uint32_t s = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    if (lane < kWarps) ws[lane] = s - w;
    if (lane == kWarps - 1) ws[kWarps] = s;
  }
  __syncthreads();
  const uint32_t r = ws[warp] + x - v;
  *total = ws[kWarps];
  __syncthreads();
  return r;
}

// Adds one histogram hit per lane with hit == true; lanes with the same digit share one atomic.
__device__ __forceinline__ void hist_add(uint32_t* hist, bool hit, uint32_t digit) {
  const int lane = threadIdx.x & 31;
  const uint32_t peers = __match_any_sync(0xffffffffu, hit ? digit : 0xFFFFFFFFu);
  if (hit && lane == __ffs(peers) - 1) atomicAdd(&hist[digit], static_cast<uint32_t>(__popc(peers)));
}

// After a histogram of the current digit: find the bin holding the krem-th largest hit.  Writes
// (bin, hits above the bin) to sel[0], sel[1].  All threads call it; ends synchronised.
__device__ __forceinline__ void find_bin(const uint32_t* hist, int nbins, uint32_t krem, uint32_t* ws, uint32_t* sel) {
  const int tid = threadIdx.x;
  const int bpt = nbins / kTopkThreads;
  uint32_t local = 0;
  for (int q = 0; q < bpt; ++q) local += hist[tid * bpt + q];
  uint32_t total;
  const uint32_t excl = block_excl_scan(local, ws, &total);
  const uint32_t above = total - excl - local;   // hits in the bins above this thread's range
  if (above < krem && above + local >= krem) {
    uint32_t acc = above;
    for (int q = bpt - 1; q >= 0; --q) {
      const uint32_t h = hist[tid * bpt + q];
      if (acc + h >= krem) {
        sel[0] = static_cast<uint32_t>(tid * bpt + q);
        sel[1] = acc;
        break;
      }
      acc += h;
    }
  }
  __syncthreads();
}

// As find_bin, but the bins are scanned by warp 0 alone (no block-wide scan): lane l owns bins
// [l*nbins/32, (l+1)*nbins/32).  All threads call it; ends synchronised.
__device__ __forceinline__ void find_bin_warp(const uint32_t* hist, int nbins, uint32_t krem, uint32_t* sel) {
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    const int bpl = nbins / 32;
    const uint32_t* hp = hist + lane * bpl;
    uint32_t local = 0;
#pragma unroll 8
    for (int q = 0; q < bpl; ++q) local += hp[q];
    uint32_t incl = local;   // hits in this lane's bins and every higher lane's
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_down_sync(0xffffffffu, incl, o);
      if (lane + o < 32) incl += y;
    }
    const uint32_t above = incl - local;
    if (above < krem && above + local >= krem) {
      uint32_t acc = above;
      for (int q = bpl - 1; q >= 0; --q) {
        const uint32_t h = hp[q];
        if (acc + h >= krem) {
          sel[0] = static_cast<uint32_t>(lane * bpl + q);
          sel[1] = acc;
          break;
        }
        acc += h;
      }
    }
  }
  __syncthreads();
}

// Radix select over values in shared memory: the krem-th largest of vals[0..m), resolving
// `passes` 8-bit digits from the top (4 passes resolve the whole key; unresolved low bits are
// returned as zero).  *left = how many values equal to the result (on the resolved bits) are still
// to be taken.  After the last pass hist[] holds that pass's histogram.  Needs >= 256 threads.
__device__ uint32_t smem_select(const uint32_t* vals, int m, uint32_t krem, int passes, uint32_t* hist, uint32_t* ws,
                                uint32_t* sel, uint32_t* left) {
  (void)ws;
  uint32_t prefix = 0, pmask = 0;
  for (int pass = 0; pass < passes; ++pass) {
    const int shift = 24 - 8 * pass;
    if (threadIdx.x < 256) hist[threadIdx.x] = 0;
    __syncthreads();
    for (int base = 0; base < m; base += kTopkThreads) {
      const int i = base + threadIdx.x;
      const uint32_t v = i < m ? vals[i] : 0u;
      const bool hit = i < m && (v & pmask) == prefix;
      hist_add(hist, hit, (v >> shift) & 0xFFu);
    }
    __syncthreads();
    find_bin_warp(hist, 256, krem, sel);   // ends synchronised
    prefix |= sel[0] << shift;
    pmask |= 0xFFu << shift;
    krem -= sel[1];
  }
  *left = krem;
  return prefix;
}

// Exact fallback: three radix passes over the row in global memory, then an ordered emission.
__device__ void topk_global(const float* s, int n, int k, int32_t* out, uint32_t* hist, uint32_t* ws, uint32_t* sel) {
  const int tid = threadIdx.x;
  const int shifts[3] = {21, 10, 0};
  const int widths[3] = {11, 11, 10};
  uint32_t prefix = 0, pmask = 0, krem = static_cast<uint32_t>(k);
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = shifts[pass], nbins = 1 << widths[pass];
    const uint32_t dmask = static_cast<uint32_t>(nbins - 1);
    for (int i = tid; i < nbins; i += kTopkThreads) hist[i] = 0;
    __syncthreads();
    for (int base = 0; base < n; base += kTopkThreads) {
      const int i = base + tid;
      const uint32_t key = i < n ? key_of(s[i]) : 0u;
      const bool hit = i < n && (key & pmask) == prefix;
      hist_add(hist, hit, (key >> shift) & dmask);
    }
    __syncthreads();
    find_bin(hist, nbins, krem, ws, sel);
    prefix |= sel[0] << shift;
    pmask |= dmask << shift;
    krem -= sel[1];
    __syncthreads();
  }
  const uint32_t kth = prefix, need_eq = krem;
  uint32_t gt_tot = 0, eq_tot = 0;
  for (int base = 0; base < n; base += 4 * kTopkThreads) {
    const int i0 = base + 4 * tid;
    uint32_t gt_m = 0, eq_m = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (i0 + e < n) {
        const uint32_t key = key_of(s[i0 + e]);
        gt_m |= (key > kth ? 1u : 0u) << e;
        eq_m |= (key == kth ? 1u : 0u) << e;
      }
    }
    const uint32_t packed = (static_cast<uint32_t>(__popc(gt_m)) << 16) | static_cast<uint32_t>(__popc(eq_m));
    uint32_t total;
    const uint32_t ex = block_excl_scan(packed, ws, &total);
    uint32_t gt_run = gt_tot + (ex >> 16), eq_run = eq_tot + (ex & 0xFFFFu);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (gt_m & (1u << e)) {
        const uint32_t p = gt_run + min(eq_run, need_eq);
        if (p < static_cast<uint32_t>(k)) out[p] = i0 + e;
        ++gt_run;
      } else if (eq_m & (1u << e)) {
        const uint32_t p = gt_run + eq_run;
        if (eq_run < need_eq && p < static_cast<uint32_t>(k)) out[p] = i0 + e;
        ++eq_run;
      }
    }
    gt_tot += total >> 16;
    eq_tot += total & 0xFFFFu;
  }
}

// Shared-memory layout of the CTA-per-row kernels.
struct TopkSmem {
  uint32_t* cand_key;   // kCap
  uint32_t* cand_idx;   // kCap
  uint32_t* hist;       // kBins
  uint32_t* samp;       // kSamples
  uint32_t* ws;         // kWarps + 1
  uint32_t* sel;        // 2
  uint32_t* misc;       // 5 counters / flags
  uint32_t* bitmap;     // bitmap words of the row
};

__device__ __forceinline__ TopkSmem topk_smem(uint32_t* sm) {
  TopkSmem t;
  t.cand_key = sm;
  t.cand_idx = t.cand_key + kCap;
  t.hist = t.cand_idx + kCap;
  t.samp = t.hist + kBins;
  t.ws = t.samp + kSamples;
  t.sel = t.ws + kWarps + 1;
  t.misc = t.sel + 2;
  t.bitmap = t.misc + 5;
  return t;
}

// kSamples keys of the row: kSamples/128 evenly spaced runs of 128 consecutive scores (one 16-byte
// load per thread; coalesced per warp).  Ends synchronised.
__device__ __forceinline__ void load_samples(const float* s, int n, uint32_t* samp) {
  constexpr int kRuns = kSamples / 128;
  for (int j = threadIdx.x; j < kSamples / 4; j += kTopkThreads) {
    const int run = j >> 5, off = (j & 31) * 4;
    const int i0 = (static_cast<int>((static_cast<long long>(run) * n) / kRuns) & ~3) + off;
    float4 f;
    if ((reinterpret_cast<uintptr_t>(s) & 15u) == 0 && i0 + 3 < n) {
      f = __ldcs(reinterpret_cast<const float4*>(s + i0));
    } else {
      f.x = s[min(i0, n - 1)];
      f.y = s[min(i0 + 1, n - 1)];
      f.z = s[min(i0 + 2, n - 1)];
      f.w = s[min(i0 + 3, n - 1)];
    }
    samp[4 * j] = key_of(f.x);
    samp[4 * j + 1] = key_of(f.y);
    samp[4 * j + 2] = key_of(f.z);
    samp[4 * j + 3] = key_of(f.w);
  }
  __syncthreads();
}

// Sample rank whose key is expected to have ~2.5k + 128 scores of the row at or above it.
__device__ __forceinline__ long long initial_rank(int n, int k) {
  const long long target = min(static_cast<long long>(k) * 5 / 2 + 128, static_cast<long long>(k + kCap) / 2);
  return (static_cast<long long>(kSamples) * target + n - 1) / n;
}

// The float whose key is the rank-th largest sample's key, resolved on its top 16 bits (a little
// below that sample, so the candidates it admits include it).  Ends synchronised.
__device__ __forceinline__ float tau_of_rank(long long rank, const TopkSmem& t) {
  uint32_t dummy;
  const uint32_t tau = smem_select(t.samp, kSamples, static_cast<uint32_t>(rank), 2, t.hist, t.ws, t.sel, &dummy);
  // keys of finite floats are never 0x7FFFFFFF..0, so this inverts key_of on the resolved bits
  return __uint_as_float((tau & 0x80000000u) ? (tau & 0x7FFFFFFFu) : ~tau);
}

// Appends every (key, index) of s[lo, hi) with score >= tau_f to the candidate arrays (unordered;
// t.misc[0] counts them, including any beyond kCap, which are dropped).  lo is a multiple of 4.
// KU independent 16-byte loads per thread are in flight before any of them is used.
template <int KU>
__device__ __forceinline__ void collect(const float* s, int lo, int hi, bool vec, float tau_f, const TopkSmem& t) {
  const int tid = threadIdx.x;
  for (int base = lo; base < hi; base += 4 * kTopkThreads * KU) {
    float v[KU][4];
#pragma unroll
    for (int u = 0; u < KU; ++u) {
      const int i0 = base + 4 * (u * kTopkThreads + tid);
      if (vec && i0 + 3 < hi) {
        const float4 f = __ldcs(reinterpret_cast<const float4*>(s + i0));
        v[u][0] = f.x;
        v[u][1] = f.y;
        v[u][2] = f.z;
        v[u][3] = f.w;
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) v[u][e] = i0 + e < hi ? s[i0 + e] : -INFINITY;
      }
    }
#pragma unroll
    for (int u = 0; u < KU; ++u) {
      const int i0 = base + 4 * (u * kTopkThreads + tid);
      const int nvalid = min(4, max(0, hi - i0));
      const uint32_t hm = ((v[u][0] >= tau_f ? 1u : 0u) | (v[u][1] >= tau_f ? 2u : 0u) |
                           (v[u][2] >= tau_f ? 4u : 0u) | (v[u][3] >= tau_f ? 8u : 0u)) &
                          ((1u << nvalid) - 1u);
#if QSA_TOPK_APPEND == 1
      if (hm) {   // a shared-memory atomic per thread that has candidates
        uint32_t p = atomicAdd(&t.misc[0], static_cast<uint32_t>(__popc(hm)));
#else
      const int lane = tid & 31;
      const uint32_t nh = static_cast<uint32_t>(__popc(hm));
      if (__ballot_sync(0xffffffffu, nh != 0) != 0u) {   // warp-uniform
        uint32_t incl = nh;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        uint32_t wbase = 0;
        if (lane == 31) wbase = atomicAdd(&t.misc[0], incl);
        uint32_t p = __shfl_sync(0xffffffffu, wbase, 31) + incl - nh;
#endif
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if (hm & (1u << e)) {
            if (p < static_cast<uint32_t>(kCap)) {
              t.cand_key[p] = key_of(v[u][e]);
              t.cand_idx[p] = static_cast<uint32_t>(i0 + e);
            }
            ++p;
          }
        }
      }
    }
  }
}

// Steps 3-5 on m candidates (k <= m <= kCap) in t.cand_key / t.cand_idx: the exact k-th key, the
// index cutoff among equal keys, the bitmap of the kept set and its ascending emission.  Returns
// false (nothing written) when more than kSamples candidates equal the k-th key; the caller then
// selects over the row in memory.  All threads call it; starts and ends synchronised.
__device__ bool select_emit(int m, int k, int words, int32_t* out, const TopkSmem& t) {
  const int tid = threadIdx.x;
  uint32_t need_eq;
  const uint32_t kth = smem_select(t.cand_key, m, static_cast<uint32_t>(k), 4, t.hist, t.ws, t.sel, &need_eq);
  const uint32_t n_eq = t.hist[kth & 0xFFu];   // last pass: hits in the K* bin = keys equal to K*
  uint32_t icut = 0xFFFFFFFFu;
  if (need_eq < n_eq) {
    // the need_eq smallest indices among the keys equal to K*: select on ~index among them
    uint32_t* inv = t.samp;   // reuse: up to kSamples entries
    if (tid == 0) t.misc[1] = 0;
    __syncthreads();
    for (int i = tid; i < m; i += kTopkThreads) {
      if (t.cand_key[i] == kth) {
        const uint32_t p = atomicAdd(&t.misc[1], 1u);
        if (p < static_cast<uint32_t>(kSamples)) inv[p] = ~t.cand_idx[i];
      }
    }
    __syncthreads();
    const int ne = static_cast<int>(t.misc[1]);
    __syncthreads();
    if (ne > kSamples) return false;
    uint32_t dummy;
    icut = ~smem_select(inv, ne, need_eq, 4, t.hist, t.ws, t.sel, &dummy);
  }
  for (int wd = tid; wd < words; wd += kTopkThreads) t.bitmap[wd] = 0u;
  __syncthreads();
  for (int i = tid; i < m; i += kTopkThreads) {
    const uint32_t key = t.cand_key[i], id = t.cand_idx[i];
    if (key > kth || (key == kth && id <= icut)) atomicOr(&t.bitmap[id >> 5], 1u << (id & 31));
  }
  __syncthreads();
  const int wpt = (words + kTopkThreads - 1) / kTopkThreads;
  const int w0 = tid * wpt, w1 = min(words, w0 + wpt);
  uint32_t cnt = 0;
  for (int wd = w0; wd < w1; ++wd) cnt += static_cast<uint32_t>(__popc(t.bitmap[wd]));
  uint32_t total;
  uint32_t p = block_excl_scan(cnt, t.ws, &total);
  for (int wd = w0; wd < w1; ++wd) {
    uint32_t bits = t.bitmap[wd];
    while (bits) {
      const int bit = __ffs(bits) - 1;
      bits &= bits - 1;
      if (p < static_cast<uint32_t>(k)) out[p] = wd * 32 + bit;
      ++p;
    }
  }
  __syncthreads();
  return true;
}

// The whole selection of one row with n > k by one CTA (steps 1-5, threshold retries, and the
// radix select over memory as the last resort).
template <int KU>
__device__ void topk_row(const float* s, int n, int k, int words, int bitmap_words, int32_t* out, const TopkSmem& t) {
  const int tid = threadIdx.x;
  if (k >= kCap || words > bitmap_words) {
    topk_global(s, n, k, out, t.hist, t.ws, t.sel);
    return;
  }
  int m = 0;
  if (n <= kCap) {
    for (int i = tid; i < n; i += kTopkThreads) {
      t.cand_key[i] = key_of(s[i]);
      t.cand_idx[i] = static_cast<uint32_t>(i);
    }
    m = n;
    __syncthreads();
  } else {
    load_samples(s, n, t.samp);
    long long rank = initial_rank(n, k);
    const bool vec = ((reinterpret_cast<uintptr_t>(s) & 15u) == 0);
    bool ok = false;
    for (int attempt = 0; attempt < 3 && !ok; ++attempt) {
      rank = max(1ll, min(rank, static_cast<long long>(kSamples)));
      const float tau_f = tau_of_rank(rank, t);
      if (tid == 0) t.misc[0] = 0;
      __syncthreads();
      collect<KU>(s, 0, n, vec, tau_f, t);
      __syncthreads();
      const uint32_t got = t.misc[0];
      __syncthreads();
      if (got >= static_cast<uint32_t>(k) && got <= static_cast<uint32_t>(kCap)) {
        ok = true;
        m = static_cast<int>(got);
      } else if (got < static_cast<uint32_t>(k)) {
        rank *= 4;          // threshold too high: take it lower
      } else {
        rank /= 4;          // too many candidates: take it higher
      }
    }
    if (!ok) {
      topk_global(s, n, k, out, t.hist, t.ws, t.sel);
      return;
    }
  }
  if (!select_emit(m, k, words, out, t)) topk_global(s, n, k, out, t.hist, t.ws, t.sel);
}

// KU: 16-byte loads per thread in flight in the filter pass.  Launches with fewer rows than SMs
// take KU = 16 at one CTA per SM, so a long row is read in few round trips; many-row launches keep
// KU small for three CTAs per SM.
template <int KU, int MINB>
__global__ void __launch_bounds__(kTopkThreads, MINB) topk_kernel(const float* __restrict__ scores, long long ld,
                                                            long long batch_stride, const int32_t* __restrict__ seqlens,
                                                            int Tq, int NBk, int blk, long long q_pos0, int b0,
                                                            int row0, int k, int32_t* __restrict__ idx,
                                                            int bitmap_words, KernelCtl ctl) {
  extern __shared__ uint32_t sm[];
  const TopkSmem t = topk_smem(sm);
  const int tid = threadIdx.x;
  const int r = row0 + static_cast<int>(blockIdx.x);
  const int bz = blockIdx.y;
  const int b = b0 + bz;
  long long pos;
  if (seqlens) {
    pos = static_cast<long long>(seqlens[b]) - 1;
    if (pos < 0 && tid == 0) record_status(ctl, kStBadArg);
  } else {
    pos = q_pos0 + r;
  }
  const int n = pos < 0 ? 0 : static_cast<int>(min(static_cast<long long>(NBk), pos / blk));
  const float* s = scores + static_cast<long long>(bz) * batch_stride + static_cast<long long>(r - row0) * ld;
  int32_t* out = idx + (static_cast<long long>(b) * Tq + r) * k;
  if (n <= k) {
    for (int i = tid; i < k; i += kTopkThreads) out[i] = i < n ? i : -1;
    return;
  }
  topk_row<KU>(s, n, k, (n + 31) >> 5, bitmap_words, out, t);
}

// ======================================================================================
// Warp-per-row variant (used when there are many rows): one warp owns a row end to end, so no
// phase needs a block-wide barrier, and the 16 warps of an SM work on 16 rows at once.
//   1. 1024 samples (32 runs of 32 consecutive scores) give tau, a little below the k-th largest
//      (about 1.8k + 64 scores expected above it; two 8-bit radix passes on the samples);
//   2. one pass over the row (kWU 16-byte loads per lane in flight) appends every score >= tau to
//      the warp's shared-memory list IN INDEX ORDER (ballot-based compaction);
//   3. four 8-bit radix passes over the list give the k-th key K* and how many keys equal to K* are
//      kept (the lowest indices, since the list is in index order);
//   4. one ordered pass over the list emits the kept indices ascending.
// A row whose list would overflow (or hold fewer than k) moves tau by bisection on its sample rank
// and retries; if no rank works (heavy ties) the warp falls back to four radix passes over the
// whole row in memory.
#ifndef QSA_TOPK_WROWS
#define QSA_TOPK_WROWS 8
#endif
constexpr int kWarpRowsPerCta = QSA_TOPK_WROWS;
#ifndef QSA_TOPK_WLOAD
#define QSA_TOPK_WLOAD 0
#endif
#ifndef QSA_TOPK_WU
#define QSA_TOPK_WU 8
#endif
constexpr int kWU = QSA_TOPK_WU;   // 16-byte loads in flight per lane in the filter pass
constexpr int kWSamples = 1024;
// Rows longer than this go to the CTA-per-row kernel, whose filter pass streams faster.
constexpr int kWarpRowMax = 8192;

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Warp-level select, one bit at a time from the top: the krem-th largest of vals[0..m), resolving
// the top 8*passes bits (unresolved low bits returned as zero).  Each bit costs one ballot + popc
// per 32 values (no histogram, no atomics).  *left = how many values equal to the result (on the
// resolved bits) remain to be taken.
__device__ uint32_t warp_select(const uint32_t* vals, int m, uint32_t krem, int passes, uint32_t* hist,
                                uint32_t* left) {
  (void)hist;
  const int lane = threadIdx.x & 31;
  uint32_t prefix = 0;
  const int lowest = 32 - 8 * passes;
  for (int bit = 31; bit >= lowest; --bit) {
    const uint32_t want = (prefix >> bit) | 1u;   // top bits of prefix with this bit set
    uint32_t cnt = 0;
    for (int base = 0; base < m; base += 32) {
      const int i = base + lane;
      const bool hit = i < m && (vals[i] >> bit) == want;
      cnt += __popc(__ballot_sync(0xffffffffu, hit));
    }
    if (cnt >= krem)
      prefix |= 1u << bit;
    else
      krem -= cnt;
  }
  *left = krem;
  return prefix;
}

__global__ void __launch_bounds__(kWarpRowsPerCta * 32) topk_warp_kernel(
    const float* __restrict__ scores, long long ld, long long batch_stride, int Tq, int NBk, long long q_pos0, int b0,
    int row0, int rows, int k, int cap, int32_t* __restrict__ idx) {
  extern __shared__ uint32_t smw[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint32_t* ckey = smw + warp * (2 * cap + 256);   // cap keys, then cap indices, then 256 hist words
  uint32_t* cidx = ckey + cap;
  uint32_t* hist = cidx + cap;
  const int r = row0 + static_cast<int>(blockIdx.x) * kWarpRowsPerCta + warp;
  if (r >= row0 + rows) return;
  const int bz = blockIdx.y;
  const int b = b0 + bz;
  const long long pos = q_pos0 + r;
  const int n = static_cast<int>(min(static_cast<long long>(NBk), pos / 4));
  const float* s = scores + static_cast<long long>(bz) * batch_stride + static_cast<long long>(r - row0) * ld;
  int32_t* out = idx + (static_cast<long long>(b) * Tq + r) * k;
  if (n <= k) {
    for (int i = lane; i < k; i += 32) out[i] = i < n ? i : -1;
    return;
  }
  const bool vec = (reinterpret_cast<uintptr_t>(s) & 15u) == 0;
  const uint32_t lt = lanemask_lt();

  // ---- candidates in index order
  float tau_f = -INFINITY;
  int m = 0;
  bool ok = false;
  // rank of tau among the samples: a larger rank gives a lower tau and more candidates.  A failed
  // pass narrows (rlo, rhi), the open interval that must hold a working rank.
  long long rank = 0, rlo = 0, rhi = kWSamples + 1;
  auto draw_samples = [&]() {
#pragma unroll 4
    for (int run = 0; run < 32; ++run) {
      const int i = static_cast<int>((static_cast<long long>(run) * (n - 32)) / 31) + lane;
      ckey[run * 32 + lane] = key_of(s[i]);
    }
    __syncwarp();
  };
  if (n > cap) {
    draw_samples();
    const long long target = (9ll * k) / 5 + 64;
    rank = (static_cast<long long>(kWSamples) * target + n - 1) / n;
  }
  for (int attempt = 0; attempt < 6 && !ok; ++attempt) {
    if (n > cap) {
      rank = max(rlo + 1, min(rank, rhi - 1));
      if (rank <= rlo || rank >= rhi) break;   // no rank left to try
      uint32_t dummy;
      const uint32_t tau = warp_select(ckey, kWSamples, static_cast<uint32_t>(rank), 2, hist, &dummy);
      tau_f = __uint_as_float((tau & 0x80000000u) ? (tau & 0x7FFFFFFFu) : ~tau);
    }
    uint32_t cnt = 0;
    bool over = false;
    for (int base = 0; base < n; base += 128 * kWU) {
      float v[kWU][4];
#pragma unroll
      for (int u = 0; u < kWU; ++u) {
        const int i0 = base + (u * 32 + lane) * 4;
        if (vec && i0 + 3 < n) {
#if QSA_TOPK_WLOAD == 1
          const float4 f = __ldg(reinterpret_cast<const float4*>(s + i0));
#else
          const float4 f = __ldcs(reinterpret_cast<const float4*>(s + i0));
#endif
          v[u][0] = f.x;
          v[u][1] = f.y;
          v[u][2] = f.z;
          v[u][3] = f.w;
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e) v[u][e] = i0 + e < n ? s[i0 + e] : -INFINITY;
        }
      }
#pragma unroll
      for (int u = 0; u < kWU; ++u) {
        const int i0 = base + (u * 32 + lane) * 4;
        uint32_t hm = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) hm |= (i0 + e < n && v[u][e] >= tau_f ? 1u : 0u) << e;
        const uint32_t m0 = __ballot_sync(0xffffffffu, hm & 1u), m1 = __ballot_sync(0xffffffffu, hm & 2u);
        const uint32_t m2 = __ballot_sync(0xffffffffu, hm & 4u), m3 = __ballot_sync(0xffffffffu, hm & 8u);
        const uint32_t total = __popc(m0) + __popc(m1) + __popc(m2) + __popc(m3);
        if (total == 0) continue;
        uint32_t p = cnt + __popc(m0 & lt) + __popc(m1 & lt) + __popc(m2 & lt) + __popc(m3 & lt);
        if (cnt + total <= static_cast<uint32_t>(cap)) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            if (hm & (1u << e)) {
              ckey[p] = key_of(v[u][e]);
              cidx[p] = static_cast<uint32_t>(i0 + e);
              ++p;
            }
          }
        } else {
          over = true;
        }
        cnt += total;
      }
      if (over) break;   // warp-uniform
    }
    __syncwarp();
    if (!over && cnt >= static_cast<uint32_t>(k)) {
      ok = true;
      m = static_cast<int>(cnt);
    } else if (n > cap) {
      draw_samples();   // the list overwrote them
      if (over) {
        rhi = rank;
        rank = (rlo + rank) / 2;
      } else {
        rlo = rank;
        rank = rhi > kWSamples ? rank * 2 : (rank + rhi) / 2;
      }
    } else {
      break;
    }
  }

  uint32_t kth, need_eq;
  if (ok) {
    kth = warp_select(ckey, m, static_cast<uint32_t>(k), 4, hist, &need_eq);
  } else {
    // fallback: four radix passes over the row in memory
    uint32_t prefix = 0, pmask = 0, krem = static_cast<uint32_t>(k);
    for (int pass = 0; pass < 4; ++pass) {
      const int shift = 24 - 8 * pass;
#pragma unroll
      for (int q = 0; q < 8; ++q) hist[lane * 8 + q] = 0;
      __syncwarp();
      for (int base = 0; base < n; base += 32) {
        const int i = base + lane;
        const uint32_t key = i < n ? key_of(s[i]) : 0u;
        const bool hit = i < n && (key & pmask) == prefix;
        const uint32_t digit = (key >> shift) & 0xFFu;
        const uint32_t peers = __match_any_sync(0xffffffffu, hit ? digit : 0xFFFFFFFFu);
        if (hit && lane == __ffs(peers) - 1) hist[digit] += static_cast<uint32_t>(__popc(peers));
        __syncwarp();
      }
      const uint32_t* hp = hist + lane * 8;
      uint32_t local = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) local += hp[q];
      uint32_t incl = local;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_down_sync(0xffffffffu, incl, o);
        if (lane + o < 32) incl += y;
      }
      const uint32_t above = incl - local;
      uint32_t mybin = 0, myabove = 0;
      const bool mine = above < krem && above + local >= krem;
      if (mine) {
        uint32_t acc = above;
        for (int q = 7; q >= 0; --q) {
          if (acc + hp[q] >= krem) {
            mybin = static_cast<uint32_t>(lane * 8 + q);
            myabove = acc;
            break;
          }
          acc += hp[q];
        }
      }
      const int src = __ffs(__ballot_sync(0xffffffffu, mine)) - 1;
      prefix |= __shfl_sync(0xffffffffu, mybin, src) << shift;
      krem -= __shfl_sync(0xffffffffu, myabove, src);
      pmask |= 0xFFu << shift;
      __syncwarp();
    }
    kth = prefix;
    need_eq = krem;
  }

  // ---- ordered emission (the list, or the whole row on the fallback, is in index order)
  uint32_t out_run = 0, eq_run = 0;
  const int len = ok ? m : n;
  for (int base = 0; base < len; base += 32) {
    const int i = base + lane;
    uint32_t key = 0, id = 0;
    if (i < len) {
      if (ok) {
        key = ckey[i];
        id = cidx[i];
      } else {
        key = key_of(s[i]);
        id = static_cast<uint32_t>(i);
      }
    }
    const bool gt = i < len && key > kth;
    const bool eq = i < len && key == kth;
    const uint32_t eqm = __ballot_sync(0xffffffffu, eq);
    const uint32_t eq_rank = eq_run + __popc(eqm & lt);
    const bool keep = gt || (eq && eq_rank < need_eq);
    const uint32_t km = __ballot_sync(0xffffffffu, keep);
    if (keep) {
      const uint32_t p = out_run + __popc(km & lt);
      if (p < static_cast<uint32_t>(k)) out[p] = static_cast<int32_t>(id);
    }
    out_run += __popc(km);
    eq_run += __popc(eqm);
  }
}

// ======================================================================================
// Decode (few long rows): a thread-block cluster of P CTAs per sequence row (grid P x rows,
// cluster P x 1).  Each CTA
//   1. issues the loads of its slice of the row (a quarter, an eighth ...) and of 2048 samples of
//      the whole row (16 runs of 128), so the slice is on its way while the threshold is found;
//   2. finds the threshold from the samples as every CTA of the row does, with the same result:
//      an 11-bit histogram over the bits where the sampled keys differ; tau = the lowest key of
//      the bin holding the rank-th largest sample (~2.5 k + 128 of the row's scores expected above
//      it); rows of at most kCCap blocks keep every block;
//   3. appends the slice's (key, block) pairs with key >= tau to its shared-memory list IN BLOCK
//      ORDER (ballot compaction, one CTA-wide scan of the warps' counts per round of loads).
// After a cluster barrier, CTA 0 reads every slice's count and list through distributed shared
// memory (the slices in order, so the merged list is in block order), a second cluster barrier
// releases the other CTAs, and CTA 0 selects exactly over the merged list: an 11-bit histogram
// over the bits where the listed keys differ finds the bin of the k-th largest key, the bin's keys
// are resolved bit by bit (warp 0), and {key > K*} U {the first need_eq keys == K*} is emitted in
// list order.  If the lists together hold fewer than k or more than kCCap entries (heavy ties),
// CTA 0 selects over the row in memory instead (three radix passes), so the result never depends
// on the threshold.
constexpr int kCT = kTopkThreads;          // threads per CTA (512)
constexpr int kCWarps = kCT / 32;
constexpr int kCCap = 6144;                // list capacity of a slice, and of the merged list
constexpr int kCU = kCCap / kCT;           // merged entries per thread of CTA 0 (12)
constexpr int kCLoads = 8;                 // 16-byte loads per thread per round (16384 scores)
constexpr int kCSmem = kBins * 4 + kCCap * 8 + (kCLoads * kCWarps + 2 * kCWarps + 2 + 4 + 4) * 4;

// Block-wide min and max (ws: 2 * kCWarps words).  Ends synchronised.
__device__ __forceinline__ void block_minmax512(uint32_t& kmin, uint32_t& kmax, uint32_t* ws) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  if (lane == 0) {
    ws[2 * warp] = kmin;
    ws[2 * warp + 1] = kmax;
  }
  __syncthreads();
#pragma unroll
  for (int w = 0; w < kCWarps; ++w) {
    kmin = min(kmin, ws[2 * w]);
    kmax = max(kmax, ws[2 * w + 1]);
  }
  __syncthreads();
}

// The bin of 2048 (4 per thread, thread t holding bins 4t .. 4t + 3) that holds the rank-th
// largest hit, with two barriers: sel[0] = bin, sel[1] = hits in the bins above it.  ws: kCWarps
// words.  Ends synchronised.
__device__ __forceinline__ void find_bin2(const uint32_t* hist, uint32_t rank, uint32_t* ws, uint32_t* sel) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint4 h4 = *reinterpret_cast<const uint4*>(hist + 4 * tid);
  const uint32_t local = h4.x + h4.y + h4.z + h4.w;
  uint32_t incl = local;   // this lane's bins and those of the higher lanes of the warp
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_down_sync(0xffffffffu, incl, o);
    if (lane + o < 32) incl += y;
  }
  if (lane == 0) ws[warp] = incl;   // the warp's total
  __syncthreads();
  uint32_t above = incl - local;     // hits in the bins above this thread's four
#pragma unroll
  for (int w = 0; w < kCWarps; ++w) above += w > warp ? ws[w] : 0u;
  if (above < rank && above + local >= rank) {
    const uint32_t hb[4] = {h4.x, h4.y, h4.z, h4.w};
    uint32_t acc = above;
#pragma unroll
    for (int q = 3; q >= 0; --q) {
      if (acc < rank && acc + hb[q] >= rank) {
        sel[0] = static_cast<uint32_t>(4 * tid + q);
        sel[1] = acc;
      }
      acc += hb[q];
    }
  }
  __syncthreads();
}

// Round of slice loads: element i0 + e of load u, i0 = r0 + 4 (u kCT + tid); beyond hi: -inf.
__device__ __forceinline__ void load_round(float4 (&v)[kCLoads], const float* s, int r0, int hi, bool vec) {
#pragma unroll
  for (int u = 0; u < kCLoads; ++u) {
    const int i0 = r0 + 4 * (u * kCT + static_cast<int>(threadIdx.x));
    if (vec && i0 + 3 < hi) {
      v[u] = __ldcs(reinterpret_cast<const float4*>(s + i0));
    } else {
      v[u].x = i0 < hi ? s[i0] : -INFINITY;
      v[u].y = i0 + 1 < hi ? s[i0 + 1] : -INFINITY;
      v[u].z = i0 + 2 < hi ? s[i0 + 2] : -INFINITY;
      v[u].w = i0 + 3 < hi ? s[i0 + 3] : -INFINITY;
    }
  }
}

__global__ void __launch_bounds__(kCT, 1) topk_cluster_kernel(const float* __restrict__ scores, long long ld,
                                                            const int32_t* __restrict__ seqlens, int NBk, int blk,
                                                            int k, int32_t* __restrict__ idx, KernelCtl ctl) {
  extern __shared__ __align__(16) uint8_t csm[];
  uint32_t* hist = reinterpret_cast<uint32_t*>(csm);                        // kBins
  uint2* list = reinterpret_cast<uint2*>(csm + kBins * 4);                  // kCCap
  uint32_t* wcnt = reinterpret_cast<uint32_t*>(csm + kBins * 4 + kCCap * 8);  // kCLoads x kCWarps
  uint32_t* ws = wcnt + kCLoads * kCWarps;                                  // 2 kCWarps + 2
  uint32_t* sel = ws + 2 * kCWarps + 2;                                     // 4
  uint32_t* misc = sel + 4;                                                 // [0]: the slice's count
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t lt = lanemask_lt();
  const uint32_t part = cluster_rank();
  const int P = static_cast<int>(gridDim.x);
  const int b = blockIdx.y;
  const long long pos = static_cast<long long>(seqlens[b]) - 1;
  if (pos < 0 && tid == 0 && part == 0) record_status(ctl, kStBadArg);
  const int n = pos < 0 ? 0 : static_cast<int>(min(static_cast<long long>(NBk), pos / blk));
  const float* s = scores + static_cast<long long>(b) * ld;
  int32_t* out = idx + static_cast<long long>(b) * k;
  if (n <= k) {   // uniform over the cluster: no cluster barrier is reached
    if (part == 0)
      for (int i = tid; i < k; i += kCT) out[i] = i < n ? i : -1;
    return;
  }
  const bool vec = (reinterpret_cast<uintptr_t>(s) & 15u) == 0;
  const bool keep_every = n <= kCCap;   // every block is a candidate
  const int chunk = ((n + P - 1) / P + 3) & ~3;
  const int lo = min(n, static_cast<int>(part) * chunk), hi = min(n, lo + chunk);

  // ---- 1. the samples, then the slice's first round, in flight together (the samples first: the
  // threshold needs only them and is found while the slice is still arriving)
  float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
  if (!keep_every) {
    const int run = tid >> 5, off = (tid & 31) * 4;
    const int i0 = (static_cast<int>((static_cast<long long>(run) * n) / (kSamples / 128)) & ~3) + off;  // i0 + 3 < n
    if (vec) {
      f = __ldcs(reinterpret_cast<const float4*>(s + i0));
    } else {
      f.x = s[i0];
      f.y = s[i0 + 1];
      f.z = s[i0 + 2];
      f.w = s[i0 + 3];
    }
  }
  float4 v[kCLoads];
  load_round(v, s, lo, hi, vec);
  for (int i = tid * 4; i < kBins; i += kCT * 4) *reinterpret_cast<uint4*>(hist + i) = make_uint4(0u, 0u, 0u, 0u);
  if (tid == 0) {
    misc[2] = 0xFFFFFFFFu;   // this slice's smallest and largest candidate key
    misc[3] = 0u;
  }

  // ---- 2. threshold key
  uint32_t tkey = 0u;   // every key is >= 0
  if (!keep_every) {
    const uint32_t sk[4] = {key_of(f.x), key_of(f.y), key_of(f.z), key_of(f.w)};
    uint32_t kmin = min(min(sk[0], sk[1]), min(sk[2], sk[3]));
    uint32_t kmax = max(max(sk[0], sk[1]), max(sk[2], sk[3]));
    block_minmax512(kmin, kmax, ws);   // also orders the histogram's clearing before its use
    if (kmin == kmax) {
      tkey = kmin;
    } else {
      const int hb = 31 - __clz(kmin ^ kmax);
      const int sh = max(0, hb - 10);
#pragma unroll
      for (int e = 0; e < 4; ++e) atomicAdd(&hist[(sk[e] >> sh) & (kBins - 1)], 1u);
      __syncthreads();
      const long long target = min(static_cast<long long>(k) * 5 / 2 + 128, static_cast<long long>(k + kCCap) / 2);
      const long long rank = max(1ll, min(static_cast<long long>(kSamples), (kSamples * target + n - 1) / n));
      find_bin2(hist, static_cast<uint32_t>(rank), ws, sel);   // ends synchronised
      const uint32_t hi_mask = (sh + 11 >= 32) ? 0u : (0xFFFFFFFFu << (sh + 11));
      tkey = (kmax & hi_mask) | (sel[0] << sh);
    }
  }
  __syncthreads();   // misc[2..3] initialised (keep_every reaches no barrier above)

  // ---- 3. the slice's candidates, in block order, into this CTA's list
  const float tau_f = keep_every ? -INFINITY : key_to_float(tkey);   // key_of(x) >= tkey <=> x >= tau_f
  uint32_t count = 0;   // entries of the earlier rounds
  for (int r0 = lo; r0 < hi; r0 += 4 * kCT * kCLoads) {
    if (r0 != lo) load_round(v, s, r0, hi, vec);
    uint32_t hm[kCLoads], lp[kCLoads];
#pragma unroll
    for (int u = 0; u < kCLoads; ++u) {
      const int i0 = r0 + 4 * (u * kCT + tid);
      const uint32_t m = (v[u].x >= tau_f && i0 < hi ? 1u : 0u) | (v[u].y >= tau_f && i0 + 1 < hi ? 2u : 0u) |
                         (v[u].z >= tau_f && i0 + 2 < hi ? 4u : 0u) | (v[u].w >= tau_f && i0 + 3 < hi ? 8u : 0u);
      uint32_t before = 0, wc = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t bal = __ballot_sync(0xffffffffu, (m >> e) & 1u);
        before += static_cast<uint32_t>(__popc(bal & lt));
        wc += static_cast<uint32_t>(__popc(bal));
      }
      hm[u] = m;
      lp[u] = before;   // hits of the lower lanes of this warp in this load
      if (lane == 0) wcnt[u * kCWarps + warp] = wc;
    }
    __syncthreads();
    if (warp == 0) {   // exclusive scan of the kCLoads x kCWarps counts, (load, warp) order
      constexpr int kPer = kCLoads * kCWarps / 32;
      uint32_t c[kPer], sum = 0;
#pragma unroll
      for (int q = 0; q < kPer; ++q) {
        c[q] = wcnt[lane * kPer + q];
        sum += c[q];
      }
      uint32_t incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      uint32_t run = incl - sum;
#pragma unroll
      for (int q = 0; q < kPer; ++q) {
        wcnt[lane * kPer + q] = run;
        run += c[q];
      }
      if (lane == 31) misc[1] = incl;   // the round's total
    }
    __syncthreads();
    uint32_t cmin = 0xFFFFFFFFu, cmax = 0u;   // this thread's candidate keys
#pragma unroll
    for (int u = 0; u < kCLoads; ++u) {
      uint32_t mm = hm[u];
      if (mm == 0u) continue;   // most loads hold no candidate
      const int i0 = r0 + 4 * (u * kCT + tid);
      uint32_t p = count + wcnt[u * kCWarps + warp] + lp[u];
      while (mm) {
        const int e = __ffs(mm) - 1;
        mm &= mm - 1;
        const float x = e == 0 ? v[u].x : e == 1 ? v[u].y : e == 2 ? v[u].z : v[u].w;
        const uint32_t key = key_of(x);
        cmin = min(cmin, key);
        cmax = max(cmax, key);
        if (p < static_cast<uint32_t>(kCCap)) list[p] = make_uint2(key, static_cast<uint32_t>(i0 + e));
        ++p;
      }
    }
    cmin = __reduce_min_sync(0xffffffffu, cmin);
    cmax = __reduce_max_sync(0xffffffffu, cmax);
    if (lane == 0 && cmax >= cmin) {
      atomicMin(&misc[2], cmin);
      atomicMax(&misc[3], cmax);
    }
    count += misc[1];
    __syncthreads();   // wcnt and misc[1] are rewritten by the next round
  }
  if (tid == 0) misc[0] = count;

  // ---- 4. merge in CTA 0
  cluster_sync_all();
  if (part != 0) {
    cluster_sync_all();   // CTA 0 has read this CTA's list
    return;
  }
  uint32_t base[8], total = 0, kmin = 0xFFFFFFFFu, kmax = 0u;
  bool fits = true;
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    uint32_t cp = 0u;
    if (p < P) {
      const uint32_t a = cluster_addr(misc, p);
      cp = ld_cluster_u32(a);
      kmin = min(kmin, ld_cluster_u32(a + 8));
      kmax = max(kmax, ld_cluster_u32(a + 12));
    }
    fits = fits && cp <= static_cast<uint32_t>(kCCap);
    base[p] = total;
    total += cp;
  }
  const bool ok = fits && total >= static_cast<uint32_t>(k) && total <= static_cast<uint32_t>(kCCap);
  // merged entry j = tid + kCT u (round u of R): (key, block), in block order over (u, tid)
  const int c = ok ? static_cast<int>(total) : 0;
  const int R = (c + kCT - 1) / kCT;   // uniform
  uint2 ent[kCU];
#pragma unroll
  for (int u = 0; u < kCU; ++u) {
    ent[u] = make_uint2(0u, 0u);
    const uint32_t j = static_cast<uint32_t>(tid + u * kCT);
    if (u < R && j < static_cast<uint32_t>(c)) {
      uint32_t p = 0, rel = j;   // the slice holding merged entry j, and j's place in it
#pragma unroll
      for (int q = 1; q < 8; ++q) {
        if (q < P && j >= base[q]) {
          p = static_cast<uint32_t>(q);
          rel = j - base[q];
        }
      }
      ent[u] = ld_cluster_v2(cluster_addr(list + rel, p));
    }
  }
  cluster_sync_all();
  if (!ok) {
    topk_global(s, n, k, out, hist, ws, sel);
    return;
  }
  auto valid = [&](int u) { return u < R && tid + u * kCT < c; };
  bool keep_all = false;
  uint32_t kth = 0, need_eq = 0;
  if (c == k) {
    keep_all = true;
  } else {
    if (kmin == kmax) {   // the listed keys' range, from the slices' own minima and maxima
      kth = kmin;
      need_eq = static_cast<uint32_t>(k);
    } else {
      const int hb = 31 - __clz(kmin ^ kmax);
      const int sh = max(0, hb - 10);
      for (int i = tid * 4; i < kBins; i += kCT * 4) *reinterpret_cast<uint4*>(hist + i) = make_uint4(0u, 0u, 0u, 0u);
      __syncthreads();
#pragma unroll
      for (int u = 0; u < kCU; ++u)
        if (valid(u)) atomicAdd(&hist[(ent[u].x >> sh) & (kBins - 1)], 1u);
      __syncthreads();
      find_bin2(hist, static_cast<uint32_t>(k), ws, sel);
      const uint32_t B = sel[0];
      uint32_t krem = static_cast<uint32_t>(k) - sel[1];
      const uint32_t hi_mask = (sh + 11 >= 32) ? 0u : (0xFFFFFFFFu << (sh + 11));
      uint32_t prefix = (kmax & hi_mask) | (B << sh);   // listed keys share the bits above sh + 10
      if (sh > 0) {
        const uint32_t inbin = hist[B];   // <= c <= kCCap
        if (tid == 0) sel[2] = 0;
        __syncthreads();   // every thread has read hist[B]: the space now gathers the bin's keys
        uint32_t* buf = hist;   // kBins + 2 kCCap words (the histogram and this CTA's list) >= kCCap
#pragma unroll
        for (int u = 0; u < kCU; ++u)
          if (valid(u) && ((ent[u].x >> sh) & (kBins - 1)) == B) buf[atomicAdd(&sel[2], 1u)] = ent[u].x;
        __syncthreads();
        if (warp == 0) {
          const int mb = static_cast<int>(inbin);
          if (mb <= 32) {   // the usual case: the bin's keys in registers, one ballot per bit
            const bool have = lane < mb;
            const uint32_t key = have ? buf[lane] : 0u;
            for (int bit = sh - 1; bit >= 0; --bit) {
              const uint32_t want = (prefix >> bit) | 1u;
              const uint32_t cntb = __popc(__ballot_sync(0xffffffffu, have && (key >> bit) == want));
              if (cntb >= krem)
                prefix |= 1u << bit;
              else
                krem -= cntb;
            }
          } else {
            for (int bit = sh - 1; bit >= 0; --bit) {
              const uint32_t want = (prefix >> bit) | 1u;
              uint32_t cntb = 0;
              for (int i0 = 0; i0 < mb; i0 += 32) {
                const int i = i0 + lane;
                cntb += __popc(__ballot_sync(0xffffffffu, i < mb && (buf[i] >> bit) == want));
              }
              if (cntb >= krem)
                prefix |= 1u << bit;
              else
                krem -= cntb;
            }
          }
          if (lane == 0) {
            sel[0] = prefix;
            sel[1] = krem;
          }
        }
        __syncthreads();
        prefix = sel[0];
        krem = sel[1];
      }
      kth = prefix;
      need_eq = krem;
    }
  }
  // ordered emission: per round a warp scan of (entries > K*, entries == K*), one exchange of the
  // warps' round totals (in the list, no longer needed), then every kept entry's position
  uint32_t* xs = reinterpret_cast<uint32_t*>(list);   // [kCU][kCWarps]
  uint32_t pk[kCU], incl[kCU];
#pragma unroll
  for (int u = 0; u < kCU; ++u) {
    pk[u] = incl[u] = 0u;
    if (u < R) {   // uniform
      const bool val = valid(u);
      const bool gt = val && (keep_all || ent[u].x > kth), eq = val && !keep_all && ent[u].x == kth;
      pk[u] = (gt ? 0x10000u : 0u) | (eq ? 1u : 0u);
      uint32_t x = pk[u];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      incl[u] = x;
      if (lane == 31) xs[u * kCWarps + warp] = x;
    }
  }
  __syncthreads();
  uint32_t gt_tot = 0, eq_tot = 0;   // entries of the earlier rounds
#pragma unroll
  for (int u = 0; u < kCU; ++u) {
    if (u >= R) break;   // uniform
    uint32_t before = 0, all = 0;
#pragma unroll
    for (int w = 0; w < kCWarps; ++w) {
      const uint32_t t = xs[u * kCWarps + w];
      before += w < warp ? t : 0u;
      all += t;
    }
    const uint32_t ex = before + incl[u] - pk[u];
    const uint32_t gt_run = gt_tot + (ex >> 16), eq_run = eq_tot + (ex & 0xFFFFu);
    if (pk[u] >> 16) {
      const uint32_t p = gt_run + min(eq_run, need_eq);
      if (p < static_cast<uint32_t>(k)) out[p] = static_cast<int32_t>(ent[u].y);
    } else if (pk[u] & 1u) {
      if (eq_run < need_eq && gt_run + eq_run < static_cast<uint32_t>(k)) out[gt_run + eq_run] = static_cast<int32_t>(ent[u].y);
    }
    gt_tot += all >> 16;
    eq_tot += all & 0xFFFFu;
  }
}

// ======================================================================================
// Exact redo of the rows that the filtered selection could not settle (list shorter than k, or
// overflowing): one CTA per failed row at a time, grid-striding over the failure list
// fail[1 .. fail[0]].  The row's scores are recomputed on CUDA cores in fp32 into the CTA's
// scratch row (same formula: ReLU or linear per head, weighted sum), then selected exactly by the
// three-pass radix select over memory.  With no failure the kernel only reads fail[0].
__global__ void __launch_bounds__(kTopkThreads) topk_fallback_kernel(
    const uint16_t* __restrict__ qi, const uint16_t* __restrict__ kp, const float* __restrict__ head_w, int Hi,
    int mode, int Tq, int NBk, long long q_pos0, int b, const int* __restrict__ fail, float* __restrict__ scratch,
    int k, int32_t* __restrict__ idx) {
  __shared__ float qf[8 * 64];
  __shared__ uint32_t hist[kBins];
  __shared__ uint32_t ws[kWarps + 1];
  __shared__ uint32_t sel[2];
  const int tid = threadIdx.x;
  const int nf = fail[0];
  float* s = scratch + static_cast<long long>(blockIdx.x) * NBk;
  float w[8];
#pragma unroll
  for (int h = 0; h < 8; ++h) w[h] = h < Hi ? (head_w ? head_w[h] : 1.0f) : 0.0f;
  for (int f = blockIdx.x; f < nf; f += gridDim.x) {
    const int t = fail[1 + f];
    const int n = static_cast<int>(min(static_cast<long long>(NBk), (q_pos0 + t) >> 2));
    const uint16_t* qrow = qi + (static_cast<long long>(b) * Tq + t) * Hi * 64;
    for (int i = tid; i < Hi * 64; i += kTopkThreads) qf[i] = __uint_as_float(static_cast<uint32_t>(qrow[i]) << 16);
    __syncthreads();
    for (int j = tid; j < n; j += kTopkThreads) {
      const uint4* kr = reinterpret_cast<const uint4*>(kp + (static_cast<long long>(b) * NBk + j) * 64);
      float acc[8];
#pragma unroll
      for (int h = 0; h < 8; ++h) acc[h] = 0.0f;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint4 v = __ldg(kr + c);
        const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float x = __uint_as_float((e & 1) ? (wd[e >> 1] & 0xFFFF0000u) : (wd[e >> 1] << 16));
#pragma unroll
          for (int h = 0; h < 8; ++h)
            if (h < Hi) acc[h] = fmaf(qf[h * 64 + c * 8 + e], x, acc[h]);
        }
      }
      float sc = 0.0f;
#pragma unroll
      for (int h = 0; h < 8; ++h) {
        if (h < Hi) {
          const float x = mode == 0 ? fmaxf(acc[h], 0.0f) : acc[h];
          sc = fmaf(w[h], x, sc);
        }
      }
      s[j] = sc;
    }
    __syncthreads();
    topk_global(s, n, k, idx + (static_cast<long long>(b) * Tq + t) * k, hist, ws, sel);
    __syncthreads();
  }
}

}  // namespace

cudaError_t launch_topk(const DeviceInfo* di, const float* scores, long long ld, long long batch_stride,
                        const int32_t* seqlens, int Tq, int NBk, int blk, long long q_pos0, int b0, int nb, int row0,
                        int rows, int k, int32_t* idx, cudaStream_t s) {
  if (rows <= 0 || nb <= 0) return cudaSuccess;
  static std::once_flag once[64];
  std::call_once(once[di->device & 63], [] {
    cudaFuncSetAttribute(topk_kernel<QSA_TOPK_LOADS, 3>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         kFixedSmem + 32 + kMaxBitmapWords * 4);
    cudaFuncSetAttribute(topk_kernel<16, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         kFixedSmem + 32 + kMaxBitmapWords * 4);
  });
  // Many short rows (early prefill chunks): one warp per row.  Long rows or few rows (late chunks,
  // decode): one CTA per row.
  const int cap = std::max(3 * k, kWSamples);
  const int warp_smem = kWarpRowsPerCta * (2 * cap + 256) * 4;
  const long long n_max = std::min<long long>(NBk, (q_pos0 + row0 + rows - 1) / blk);
  if (seqlens == nullptr && static_cast<long long>(rows) * nb >= 8ll * di->num_sms && warp_smem <= 200 * 1024 &&
      n_max <= kWarpRowMax) {
    static std::once_flag wonce[64];
    std::call_once(wonce[di->device & 63], [] {
      cudaFuncSetAttribute(topk_warp_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    });
    dim3 wgrid((rows + kWarpRowsPerCta - 1) / kWarpRowsPerCta, nb);
    topk_warp_kernel<<<wgrid, kWarpRowsPerCta * 32, warp_smem, s>>>(scores, ld, batch_stride, Tq, NBk, q_pos0, b0,
                                                                    row0, rows, k, cap, idx);
    return cudaPeekAtLastError();
  }
  const int words = std::min(kMaxBitmapWords, (std::max(NBk, 1) + 31) / 32);
  const int smem = kFixedSmem + 32 + words * 4;
  dim3 grid(rows, nb);
  if (static_cast<long long>(rows) * nb < di->num_sms)
    topk_kernel<16, 1><<<grid, kTopkThreads, smem, s>>>(scores, ld, batch_stride, seqlens, Tq, NBk, blk, q_pos0, b0,
                                                         row0, k, idx, words, kernel_ctl(di));
  else
    topk_kernel<QSA_TOPK_LOADS, 3><<<grid, kTopkThreads, smem, s>>>(scores, ld, batch_stride, seqlens, Tq, NBk, blk,
                                                                     q_pos0, b0, row0, k, idx, words, kernel_ctl(di));
  return cudaPeekAtLastError();
}

int topk_cluster_parts(const DeviceInfo* di, int B, int NBk, int k) {
  if (B < 1 || k > 1024 || NBk <= kCCap) return 0;
  const int p = std::min(8, di->num_sms / B);
  return p >= 2 ? p : 0;
}

cudaError_t launch_topk_cluster(const DeviceInfo* di, const float* scores, long long ld, const int32_t* seqlens, int B,
                                int NBk, int blk, int k, int32_t* idx, int parts, cudaStream_t s) {
  if (B <= 0) return cudaSuccess;
  if (parts < 1 || parts > 8) return cudaErrorInvalidValue;
  static std::once_flag once[64];
  std::call_once(once[di->device & 63], [] {
    cudaFuncSetAttribute(topk_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kCSmem);
  });
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(parts), static_cast<unsigned>(B), 1);
  cfg.blockDim = dim3(kCT, 1, 1);
  cfg.dynamicSmemBytes = kCSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(parts);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, topk_cluster_kernel, scores, ld, seqlens, NBk, blk, k, idx, kernel_ctl(di));
}

cudaError_t launch_topk_fallback(const DeviceInfo* di, const void* qi, const void* kp, const float* head_w, int Hi,
                                 int mode, int Tq, int NBk, long long q_pos0, int b, const int* fail, float* scratch,
                                 int nctas, int k, int32_t* idx, cudaStream_t s) {
  (void)di;
  if (nctas <= 0) return cudaSuccess;
  topk_fallback_kernel<<<nctas, kTopkThreads, 0, s>>>(static_cast<const uint16_t*>(qi),
                                                      static_cast<const uint16_t*>(kp), head_w, Hi, mode, Tq, NBk,
                                                      q_pos0, b, fail, scratch, k, idx);
  return cudaPeekAtLastError();
}

}  // namespace qsa
