// Top-k selection from a filtered candidate list (prefill), the path that never writes the full
// score matrix.
//
// "Qwen3.8-Flash-Next architecture" (flozi.net), "Der Weg eines Tokens durch das Modell", item 2:
// every query keeps the 512 best-scoring micro-blocks among those it may see.  Reading fixed in
// qsa.h: the top-k of the fp32 scores, equal scores to the lower block index, ascending output.
//
// The selection runs in four steps per chunk of query rows:
//   1. sampled scores: the score of every 16th pooled block (the tensor-core score kernel on a
//      strided map of the pooled keys);
//   2. tau_kernel: per row, a threshold tau at or just below the rank-r sampled score, so that
//      about 16 r of the row's scores are expected at or above it (r ~ 2.5 k / 16, at least 64);
//   3. the score + filter kernel appends every score >= tau, in block order, to the row's list;
//   4. cand_select_kernel: the exact k-th key of the list and the kept set, emitted ascending.
// The result equals the top-k of the whole row whenever the list holds at least k entries and did
// not overflow: every block left out scores below tau, hence below k listed scores.  A row that
// fails either test is appended to a failure list and redone exactly by topk_fallback_kernel
// (scores recomputed on CUDA cores, radix select over the whole row).
#include <algorithm>
#include <mutex>

#include "launch.h"

namespace qsa {
namespace {

constexpr int kTauWarps = 4;
constexpr int kTauBins = 2048;    // bins over the bits where a row's sampled keys differ
constexpr int kSelWarps = 4;
constexpr int kSelBins = 2048;    // bins of the first select pass (11 bits)
constexpr int kSelSmemMax = 200 * 1024;

__device__ __forceinline__ uint32_t lane_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

__device__ __forceinline__ float key_to_float(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// Finds, over bins numbered 0..nbins-1 (a larger bin holds larger keys), the bin holding the
// rank-th largest entry; returns it and the number of entries in higher bins.  Lane l scans
// bins [nbins - (l + 1) * per, nbins - l * per) with per = nbins / 32; all lanes get the result.
__device__ __forceinline__ uint32_t warp_find_bin(const uint32_t* hist, int nbins, uint32_t rank, uint32_t* above_out) {
  const int lane = threadIdx.x & 31;
  const int per = nbins / 32;
  const int lo = nbins - (lane + 1) * per;
  uint32_t local = 0;
  for (int q = 0; q < per; q += 4) {
    const uint4 v = *reinterpret_cast<const uint4*>(hist + lo + q);
    local += v.x + v.y + v.z + v.w;
  }
  uint32_t incl = local;   // entries in this lane's bins and every higher bin
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  const uint32_t above = incl - local;
  const uint32_t win = __ballot_sync(0xffffffffu, above < rank && incl >= rank);
  const int wl = win ? __ffs(win) - 1 : 31;
  uint32_t acc = __shfl_sync(0xffffffffu, above, wl);
  // the winning lane's bins, one per lane from its top (per <= 128 handled in chunks of 32)
  const int wlo = nbins - (wl + 1) * per;
  for (int top = wlo + per - 1; top >= wlo; top -= 32) {
    const int bin = top - lane;
    const uint32_t h = bin >= wlo ? hist[bin] : 0u;
    uint32_t inc = h;   // entries in bins top-lane .. top
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += y;
    }
    const uint32_t hit = __ballot_sync(0xffffffffu, acc + inc >= rank && bin >= wlo);
    if (hit) {
      const int src = __ffs(hit) - 1;
      *above_out = acc + __shfl_sync(0xffffffffu, inc - h, src);
      return static_cast<uint32_t>(top - src);
    }
    acc += __shfl_sync(0xffffffffu, inc, 31);
  }
  *above_out = acc;   // unreachable when rank <= the total
  return static_cast<uint32_t>(wlo);
}

// ---------------------------------------------------------------------------------------------
// Step 2: one warp per row.  tau = the lowest key of the histogram bin that holds the rank-th
// largest sampled score (so at least `rank` samples are >= tau); -inf for rows of at most `cap`
// blocks, whose lists keep every block.  The 2048 bins span the bits where the row's sampled keys
// differ, so the samples spread over the bins whatever the scale of the scores.
template <typename F>
__device__ __forceinline__ void for_each_sample(const float* s, int m, F&& f) {
  const int lane = threadIdx.x & 31;
  // rows start 16-byte aligned (ld is a multiple of 4): 16-byte loads, eight in flight per lane
  for (int base = 0; base < m; base += 32 * 4 * 8) {
    float4 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i0 = base + (u * 32 + lane) * 4;
      v[u] = i0 < m ? __ldcg(reinterpret_cast<const float4*>(s + i0)) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i0 = base + (u * 32 + lane) * 4;
      const float e[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (i0 + j < m) f(score_key(e[j] + 0.0f));
    }
  }
}

__global__ void __launch_bounds__(kTauWarps * 32) tau_kernel(const float* __restrict__ samp, long long ld, int NBk,
                                                             long long q_pos0, int row0, int rows, int cap, int rank,
                                                             int kshift, int koff, float* __restrict__ tau,
                                                             int* __restrict__ fail) {
  extern __shared__ uint32_t tsm[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (blockIdx.x == 0 && threadIdx.x == 0) fail[0] = 0;   // the failure list of this chunk starts empty
  const int L = static_cast<int>(blockIdx.x) * kTauWarps + warp;
  if (L >= rows) return;
  const int n = static_cast<int>(min(static_cast<long long>(NBk), (q_pos0 + row0 + L) >> 2));
  if (n <= cap) {
    if (lane == 0) tau[L] = -INFINITY;
    return;
  }
  const int m = n > koff ? ((n - koff - 1) >> kshift) + 1 : 0;
  const float* s = samp + static_cast<long long>(L) * ld;
  uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
  for_each_sample(s, m, [&](uint32_t key) {
    kmin = min(kmin, key);
    kmax = max(kmax, key);
  });
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  if (kmin == kmax) {   // every sample equal
    if (lane == 0) tau[L] = key_to_float(kmin);
    return;
  }
  const int hb = 31 - __clz(kmin ^ kmax);
  const int sh = max(0, hb - 10);
  uint32_t* h = tsm + warp * kTauBins;
  for (int i = lane * 4; i < kTauBins; i += 128) *reinterpret_cast<uint4*>(h + i) = make_uint4(0, 0, 0, 0);
  __syncwarp();
  for_each_sample(s, m, [&](uint32_t key) { atomicAdd(&h[(key >> sh) & (kTauBins - 1)], 1u); });
  __syncwarp();
  uint32_t above;
  const uint32_t r = static_cast<uint32_t>(min(rank, m));
  const uint32_t bin = warp_find_bin(h, kTauBins, r, &above);
  const uint32_t hi_mask = (sh + 11 >= 32) ? 0u : (0xFFFFFFFFu << (sh + 11));
  if (lane == 0) tau[L] = key_to_float((kmax & hi_mask) | (bin << sh));
}

// ---------------------------------------------------------------------------------------------
// Step 4: one warp per row.  The list holds (key, block) pairs in block order.  An 11-bit radix
// pass over the bits where the listed keys differ finds the bin of the k-th largest key; the keys
// of that bin are gathered and their remaining low bits resolved one at a time with ballots.  The
// kept set {key > K*} U {the lowest-block keys == K*} is then emitted in list (= block) order.
__device__ void fail_row(int* fail, int t) {
  if ((threadIdx.x & 31) == 0) {
    const int slot = atomicAdd(&fail[0], 1);
    fail[1 + slot] = t;
  }
}

__global__ void __launch_bounds__(kSelWarps * 32) cand_select_kernel(const uint2* __restrict__ cand,
                                                                     const int* __restrict__ cnt, int cap, int Tq,
                                                                     int NBk, long long q_pos0, int b, int row0,
                                                                     int rows, int k, int32_t* __restrict__ idx,
                                                                     int* __restrict__ fail) {
  extern __shared__ uint32_t csm[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int L = static_cast<int>(blockIdx.x) * (blockDim.x >> 5) + warp;
  if (L >= rows) return;
  const int t = row0 + L;
  const int n = static_cast<int>(min(static_cast<long long>(NBk), (q_pos0 + t) >> 2));
  int32_t* out = idx + (static_cast<long long>(b) * Tq + t) * k;
  if (n <= k) {
    for (int i = lane; i < k; i += 32) out[i] = i < n ? i : -1;
    return;
  }
  const int c = cnt[L];
  if (c < k || c > cap) {
    fail_row(fail, t);
    return;
  }
  const uint2* lst = cand + static_cast<long long>(L) * cap;
  uint32_t* keys = csm + warp * (cap + kSelBins);   // the list's keys
  uint32_t* hist = keys + cap;                       // 11-bit histogram, then the k-th bin's keys
  const uint32_t lt = lane_lt();

  // keys into shared memory (eight 8-byte loads in flight per lane), with their min and max
  uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
  for (int base = 0; base < c; base += 32 * 8) {
    uint32_t v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = base + u * 32 + lane;
      v[u] = i < c ? __ldcs(&lst[i].x) : 0u;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = base + u * 32 + lane;
      if (i < c) {
        keys[i] = v[u];
        kmin = min(kmin, v[u]);
        kmax = max(kmax, v[u]);
      }
    }
  }
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  __syncwarp();

  bool keep_all = false;
  uint32_t kth = 0, need_eq = 0;
  if (c == k) {
    keep_all = true;
  } else if (kmin == kmax) {
    kth = kmin;
    need_eq = static_cast<uint32_t>(k);
  } else {
    const int hb = 31 - __clz(kmin ^ kmax);      // highest bit where listed keys differ
    const int sh = max(0, hb - 10);              // the 11-bit digit covers bits sh .. sh + 10
    for (int i = lane * 4; i < kSelBins; i += 128) *reinterpret_cast<uint4*>(hist + i) = make_uint4(0, 0, 0, 0);
    __syncwarp();
    for (int i = lane; i < c; i += 32) atomicAdd(&hist[(keys[i] >> sh) & (kSelBins - 1)], 1u);
    __syncwarp();
    uint32_t above;
    const uint32_t B = warp_find_bin(hist, kSelBins, static_cast<uint32_t>(k), &above);
    uint32_t krem = static_cast<uint32_t>(k) - above;
    // every listed key shares the bits above bit sh + 10 with kmax
    const uint32_t hi_mask = (sh + 11 >= 32) ? 0u : (0xFFFFFFFFu << (sh + 11));
    uint32_t prefix = (kmax & hi_mask) | (B << sh);
    if (sh > 0) {
      const uint32_t inbin = hist[B];   // <= c <= cap; the histogram space holds kSelBins keys
      __syncwarp();
      if (inbin > static_cast<uint32_t>(kSelBins)) {
        fail_row(fail, t);
        return;
      }
      uint32_t* buf = hist;
      uint32_t pos = 0;
      for (int base = 0; base < c; base += 32) {
        const int i = base + lane;
        const uint32_t key = i < c ? keys[i] : 0u;
        const bool in = i < c && ((key >> sh) & (kSelBins - 1)) == B;
        const uint32_t bm = __ballot_sync(0xffffffffu, in);
        if (in) buf[pos + __popc(bm & lt)] = key;
        pos += __popc(bm);
      }
      __syncwarp();
      const int mb = static_cast<int>(inbin);
      for (int bit = sh - 1; bit >= 0; --bit) {
        const uint32_t want = (prefix >> bit) | 1u;
        uint32_t cntb = 0;
        for (int base = 0; base < mb; base += 32) {
          const int i = base + lane;
          cntb += __popc(__ballot_sync(0xffffffffu, i < mb && (buf[i] >> bit) == want));
        }
        if (cntb >= krem)
          prefix |= 1u << bit;
        else
          krem -= cntb;
      }
    }
    kth = prefix;
    need_eq = krem;
  }

  // ordered emission: keys from shared memory, block indices from the list (batched loads)
  uint32_t out_run = 0, eq_run = 0;
  for (int base = 0; base < c; base += 32 * 8) {
    uint32_t id[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = base + u * 32 + lane;
      id[u] = i < c ? __ldcs(&lst[i].y) : 0u;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = base + u * 32 + lane;
      const uint32_t key = i < c ? keys[i] : 0u;
      const bool gt = i < c && (keep_all || key > kth);
      const bool eq = i < c && !keep_all && key == kth;
      const uint32_t eqm = __ballot_sync(0xffffffffu, eq);
      const uint32_t eq_rank = eq_run + __popc(eqm & lt);
      const bool keep = gt || (eq && eq_rank < need_eq);
      const uint32_t km = __ballot_sync(0xffffffffu, keep);
      if (keep) {
        const uint32_t p = out_run + __popc(km & lt);
        if (p < static_cast<uint32_t>(k)) out[p] = static_cast<int32_t>(id[u]);
      }
      out_run += __popc(km);
      eq_run += __popc(eqm);
    }
  }
}

}  // namespace

cudaError_t launch_select_tau(const DeviceInfo* di, const float* samp, long long ld, int NBk, long long q_pos0,
                              int row0, int rows, int cap, int rank, int kshift, int koff, float* tau, int* fail,
                              cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  constexpr int smem = kTauWarps * kTauBins * 4;
  static std::once_flag once[64];
  std::call_once(once[di->device & 63],
                 [] { cudaFuncSetAttribute(tau_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem); });
  tau_kernel<<<(rows + kTauWarps - 1) / kTauWarps, kTauWarps * 32, smem, s>>>(samp, ld, NBk, q_pos0, row0, rows, cap,
                                                                            rank, kshift, koff, tau, fail);
  return cudaPeekAtLastError();
}

cudaError_t launch_select_candidates(const DeviceInfo* di, const uint2* cand, const int* cnt, int cap, int Tq, int NBk,
                                     long long q_pos0, int b, int row0, int rows, int k, int32_t* idx, int* fail,
                                     cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  static std::once_flag once[64];
  std::call_once(once[di->device & 63], [] {
    cudaFuncSetAttribute(cand_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSelSmemMax);
  });
  const int per_warp = (cap + kSelBins) * 4;
  const int warps = std::max(1, std::min(kSelWarps, kSelSmemMax / per_warp));
  if (per_warp > kSelSmemMax) return cudaErrorInvalidValue;
  cand_select_kernel<<<(rows + warps - 1) / warps, warps * 32, warps * per_warp, s>>>(cand, cnt, cap, Tq, NBk, q_pos0,
                                                                                    b, row0, rows, k, idx, fail);
  return cudaPeekAtLastError();
}

}  // namespace qsa
