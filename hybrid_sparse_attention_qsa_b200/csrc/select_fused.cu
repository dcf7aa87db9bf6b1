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

constexpr int kSelBins = 2048;    // bins of the first select pass (11 bits)

constexpr int kSelThreads = 128;
constexpr int kSelWarpsPerRow = kSelThreads / 32;

// Exclusive block scan of one value per thread; also returns the block total.  Ends synchronised.
__device__ __forceinline__ uint32_t sel_block_scan(uint32_t v, uint32_t* ws, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) ws[warp] = x;
  __syncthreads();
  uint32_t before = 0, all = 0;
#pragma unroll
  for (int w = 0; w < kSelWarpsPerRow; ++w) {
    const uint32_t t = ws[w];
    before += w < warp ? t : 0u;
    all += t;
  }
  __syncthreads();
  *total = all;
  return before + x - v;
}

// Finds, over kSelBins bins in shared memory (a larger bin holds larger keys), the bin holding the
// rank-th largest entry with the whole CTA; returns (bin, entries in higher bins) in sel[0], sel[1].
// Ends synchronised.
__device__ __forceinline__ void block_find_bin(const uint32_t* hist, uint32_t rank, uint32_t* ws, uint32_t* sel) {
  constexpr int per = kSelBins / kSelThreads;
  const int tid = threadIdx.x;
  const int lo = kSelBins - per * (tid + 1);   // thread 0 holds the top bins
  uint32_t local = 0;
#pragma unroll
  for (int q = 0; q < per; q += 4) {
    const uint4 h4 = *reinterpret_cast<const uint4*>(hist + lo + q);
    local += h4.x + h4.y + h4.z + h4.w;
  }
  uint32_t total;
  const uint32_t above = sel_block_scan(local, ws, &total);   // entries in bins above this range
  if (above < rank && above + local >= rank) {
    uint32_t acc = above;
    for (int q = per - 1; q >= 0; --q) {
      const uint32_t h = hist[lo + q];
      if (acc + h >= rank) {
        sel[0] = static_cast<uint32_t>(lo + q);
        sel[1] = acc;
        break;
      }
      acc += h;
    }
  }
  __syncthreads();
}

// Block-wide min and max of one key per thread (ws: 2 * kSelWarpsPerRow words).  Ends synchronised.
__device__ __forceinline__ void block_minmax(uint32_t& kmin, uint32_t& kmax, uint32_t* ws) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  if (lane == 0) {
    ws[2 * warp] = kmin;
    ws[2 * warp + 1] = kmax;
  }
  __syncthreads();
#pragma unroll
  for (int w = 0; w < kSelWarpsPerRow; ++w) {
    kmin = min(kmin, ws[2 * w]);
    kmax = max(kmax, ws[2 * w + 1]);
  }
  __syncthreads();
}

// ---------------------------------------------------------------------------------------------
// Step 2: one CTA of kSelThreads per row.  tau = the lowest key of the histogram bin that holds
// the rank-th largest sampled score (so at least `rank` samples are >= tau); -inf for rows of at
// most `cap` blocks, whose lists keep every block.  The kSelBins bins span the bits where the
// row's sampled keys differ, so the samples spread over the bins whatever the scale of the scores.
// Up to kTauRegs * kSelThreads samples are read once into registers; longer rows are read twice.
constexpr int kTauRegs = 16;

__global__ void __launch_bounds__(kSelThreads) tau_kernel(const float* __restrict__ samp, long long ld, int NBk,
                                                          long long q_pos0, int row0, int cap, int rank, int kshift,
                                                          int koff, float* __restrict__ tau, int* __restrict__ fail) {
  __shared__ __align__(16) uint32_t hist[kSelBins];
  __shared__ uint32_t ws[2 * kSelWarpsPerRow];
  __shared__ uint32_t sel[2];
  const int tid = threadIdx.x;
  const int L = static_cast<int>(blockIdx.x);
  if (L == 0 && tid == 0) fail[0] = 0;   // the failure list of this chunk starts empty
  const int n = static_cast<int>(min(static_cast<long long>(NBk), (q_pos0 + row0 + L) >> 2));
  if (n <= cap) {
    if (tid == 0) tau[L] = -INFINITY;
    return;
  }
  const int m = n > koff ? ((n - koff - 1) >> kshift) + 1 : 0;
  const float* s = samp + static_cast<long long>(L) * ld;   // 16-byte aligned (ld is a multiple of 4)
  const bool in_regs = m <= kTauRegs * kSelThreads;
  uint32_t key[kTauRegs];
  uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
  if (in_regs) {
    float4 f[kTauRegs / 4];
#pragma unroll
    for (int u = 0; u < kTauRegs / 4; ++u) {
      const int i0 = (tid + u * kSelThreads) * 4;
      f[u] = i0 < m ? __ldcs(reinterpret_cast<const float4*>(s + i0)) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < kTauRegs / 4; ++u) {
      const int i0 = (tid + u * kSelThreads) * 4;
      const float e[4] = {f[u].x, f[u].y, f[u].z, f[u].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        key[u * 4 + j] = score_key(e[j] + 0.0f);
        if (i0 + j < m) {
          kmin = min(kmin, key[u * 4 + j]);
          kmax = max(kmax, key[u * 4 + j]);
        }
      }
    }
  } else {
    for (int i = tid; i < m; i += kSelThreads) {
      const uint32_t k1 = score_key(s[i] + 0.0f);
      kmin = min(kmin, k1);
      kmax = max(kmax, k1);
    }
  }
  block_minmax(kmin, kmax, ws);
  if (kmin == kmax) {   // every sample equal
    if (tid == 0) tau[L] = key_to_float(kmin);
    return;
  }
  const int hb = 31 - __clz(kmin ^ kmax);
  const int sh = max(0, hb - 10);
  for (int i = tid * 4; i < kSelBins; i += kSelThreads * 4)
    *reinterpret_cast<uint4*>(hist + i) = make_uint4(0u, 0u, 0u, 0u);
  __syncthreads();
  if (in_regs) {
#pragma unroll
    for (int u = 0; u < kTauRegs / 4; ++u) {
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if ((tid + u * kSelThreads) * 4 + j < m) atomicAdd(&hist[(key[u * 4 + j] >> sh) & (kSelBins - 1)], 1u);
    }
  } else {
    for (int i = tid; i < m; i += kSelThreads) atomicAdd(&hist[(score_key(s[i] + 0.0f) >> sh) & (kSelBins - 1)], 1u);
  }
  __syncthreads();
  block_find_bin(hist, static_cast<uint32_t>(min(rank, m)), ws, sel);
  const uint32_t hi_mask = (sh + 11 >= 32) ? 0u : (0xFFFFFFFFu << (sh + 11));
  if (tid == 0) tau[L] = key_to_float((kmax & hi_mask) | (sel[0] << sh));
}

// ---------------------------------------------------------------------------------------------
// Step 4: one CTA of kSelThreads per row.  The list holds (fp32 score bits, block) pairs in block
// order; it is read once into registers (thread t holds entries 2 (t + 128 u) and 2 (t + 128 u) + 1)
// and the scores turned into order-preserving keys.  An
// 11-bit histogram over the bits where the listed keys differ finds the bin of the k-th largest
// key; the keys of that bin are gathered and their remaining low bits resolved one at a time with
// ballots (warp 0).  The kept set {key > K*} U {the first need_eq keys == K*} is then emitted in
// list (= block) order with block-wide scans.
__device__ void fail_row(int* fail, int t) {
  const int slot = atomicAdd(&fail[0], 1);
  fail[1 + slot] = t;
}

template <int U>
__device__ __forceinline__ void select_row(const uint2* __restrict__ cand, const int* __restrict__ cnt, int cap,
                                           int Tq, int NBk, long long q_pos0, int b, int row0, int k,
                                           int32_t* __restrict__ idx, int* __restrict__ fail, int L, uint32_t* hist,
                                           uint32_t* ws, uint32_t* sel) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int t = row0 + L;
  const int n = static_cast<int>(min(static_cast<long long>(NBk), (q_pos0 + t) >> 2));
  int32_t* out = idx + (static_cast<long long>(b) * Tq + t) * k;
  if (n <= k) {
    for (int i = tid; i < k; i += kSelThreads) out[i] = i < n ? i : -1;
    return;
  }
  const int c = cnt[L];
  if (c < k || c > cap || c > 2 * U * kSelThreads) {
    if (tid == 0) fail_row(fail, t);
    return;
  }
  // the whole list into registers: U 16-byte loads in flight per thread (cap is even, so every
  // list starts 16-byte aligned)
  const uint4* src = reinterpret_cast<const uint4*>(cand + static_cast<long long>(L) * cap);
  const int c2 = (c + 1) >> 1;
  const int rounds = (c + 2 * kSelThreads - 1) / (2 * kSelThreads);   // rounds holding entries
  uint4 v[U];
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int j = tid + u * kSelThreads;
    v[u] = (u < rounds && j < c2) ? __ldcs(src + j) : make_uint4(0u, 0u, 0u, 0u);
  }
  // entry 2j is (v.x, v.y), entry 2j + 1 is (v.z, v.w): fp32 score bits, turned into
  // order-preserving keys here; invalid entries get key 0 (below any score)
  uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
#pragma unroll
  for (int u = 0; u < U; ++u) {
    if (u >= rounds) break;   // uniform
    const int j = tid + u * kSelThreads;
    v[u].x = score_key(__uint_as_float(v[u].x) + 0.0f);
    v[u].z = score_key(__uint_as_float(v[u].z) + 0.0f);
    if (2 * j + 1 >= c) v[u].z = 0u;
    if (2 * j < c) {
      kmin = min(kmin, v[u].x);
      kmax = max(kmax, v[u].x);
    }
    if (2 * j + 1 < c) {
      kmin = min(kmin, v[u].z);
      kmax = max(kmax, v[u].z);
    }
  }
  block_minmax(kmin, kmax, ws);

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
    for (int i = tid * 4; i < kSelBins; i += kSelThreads * 4)
      *reinterpret_cast<uint4*>(hist + i) = make_uint4(0u, 0u, 0u, 0u);
    __syncthreads();
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (u >= rounds) break;   // uniform
      const int j = tid + u * kSelThreads;
      if (2 * j < c) atomicAdd(&hist[(v[u].x >> sh) & (kSelBins - 1)], 1u);
      if (2 * j + 1 < c) atomicAdd(&hist[(v[u].z >> sh) & (kSelBins - 1)], 1u);
    }
    __syncthreads();
    block_find_bin(hist, static_cast<uint32_t>(k), ws, sel);
    const uint32_t B = sel[0];
    uint32_t krem = static_cast<uint32_t>(k) - sel[1];
    const uint32_t hi_mask = (sh + 11 >= 32) ? 0u : (0xFFFFFFFFu << (sh + 11));
    uint32_t prefix = (kmax & hi_mask) | (B << sh);   // listed keys share the bits above sh + 10
    if (sh > 0) {
      const uint32_t inbin = hist[B];
      if (tid == 0) sel[2] = 0;
      __syncthreads();   // every thread has read hist[B]: the space now gathers the bin's keys
      if (inbin > static_cast<uint32_t>(kSelBins)) {
        if (tid == 0) fail_row(fail, t);
        return;
      }
      uint32_t* buf = hist;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        if (u >= rounds) break;   // uniform
        const int j = tid + u * kSelThreads;
        if (2 * j < c && ((v[u].x >> sh) & (kSelBins - 1)) == B) buf[atomicAdd(&sel[2], 1u)] = v[u].x;
        if (2 * j + 1 < c && ((v[u].z >> sh) & (kSelBins - 1)) == B) buf[atomicAdd(&sel[2], 1u)] = v[u].z;
      }
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

  // ordered emission: round u covers entries [256 u, 256 u + 256), two consecutive per thread.
  // One pass of warp scans over all rounds at once and one exchange of the warps' round totals
  // give every entry its number of kept entries before it.
  uint32_t pk[U];   // per round: (entries > K*) << 16 | (entries == K*) among this thread's two
#pragma unroll
  for (int u = 0; u < U; ++u) {
    pk[u] = 0;
    if (u >= rounds) continue;   // uniform
    const int j = tid + u * kSelThreads;
    const bool ok0 = 2 * j < c, ok1 = 2 * j + 1 < c;
    const bool gt0 = ok0 && (keep_all || v[u].x > kth), gt1 = ok1 && (keep_all || v[u].z > kth);
    const bool eq0 = ok0 && !keep_all && v[u].x == kth, eq1 = ok1 && !keep_all && v[u].z == kth;
    pk[u] = ((static_cast<uint32_t>(gt0) + gt1) << 16) | (static_cast<uint32_t>(eq0) + eq1);
  }
  uint32_t incl[U];
#pragma unroll
  for (int u = 0; u < U; ++u) {
    if (u >= rounds) {   // uniform
      incl[u] = 0;
      continue;
    }
    uint32_t x = pk[u];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    incl[u] = x;
  }
  if (lane == 31) {
#pragma unroll
    for (int u = 0; u < U; ++u)
      if (u < rounds) hist[u * kSelWarpsPerRow + warp] = incl[u];   // the histogram is no longer needed
  }
  __syncthreads();
  uint32_t gt_tot = 0, eq_tot = 0;   // entries of earlier rounds
#pragma unroll
  for (int u = 0; u < U; ++u) {
    if (u >= rounds) break;   // uniform
    uint32_t before = 0, all = 0;
#pragma unroll
    for (int w = 0; w < kSelWarpsPerRow; ++w) {
      const uint32_t t = hist[u * kSelWarpsPerRow + w];
      before += w < warp ? t : 0u;
      all += t;
    }
    const uint32_t ex = before + incl[u] - pk[u];
    uint32_t gt_run = gt_tot + (ex >> 16), eq_run = eq_tot + (ex & 0xFFFFu);
    const int j = tid + u * kSelThreads;
    const bool ok0 = 2 * j < c, ok1 = 2 * j + 1 < c;
    const bool gt0 = ok0 && (keep_all || v[u].x > kth), gt1 = ok1 && (keep_all || v[u].z > kth);
    const bool eq0 = ok0 && !keep_all && v[u].x == kth, eq1 = ok1 && !keep_all && v[u].z == kth;
    if (gt0) {
      const uint32_t p = gt_run + min(eq_run, need_eq);
      if (p < static_cast<uint32_t>(k)) out[p] = static_cast<int32_t>(v[u].y);
      ++gt_run;
    } else if (eq0) {
      if (eq_run < need_eq && gt_run + eq_run < static_cast<uint32_t>(k)) out[gt_run + eq_run] = static_cast<int32_t>(v[u].y);
      ++eq_run;
    }
    if (gt1) {
      const uint32_t p = gt_run + min(eq_run, need_eq);
      if (p < static_cast<uint32_t>(k)) out[p] = static_cast<int32_t>(v[u].w);
    } else if (eq1) {
      if (eq_run < need_eq && gt_run + eq_run < static_cast<uint32_t>(k)) out[gt_run + eq_run] = static_cast<int32_t>(v[u].w);
    }
    gt_tot += all >> 16;
    eq_tot += all & 0xFFFFu;
  }
}

// One CTA per row (a grid-strided loop over rows held ~40 more registers per thread live and cut
// the resident CTAs per SM from 6 to 4).  At most 64 registers, for 8 resident rows per SM: the few
// spills that costs are cheaper than the rows it adds in flight.
template <int U>
__global__ void __launch_bounds__(kSelThreads, 8) cand_select_kernel(const uint2* __restrict__ cand,
                                                                  const int* __restrict__ cnt, int cap, int Tq, int NBk,
                                                                  long long q_pos0, int b, int row0, int k,
                                                                  int32_t* __restrict__ idx, int* __restrict__ fail) {
  __shared__ __align__(16) uint32_t hist[kSelBins];   // histogram, then the k-th bin's keys
  __shared__ uint32_t ws[2 * kSelWarpsPerRow];
  __shared__ uint32_t sel[4];
  select_row<U>(cand, cnt, cap, Tq, NBk, q_pos0, b, row0, k, idx, fail, static_cast<int>(blockIdx.x), hist, ws, sel);
}

}  // namespace

cudaError_t launch_select_tau(const DeviceInfo* di, const float* samp, long long ld, int NBk, long long q_pos0,
                              int row0, int rows, int cap, int rank, int kshift, int koff, float* tau, int* fail,
                              cudaStream_t s) {
  (void)di;
  if (rows <= 0) return cudaSuccess;
  tau_kernel<<<rows, kSelThreads, 0, s>>>(samp, ld, NBk, q_pos0, row0, cap, rank, kshift, koff, tau, fail);
  return cudaPeekAtLastError();
}

cudaError_t launch_select_candidates(const DeviceInfo* di, const uint2* cand, const int* cnt, int cap, int Tq, int NBk,
                                     long long q_pos0, int b, int row0, int rows, int k, int32_t* idx, int* fail,
                                     cudaStream_t s) {
  (void)di;
  if (rows <= 0) return cudaSuccess;
  // lists of up to 2 * U * kSelThreads entries fit the registers; longer ones are refused (the
  // caller only plans caps that fit)
  if (cap <= 2 * 8 * kSelThreads)   // k <= 512: no spills within the 64 registers
    cand_select_kernel<8><<<rows, kSelThreads, 0, s>>>(cand, cnt, cap, Tq, NBk, q_pos0, b, row0, k, idx, fail);
  else if (cap <= 2 * 10 * kSelThreads)
    cand_select_kernel<10><<<rows, kSelThreads, 0, s>>>(cand, cnt, cap, Tq, NBk, q_pos0, b, row0, k, idx, fail);
  else if (cap <= 2 * 20 * kSelThreads)
    cand_select_kernel<20><<<rows, kSelThreads, 0, s>>>(cand, cnt, cap, Tq, NBk, q_pos0, b, row0, k, idx, fail);
  else
    return cudaErrorInvalidValue;
  return cudaPeekAtLastError();
}

}  // namespace qsa
