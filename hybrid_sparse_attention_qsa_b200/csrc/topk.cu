// Per-query top-k block selection.
//
// "Qwen3.8-Flash-Next architecture" (flozi.net), "Der Weg eines Tokens durch das Modell", item 2:
// each query keeps a budget of 512 fully selected micro-blocks (2048 tokens) plus its own,
// possibly incomplete, block.  Reading fixed in qsa.h: the top-k of the fp32 scores over the
// candidates b < floor(p/blk), equal scores to the lower index, ascending output, -1 padded.
//
// One CTA per score row.  The k-th largest score is found exactly by a radix select on the
// order-preserving 32-bit keys of the fp32 scores (three passes of 11, 11 and 10 bits over the
// row, shared-memory histograms; the lanes of a warp that hit the same bin are merged with
// match.any so one atomic per distinct bin is issued).  A final pass in index order emits every
// key above the threshold and the first (k - #above) keys equal to it, with a block-wide scan for
// the output positions, so the list comes out ascending without a sort.
#include "launch.h"

namespace qsa {
namespace {

constexpr int kTopkThreads = 512;
constexpr int kWarps = kTopkThreads / 32;
constexpr int kMaxBins = 2048;

__device__ __forceinline__ uint32_t key_of(float s) {
  return score_key(s + 0.0f);   // -0 -> +0, so the two zeros compare equal as in fp32
}

// Exclusive scan of one value per thread over the block; returns the exclusive prefix and writes
// the block total to *total.  Uses `ws` (kWarps + 1 words); ends with the block synchronised.
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

__global__ void __launch_bounds__(kTopkThreads) topk_kernel(const float* __restrict__ scores, long long ld,
                                                            long long batch_stride, const int32_t* __restrict__ seqlens,
                                                            int Tq, int NBk, int blk, long long q_pos0, int b0,
                                                            int row0, int k, int32_t* __restrict__ idx,
                                                            KernelCtl ctl) {
  __shared__ uint32_t hist[kMaxBins];
  __shared__ uint32_t scan_ws[kWarps + 1];
  __shared__ uint32_t sel_bin, sel_above;

  const int tid = threadIdx.x, lane = tid & 31;
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

  // ---- radix select of the k-th largest key
  uint32_t prefix = 0, pmask = 0, krem = static_cast<uint32_t>(k);
  const int shifts[3] = {21, 10, 0};
  const int widths[3] = {11, 11, 10};
#pragma unroll 1
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = shifts[pass];
    const int nbins = 1 << widths[pass];
    const uint32_t dmask = static_cast<uint32_t>(nbins - 1);
    for (int i = tid; i < nbins; i += kTopkThreads) hist[i] = 0;
    __syncthreads();
    for (int base = 0; base < n; base += kTopkThreads) {
      const int i = base + tid;
      bool hit = false;
      uint32_t digit = 0xFFFFFFFFu;
      if (i < n) {
        const uint32_t key = key_of(s[i]);
        if ((key & pmask) == prefix) {
          hit = true;
          digit = (key >> shift) & dmask;
        }
      }
      const uint32_t peers = __match_any_sync(0xffffffffu, digit);
      if (hit && lane == __ffs(peers) - 1) atomicAdd(&hist[digit], static_cast<uint32_t>(__popc(peers)));
    }
    __syncthreads();
    // Bin of the krem-th largest among the hits: thread t owns bins [t*bpt, (t+1)*bpt).
    const int bpt = nbins / kTopkThreads;
    uint32_t local = 0;
    for (int q = 0; q < bpt; ++q) local += hist[tid * bpt + q];
    // count of hits in bins above this thread's range = total - inclusive prefix
    uint32_t total;
    const uint32_t excl = block_excl_scan(local, scan_ws, &total);
    const uint32_t above = total - excl - local;
    if (above < krem && above + local >= krem) {
      uint32_t acc = above;
      for (int q = bpt - 1; q >= 0; --q) {
        const uint32_t h = hist[tid * bpt + q];
        if (acc + h >= krem) {
          sel_bin = static_cast<uint32_t>(tid * bpt + q);
          sel_above = acc;
          break;
        }
        acc += h;
      }
    }
    __syncthreads();
    prefix |= sel_bin << shift;
    pmask |= dmask << shift;
    krem -= sel_above;
    __syncthreads();
  }
  const uint32_t kth = prefix;      // the exact k-th largest key
  const uint32_t need_eq = krem;    // how many keys equal to kth are taken (lowest indices)

  // ---- ordered emission: 4 consecutive elements per thread per chunk
  uint32_t gt_tot = 0, eq_tot = 0;
  for (int base = 0; base < n; base += 4 * kTopkThreads) {
    const int i0 = base + 4 * tid;
    uint32_t gt_m = 0, eq_m = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int i = i0 + e;
      if (i < n) {
        const uint32_t key = key_of(s[i]);
        gt_m |= (key > kth ? 1u : 0u) << e;
        eq_m |= (key == kth ? 1u : 0u) << e;
      }
    }
    const uint32_t packed = (static_cast<uint32_t>(__popc(gt_m)) << 16) | static_cast<uint32_t>(__popc(eq_m));
    uint32_t total;
    const uint32_t ex = block_excl_scan(packed, scan_ws, &total);
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

}  // namespace

cudaError_t launch_topk(const DeviceInfo* di, const float* scores, long long ld, long long batch_stride,
                        const int32_t* seqlens, int Tq, int NBk, int blk, long long q_pos0, int b0, int nb, int row0,
                        int rows, int k, int32_t* idx, cudaStream_t s) {
  if (rows <= 0 || nb <= 0) return cudaSuccess;
  dim3 grid(rows, nb);
  topk_kernel<<<grid, kTopkThreads, 0, s>>>(scores, ld, batch_stride, seqlens, Tq, NBk, blk, q_pos0, b0, row0, k, idx,
                                            kernel_ctl(di));
  return cudaPeekAtLastError();
}

}  // namespace qsa
