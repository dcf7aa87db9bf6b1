// The C ABI (include/qsa.h): argument checks on the host, then launches on the caller's stream.
#include <algorithm>
#include <cmath>
#include <atomic>
#include <cstdint>
#include <mutex>

#include "launch.h"
#include "qsa.h"

namespace qsa {

__device__ unsigned int g_status_word;   // one per device that loads the library

namespace {
constexpr int kMaxDevices = 64;
constexpr unsigned long long kDefaultWaitNs = 2000000000ull;
std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];
bool g_dev_ok[kMaxDevices];
std::atomic<unsigned long long> g_wait_ns{kDefaultWaitNs};

// Per-device side stream and events used by qsa_select_topk to overlap chunks (created on first
// use with the device current; kept until the process exits).
struct SideStream {
  std::mutex mu;
  cudaStream_t stream = nullptr;
  cudaEvent_t begin = nullptr, end = nullptr, score_done[2] = {nullptr, nullptr}, topk_done[2] = {nullptr, nullptr};
};
SideStream g_side[kMaxDevices];
std::once_flag g_side_once[kMaxDevices];
bool g_side_ok[kMaxDevices];

SideStream* side_stream(int dev) {
  std::call_once(g_side_once[dev], [dev] {
    SideStream& ss = g_side[dev];
    bool ok = cudaStreamCreateWithFlags(&ss.stream, cudaStreamNonBlocking) == cudaSuccess;
    cudaEvent_t* evs[] = {&ss.begin, &ss.end, &ss.score_done[0], &ss.score_done[1], &ss.topk_done[0],
                          &ss.topk_done[1]};
    for (cudaEvent_t* ev : evs) ok = ok && cudaEventCreateWithFlags(ev, cudaEventDisableTiming) == cudaSuccess;
    g_side_ok[dev] = ok;
  });
  return g_side_ok[dev] ? &g_side[dev] : nullptr;
}

__global__ void wait_selftest_kernel(KernelCtl ctl) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, ctl);   // nothing ever arrives: the wait must give up
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool ok_ptr(const void* p) { return p != nullptr && aligned16(p); }
cudaStream_t S(void* s) { return static_cast<cudaStream_t>(s); }
qsa_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? QSA_OK : QSA_ERR_CUDA; }
bool hi_supported(int Hi) { return Hi == 1 || Hi == 2 || Hi == 4 || Hi == 8; }

// ---- filtered selection (prefill without materialised scores)
std::atomic<int> g_select_path{0};    // 0 automatic, 1 materialised scores, 2 filtered
std::atomic<int> g_attn_path{0};      // prefill attention: 0 automatic, 1 row by row, 2 query tiles
std::atomic<int> g_sample_rank{0};    // 0: the default rank of the threshold among the samples
constexpr int kSampleShift = 4;       // every 16th pooled block is sampled ...
constexpr int kSampleOff = 8;         // ... starting at block 8
constexpr int kFallbackCtas = 128;    // CTAs (and scratch rows) of the exact redo of failed rows
constexpr long long kFusedTarget = 4ll << 30;   // workspace the size query plans the filtered path in
constexpr int kFusedMinRows = 16384;  // automatic choice: row length (last position) from which it pays
constexpr int kFusedMaxCap = 5120;    // longest candidate list the select kernel holds (k <= 1024)

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct FusedPlan {
  int rank, cap, ns, ld_s;
  long long per_row, fixed;
};
// rank r of the threshold among the row's samples (about 16 r scores expected above it, at least
// 2 k: the sample rank's relative spread is about 1 / sqrt(r), so a list shorter than k is a
// four-sigma event or rarer) and the list capacity 32 r.  (2.5 k took 3 % longer at 128K, 1.5 k
// sent enough rows to the exact redo to cost more.)
FusedPlan fused_plan(int NBk, int k) {
  FusedPlan p;
  p.rank = std::max(64, (2 * k + 15) / 16);
  p.cap = 32 * p.rank;
  p.ns = NBk > kSampleOff ? ((NBk - kSampleOff - 1) >> kSampleShift) + 1 : 0;
  p.ld_s = (std::max(p.ns, 1) + 3) & ~3;
  p.per_row = static_cast<long long>(p.ld_s) * 4 + 12 + static_cast<long long>(p.cap) * 8;
  p.fixed = 12 * 256 + 4 + static_cast<long long>(kFallbackCtas) * std::max(NBk, 1) * 4;
  return p;
}
long long fused_rows_fit(const FusedPlan& p, size_t ws_bytes) {
  const long long avail = static_cast<long long>(ws_bytes) - p.fixed;
  return avail > 0 ? avail / p.per_row : 0;
}
}  // namespace

const DeviceInfo* device_info() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_dev_ok[dev]) {
    int sms = 0;
    void* p = nullptr;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return nullptr;
    if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return nullptr;
    g_dev[dev] = DeviceInfo{dev, sms, static_cast<unsigned*>(p)};
    g_dev_ok[dev] = true;
  }
  return &g_dev[dev];
}

KernelCtl kernel_ctl(const DeviceInfo* di) { return KernelCtl{di->status, g_wait_ns.load()}; }

int attn_path() { return g_attn_path.load(); }

}  // namespace qsa

using namespace qsa;

extern "C" {

const char* qsa_status_string(qsa_status_t status) {
  switch (status) {
    case QSA_OK: return "QSA_OK";
    case QSA_ERR_INVALID_ARGUMENT: return "QSA_ERR_INVALID_ARGUMENT";
    case QSA_ERR_UNSUPPORTED: return "QSA_ERR_UNSUPPORTED";
    case QSA_ERR_WORKSPACE_TOO_SMALL: return "QSA_ERR_WORKSPACE_TOO_SMALL";
    case QSA_ERR_CUDA: return "QSA_ERR_CUDA";
    case QSA_ERR_TIMEOUT: return "QSA_ERR_TIMEOUT";
    case QSA_ERR_DEVICE_CHECK: return "QSA_ERR_DEVICE_CHECK";
  }
  return "QSA_ERR_UNKNOWN";
}

int qsa_abi_version(void) { return QSA_ABI_VERSION; }

qsa_status_t qsa_set_select_options(int path, int sample_rank) {
  if (path < 0 || path > 2 || sample_rank < 0) return QSA_ERR_INVALID_ARGUMENT;
  g_select_path.store(path);
  g_sample_rank.store(sample_rank);
  return QSA_OK;
}

void qsa_set_wait_timeout_ns(uint64_t ns) { g_wait_ns.store(ns ? ns : kDefaultWaitNs); }

// Checks and resolves the rotary parameters (NULL or theta <= 0: no rotation).
static qsa_status_t resolve_rope(const qsa_rope_params_t* in, RopeParams* out) {
  *out = RopeParams{0.0, 1.0, 0.0, 1.0, 32.0, 1.0};
  if (in == nullptr || !(in->theta > 0.0)) return QSA_OK;
  out->theta = in->theta;
  if (in->yarn_factor > 1.0) {
    if (!(in->yarn_orig_ctx > 0.0) || !(in->yarn_beta > in->yarn_alpha)) return QSA_ERR_INVALID_ARGUMENT;
    out->factor = in->yarn_factor;
    out->orig_ctx = in->yarn_orig_ctx;
    out->alpha = in->yarn_alpha;
    out->beta = in->yarn_beta;
    out->mscale = in->yarn_mscale > 0.0 ? in->yarn_mscale : 0.1 * std::log(in->yarn_factor) + 1.0;
  } else if (!(in->yarn_factor >= 0.0)) {
    return QSA_ERR_INVALID_ARGUMENT;
  }
  return QSA_OK;
}

qsa_status_t qsa_pool_block_keys_rope(const void* ki, void* kp, int B, int L, int Di, int blk,
                                      const qsa_rope_params_t* rope, int64_t pos0, int64_t ki_batch_stride,
                                      int64_t kp_batch_stride, void* stream) {
  QSA_NVTX();
  if (B < 0 || L < 0 || Di < 2 || Di > 256 || (Di & 1) || pos0 < 0) return QSA_ERR_INVALID_ARGUMENT;
  if (ki_batch_stride < 0 || kp_batch_stride < 0) return QSA_ERR_INVALID_ARGUMENT;
  RopeParams rp;
  if (resolve_rope(rope, &rp) != QSA_OK) return QSA_ERR_INVALID_ARGUMENT;
  const long long kis = ki_batch_stride ? ki_batch_stride : static_cast<long long>(L) * Di;
  const long long kps = kp_batch_stride ? kp_batch_stride : static_cast<long long>(L / 4) * Di;
  if (kis < static_cast<long long>(L) * Di || kps < static_cast<long long>(L / 4) * Di) return QSA_ERR_INVALID_ARGUMENT;
  if (blk != 4) return QSA_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * (L / blk) == 0) return QSA_OK;
  if (!ok_ptr(ki) || !ok_ptr(kp)) return QSA_ERR_INVALID_ARGUMENT;
  if (!device_info()) return QSA_ERR_CUDA;
  return cuda_status(launch_pool(ki, kp, B, L, Di, blk, rp, pos0, kis, kps, S(stream)));
}

qsa_status_t qsa_pool_block_keys(const void* ki, void* kp, int B, int L, int Di, int blk, float rope_theta,
                                 int64_t pos0, int64_t ki_batch_stride, int64_t kp_batch_stride, void* stream) {
  QSA_NVTX();
  const qsa_rope_params_t rope{rope_theta > 0.f ? static_cast<double>(rope_theta) : 0.0, 1.0, 0.0, 1.0, 32.0, 0.0};
  return qsa_pool_block_keys_rope(ki, kp, B, L, Di, blk, &rope, pos0, ki_batch_stride, kp_batch_stride, stream);
}

qsa_status_t qsa_rope_index_queries_rope(const void* qi, void* qi_out, int B, int Tq, int Hi, int Di, int64_t q_pos0,
                                         const int32_t* seqlens, const qsa_rope_params_t* rope, void* stream) {
  QSA_NVTX();
  RopeParams rp;
  if (B < 0 || Tq < 0 || Hi < 1 || Di < 2 || Di > 256 || (Di & 1) || q_pos0 < 0) return QSA_ERR_INVALID_ARGUMENT;
  if (resolve_rope(rope, &rp) != QSA_OK || !(rp.theta > 0.0)) return QSA_ERR_INVALID_ARGUMENT;
  if (seqlens && Tq != 1) return QSA_ERR_INVALID_ARGUMENT;
  if (static_cast<long long>(B) * Tq == 0) return QSA_OK;
  if (!ok_ptr(qi) || !ok_ptr(qi_out)) return QSA_ERR_INVALID_ARGUMENT;
  if (!device_info()) return QSA_ERR_CUDA;
  return cuda_status(launch_rope_queries(qi, qi_out, B, Tq, Hi, Di, q_pos0, seqlens, rp, S(stream)));
}

qsa_status_t qsa_rope_index_queries(const void* qi, void* qi_out, int B, int Tq, int Hi, int Di, int64_t q_pos0,
                                    const int32_t* seqlens, float rope_theta, void* stream) {
  QSA_NVTX();
  if (!(rope_theta > 0.f)) return QSA_ERR_INVALID_ARGUMENT;
  const qsa_rope_params_t rope{static_cast<double>(rope_theta), 1.0, 0.0, 1.0, 32.0, 0.0};
  return qsa_rope_index_queries_rope(qi, qi_out, B, Tq, Hi, Di, q_pos0, seqlens, &rope, stream);
}

static qsa_status_t check_score_args(const void* qi, const void* kp, const int32_t* seqlens, int B, int Tq, int NBk,
                                     int Hi, int Di, int blk, int64_t q_pos0, int mode) {
  if (B < 0 || Tq < 0 || NBk < 0 || q_pos0 < 0 || (mode != 0 && mode != 1)) return QSA_ERR_INVALID_ARGUMENT;
  if (Di != 64 || !hi_supported(Hi) || blk != 4) return QSA_ERR_UNSUPPORTED;
  if (seqlens) {
    if (Tq != 1) return QSA_ERR_INVALID_ARGUMENT;
  } else if (Tq > 0 && (q_pos0 + Tq - 1) / blk > NBk) {
    return QSA_ERR_INVALID_ARGUMENT;   // the pooled keys do not cover the queries' candidates
  }
  if (static_cast<long long>(B) * Tq > 0 && NBk > 0 && (!ok_ptr(qi) || !ok_ptr(kp))) return QSA_ERR_INVALID_ARGUMENT;
  return QSA_OK;
}

qsa_status_t qsa_index_score(const void* qi, const void* kp, const float* head_w, const int32_t* seqlens, int B,
                             int Tq, int NBk, int Hi, int Di, int blk, int64_t q_pos0, qsa_score_mode_t mode,
                             float* scores, int64_t ld_scores, void* stream) {
  QSA_NVTX();
  qsa_status_t st = check_score_args(qi, kp, seqlens, B, Tq, NBk, Hi, Di, blk, q_pos0, mode);
  if (st != QSA_OK) return st;
  if (ld_scores < std::max(NBk, 1)) return QSA_ERR_INVALID_ARGUMENT;
  if (static_cast<long long>(B) * Tq == 0 || NBk == 0) return QSA_OK;
  if (scores == nullptr) return QSA_ERR_INVALID_ARGUMENT;
  const DeviceInfo* di = device_info();
  if (!di) return QSA_ERR_CUDA;
  if (seqlens)
    return cuda_status(launch_score_decode(di, qi, kp, head_w, seqlens, B, NBk, Hi, Di, blk, mode, scores, ld_scores,
                                           S(stream)));
  return cuda_status(launch_score_prefill(di, qi, kp, head_w, B, Tq, NBk, Hi, Di, blk, q_pos0, mode, 0, B, 0, Tq,
                                          scores, ld_scores, static_cast<long long>(Tq) * ld_scores, S(stream)));
}

qsa_status_t qsa_select_topk(const float* scores, int64_t ld_scores, const void* qi, const void* kp,
                             const float* head_w, const int32_t* seqlens, int B, int Tq, int NBk, int Hi, int Di,
                             int blk, int64_t q_pos0, qsa_score_mode_t mode, int k, int32_t* idx, void* workspace,
                             size_t ws_bytes, void* stream) {
  QSA_NVTX();
  if (k < 1 || B < 0 || Tq < 0 || NBk < 0 || q_pos0 < 0) return QSA_ERR_INVALID_ARGUMENT;
  if (blk != 4) return QSA_ERR_UNSUPPORTED;
  if (seqlens && Tq != 1) return QSA_ERR_INVALID_ARGUMENT;
  if (!seqlens && Tq > 0 && (q_pos0 + Tq - 1) / blk > NBk) return QSA_ERR_INVALID_ARGUMENT;
  if (static_cast<long long>(B) * Tq == 0) return QSA_OK;
  if (idx == nullptr) return QSA_ERR_INVALID_ARGUMENT;
  cudaStream_t s = S(stream);
  if (scores) {
    if (ld_scores < std::max(NBk, 1)) return QSA_ERR_INVALID_ARGUMENT;
    const DeviceInfo* di = device_info();
    if (!di) return QSA_ERR_CUDA;
    return cuda_status(launch_topk(di, scores, ld_scores, static_cast<long long>(Tq) * ld_scores, seqlens, Tq, NBk, blk,
                                   q_pos0, 0, B, 0, Tq, k, idx, s));
  }
  qsa_status_t st = check_score_args(qi, kp, seqlens, B, Tq, NBk, Hi, Di, blk, q_pos0, mode);
  if (st != QSA_OK) return st;
  float* ws = static_cast<float*>(workspace);
  const long long row_bytes = static_cast<long long>(std::max(NBk, 1)) * 4;
  if (NBk > 0 && seqlens && (ws == nullptr || static_cast<long long>(ws_bytes) < row_bytes * B))
    return QSA_ERR_WORKSPACE_TOO_SMALL;
  const long long R = ws ? static_cast<long long>(ws_bytes) / row_bytes : 0;
  if (NBk > 0 && !seqlens && R < 1) return QSA_ERR_WORKSPACE_TOO_SMALL;
  const DeviceInfo* di = device_info();
  if (!di) return QSA_ERR_CUDA;
  if (NBk == 0) {   // no candidates anywhere: the lists are all -1
    return cuda_status(launch_topk(di, nullptr, 1, 0, seqlens, Tq, 0, blk, q_pos0, 0, B, 0, Tq, k, idx, s));
  }
  if (seqlens) {
    // Decode: the scores of every sequence, then the top-k with a cluster of CTAs per sequence
    // (one CTA per sequence for many sequences or short caches).
    const int parts = topk_cluster_parts(di, B, NBk, k);
    cudaError_t e = launch_score_decode(di, qi, kp, head_w, seqlens, B, NBk, Hi, Di, blk, mode, ws, NBk, s);
    if (e == cudaSuccess)
      e = parts > 0 ? launch_topk_cluster(di, ws, NBk, seqlens, B, NBk, blk, k, idx, parts, s)
                    : launch_topk(di, ws, NBk, NBk, seqlens, 1, NBk, blk, 0, 0, B, 0, 1, k, idx, s);
    return cuda_status(e);
  }
  // Filtered selection: sampled scores -> thresholds -> score + filter -> select over the lists
  // -> exact redo of failed rows, per chunk of rows of one sequence.
  {
    const FusedPlan fp = fused_plan(NBk, k);
    const long long fit = fused_rows_fit(fp, ws_bytes);
    const int path = g_select_path.load();
    const bool able = (Hi == 4 || Hi == 8) && k <= 1024 && fp.cap <= kFusedMaxCap;
    if (path == 2 && !able) return QSA_ERR_UNSUPPORTED;
    if (path == 2 && fit < 1) return QSA_ERR_WORKSPACE_TOO_SMALL;
    // automatic: rows long enough (the chunk's last row sees 16384 positions or more), and a
    // workspace holding 4096 rows or all of them
    if (path == 2 || (path == 0 && able && q_pos0 + Tq >= kFusedMinRows && fit >= std::min(Tq, 4096))) {
      long long R = std::min<long long>(Tq, fit);
      if (R < Tq && R >= 64) R &= ~63ll;
      uint8_t* w8 = static_cast<uint8_t*>(workspace);
      float* samp = reinterpret_cast<float*>(w8);
      size_t off = align256(static_cast<size_t>(R) * fp.ld_s * 4);
      float* tau = reinterpret_cast<float*>(w8 + off);
      off += align256(static_cast<size_t>(R) * 4);
      int* cnt = reinterpret_cast<int*>(w8 + off);
      off += align256(static_cast<size_t>(R) * 4);
      int* fail = reinterpret_cast<int*>(w8 + off);
      off += align256(static_cast<size_t>(R + 1) * 4);
      uint2* cand = reinterpret_cast<uint2*>(w8 + off);
      off += align256(static_cast<size_t>(R) * fp.cap * 8);
      float* scratch = reinterpret_cast<float*>(w8 + off);
      const int rank = g_sample_rank.load() > 0 ? g_sample_rank.load() : fp.rank;
      const size_t qi_b = static_cast<size_t>(Tq) * Hi * Di * 2, kp_b = static_cast<size_t>(NBk) * Di * 2;
      cudaError_t e = cudaSuccess;
      for (int b = 0; e == cudaSuccess && b < B; ++b) {
        const uint8_t* qib = static_cast<const uint8_t*>(qi) + b * qi_b;
        const uint8_t* kpb = static_cast<const uint8_t*>(kp) + b * kp_b;
        for (int r0 = 0; e == cudaSuccess && r0 < Tq; r0 += static_cast<int>(R)) {
          const int rows = static_cast<int>(std::min<long long>(R, Tq - r0));
          e = launch_score_prefill(di, qib, kpb, head_w, 1, Tq, NBk, Hi, Di, blk, q_pos0, mode, 0, 1, r0, rows, samp,
                                   fp.ld_s, 0, s, kSampleShift, kSampleOff);
          if (e == cudaSuccess)
            e = launch_select_tau(di, samp, fp.ld_s, NBk, q_pos0, r0, rows, fp.cap, rank, kSampleShift, kSampleOff,
                                  tau, fail, s);
          if (e == cudaSuccess)
            e = launch_score_filter(di, qib, kpb, head_w, Tq, NBk, Hi, q_pos0, mode, 0, 1, r0, rows, tau, cand, cnt,
                                    fp.cap, s);
          if (e == cudaSuccess)
            e = launch_select_candidates(di, cand, cnt, fp.cap, Tq, NBk, q_pos0, b, r0, rows, k, idx, fail, s);
          if (e == cudaSuccess)
            e = launch_topk_fallback(di, qi, kp, head_w, Hi, mode, Tq, NBk, q_pos0, b, fail, scratch, kFallbackCtas, k,
                                     idx, s);
        }
      }
      return cuda_status(e);
    }
  }
  const long long chunks = static_cast<long long>(B) * ((Tq + R - 1) / R);
  SideStream* side = chunks > 1 && R >= 2 ? side_stream(di->device) : nullptr;
  if (side == nullptr) {
    for (int b = 0; b < B; ++b) {
      for (int r0 = 0; r0 < Tq; r0 += static_cast<int>(std::min<long long>(R, Tq))) {
        const int rows = static_cast<int>(std::min<long long>(R, Tq - r0));
        cudaError_t e = launch_score_prefill(di, qi, kp, head_w, B, Tq, NBk, Hi, Di, blk, q_pos0, mode, b, 1, r0,
                                             rows, ws, NBk, 0, s);
        if (e == cudaSuccess) e = launch_topk(di, ws, NBk, 0, nullptr, Tq, NBk, blk, q_pos0, b, 1, r0, rows, k, idx, s);
        if (e != cudaSuccess) return QSA_ERR_CUDA;
      }
    }
    return QSA_OK;
  }
  // Two halves of the workspace: the scores of chunk i+1 are computed on the caller's stream while
  // the top-k of chunk i runs on a side stream (the kernels fit on an SM together).  Events order
  // every reuse of a half and join the side stream back into the caller's stream.
  const long long R2 = R / 2;
  std::lock_guard<std::mutex> lk(side->mu);
  cudaError_t e = cudaEventRecord(side->begin, s);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(side->stream, side->begin, 0);
  long long c = 0;
  for (int b = 0; e == cudaSuccess && b < B; ++b) {
    for (int r0 = 0; e == cudaSuccess && r0 < Tq; r0 += static_cast<int>(R2), ++c) {
      const int rows = static_cast<int>(std::min<long long>(R2, Tq - r0));
      const int buf = static_cast<int>(c & 1);
      float* half = ws + buf * R2 * NBk;
      if (c >= 2) e = cudaStreamWaitEvent(s, side->topk_done[buf], 0);
      if (e == cudaSuccess)
        e = launch_score_prefill(di, qi, kp, head_w, B, Tq, NBk, Hi, Di, blk, q_pos0, mode, b, 1, r0, rows, half, NBk,
                                 0, s);
      if (e == cudaSuccess) e = cudaEventRecord(side->score_done[buf], s);
      if (e == cudaSuccess) e = cudaStreamWaitEvent(side->stream, side->score_done[buf], 0);
      if (e == cudaSuccess)
        e = launch_topk(di, half, NBk, 0, nullptr, Tq, NBk, blk, q_pos0, b, 1, r0, rows, k, idx, side->stream);
      if (e == cudaSuccess) e = cudaEventRecord(side->topk_done[buf], side->stream);
    }
  }
  if (e == cudaSuccess) e = cudaEventRecord(side->end, side->stream);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(s, side->end, 0);
  return cuda_status(e);
}

static qsa_status_t check_attn_shape(int Hq, int Hkv, int D, int blk, int k_blocks) {
  if (Hq < 1 || Hkv < 1 || k_blocks < 0) return QSA_ERR_INVALID_ARGUMENT;
  if (Hq % Hkv) return QSA_ERR_INVALID_ARGUMENT;
  if ((D != 128 && D != 256) || blk != 4 || Hkv > 2 || Hq / Hkv > 16) return QSA_ERR_UNSUPPORTED;
  return QSA_OK;
}

qsa_status_t qsa_decode_select(const void* qi, void* kp, const void* ki, int64_t ki_batch_stride,
                               const float* head_w, const int32_t* seqlens, int B, int NBk, int Hi, int Di, int blk,
                               qsa_score_mode_t mode, const qsa_rope_params_t* rope, int k, int32_t* idx,
                               void* workspace, size_t ws_bytes, void* stream) {
  QSA_NVTX();
  if (k < 1 || B < 0 || NBk < 0 || ki_batch_stride < 0) return QSA_ERR_INVALID_ARGUMENT;
  if (blk != 4) return QSA_ERR_UNSUPPORTED;
  if (B == 0) return QSA_OK;
  if (seqlens == nullptr || idx == nullptr || !ok_ptr(ki)) return QSA_ERR_INVALID_ARGUMENT;
  RopeParams rp;
  if (resolve_rope(rope, &rp) != QSA_OK) return QSA_ERR_INVALID_ARGUMENT;
  const long long kis = ki_batch_stride ? ki_batch_stride : static_cast<long long>(NBk) * blk * Di;
  if (kis < static_cast<long long>(NBk) * blk * Di) return QSA_ERR_INVALID_ARGUMENT;
  qsa_status_t st = check_score_args(qi, kp, seqlens, B, 1, NBk, Hi, Di, blk, 0, mode);
  if (st != QSA_OK) return st;
  if (NBk == 0) return qsa_select_topk(nullptr, 0, qi, kp, head_w, seqlens, B, 1, NBk, Hi, Di, blk, 0, mode, k, idx,
                                       workspace, ws_bytes, stream);
  float* ws = static_cast<float*>(workspace);
  const long long row_bytes = static_cast<long long>(NBk) * 4;
  if (ws == nullptr || static_cast<long long>(ws_bytes) < row_bytes * B) return QSA_ERR_WORKSPACE_TOO_SMALL;
  const DeviceInfo* di = device_info();
  if (!di) return QSA_ERR_CUDA;
  cudaStream_t s = S(stream);
  const NewBlockPool np{static_cast<const uint16_t*>(ki), static_cast<uint16_t*>(kp), kis,
                        static_cast<long long>(NBk) * Di, rp};
  const int parts = topk_cluster_parts(di, B, NBk, k);
  cudaError_t e = launch_score_decode(di, qi, kp, head_w, seqlens, B, NBk, Hi, Di, blk, mode, ws, NBk, s, &np);
  if (e == cudaSuccess)
    e = parts > 0 ? launch_topk_cluster(di, ws, NBk, seqlens, B, NBk, blk, k, idx, parts, s)
                  : launch_topk(di, ws, NBk, NBk, seqlens, 1, NBk, blk, 0, 0, B, 0, 1, k, idx, s);
  return cuda_status(e);
}

qsa_status_t qsa_sparse_attn_prefill(const void* q, const void* k, const void* v, const int32_t* idx, int B, int Tq,
                                     int Tk, int Hq, int Hkv, int D, int k_blocks, int blk, int64_t q_pos0,
                                     float scale, void* out, float* lse, void* stream) {
  QSA_NVTX();
  qsa_status_t st = check_attn_shape(Hq, Hkv, D, blk, k_blocks);
  if (st != QSA_OK) return st;
  if (B < 0 || Tq < 0 || Tk < 0 || q_pos0 < 0 || q_pos0 + Tq > Tk) return QSA_ERR_INVALID_ARGUMENT;
  if (static_cast<long long>(B) * Tq == 0) return QSA_OK;
  if (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(out) || (k_blocks > 0 && idx == nullptr))
    return QSA_ERR_INVALID_ARGUMENT;
  if (static_cast<long long>(B) * Tq > 0x7fffffffLL) return QSA_ERR_UNSUPPORTED;
  const DeviceInfo* di = device_info();
  if (!di) return QSA_ERR_CUDA;
  return cuda_status(
      launch_attn_prefill(di, q, k, v, idx, B, Tq, Tk, Hq, Hkv, D, k_blocks, q_pos0, scale, out, lse, S(stream)));
}

qsa_status_t qsa_sparse_attn_prefill_ws(const void* q, const void* k, const void* v, const int32_t* idx, int B,
                                        int Tq, int Tk, int Hq, int Hkv, int D, int k_blocks, int blk,
                                        int64_t q_pos0, float scale, void* out, float* lse, void* workspace,
                                        size_t ws_bytes, void* stream) {
  QSA_NVTX();
  qsa_status_t st = check_attn_shape(Hq, Hkv, D, blk, k_blocks);
  if (st != QSA_OK) return st;
  if (B < 0 || Tq < 0 || Tk < 0 || q_pos0 < 0 || q_pos0 + Tq > Tk) return QSA_ERR_INVALID_ARGUMENT;
  if (static_cast<long long>(B) * Tq == 0) return QSA_OK;
  if (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(out) || (k_blocks > 0 && idx == nullptr))
    return QSA_ERR_INVALID_ARGUMENT;
  if (static_cast<long long>(B) * Tq > 0x7fffffffLL) return QSA_ERR_UNSUPPORTED;
  const DeviceInfo* di = device_info();
  if (!di) return QSA_ERR_CUDA;
  // Automatic choice: row by row.  On the measured workloads (random queries, whose consecutive
  // rows share little of their selections: the union of 16 rows is 0.38-0.46 of their lists) the
  // row kernel is the faster one; the query tiles are chosen with qsa_set_attn_options.  When the
  // workspace holds K and V interleaved by block (and the shape is the 16-slot kernel's), the
  // automatic choice first interleaves the positions the rows can see and gathers each block's K
  // and V with one copy: 4 KB copies instead of two of 2 KB, a higher per-SM gather rate.
  const int path = g_attn_path.load();
  const bool tiles_ok = attn_tc_supported(Hq, Hkv, D, k_blocks) && path == 2 && workspace != nullptr &&
                        ok_ptr(workspace) && ws_bytes >= 512 + attn_tc_tile_bytes(k_blocks);
  if (path == 2 && !tiles_ok)
    return attn_tc_supported(Hq, Hkv, D, k_blocks) ? QSA_ERR_WORKSPACE_TOO_SMALL : QSA_ERR_UNSUPPORTED;
  if (path == 0 && attn_kv_supported(Hq, Hkv, D) && B <= 65535 && workspace != nullptr && ok_ptr(workspace) &&
      ws_bytes >= attn_kv_bytes(B, Tk, Hkv, D)) {
    const long long j1 = (q_pos0 + Tq + 3) / 4;
    cudaError_t e = launch_interleave_kv(di, k, v, workspace, B, Tk, Hkv, D, 0, j1, S(stream));
    if (e == cudaSuccess)
      e = launch_attn_prefill_kv(di, q, workspace, idx, B, Tq, Tk, Hq, Hkv, k_blocks, q_pos0, scale, out, lse,
                                 S(stream));
    return cuda_status(e);
  }
  if (!tiles_ok)
    return cuda_status(
        launch_attn_prefill(di, q, k, v, idx, B, Tq, Tk, Hq, Hkv, D, k_blocks, q_pos0, scale, out, lse, S(stream)));
  return cuda_status(launch_attn_prefill_tc(di, q, k, v, idx, B, Tq, Tk, Hq, Hkv, k_blocks, q_pos0, scale, out, lse,
                                            workspace, ws_bytes, S(stream)));
}

qsa_status_t qsa_interleave_kv(const void* k, const void* v, void* kv, int B, int Tk, int Hkv, int D, int blk,
                               int64_t pos_lo, int64_t pos_hi, void* stream) {
  QSA_NVTX();
  if (blk != 4 || B < 0 || Tk < 0 || pos_lo < 0 || pos_lo > pos_hi || pos_hi > Tk) return QSA_ERR_INVALID_ARGUMENT;
  if (D != 128 || (Hkv != 1 && Hkv != 2)) return QSA_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * (pos_hi - pos_lo) == 0) return QSA_OK;
  if (!ok_ptr(k) || !ok_ptr(v) || !ok_ptr(kv) || B > 65535) return QSA_ERR_INVALID_ARGUMENT;
  const DeviceInfo* di = device_info();
  if (!di) return QSA_ERR_CUDA;
  return cuda_status(launch_interleave_kv(di, k, v, kv, B, Tk, Hkv, D, pos_lo / 4, (pos_hi + 3) / 4, S(stream)));
}

qsa_status_t qsa_sparse_attn_prefill_kv(const void* q, const void* kv, const int32_t* idx, int B, int Tq, int Tk,
                                        int Hq, int Hkv, int D, int k_blocks, int blk, int64_t q_pos0, float scale,
                                        void* out, float* lse, void* stream) {
  QSA_NVTX();
  qsa_status_t st = check_attn_shape(Hq, Hkv, D, blk, k_blocks);
  if (st != QSA_OK) return st;
  if (!attn_kv_supported(Hq, Hkv, D)) return QSA_ERR_UNSUPPORTED;
  if (B < 0 || Tq < 0 || Tk < 0 || q_pos0 < 0 || q_pos0 + Tq > Tk) return QSA_ERR_INVALID_ARGUMENT;
  if (static_cast<long long>(B) * Tq == 0) return QSA_OK;
  if (!ok_ptr(q) || !ok_ptr(kv) || !ok_ptr(out) || (k_blocks > 0 && idx == nullptr)) return QSA_ERR_INVALID_ARGUMENT;
  if (static_cast<long long>(B) * Tq > 0x7fffffffLL) return QSA_ERR_UNSUPPORTED;
  const DeviceInfo* di = device_info();
  if (!di) return QSA_ERR_CUDA;
  return cuda_status(
      launch_attn_prefill_kv(di, q, kv, idx, B, Tq, Tk, Hq, Hkv, k_blocks, q_pos0, scale, out, lse, S(stream)));
}

size_t qsa_attn_prefill_workspace_size(int B, int Tq, int Tk, int Hq, int Hkv, int D, int k_blocks) {
  if (B < 0 || Tq < 0 || Tk < 0 || Hq < 1 || Hkv < 1 || D < 1 || k_blocks < 1) return 0;
  size_t n = qsa_workspace_size(QSA_OP_SPARSE_ATTN_PREFILL, B, Tq, 0, k_blocks, Hq, D, 0);
  if (attn_kv_supported(Hq, Hkv, D)) n = std::max(n, attn_kv_bytes(B, Tk, Hkv, D));
  return n;
}

qsa_status_t qsa_set_attn_options(int path) {
  if (path < 0 || path > 2) return QSA_ERR_INVALID_ARGUMENT;
  g_attn_path.store(path);
  return QSA_OK;
}

int qsa_decode_default_splits(int B, int k_blocks) {
  const DeviceInfo* di = device_info();
  if (!di || B < 1) return 1;
  return decode_default_splits(di, B, std::max(k_blocks, 1));
}

int qsa_decode_split_merge(int B, int Hq, int Hkv, int D, int num_splits) {
  if (B < 1 || Hq < 1 || Hkv < 1 || D < 1 || num_splits < 1 || Hq % Hkv) return -1;
  if (num_splits == 1) return 0;
  const DeviceInfo* di = device_info();
  if (!di) return -1;
  return decode_cluster_ok(di, B, Hq, Hkv, D, num_splits) ? 1 : 2;
}

qsa_status_t qsa_sparse_attn_decode(const void* q, const void* kcache, const void* vcache, const int32_t* seqlens,
                                    const int32_t* idx, int B, int Lmax, int Hq, int Hkv, int D, int k_blocks, int blk,
                                    float scale, int num_splits, void* out, float* lse, void* workspace,
                                    size_t ws_bytes, void* stream) {
  QSA_NVTX();
  qsa_status_t st = check_attn_shape(Hq, Hkv, D, blk, k_blocks);
  if (st != QSA_OK) return st;
  if (B < 0 || Lmax < 1 || num_splits < 0) return QSA_ERR_INVALID_ARGUMENT;
  if (B == 0) return QSA_OK;
  if (!ok_ptr(q) || !ok_ptr(kcache) || !ok_ptr(vcache) || !ok_ptr(out) || seqlens == nullptr ||
      (k_blocks > 0 && idx == nullptr))
    return QSA_ERR_INVALID_ARGUMENT;
  const DeviceInfo* di = device_info();
  if (!di) return QSA_ERR_CUDA;
  int splits = num_splits == 0 ? decode_default_splits(di, B, std::max(k_blocks, 1)) : num_splits;
  splits = std::max(1, std::min(splits, std::max(k_blocks, 1)));
  float* part = nullptr;
  if (splits > 1) {
    const size_t need = static_cast<size_t>(B) * splits * Hq * (D + 2) * sizeof(float);
    if (workspace == nullptr || ws_bytes < need) return QSA_ERR_WORKSPACE_TOO_SMALL;
    part = static_cast<float*>(workspace);
  }
  return cuda_status(launch_attn_decode(di, q, kcache, vcache, seqlens, idx, B, Lmax, Hq, Hkv, D, k_blocks, scale,
                                        splits, out, lse, part, S(stream)));
}

size_t qsa_workspace_size(qsa_op_t op, int B, int Tq, int NBk, int k, int Hq, int D, int num_splits) {
  if (op == QSA_OP_SELECT_TOPK) {
    if (B < 0 || Tq < 0 || NBk < 0) return 0;
    const long long row = static_cast<long long>(std::max(NBk, 1)) * 4;
    if (Tq <= 1) return static_cast<size_t>(row * std::max(B, 1));
    const long long cap = 512ll << 20;   // chunk of score rows kept at or below 512 MiB
    const long long rows = std::max(1ll, std::min<long long>(Tq, cap / row));
    long long bytes = rows * row;
    if (k >= 1) {   // room for the filtered path: all rows of a sequence, or chunks within ~4 GiB
      const FusedPlan fp = fused_plan(NBk, k);
      const long long frows = std::max(64ll, std::min<long long>(Tq, (kFusedTarget - fp.fixed) / fp.per_row));
      bytes = std::max(bytes, fp.fixed + frows * fp.per_row);
    }
    return static_cast<size_t>(bytes);
  }
  if (op == QSA_OP_SPARSE_ATTN_PREFILL) {
    // the tile unions of up to 4096 tiles of 16 rows (all tiles when fewer)
    if (B < 0 || Tq < 0 || k < 1) return 0;
    const long long tiles = static_cast<long long>(B) * ((Tq + 15) / 16);
    const long long n = std::max(1ll, std::min(tiles, 4096ll));
    return static_cast<size_t>(1024 + n * static_cast<long long>(attn_tc_tile_bytes(k)));
  }
  if (op == QSA_OP_SPARSE_ATTN_DECODE) {
    if (B < 1 || Hq < 1 || D < 1) return 0;
    int splits = num_splits > 0 ? num_splits : qsa_decode_default_splits(B, k);
    splits = std::max(1, std::min(splits, std::max(k, 1)));
    return static_cast<size_t>(B) * splits * Hq * (D + 2) * sizeof(float);
  }
  return 0;
}

qsa_status_t qsa_get_device_status(void* stream) {
  if (cudaStreamSynchronize(S(stream)) != cudaSuccess) return QSA_ERR_CUDA;
  unsigned v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_status_word, sizeof v) != cudaSuccess) return QSA_ERR_CUDA;
  if (v != 0 && cudaMemcpyToSymbol(g_status_word, &zero, sizeof zero) != cudaSuccess) return QSA_ERR_CUDA;
  return static_cast<qsa_status_t>(v);
}

qsa_status_t qsa_wait_timeout_selftest(uint64_t timeout_ns, void* stream) {
  const DeviceInfo* di = device_info();
  if (!di) return QSA_ERR_CUDA;
  KernelCtl ctl{di->status, timeout_ns ? timeout_ns : 1000000ull};
  wait_selftest_kernel<<<1, 32, 0, S(stream)>>>(ctl);
  return cuda_status(cudaPeekAtLastError());
}

}  // extern "C"
