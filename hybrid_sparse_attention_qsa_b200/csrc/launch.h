// Internal launchers behind the C ABI (one per kernel family).  Arguments are validated by the
// ABI layer before any of these is called.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <nvtx3/nvToolsExt.h>

#include "common.cuh"

namespace qsa {

// An NVTX range around a C-ABI call (header-only NVTX v3: one pointer test when no tool listens).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};
#define QSA_NVTX() ::qsa::NvtxRange qsa_nvtx_range_(__func__)

struct DeviceInfo {
  int device;
  int num_sms;
  unsigned* status;   // device address of the status word
};
// Per-device cached attributes of the current device (nullptr on a runtime error).
const DeviceInfo* device_info();
KernelCtl kernel_ctl(const DeviceInfo* di);
// The prefill attention path chosen with qsa_set_attn_options (0 automatic, 1 rows, 2 tiles).
int attn_path();

// Rotary parameters of the indexer (theta <= 0: no rotation); factor > 1 turns on YaRN scaling
// with the given original context, ramp bounds and magnitude factor (already resolved).
struct RopeParams {
  double theta, factor, orig_ctx, alpha, beta, mscale;
};

cudaError_t launch_pool(const void* ki, void* kp, int B, int L, int Di, int blk, const RopeParams& rp, long long pos0,
                        long long ki_bs, long long kp_bs, cudaStream_t s);
cudaError_t launch_rope_queries(const void* qi, void* qo, int B, int Tq, int Hi, int Di, long long q_pos0,
                                const int32_t* seqlens, const RopeParams& rp, cudaStream_t s);

// Prefill scores for query rows [row0, row0 + rows) of batches [b0, b0 + nb) into
// scores + (b - b0) * batch_stride + (t - row0) * ld.
// With kshift > 0, column c of a row is the score of pooled block (c << kshift) + koff (the sampled
// scores behind the selection thresholds); columns past the row's visible blocks are not written.
cudaError_t launch_score_prefill(const DeviceInfo* di, const void* qi, const void* kp, const float* head_w, int B,
                                 int Tq, int NBk, int Hi, int Di, int blk, long long q_pos0, int mode, int b0, int nb,
                                 int row0, int rows, float* scores, long long ld, long long batch_stride,
                                 cudaStream_t s, int kshift = 0, int koff = 0);
// Scores of rows [row0, row0 + rows) of batches [b0, b0 + nb) compared with tau[list] on the fly;
// the survivors go to cand[list][0 .. cap) in block order and their number to cnt[list], where
// list = (b - b0) * rows + (t - row0).  Hi must be 4 or 8.
cudaError_t launch_score_filter(const DeviceInfo* di, const void* qi, const void* kp, const float* head_w, int Tq,
                                int NBk, int Hi, long long q_pos0, int mode, int b0, int nb, int row0, int rows,
                                const float* tau, uint2* cand, int* cnt, int cap, cudaStream_t s);
// Optional pooling of each sequence's newest completed block by the decode score kernel (ki
// nullptr: none).  ki/kp batch strides in elements; kp rows of Di = 64 keys.
struct NewBlockPool {
  const uint16_t* ki;
  uint16_t* kp;
  long long ki_bs, kp_bs;
  RopeParams rp;
};
cudaError_t launch_score_decode(const DeviceInfo* di, const void* qi, const void* kp, const float* head_w,
                                const int32_t* seqlens, int B, int NBk, int Hi, int Di, int blk, int mode,
                                float* scores, long long ld, cudaStream_t s, const NewBlockPool* np = nullptr);

// Top-k over score rows: row r of batch b (b0 <= b < b0 + nb, row0 <= r < row0 + rows) reads
// scores + (b - b0) * batch_stride + (r - row0) * ld and writes idx + (b * Tq + r) * k.
cudaError_t launch_topk(const DeviceInfo* di, const float* scores, long long ld, long long batch_stride,
                        const int32_t* seqlens, int Tq, int NBk, int blk, long long q_pos0, int b0, int nb, int row0,
                        int rows, int k, int32_t* idx, cudaStream_t s);
// Decode top-k with a thread-block cluster of `parts` CTAs per sequence row (row b reads
// scores + b * ld).  topk_cluster_parts gives the cluster size for this device and shape, or 0
// when the one-CTA-per-row kernel is the better choice (many rows, short rows, k > 1024).
int topk_cluster_parts(const DeviceInfo* di, int B, int NBk, int k);
cudaError_t launch_topk_cluster(const DeviceInfo* di, const float* scores, long long ld, const int32_t* seqlens, int B,
                                int NBk, int blk, int k, int32_t* idx, int parts, cudaStream_t s);

// Filtered selection (prefill): thresholds from sampled scores, the exact select over each row's
// candidate list, and the exact redo of the rows listed in fail[1 .. fail[0]].
cudaError_t launch_select_tau(const DeviceInfo* di, const float* samp, long long ld, int NBk, long long q_pos0,
                              int row0, int rows, int cap, int rank, int kshift, int koff, float* tau, int* fail,
                              cudaStream_t s);
cudaError_t launch_select_candidates(const DeviceInfo* di, const uint2* cand, const int* cnt, int cap, int Tq, int NBk,
                                     long long q_pos0, int b, int row0, int rows, int k, int32_t* idx, int* fail,
                                     cudaStream_t s);
cudaError_t launch_topk_fallback(const DeviceInfo* di, const void* qi, const void* kp, const float* head_w, int Hi,
                                 int mode, int Tq, int NBk, long long q_pos0, int b, const int* fail, float* scratch,
                                 int nctas, int k, int32_t* idx, cudaStream_t s);

cudaError_t launch_attn_prefill(const DeviceInfo* di, const void* q, const void* k, const void* v, const int32_t* idx,
                                int B, int Tq, int Tk, int Hq, int Hkv, int D, int k_blocks, long long q_pos0,
                                float scale, void* out, float* lse, cudaStream_t s);
// Row-by-row prefill attention over K and V interleaved by block (kv [B][ceil(Tk/4)][2][4][Hkv][D]:
// one copy fetches a block's K and V): D = 128, Hkv in {1, 2}, groups of up to 8 query heads.
bool attn_kv_supported(int Hq, int Hkv, int D);
size_t attn_kv_bytes(int B, int Tk, int Hkv, int D);
// Writes the interleaved blocks [j0, j1) of every sequence from k and v ([B][Tk][Hkv][D]).
cudaError_t launch_interleave_kv(const DeviceInfo* di, const void* k, const void* v, void* kv, int B, int Tk, int Hkv,
                                 int D, long long j0, long long j1, cudaStream_t s);
cudaError_t launch_attn_prefill_kv(const DeviceInfo* di, const void* q, const void* kv, const int32_t* idx, int B,
                                   int Tq, int Tk, int Hq, int Hkv, int k_blocks, long long q_pos0, float scale,
                                   void* out, float* lse, cudaStream_t s);
// Query-tile prefill attention on tcgen05 (sparse_attn_tc.cu): D = 128, groups of 8 query heads,
// k_blocks <= 1024.  The workspace holds the tile unions of as many 16-row tiles as fit (at least
// one: 256 + attn_tc_tile_bytes(k_blocks) bytes); the call walks the tiles in ranges of that many.
bool attn_tc_supported(int Hq, int Hkv, int D, int k_blocks);
size_t attn_tc_tile_bytes(int k_blocks);
cudaError_t launch_attn_prefill_tc(const DeviceInfo* di, const void* q, const void* k, const void* v,
                                   const int32_t* idx, int B, int Tq, int Tk, int Hq, int Hkv, int k_blocks,
                                   long long q_pos0, float scale, void* out, float* lse, void* ws, size_t ws_bytes,
                                   cudaStream_t s);
cudaError_t launch_attn_decode(const DeviceInfo* di, const void* q, const void* kc, const void* vc,
                               const int32_t* seqlens, const int32_t* idx, int B, int Lmax, int Hq, int Hkv, int D,
                               int k_blocks, float scale, int num_splits, void* out, float* lse, float* part,
                               cudaStream_t s);
int decode_default_splits(const DeviceInfo* di, int B, int k_blocks);
// Whether a decode launch with these sizes merges its splits inside thread-block clusters.
bool decode_cluster_ok(const DeviceInfo* di, int B, int Hq, int Hkv, int D, int splits);

cudaError_t launch_wait_selftest(const DeviceInfo* di, unsigned long long timeout_ns, cudaStream_t s);

}  // namespace qsa
