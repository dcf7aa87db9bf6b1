// Micro-block key pooling with RoPE after pooling, and RoPE of the indexer queries.
//
// "Qwen3.8-Flash-Next architecture" (flozi.net), "Der Weg eines Tokens durch das Modell", item 2:
// groups of four indexer keys are averaged into one micro-block key, and the rotary embedding is
// applied after the averaging so that keys of different positions are not mixed at different
// rotation phases.  For contexts beyond the trained one the frequencies can be YaRN-scaled.
//
// Bandwidth-bound and tiny next to the rest of the path (at 131072 tokens: 16.8 MB read, 4.2 MB
// written).  One warp per output row; lane i owns the rotation pair (i, i + Di/2), so the pair
// never leaves a thread.  The mean is formed exactly in double (a sum of four bf16 values) and
// rounded once to bf16, which makes the result bit-identical to the CPU oracle without RoPE.
#include "pool_math.cuh"

namespace qsa {
namespace {

__global__ void __launch_bounds__(256) pool_kernel(const uint16_t* __restrict__ ki, uint16_t* __restrict__ kp,
                                                   int B, int L, int Di, int blk, RopeParams rp, long long pos0,
                                                   long long ki_bs, long long kp_bs) {
  const int nb = L / blk;
  const long long row = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (row >= static_cast<long long>(B) * nb) return;
  const long long b = row / nb, j = row % nb;
  const uint16_t* src = ki + b * ki_bs + j * blk * Di;
  uint16_t* dst = kp + b * kp_bs + j * Di;
  pool_row_warp(src, dst, Di, blk, rp, static_cast<double>(pos0 + j * blk));
}

__global__ void __launch_bounds__(256) rope_q_kernel(const uint16_t* qi, uint16_t* qo,
                                                     int B, int Tq, int Hi, int Di, long long q_pos0,
                                                     const int32_t* __restrict__ seqlens, RopeParams rp) {
  const long long row = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);   // (b, t, h)
  if (row >= static_cast<long long>(B) * Tq * Hi) return;
  const int lane = threadIdx.x & 31;
  const long long bt = row / Hi;
  const long long b = bt / Tq, t = bt % Tq;
  const double pos = seqlens ? static_cast<double>(seqlens[b] - 1) : static_cast<double>(q_pos0 + t);
  const int half = Di / 2;
  // Each rotation pair is read and written by one thread only, so qo may alias qi.
  for (int i = lane; i < half; i += 32) {
    double y1, y2;
    rope_rotate(bf16_to_f64(qi[row * Di + i]), bf16_to_f64(qi[row * Di + i + half]), pos, i, Di, rp, &y1, &y2);
    qo[row * Di + i] = bf16_bits_rne_f64(y1);
    qo[row * Di + i + half] = bf16_bits_rne_f64(y2);
  }
}

}  // namespace

cudaError_t launch_pool(const void* ki, void* kp, int B, int L, int Di, int blk, const RopeParams& rp, long long pos0,
                        long long ki_bs, long long kp_bs, cudaStream_t s) {
  const long long rows = static_cast<long long>(B) * (L / blk);
  if (rows == 0) return cudaSuccess;
  const unsigned grid = static_cast<unsigned>((rows + 7) / 8);
  pool_kernel<<<grid, 256, 0, s>>>(static_cast<const uint16_t*>(ki), static_cast<uint16_t*>(kp), B, L, Di, blk,
                                   rp, pos0, ki_bs, kp_bs);
  return cudaPeekAtLastError();
}

cudaError_t launch_rope_queries(const void* qi, void* qo, int B, int Tq, int Hi, int Di, long long q_pos0,
                                const int32_t* seqlens, const RopeParams& rp, cudaStream_t s) {
  const long long rows = static_cast<long long>(B) * Tq * Hi;
  if (rows == 0) return cudaSuccess;
  const unsigned grid = static_cast<unsigned>((rows + 7) / 8);
  rope_q_kernel<<<grid, 256, 0, s>>>(static_cast<const uint16_t*>(qi), static_cast<uint16_t*>(qo), B, Tq, Hi, Di,
                                     q_pos0, seqlens, rp);
  return cudaPeekAtLastError();
}

}  // namespace qsa
