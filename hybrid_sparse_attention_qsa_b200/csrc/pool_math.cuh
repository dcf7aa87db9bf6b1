// Micro-block key pooling arithmetic shared by the pooling kernel and the decode score kernel
// (which pools the newest completed block of each sequence in its prologue).
//
// "Qwen3.8-Flash-Next architecture" (flozi.net), "Der Weg eines Tokens durch das Modell", item 2:
// groups of four indexer keys are averaged into one micro-block key, and the rotary embedding is
// applied after the averaging.  The mean is formed exactly in double (a sum of four bf16 values)
// and rounded once to bf16; with RoPE the rotation is applied in double before that rounding.
#pragma once

#include "launch.h"

namespace qsa {

__device__ __forceinline__ double bf16_to_f64(uint16_t h) {
  return static_cast<double>(__uint_as_float(static_cast<uint32_t>(h) << 16));
}

// YaRN context extension of the rotary frequencies ("YaRN: Efficient Context Window Extension of
// Large Language Models", Peng et al. 2023, sections 3.2 and 3.4): with r = orig_ctx * f / 2 pi
// rotations of a pair over the original context and g = clamp((r - alpha) / (beta - alpha), 0, 1),
// the frequency f becomes (1 - g) f / factor + g f, and the rotated pair is scaled by mscale.
// factor <= 1 leaves plain RoPE.
__device__ __forceinline__ void rope_rotate(double x1, double x2, double pos, int i, int Di, const RopeParams& rp,
                                            double* y1, double* y2) {
  double inv_freq = pow(rp.theta, -2.0 * static_cast<double>(i) / static_cast<double>(Di));
  double m = 1.0;
  if (rp.factor > 1.0) {
    const double r = rp.orig_ctx * inv_freq / 6.283185307179586476925286766559;
    const double g = fmin(1.0, fmax(0.0, (r - rp.alpha) / (rp.beta - rp.alpha)));
    inv_freq = (1.0 - g) * inv_freq / rp.factor + g * inv_freq;
    m = rp.mscale;
  }
  double s, c;
  sincos(pos * inv_freq, &s, &c);
  *y1 = m * (x1 * c - x2 * s);
  *y2 = m * (x2 * c + x1 * s);
}

// One pooled key row by one warp: src = blk consecutive rows of Di bf16 keys, dst = Di bf16;
// lane i owns the rotation pair (i, i + Di/2) (so the pair never leaves a thread); pos = the
// position of the block's first token.
__device__ __forceinline__ void pool_row_warp(const uint16_t* src, uint16_t* dst, int Di, int blk, const RopeParams& rp,
                                              double pos) {
  const int lane = threadIdx.x & 31;
  const int half = Di / 2;
  for (int i = lane; i < half; i += 32) {
    double m1 = 0.0, m2 = 0.0;
    for (int t = 0; t < blk; ++t) {
      m1 += bf16_to_f64(src[t * Di + i]);
      m2 += bf16_to_f64(src[t * Di + i + half]);
    }
    m1 /= static_cast<double>(blk);
    m2 /= static_cast<double>(blk);
    if (rp.theta > 0.0) {
      double y1, y2;
      rope_rotate(m1, m2, pos, i, Di, rp, &y1, &y2);
      m1 = y1;
      m2 = y2;
    }
    dst[i] = bf16_bits_rne_f64(m1);
    dst[i + half] = bf16_bits_rne_f64(m2);
  }
}

}  // namespace qsa
