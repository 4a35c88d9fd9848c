// MXFP8 (OCP Microscaling format v1.0 with E4M3 elements): blocks of 32
// consecutive elements along the contraction dimension share one E8M0 scale
// X = 2^(code - 127).  The format is the one the Olmo-core 3 news piece names
// ("MXFP8 low-precision switch") and the SonicMoE summary lists as future
// work; the pages do not define it, so this follows the public specification:
//   shared exponent = floor(log2(max |v|)) - 8   (8 = exponent of 448, the
//                     largest E4M3 value), clamped to the E8M0 range,
//   element         = E4M3 round-to-nearest-even of v / X, saturated to +-448.
//
// Scale layout (the one tcgen05 block-scaled MMAs read through tcgen05.cp
// .32x128b.warpx4): for a matrix of R rows (MN dimension, R a multiple of 128)
// and K columns, 512-byte blocks [R/128][K/128]; inside a block the scale of
// row r and 32-element K-block j sits at byte
//   (r % 32) * 16 + ((r / 32) % 4) * 4 + (j % 4).
#pragma once

#include <stdint.h>

#include "common.cuh"

namespace moe {

// Byte offset of the scale of row r, 32-element K-block kb, in a scale array
// with `kchunks` = K / 128 blocks per 128 rows.
__host__ __device__ __forceinline__ size_t mx_sf_offset(int r, int kb, int kchunks) {
  return ((size_t)(r >> 7) * kchunks + (kb >> 2)) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 +
         (kb & 3);
}

// E8M0 code of a block whose largest magnitude is amax (finite, >= 0):
// floor(log2 amax) - 8 + 127 = (biased fp32 exponent of amax) - 8, clamped at
// 0 (also for amax = 0 and fp32-subnormal amax, whose shared exponent is at
// or below the E8M0 floor 2^-127).
__device__ __forceinline__ uint32_t mx_scale_code(float amax) {
  const uint32_t ef = (__float_as_uint(amax) >> 23) & 0xFFu;
  return ef > 8u ? ef - 8u : 0u;
}

// 1 / X = 2^(127 - code), exact (a normal fp32 for every code in [0, 246]).
__device__ __forceinline__ float mx_inv_scale(uint32_t code) {
  return __uint_as_float((254u - code) << 23);
}

// Two E4M3 codes (round to nearest even, saturated to +-448): lo in the low byte.
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// Quantise 32 consecutive values (rounded to bf16 first, as stored) as one
// MXFP8 block: 32 E4M3 bytes to dst (16-byte aligned) and the code to *sf.
__device__ __forceinline__ void mx_store_block(const float* v, uint8_t* dst, uint8_t* sf) {
  float b[32];
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    b[i] = __bfloat162float(__float2bfloat16_rn(v[i]));
    amax = fmaxf(amax, fabsf(b[i]));
  }
  const uint32_t code = mx_scale_code(amax);
  const float inv = mx_inv_scale(code);
  uint32_t w[8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
    w[i] = cvt_e4m3x2(b[4 * i] * inv, b[4 * i + 1] * inv) |
           (cvt_e4m3x2(b[4 * i + 2] * inv, b[4 * i + 3] * inv) << 16);
  reinterpret_cast<uint4*>(dst)[0] = make_uint4(w[0], w[1], w[2], w[3]);
  reinterpret_cast<uint4*>(dst)[1] = make_uint4(w[4], w[5], w[6], w[7]);
  *sf = (uint8_t)code;
}

}  // namespace moe
