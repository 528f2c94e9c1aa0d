// MXFP8 encoding of one 32-element block (OCP Microscaling, E4M3 elements,
// UE8M0 shared exponent), shared by the stand-alone quantiser and the
// epilogues that write the projection operand straight in MXFP8.
//
// "Video DeltaNet: A Video-Native Hybrid Attention for Livestream Video
// Generation", implementation section ("Other optimizations": MXFP8 GEMMs).
// The block's shared exponent is e = floor(log2(max |v|)) - 8 (8 = exponent of
// the largest normal E4M3 value, 448), stored as e + 127; an all-zero block
// takes e = -127.  Each element is v * 2^-e rounded to E4M3, to nearest with
// ties to even, saturating at +-448.  The values handed in here are fp16
// values (as float), so max |v| is zero or a normal float32 and e comes from
// its exponent field exactly.
#pragma once
#include <cuda_fp16.h>
#include <stddef.h>
#include <stdint.h>

namespace vdn {
namespace mx {

// e of a block whose largest magnitude is amax (amax zero or normal)
__device__ __forceinline__ int block_exp(float amax) {
  int e = amax > 0.f ? (int)((__float_as_uint(amax) >> 23) & 0xFF) - 127 - 8 : -127;
  return e < -127 ? -127 : (e > 127 ? 127 : e);
}

// 2^-e for e in [-127, 127] (exact)
__device__ __forceinline__ float inv_scale(int e) { return ldexpf(1.f, -e); }

// E4M3 codes of (lo, hi): lo in the low byte
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// Byte offset of the scale of row r, block j (32 elements) in the scale
// atoms of a matrix with K contraction columns: 512-byte atoms of 128 rows x
// 4 blocks, atom (r / 128) * (K / 128) + j / 4, byte 16 (r % 32) +
// 4 ((r % 128) / 32) + j % 4.
__device__ __forceinline__ size_t sf_offset(size_t r, int j, int K) {
  return ((r / 128) * (size_t)(K / 128) + (size_t)(j / 4)) * 512u + 16u * (r % 32) +
         4u * ((r % 128) / 32) + (size_t)(j % 4);
}

// Encodes 32 fp16 values (16 half2 words, element 2i in the low half of word
// i) into 32 E4M3 codes (8 words, element 4i in the low byte of word i);
// returns e + 127.
__device__ __forceinline__ uint32_t encode32(const uint32_t (&hw)[16], uint32_t (&cw)[8]) {
  float v[32];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const __half2 h = *reinterpret_cast<const __half2*>(&hw[i]);
    const float2 f = __half22float2(h);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const int e = block_exp(amax);
  const float inv = inv_scale(e);
#pragma unroll
  for (int i = 0; i < 8; ++i)
    cw[i] = e4m3x2(v[4 * i] * inv, v[4 * i + 1] * inv) |
            (e4m3x2(v[4 * i + 2] * inv, v[4 * i + 3] * inv) << 16);
  return (uint32_t)(e + 127);
}

}  // namespace mx
}  // namespace vdn
