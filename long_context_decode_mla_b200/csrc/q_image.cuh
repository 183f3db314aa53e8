// Q operand image of one request for the e4m3 kernel (the exact-score split
// of the query, built once per request outside the decode kernel).
//
// Layout (kQImageBytes): the e4m3 hi codes of the latent times 2^a (four
// 8 KB chunks of 64 head rows x 128 values), the e4m3 lo codes of what hi
// leaves (four chunks), the bf16 rope (one chunk of 64 rows x 64 values),
// each chunk in the decode kernel's 128-byte-swizzled shared-memory order;
// then the 64 frame factors 2^-a (fp32).  The frame 2^a of a head puts the
// largest |q| of its latent in [128, 256), where q times 2^a is hi + lo for
// every bf16 value above 2^-9 of that largest one.  Head rows past the call's
// head count are zero.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "common.cuh"

namespace dcpmla {
namespace qimg {

constexpr uint32_t kChunk = 8192;                  // 64 rows x 128 bytes
constexpr uint32_t kHi = 0, kLo = 4 * kChunk, kRope = 8 * kChunk;
constexpr uint32_t kFrame = 9 * kChunk;            // 64 x fp32 2^-a
static_assert(kFrame + 64 * 4 == (uint32_t)kQImageBytes, "Q image layout");

// byte offset of 16-byte unit u of row r in a 128-byte-swizzled chunk
__device__ __forceinline__ uint32_t sw128(int r, int u) {
  return (uint32_t)((r >> 3) * 1024 + (r & 7) * 128 + ((u ^ (r & 7)) << 4));
}

// two fp32 -> two e4m3 (lo -> low byte), round to nearest even, saturated
__device__ __forceinline__ uint32_t e4m3x2_f32(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}
// two e4m3 (low byte first) -> two fp32, exact
__device__ __forceinline__ float2 e4m3x2_to_f32(uint32_t pair) {
  uint32_t h;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"((uint16_t)pair));
  float lo, hi;
  asm("{\n .reg .f16 a, b;\n mov.b32 {a, b}, %2;\n cvt.f32.f16 %0, a;\n cvt.f32.f16 %1, b;\n}\n"
      : "=f"(lo), "=f"(hi)
      : "r"(h));
  return make_float2(lo, hi);
}

// Two words of bf16 pairs (four values) times the frame 2^a -> the e4m3 codes
// of the four values (hi) and the e4m3 codes of what hi leaves of them (lo),
// first value in the low byte.  The product is exact (a power of two within
// range) and so is the remainder.
__device__ __forceinline__ void split_q4(uint32_t w0, uint32_t w1, float fa, uint32_t& hi,
                                         uint32_t& lo) {
  const float f0 = __uint_as_float(w0 << 16) * fa;
  const float f1 = __uint_as_float(w0 & 0xFFFF0000u) * fa;
  const float f2 = __uint_as_float(w1 << 16) * fa;
  const float f3 = __uint_as_float(w1 & 0xFFFF0000u) * fa;
  const uint32_t h01 = e4m3x2_f32(f0, f1), h23 = e4m3x2_f32(f2, f3);
  const float2 b01 = e4m3x2_to_f32(h01), b23 = e4m3x2_to_f32(h23);
  hi = h01 | (h23 << 16);
  lo = e4m3x2_f32(f0 - b01.x, f1 - b01.y) | (e4m3x2_f32(f2 - b23.x, f3 - b23.y) << 16);
}

// One thread's share of request b's image: head row h (< 64), part t (0..7,
// the eight threads of a head in consecutive lanes of one warp, all eight
// calling together): latent values [64 t, 64 t + 64) (four 16-value units of
// group t / 2) and rope unit t.  All of the thread's loads are issued before
// any use.
__device__ __forceinline__ void build_q_image_row(const __nv_bfloat16* q, int rows_q, int heads,
                                                  int b, int h, int t, uint8_t* image) {
  const bool live = h < heads;
  const uint4* src =
      reinterpret_cast<const uint4*>(q + ((size_t)b * rows_q + (live ? h : 0)) * kHeadDim);
  const uint4 zero = make_uint4(0, 0, 0, 0);
  uint4 v[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) v[k] = live ? __ldg(src + 8 * t + k) : zero;
  const uint4 rope = live ? __ldg(src + 64 + t) : zero;
  float amax = 0.f;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint32_t w[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
#pragma unroll
    for (int e = 0; e < 4; ++e)
      amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(w[e] << 16)),
                               fabsf(__uint_as_float(w[e] & 0xFFFF0000u))));
  }
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  int a = 0;
  if (amax > 0.f) {
    const int e = (int)((__float_as_uint(amax) >> 23) & 0xFF) - 127;
    a = min(120, max(-120, 7 - e));
  }
  const float fa = __uint_as_float((uint32_t)(127 + a) << 23);
  uint8_t* img = image + (size_t)b * kQImageBytes;
  if (t == 0) reinterpret_cast<float*>(img + kFrame)[h] = __uint_as_float((uint32_t)(127 - a) << 23);
  const int g = t >> 1;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int un = (t & 1) * 4 + j;
    const uint4 x0 = v[2 * j], x1 = v[2 * j + 1];
    uint4 hi, lo;
    split_q4(x0.x, x0.y, fa, hi.x, lo.x);
    split_q4(x0.z, x0.w, fa, hi.y, lo.y);
    split_q4(x1.x, x1.y, fa, hi.z, lo.z);
    split_q4(x1.z, x1.w, fa, hi.w, lo.w);
    *reinterpret_cast<uint4*>(img + kHi + g * kChunk + sw128(h, un)) = hi;
    *reinterpret_cast<uint4*>(img + kLo + g * kChunk + sw128(h, un)) = lo;
  }
  *reinterpret_cast<uint4*>(img + kRope + sw128(h, t)) = rope;
}

}  // namespace qimg
}  // namespace dcpmla
