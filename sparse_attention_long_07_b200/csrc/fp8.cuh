// fp8.cuh -- inputs of the FP8 lightning indexer: Hadamard rotation and e4m3
// quantization with power-of-two scales.
//
// "DeepSeek-V3.2" (transformers model doc), "DeepSeek Sparse Attention (DSA)",
// item 1: DeepSeek's own indexer scores in e4m3 after a Hadamard rotation of
// queries and keys (rotate_activation); "DeepSeek-V3.2-Exp" token-ids page,
// released config: scale_fmt "ue8m0" (power-of-two scales).
//
// Every vector of 128 values (one index-head query, or one index key) is
// rotated by the Sylvester-Hadamard matrix H (entries +-1, H[i][j] =
// (-1)^popcount(i & j)) and quantized to e4m3 with one scale s = 2^e per
// vector, e the smallest integer with max|Hx| <= 448 s; the bytes are
// e4m3(Hx / s), rounded to nearest even.  Both operands of a score are
// rotated by the same H, so (Hq).(Hk) = 128 (q.k): the indexer divides the
// factor 128 back out of the score (exact, a power of two).  The rotation is
// not normalised by 1/sqrt(128), which would need an inexact product.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace dsa {

constexpr int FP8_DIM = 128;              // vector length of the rotation
constexpr int FP8_HADAMARD_LOG2 = 7;      // (Hq).(Hk) = 2^7 (q.k)

// Butterfly of the fast Walsh-Hadamard transform: (a, b) -> (a + b, a - b).
__device__ __forceinline__ void wht_pair(float& a, float& b) {
  const float s = a + b, d = a - b;
  a = s;
  b = d;
}

// Power-of-two exponent e with amax <= 448 * 2^e < 2 * amax (amax > 0, finite):
// amax = m 2^E with m in [1, 2); 448 = 1.75 * 2^8, so e = E - 8 when m <= 1.75
// and E - 7 when m > 1.75.  Exact, from the bits of amax.
__device__ __forceinline__ int pow2_scale_exponent(float amax) {
  const uint32_t u = __float_as_uint(amax);
  int E = static_cast<int>((u >> 23) & 0xFF) - 127;
  uint32_t frac = u & 0x7FFFFFu;
  if (E == -127) {   // subnormal amax: normalise
    const int lz = __clz(frac) - 8;   // leading zeros inside the 23-bit field
    E = -126 - (lz + 1);
    frac = (frac << (lz + 1)) & 0x7FFFFFu;
  }
  return E - 8 + (frac > 0x600000u ? 1 : 0);   // 0x600000 / 2^23 = 0.75
}

// The four values of lane l (elements 4l .. 4l+3 of a 128-value vector) as
// fp32, from their bf16 bits.
__device__ __forceinline__ void load_bf16x4(const __nv_bfloat16* x, int lane, float a[4]) {
  const uint2 raw = *reinterpret_cast<const uint2*>(x + lane * 4);
  a[0] = __uint_as_float(raw.x << 16);
  a[1] = __uint_as_float(raw.x & 0xFFFF0000u);
  a[2] = __uint_as_float(raw.y << 16);
  a[3] = __uint_as_float(raw.y & 0xFFFF0000u);
}

// e4m3 bytes (round to nearest even, saturating) of the four values, packed
// in element order.
__device__ __forceinline__ uint32_t e4m3x4(float a0, float a1, float a2, float a3) {
  uint16_t lo, hi;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(a1), "f"(a0));
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(a3), "f"(a2));
  return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
}

__device__ __forceinline__ float warp_amax(float v) {
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, m));
  return v;
}

// One warp rotates and quantizes one vector (see the file comment): x bf16
// [128] -> q e4m3 [128], *scale = 2^e.  All 32 lanes take part.
__device__ __forceinline__ void hadamard_quantize_warp(const __nv_bfloat16* __restrict__ x, uint8_t* __restrict__ q,
                                                       float* __restrict__ scale) {
  const int lane = threadIdx.x & 31;
  float a[4];
  load_bf16x4(x, lane, a);
  // index bits 0 and 1 live inside the lane, bits 2..6 across lanes
  wht_pair(a[0], a[1]);
  wht_pair(a[2], a[3]);
  wht_pair(a[0], a[2]);
  wht_pair(a[1], a[3]);
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
    const bool upper = (lane & m) != 0;   // this lane holds the element with the index bit set
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float o = __shfl_xor_sync(0xFFFFFFFFu, a[e], m);
      a[e] = upper ? o - a[e] : a[e] + o;
    }
  }
  const float amax = warp_amax(fmaxf(fmaxf(fabsf(a[0]), fabsf(a[1])), fmaxf(fabsf(a[2]), fabsf(a[3]))));
  // (vectors so small that 2^-e would overflow fp32 keep e = -126)
  const int e = amax > 0.f ? max(pow2_scale_exponent(amax), -126) : 0;
  const float inv = ldexpf(1.f, -e);    // exact: x * 2^-e only moves the exponent
  reinterpret_cast<uint32_t*>(q)[lane] = e4m3x4(a[0] * inv, a[1] * inv, a[2] * inv, a[3] * inv);
  if (lane == 0) *scale = ldexpf(1.f, e);
}

// e4m3 with one fp32 scale per vector, scale = amax / 448 (1 for a zero
// vector), bytes = e4m3 (nearest even) of the fp32 quotient x / scale; no
// rotation.  One warp per vector of 128 values, as above.
__device__ __forceinline__ void amax_quantize_warp(const __nv_bfloat16* __restrict__ x, uint8_t* __restrict__ q,
                                                   float* __restrict__ scale) {
  const int lane = threadIdx.x & 31;
  float a[4];
  load_bf16x4(x, lane, a);
  const float amax = warp_amax(fmaxf(fmaxf(fabsf(a[0]), fabsf(a[1])), fmaxf(fabsf(a[2]), fabsf(a[3]))));
  const float s = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
  reinterpret_cast<uint32_t*>(q)[lane] =
      e4m3x4(__fdiv_rn(a[0], s), __fdiv_rn(a[1], s), __fdiv_rn(a[2], s), __fdiv_rn(a[3], s));
  if (lane == 0) *scale = s;
}

// One warp per vector.  x: bf16 [n, 128]; q: e4m3 bytes [n, 128]; scale: fp32 [n] (= 2^e).
__global__ void __launch_bounds__(256) hadamard_quantize_kernel(const __nv_bfloat16* __restrict__ x, int64_t n,
                                                                uint8_t* __restrict__ q, float* __restrict__ scale) {
  const int64_t v = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (v >= n) return;
  hadamard_quantize_warp(x + v * FP8_DIM, q + v * FP8_DIM, scale + v);
}

}  // namespace dsa
