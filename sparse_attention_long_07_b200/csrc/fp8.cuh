// fp8.cuh -- inputs of the FP8 lightning indexer: Hadamard rotation and e4m3
// quantization with power-of-two scales.
//
// "DeepSeek-V3.2" (transformers model doc), "DeepSeek Sparse Attention
// (DSA)", item 1: the reference indexer runs in FP8 with a Hadamard
// (rotate_activation) transform; "DeepSeek-V3.2-Exp" token-ids page, released
// config: scale_fmt "ue8m0" (power-of-two scales).
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

// One warp per vector: lane l holds elements 4l .. 4l+3.  x: bf16 [n, 128];
// q: e4m3 bytes [n, 128]; scale: fp32 [n] (= 2^e).
__global__ void __launch_bounds__(256) hadamard_quantize_kernel(const __nv_bfloat16* __restrict__ x, int64_t n,
                                                                uint8_t* __restrict__ q, float* __restrict__ scale) {
  const int64_t v = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (v >= n) return;
  const uint2 raw = *reinterpret_cast<const uint2*>(x + v * FP8_DIM + lane * 4);
  float a[4];
  a[0] = __uint_as_float(raw.x << 16);
  a[1] = __uint_as_float(raw.x & 0xFFFF0000u);
  a[2] = __uint_as_float(raw.y << 16);
  a[3] = __uint_as_float(raw.y & 0xFFFF0000u);
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
  float amax = fmaxf(fmaxf(fabsf(a[0]), fabsf(a[1])), fmaxf(fabsf(a[2]), fabsf(a[3])));
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, m));
  // (vectors so small that 2^-e would overflow fp32 keep e = -126)
  const int e = amax > 0.f ? max(pow2_scale_exponent(amax), -126) : 0;
  const float inv = ldexpf(1.f, -e);    // exact: x * 2^-e only moves the exponent
  uint16_t lo, hi;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(a[1] * inv), "f"(a[0] * inv));
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(a[3] * inv), "f"(a[2] * inv));
  reinterpret_cast<uint32_t*>(q + v * FP8_DIM)[lane] = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
  if (lane == 0) scale[v] = ldexpf(1.f, e);
}

}  // namespace dsa
