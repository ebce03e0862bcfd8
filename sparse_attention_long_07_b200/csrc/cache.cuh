// cache.cuh -- appending a step's new tokens to the index-key and latent caches.
//
// "DeepSeek-V3.2" (transformers model doc), "DeepSeek Sparse Attention
// (DSA)": besides the main cache, the indexer stores one index_head_dim key
// per token in a cache of its own, refreshed each step (update_indexer), in a
// growing or a preallocated cache layer; MLA caches one compressed latent per
// token, whose RoPE part carries the token's position ("DeepSeek-V3.2-Exp"
// token-ids page, released config: kv_lora_rank 512, qk_rope_head_dim 64,
// index_head_dim 128).
//
// The new tokens of a step are its query rows: row t is entry pos(t) of its
// sequence, whose cache row the PageMap gives (packed or paged).  One warp
// per new token writes
//   - the latent row (bf16 copy; with a RoPE table, the columns from d_v on
//     rotated at pos(t): pair (2i, 2i+1) times (cos, sin) of entry [pos][i]);
//   - the index-key row: a bf16 copy, or e4m3 with one fp32 scale per key,
//     either amax / 448 on the values as they are, or a power of two after the
//     Sylvester-Hadamard rotation (the FP8 indexer's keys, fp8.cuh).
#pragma once

#include <cuda_bf16.h>

#include "common.cuh"
#include "fp8.cuh"
#include "sm100.cuh"

namespace dsa {

enum KeyQuant : int { kKeyBf16 = 0, kKeyE4m3Amax = 1, kKeyE4m3Hadamard = 2 };

struct AppendParams {
  const __nv_bfloat16* latent_new;   // [T, dqk] or null
  const __nv_bfloat16* kidx_new;     // [T, di] or null
  const int32_t* cu_q;
  const int32_t* cu_k;
  int B;
  int64_t T;
  PageMap pages;
  int cache_rows;                    // rows of the caches (checked builds)
  const float2* rope;                // null, or [max_pos, (dqk - dv) / 2] (cos, sin)
  int dqk, dv, di;
  int k_quant;                       // KeyQuant
  __nv_bfloat16* latent_cache;       // [cache rows, dqk]
  void* k_cache;                     // [cache rows, di] bf16 or e4m3 bytes
  float* k_scale;                    // [cache rows] (e4m3 forms)
};

__global__ void __launch_bounds__(256) cache_append_kernel(const AppendParams p) {
  const int64_t t = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= p.T) return;
  const RowInfo ri = locate_row(p.cu_q, p.cu_k, p.B, t);
  const int r = p.pages.row(ri.b, ri.k_base, ri.pos);
  if (r < 0) {   // no valid page for this entry: nothing is written
    if (lane == 0) record_device_error(kErrMissingPage | (24 << 8));
    return;
  }
  if (!in_bounds(r < p.cache_rows, 87)) return;
  if (p.latent_new != nullptr) {
    const uint4* src = reinterpret_cast<const uint4*>(p.latent_new + t * p.dqk);
    uint4* dst = reinterpret_cast<uint4*>(p.latent_cache + static_cast<int64_t>(r) * p.dqk);
    for (int i = lane; i < p.dqk / 8; i += 32) {
      uint4 v = src[i];
      if (p.rope != nullptr && 8 * i >= p.dv) {
        const float2* cs = p.rope + static_cast<int64_t>(ri.pos) * ((p.dqk - p.dv) / 2) + (8 * i - p.dv) / 2;
        uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float re = __uint_as_float(w[j] << 16), im = __uint_as_float(w[j] & 0xFFFF0000u);
          const float2 c = __ldg(cs + j);
          const __nv_bfloat162 b2 = __floats2bfloat162_rn(fmaf(re, c.x, -im * c.y), fmaf(re, c.y, im * c.x));
          w[j] = *reinterpret_cast<const uint32_t*>(&b2);
        }
        v = make_uint4(w[0], w[1], w[2], w[3]);
      }
      dst[i] = v;
    }
  }
  if (p.kidx_new != nullptr) {
    const __nv_bfloat16* src = p.kidx_new + t * p.di;
    if (p.k_quant == kKeyBf16) {
      uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.k_cache) + static_cast<int64_t>(r) * p.di);
      for (int i = lane; i < p.di / 8; i += 32) dst[i] = reinterpret_cast<const uint4*>(src)[i];
    } else {
      uint8_t* dst = static_cast<uint8_t*>(p.k_cache) + static_cast<int64_t>(r) * FP8_DIM;
      if (p.k_quant == kKeyE4m3Hadamard) hadamard_quantize_warp(src, dst, p.k_scale + r);
      else amax_quantize_warp(src, dst, p.k_scale + r);
    }
  }
}

}  // namespace dsa
