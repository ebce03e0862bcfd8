// up_proj.cuh -- per-head up-projection of the absorbed attention output out
// of latent space.
//
// "DeepSeek-V3.2-Exp" (token-ids page), released config: kv_lora_rank 512,
// v_head_dim 128, n_heads 128; "DeepSeek-V3.2" (transformers model doc),
// "DeepSeek Sparse Attention (DSA)": MLA attention whose cached entries (the
// compressed latents) are shared by all heads.  The absorbed attention leaves
// each head's output in the 512-wide latent space; its value up-projection
// W_UV[h] (512 x 128 per head) maps it to the head's 128 value dimensions:
//     y[t, h, :] = o[t, h, :] @ W_UV[h].
//
// sm_100a mapping: one CTA per (head, tile of 128 query rows): a tcgen05 GEMM
// with M = 128 query rows, N = 128, K = 512, fed by TMA through a four-stage
// ring of 64-wide K chunks (o rows K-major, W_UV rows N-major, both 128-byte
// swizzled), fp32 accumulation in tensor memory, bf16 out.  W_UV[h] is read
// once per query tile, so a decode batch reads every weight once.
#pragma once

#include <cuda_bf16.h>

#include "sm100.cuh"

namespace dsa {

struct UpProjCfg {
  static constexpr int H = 128, DC = 512, DV = 128;
  static constexpr int BM = 128;                 // query rows per CTA (MMA M)
  static constexpr int BKC = 64;                 // K chunk (one 128-byte atom of o)
  static constexpr int NCHUNK = DC / BKC;        // 8
  static constexpr int NSTG = 4;
  static constexpr int A_BYTES = BM * BKC * 2;   // 16 KB: 128 rows x 128 B
  static constexpr int B_ATOM = BKC * 128;       // 8 KB: 64 K rows x 64 N columns
  static constexpr int B_BYTES = 2 * B_ATOM;     // N = 128: two 64-column atoms
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int OFF_BAR = NSTG * STAGE;
  static constexpr int SMEM_BYTES = OFF_BAR + (2 * NSTG + 2) * 8 + 16 + 1024;
  static constexpr int NT = 6 * 32;              // producer, MMA, four epilogue warps
  static constexpr uint32_t IDESC = idesc_bf16_f32(BM, DV, false, true);
  static_assert(STAGE % 1024 == 0 && A_BYTES % 1024 == 0 && B_ATOM % 1024 == 0, "swizzle atoms");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

// tm_o: o as (c, h, t) with box (64, 1, 128); tm_w: W_UV as (e, c, h) with box (64, 64, 1).
__global__ void __launch_bounds__(UpProjCfg::NT, 1)
    up_proj_kernel(const __grid_constant__ CUtensorMap tm_o, const __grid_constant__ CUtensorMap tm_w,
                   __nv_bfloat16* __restrict__ y, int64_t T) {
  using C = UpProjCfg;
  const int h = blockIdx.x;
  const int64_t t0 = static_cast<int64_t>(blockIdx.y) * C::BM;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + C::OFF_BAR;
  auto bar_full = [&](int s) { return bar0 + 8 * s; };
  auto bar_empty = [&](int s) { return bar0 + 8 * (C::NSTG + s); };
  const uint32_t bar_acc = bar0 + 8 * (2 * C::NSTG);
  const uint32_t bar_drain = bar0 + 8 * (2 * C::NSTG + 1);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::OFF_BAR + (2 * C::NSTG + 2) * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (device_error_pending()) return;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NSTG; ++s) {
      mbar_init(bar_full(s), 1);
      mbar_init(bar_empty(s), 1);
    }
    mbar_init(bar_acc, 1);
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), 128);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_o);
    tma_prefetch_desc(&tm_w);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int k = 0;
      for (; k < C::NCHUNK; ++k) {
        const int s = k % C::NSTG;
        if (!mbar_wait(bar_empty(s), ((k / C::NSTG) & 1) ^ 1, abort_flag, 70)) break;
        const uint32_t st = sbase + s * C::STAGE;
        mbar_arrive_expect_tx(bar_full(s), C::STAGE);
        tma_load_3d(st, &tm_o, bar_full(s), k * C::BKC, h, static_cast<int32_t>(t0));
        tma_load_3d(st + C::A_BYTES, &tm_w, bar_full(s), 0, k * C::BKC, h);
        tma_load_3d(st + C::A_BYTES + C::B_ATOM, &tm_w, bar_full(s), 64, k * C::BKC, h);
      }
      if (*abort_flag) {   // let copies in flight land
        long long tw = clock64();
        for (int j = (k > C::NSTG ? k - C::NSTG : 0); j < k; ++j)
          while (!mbar_try_wait(bar_full(j % C::NSTG), (j / C::NSTG) & 1) && clock64() - tw < kWaitLimitCycles) {
          }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      for (int k = 0; k < C::NCHUNK; ++k) {
        const int s = k % C::NSTG;
        if (!mbar_wait(bar_full(s), (k / C::NSTG) & 1, abort_flag, 71)) break;
        tc_fence_after();
        const uint32_t st = sbase + s * C::STAGE;
#pragma unroll
        for (int kk = 0; kk < C::BKC / 16; ++kk) {
          // A: 128 rows x 128 B, K-major; B: two 64-column atoms of 64 K rows, N-major
          const uint64_t ad = smem_desc(st + kk * 32, 16, 1024, 2);
          const uint64_t bd = smem_desc(st + C::A_BYTES + kk * 16 * 128, C::B_ATOM, 1024, 2);
          umma_ss(tmem, ad, bd, C::IDESC, (k > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(bar_empty(s));
        if (k == C::NCHUNK - 1) umma_commit(bar_acc);
      }
      umma_commit(bar_drain);
      long long tw = clock64();
      while (!mbar_try_wait(bar_drain, 0) && clock64() - tw < kWaitLimitCycles) {
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue: TMEM -> bf16 y
    const int q = warp & 3;                 // TMEM lane quarter of this warp
    const int64_t t = t0 + q * 32 + lane;   // query row of this thread
    if (mbar_wait_warp(bar_acc, 0, abort_flag, 72)) {
      tc_fence_after();
      __nv_bfloat16* yrow = y + (t * C::H + h) * C::DV;
#pragma unroll 1
      for (int c0 = 0; c0 < C::DV; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(tmem + (static_cast<uint32_t>(q * 32) << 16) + c0, v);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(v[2 * j]), __uint_as_float(v[2 * j + 1]));
          pk[j] = *reinterpret_cast<const uint32_t*>(&b2);
        }
        if (t < T) {
          uint4* dst = reinterpret_cast<uint4*>(yrow + c0);
#pragma unroll
          for (int j = 0; j < 4; ++j) dst[j] = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

}  // namespace dsa
