// topk.cuh -- per-query top-k token selection (radix select).
//
// "DeepSeek-V3.2" (transformers model doc), "DeepSeek Sparse Attention (DSA)",
// item 2: every query keeps the index_topk highest-scoring earlier tokens.
//
// One CTA per query row.  Scores are mapped to order-preserving 32-bit keys
// and the k-th largest key is found digit by digit (4 passes of 8 bits, a
// 256-bin shared-memory histogram per pass, restricted to keys that match the
// digits found so far).  A last pass over the row, in index order, emits every
// key above that threshold and the lowest-index keys equal to it; ranks come
// from warp ballots and a block scan, so the output is deterministic:
// [keys > thr in index order][first keys == thr in index order][-1 ...].
// Rows are read from global memory (L2-resident right after the indexer
// wrote them) with 16-byte loads.
#pragma once

#include "common.cuh"

namespace dsa {

template <int NT>
__global__ void __launch_bounds__(NT) topk_radix_kernel(const float* __restrict__ scores,
                                                        int64_t ld, const int32_t* __restrict__ cu_q,
                                                        const int32_t* __restrict__ cu_k, int B,
                                                        int64_t q_begin, int topk,
                                                        int32_t* __restrict__ idx) {
  constexpr int NW = NT / 32;
  __shared__ uint32_t hist[256];
  __shared__ uint32_t s_digit, s_above;
  __shared__ uint32_t warp_cnt[NW];

  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int64_t r = blockIdx.x;
  const RowInfo ri = locate_row(cu_q, cu_k, B, q_begin + r);
  const int n = ri.pos + 1;
  const float* __restrict__ row = scores + r * ld;
  int32_t* __restrict__ out = idx + r * topk;

  if (n <= topk) {  // every candidate is selected
    for (int i = tid; i < topk; i += NT) out[i] = i < n ? i : -1;
    return;
  }

  const int n4 = n >> 2;  // rows start 16-byte aligned (ld % 4 == 0)
  const float4* __restrict__ row4 = reinterpret_cast<const float4*>(row);

  uint32_t prefix = 0;
  int remaining = topk;
#pragma unroll 1
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    const uint32_t hi_mask = pass == 0 ? 0u : (0xFFFFFFFFu << (shift + 8));
    for (int i = tid; i < 256; i += NT) hist[i] = 0u;
    __syncthreads();
    auto count = [&](uint32_t key, bool valid) {
      const bool m = valid && ((key & hi_mask) == prefix);
      const uint32_t bin = (key >> shift) & 255u;
      const uint32_t active = __ballot_sync(0xFFFFFFFFu, m);
      if (m) {
        const uint32_t peers = __match_any_sync(active, bin);
        if (lane == __ffs(peers) - 1) atomicAdd(&hist[bin], static_cast<uint32_t>(__popc(peers)));
      }
    };
    for (int base = 0; base < n4; base += NT) {
      const int i4 = base + tid;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      const bool ok = i4 < n4;
      if (ok) v = row4[i4];
      count(order_key(v.x), ok);
      count(order_key(v.y), ok);
      count(order_key(v.z), ok);
      count(order_key(v.w), ok);
    }
    {  // ragged tail (fewer than 4 elements)
      const int i = 4 * n4 + tid;
      const bool ok = tid < 32 && i < n;
      if (warp == 0) count(ok ? order_key(row[i]) : 0u, ok);
    }
    __syncthreads();
    if (warp == 0) {
      // lane l owns bins 255-8l .. 248-8l (descending); scan counts from the top
      uint32_t c[8], sum = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        c[j] = hist[255 - 8 * lane - j];
        sum += c[j];
      }
      uint32_t incl = sum;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, off);
        if (lane >= off) incl += v;
      }
      const uint32_t excl = incl - sum;
      const uint32_t need = static_cast<uint32_t>(remaining);
      if (excl < need && need <= incl) {
        uint32_t acc = excl;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (acc + c[j] >= need) {
            s_digit = 255u - 8u * lane - j;
            s_above = acc;
            break;
          }
          acc += c[j];
        }
      }
    }
    __syncthreads();
    prefix |= s_digit << shift;
    remaining -= static_cast<int>(s_above);
  }

  // keys > prefix: exactly topk - remaining of them; keys == prefix: take the
  // first `remaining` in index order.
  const uint32_t thr = prefix;
  const int need_eq = remaining;
  const int n_gt = topk - remaining;
  const uint32_t lt_mask = (1u << lane) - 1u;
  int gt_base = 0, eq_base = 0;
#pragma unroll 1
  for (int base = 0; base < n; base += NT) {
    const int i = base + tid;
    const uint32_t key = i < n ? order_key(row[i]) : 0u;
    const bool gt = i < n && key > thr;
    const bool eq = i < n && key == thr;
    const uint32_t bg = __ballot_sync(0xFFFFFFFFu, gt);
    const uint32_t be = __ballot_sync(0xFFFFFFFFu, eq);
    if (lane == 0) warp_cnt[warp] = (static_cast<uint32_t>(__popc(bg)) << 16) | __popc(be);
    __syncthreads();
    uint32_t off = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const uint32_t v = warp_cnt[w];
      off += w < warp ? v : 0u;
      tot += v;
    }
    if (gt) out[gt_base + static_cast<int>(off >> 16) + __popc(bg & lt_mask)] = i;
    if (eq) {
      const int rk = eq_base + static_cast<int>(off & 0xFFFFu) + __popc(be & lt_mask);
      if (rk < need_eq) out[n_gt + rk] = i;
    }
    gt_base += static_cast<int>(tot >> 16);
    eq_base += static_cast<int>(tot & 0xFFFFu);
    __syncthreads();
    if (gt_base >= n_gt && eq_base >= need_eq) break;
  }
}

}  // namespace dsa
