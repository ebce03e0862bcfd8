// common.cuh -- small device helpers shared by the DSA kernels.
#pragma once

#include <stdint.h>

namespace dsa {

// Keys per part of the part maxima that the indexer's epilogue emits beside
// the scores and the top-k reads: the maximum score of keys 8p .. 8p+7 of a
// row (eight consecutive keys are eight consecutive lanes of one epilogue warp).
constexpr int PART = 8;

// Where the caches keep entry s of sequence b.  Packed caches (no block
// table): row k_base + s, k_base = cu_k[b].  Paged caches: a pool of n_pages
// pages of page_size rows shared by the index-key and latent caches; entry s
// sits at row s % page_size of page block_table[b * pages_per_seq +
// s / page_size] ("DeepSeek-V3.2" transformers doc, DSA: the indexer's key
// cache lives beside the main cache, growing or preallocated).  page_size is
// a power of two of at least 64, so a 64-row span starting at a multiple of
// 64 never crosses a page.
struct PageMap {
  const int32_t* block_table;   // [B, pages_per_seq] or null (packed)
  int page_shift;               // log2(page_size)
  int pages_per_seq;
  int n_pages;

  __device__ __forceinline__ bool paged() const { return block_table != nullptr; }
  // Cache row of entry s (s >= 0) of sequence b, or -1 if its page is missing.
  __device__ __forceinline__ int row(int b, int k_base, int s) const {
    if (block_table == nullptr) return k_base + s;
    const int j = s >> page_shift;
    const int page = j < pages_per_seq ? __ldg(block_table + static_cast<int64_t>(b) * pages_per_seq + j) : -1;
    return (static_cast<unsigned>(page) < static_cast<unsigned>(n_pages))
               ? (page << page_shift) + (s & ((1 << page_shift) - 1))
               : -1;
  }
};

// Where global query row t sits: its sequence, absolute position and the
// sequence's key range.  Sequence b owns query rows [cu_q[b], cu_q[b+1]) and
// key rows [cu_k[b], cu_k[b+1]); its q_len new queries are its last tokens.
struct RowInfo {
  int b;
  int pos;       // absolute position of the query = last key index it may see
  int kv_len;
  int k_base;    // first global key row of the sequence
};

__device__ __forceinline__ RowInfo locate_row(const int32_t* __restrict__ cu_q,
                                              const int32_t* __restrict__ cu_k, int B, int64_t t) {
  // largest b with cu_q[b] <= t (then cu_q[b+1] > t, empty sequences skipped)
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (cu_q[mid] <= t) lo = mid; else hi = mid - 1;
  }
  RowInfo r;
  r.b = lo;
  int q0 = cu_q[lo], q1 = cu_q[lo + 1];
  r.k_base = cu_k[lo];
  r.kv_len = cu_k[lo + 1] - r.k_base;
  r.pos = r.kv_len - (q1 - q0) + static_cast<int>(t - q0);
  return r;
}

// locate_row with the whole CTA at once (every thread of the block must call
// it: it synchronises the block): b is the number of sequences b' >= 1 with
// cu_q[b'] <= t (cu_q is non-decreasing, so they form a prefix), counted with
// one load per thread per blockDim.x sequences instead of a chain of
// dependent loads.
__device__ __forceinline__ RowInfo locate_row_block(const int32_t* __restrict__ cu_q,
                                                    const int32_t* __restrict__ cu_k, int B, int64_t t) {
  int b = 0;
  for (int base = 1; base < B; base += static_cast<int>(blockDim.x)) {
    const int i = base + static_cast<int>(threadIdx.x);
    b += __syncthreads_count(i < B && cu_q[i] <= t);
  }
  RowInfo r;
  r.b = b;
  const int q0 = cu_q[b], q1 = cu_q[b + 1];
  r.k_base = cu_k[b];
  r.kv_len = cu_k[b + 1] - r.k_base;
  r.pos = r.kv_len - (q1 - q0) + static_cast<int>(t - q0);
  return r;
}

// Order-preserving map of a non-NaN float to uint32 (larger float -> larger
// key); -0.0 is first folded onto +0.0 so that the two tie.
__device__ __forceinline__ uint32_t order_key(float x) {
  uint32_t u = __float_as_uint(x);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

}  // namespace dsa
