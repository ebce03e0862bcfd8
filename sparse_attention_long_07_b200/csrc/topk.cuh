// topk.cuh -- per-query top-k token selection.
//
// "DeepSeek-V3.2" (transformers model doc), "DeepSeek Sparse Attention (DSA)",
// item 2: every query keeps the index_topk highest-scoring earlier tokens.
// Order: higher score first, ties to the lower index; -0.0 ties +0.0.
//
// One CTA per query row (launched as a programmatic dependent of the indexer:
// it waits for it before reading anything).  Three paths, the first that
// applies:
//   part maxima  (the indexer wrote the maximum of every 8 scores; rows of at
//                least 1.25 k parts) -- a lower bound of the k-th score from
//                the group maxima, one pass over the groups that can hold a
//                selection, the exact selection among those candidates;
//   fast         the same with part maxima taken from the streamed row;
//   exact        the passes below over the whole row.
// The row (fp32 scores, usually still in L2 after the indexer wrote it)
// streams through a 3-stage shared-memory ring of 32 KB bulk async copies
// issued by one thread, so each SM keeps ~96 KB in flight.  Scores become
// order-preserving 32-bit keys.
//   pass 1  histogram of the top 11 key bits (2048 bins; every warp counts into
//           its own copy, so the hot bins of a score distribution never see
//           atomics from two warps)  ->  the bin B that holds the k-th largest
//           key, and the count above it;
//   pass 2  every key in a bin above B is emitted; the keys of bin B are
//           compacted into shared memory (in index order);
//   refine  radix select on the remaining 21 bits among those candidates, then
//           emit the candidates above the threshold and the lowest-index ones
//           equal to it.
// If bin B holds more candidates than fit in shared memory (massive ties), the
// refinement runs over the row in global memory instead, with the same result.
// Ranks come from ballots and warp/CTA prefix sums in index order, so the
// output order is deterministic.
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace dsa {

struct TopkCfg {
  static constexpr int NT = 512, NW = NT / 32;
  static constexpr int CHUNK = 8192;                  // scores per streamed stage (32 KB)
  static constexpr int PER_WARP = CHUNK / NW;         // 512: 4 float4 per lane
  static constexpr int STAGES = 3;
  static constexpr int BITS1 = 11, BINS1 = 1 << BITS1, SHIFT1 = 32 - BITS1;
  static constexpr int CAP = 6144;                    // bin-B candidates kept in shared memory
  static constexpr int MAX_N = (65535 / PER_WARP) * CHUNK;   // 16-bit per-warp pass-1 counters
  static constexpr int PMAX_CAP = 8192;               // fast path: part maxima kept
  static constexpr int BITMAP_BITS = 262144;          // fast path: longest row (one bit per key)
  static constexpr int PM_CAP = STAGES * CHUNK;       // part-maxima path: groups kept (in the ring)
  static constexpr int PLIST_CAP = 16384;             // part-maxima path: groups that can hold a selection
  static constexpr int OFF_RING = 0;
  // union: per-warp pass-1 histograms (exact path) | part maxima + selection bitmap (fast path)
  static constexpr int OFF_WHIST = OFF_RING + STAGES * CHUNK * 4;   // per-warp pass-1 histograms
  static constexpr int OFF_PMAX = OFF_WHIST;
  static constexpr int OFF_BITMAP = OFF_WHIST + PMAX_CAP * 4;
  static constexpr int OFF_HIST = OFF_WHIST + NW * (BINS1 / 2) * 4; // two 16-bit counters per word
  static constexpr int OFF_CKEY = OFF_HIST + BINS1 * 4;
  static constexpr int OFF_CIDX = OFF_CKEY + CAP * 4;
  static constexpr int OFF_WTOT = OFF_CIDX + CAP * 4;
  static constexpr int OFF_CNT = OFF_WTOT + 2 * NW * 4;   // select: per-warp digit counts + totals
  static constexpr int OFF_BAR = OFF_CNT + 128 * 4;   // block reductions: slots and results
  static constexpr int OFF_MISC = OFF_BAR + STAGES * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 64 + 128;   // + alignment slack
  static_assert(PMAX_CAP * 4 + BITMAP_BITS / 8 <= NW * (BINS1 / 2) * 4, "fast-path union fits");
  static_assert(PLIST_CAP * 4 <= NW * (BINS1 / 2) * 4, "group list fits the histogram union");
  static_assert(OFF_RING % 128 == 0 && (CHUNK * 4) % 128 == 0, "bulk-copy destinations");
  static_assert(OFF_BAR % 8 == 0 && OFF_MISC % 8 == 0, "barrier alignment");
};

__device__ __forceinline__ uint32_t warp_excl_scan(uint32_t v, uint32_t lane, uint32_t* total) {
  uint32_t incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t u = __shfl_up_sync(0xFFFFFFFFu, incl, off);
    if (lane >= static_cast<uint32_t>(off)) incl += u;
  }
  *total = __shfl_sync(0xFFFFFFFFu, incl, 31);
  return incl - v;
}

__global__ void __launch_bounds__(TopkCfg::NT, 1)
    topk_kernel(const float* __restrict__ scores, int64_t ld, const float* __restrict__ part_max, int64_t ld_pm,
                const int32_t* __restrict__ cu_q, const int32_t* __restrict__ cu_k, int B, int64_t q_begin,
                int topk, int32_t* __restrict__ idx) {
  using C = TopkCfg;
  const uint32_t tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t r = blockIdx.x;
  // every CTA of this grid is resident once it gets here: the next kernel (the
  // attention, when launched as a dependent) may start on the free SMs; the
  // scores come from the previous kernel (the indexer), so wait for it
  grid_launch_dependents();
  grid_dependency_wait();
  const RowInfo ri = locate_row_block(cu_q, cu_k, B, q_begin + r);
  const int n = ri.pos + 1;
  const float* __restrict__ row = scores + r * ld;
  int32_t* __restrict__ out = idx + r * topk;

  if (n <= topk) {  // every candidate is selected
    for (int i = tid; i < topk; i += C::NT) out[i] = i < n ? i : -1;
    return;
  }
  if (device_error_pending()) return;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  float* ring = reinterpret_cast<float*>(smem + C::OFF_RING);
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem + C::OFF_HIST);
  uint32_t* ckey = reinterpret_cast<uint32_t*>(smem + C::OFF_CKEY);
  int32_t* cidx = reinterpret_cast<int32_t*>(smem + C::OFF_CIDX);
  uint32_t* wtot = reinterpret_cast<uint32_t*>(smem + C::OFF_WTOT);
  uint32_t* cnt = reinterpret_cast<uint32_t*>(smem + C::OFF_CNT);
  const uint32_t bar0 = smem_u32(smem + C::OFF_BAR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC);
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC + 16);

  if (tid == 0) {
    for (int s = 0; s < C::STAGES; ++s) mbar_init(bar0 + 8 * s, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  DSA_PROF_BEGIN();
  long long t_phase = clock64();
  // profiling builds: cycles of each phase (thread 0), sites 41..47
  auto phase = [&](int site) {
    if (tid == 0) DSA_PROF_SPAN(site, t_phase);
    t_phase = clock64();
  };
  uint32_t* whist = reinterpret_cast<uint32_t*>(smem + C::OFF_WHIST) + warp * (C::BINS1 / 2);
  __syncthreads();

  // ------------------------------------------------------------------ streaming
  const int nchunks = (n + C::CHUNK - 1) / C::CHUNK;
  int g = 0;           // chunks streamed before the current pass (barrier phases)
  int issued = 0;      // global chunk counter of copies issued (thread 0)
  auto issue = [&](int c, int gg) {
    const int s = gg % C::STAGES;
    const int cnt = min(C::CHUNK, n - c * C::CHUNK);
    const uint32_t bytes = static_cast<uint32_t>((cnt + 3) & ~3) * 4u;  // rows hold ld >= n rounded up to 4
    mbar_arrive_expect_tx(bar0 + 8 * s, bytes);
    bulk_load(smem_u32(ring + s * C::CHUNK), row + static_cast<int64_t>(c) * C::CHUNK, bytes, bar0 + 8 * s);
    issued = gg + 1;
  };
  auto stream = [&](auto&& body) -> bool {
    if (tid == 0)
      for (int j = 0; j < min(C::STAGES, nchunks); ++j) issue(j, g + j);
    bool ok = true;
    int c = 0;
    for (; c < nchunks; ++c) {
      const int gg = g + c, s = gg % C::STAGES;
      const bool got = mbar_wait(bar0 + 8 * s, (gg / C::STAGES) & 1, abort_flag, 40);
      if (__syncthreads_or(!got)) { ok = false; break; }
      // every thread is done with chunk c-1: refill its stage
      if (tid == 0 && c >= 1 && c - 1 + C::STAGES < nchunks) issue(c - 1 + C::STAGES, gg - 1 + C::STAGES);
      body(c, ring + s * C::CHUNK);
    }
    if (!ok && tid == 0) {  // let copies in flight land before the CTA leaves
      long long t0 = clock64();
      for (int gg = g + c; gg < issued; ++gg)
        while (!mbar_try_wait(bar0 + 8 * (gg % C::STAGES), (gg / C::STAGES) & 1) &&
               clock64() - t0 < kWaitLimitCycles) {
        }
    }
    __syncthreads();
    g += nchunks;
    return ok;
  };

  // warp-aggregated histogram increment
  auto hist_add = [&](uint32_t* h, uint32_t bin, bool valid) {
    const uint32_t active = __ballot_sync(0xFFFFFFFFu, valid);
    if (valid) {
      const uint32_t peers = __match_any_sync(active, bin);
      if (lane == static_cast<uint32_t>(__ffs(peers) - 1)) atomicAdd(&h[bin], static_cast<uint32_t>(__popc(peers)));
    }
  };

  // pass-1 increment into this warp's private histogram (two 16-bit counters per word)
  auto whist_add = [&](uint32_t bin, bool valid) {
    const uint32_t active = __ballot_sync(0xFFFFFFFFu, valid);
    if (valid) {
      const uint32_t peers = __match_any_sync(active, bin);
      if (lane == static_cast<uint32_t>(__ffs(peers) - 1))
        atomicAdd(&whist[bin >> 1], static_cast<uint32_t>(__popc(peers)) << (16 * (bin & 1)));
    }
  };

  // Classify the chunk's elements (gt / eq flags) and emit them with ranks in
  // index order: element order inside a chunk is (warp, rr, lane, e).
  // emit_gt(rank, index, key), emit_eq(rank, index, key); bases advance by the chunk totals.
  uint32_t gt_base = 0, eq_base = 0;
  auto scan_chunk = [&](int c, const float* buf, auto&& classify, auto&& emit_gt, auto&& emit_eq) {
    uint32_t keys[16], flags = 0, rank_base[4];
    uint32_t wacc = 0;
#pragma unroll
    for (int rr = 0; rr < 4; ++rr) {
      const int off = static_cast<int>(warp) * C::PER_WARP + (static_cast<int>(lane) + 32 * rr) * 4;
      const float4 v = *reinterpret_cast<const float4*>(buf + off);
      const float vals[4] = {v.x, v.y, v.z, v.w};
      uint32_t cg = 0, ce = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int gi = c * C::CHUNK + off + e;
        const uint32_t key = order_key(vals[e]);
        keys[rr * 4 + e] = key;
        bool gt = false, eq = false;
        if (gi < n) classify(key, gt, eq);
        flags |= (gt ? 1u : 0u) << (2 * (rr * 4 + e));
        flags |= (eq ? 2u : 0u) << (2 * (rr * 4 + e));
        cg += gt;
        ce += eq;
      }
      uint32_t tot;
      const uint32_t pre = warp_excl_scan(cg | (ce << 16), lane, &tot);
      rank_base[rr] = wacc + pre;
      wacc += tot;
    }
    if (lane == 31) wtot[(c & 1) * C::NW + warp] = wacc;
    __syncthreads();
    uint32_t wpre = 0, ctot = 0;
#pragma unroll
    for (int w = 0; w < C::NW; ++w) {
      const uint32_t v = wtot[(c & 1) * C::NW + w];
      wpre += static_cast<uint32_t>(w) < warp ? v : 0u;
      ctot += v;
    }
#pragma unroll
    for (int rr = 0; rr < 4; ++rr) {
      uint32_t rg = gt_base + (wpre & 0xFFFFu) + (rank_base[rr] & 0xFFFFu);
      uint32_t re = eq_base + (wpre >> 16) + (rank_base[rr] >> 16);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t f = (flags >> (2 * (rr * 4 + e))) & 3u;
        const int gi = c * C::CHUNK + static_cast<int>(warp) * C::PER_WARP + (static_cast<int>(lane) + 32 * rr) * 4 + e;
        if (f & 1u) emit_gt(rg++, gi, keys[rr * 4 + e]);
        if (f & 2u) emit_eq(re++, gi, keys[rr * 4 + e]);
      }
    }
    gt_base += ctot & 0xFFFFu;
    eq_base += ctot >> 16;
  };

  // Digit of the `need`-th largest entry of a histogram h[nbins] (nbins <= 4 NT):
  // thread t owns the bins nbins-1-4t .. nbins-4-4t (descending), a CTA-wide
  // exclusive scan gives the count above each thread's bins, and the thread
  // whose range crosses `need` writes the digit and the count above it.
  // Called by every thread of the CTA (it contains __syncthreads).
  auto find_digit_fn = [&](const uint32_t* h, int nbins, uint32_t need, uint32_t* digit, uint32_t* above) {
    const int top = nbins - 1 - 4 * static_cast<int>(tid);
    uint32_t c4[4], sum = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      c4[j] = top - j >= 0 ? h[top - j] : 0u;
      sum += c4[j];
    }
    uint32_t wt;
    const uint32_t pre = warp_excl_scan(sum, lane, &wt);
    if (lane == 31) wtot[warp] = pre + sum;
    __syncthreads();
    uint32_t excl = pre;
    for (int w = 0; w < static_cast<int>(warp); ++w) excl += wtot[w];
    if (top >= 0 && excl < need && need <= excl + sum) {
      uint32_t acc = excl;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (acc + c4[j] >= need) {
          *digit = static_cast<uint32_t>(top - j);
          *above = acc;
          break;
        }
        acc += c4[j];
      }
    }
    __syncthreads();
  };

  // Block-wide scan.  Each warp scans with shuffles, warp 0 combines the 16
  // warp totals, and every thread reads back one word, so a call costs two
  // barriers and a couple of shared loads per thread.
  uint32_t red_phase = 0;   // alternates the result words between calls
  // block_scan(v, &total): exclusive prefix of v over the threads in order.
  auto block_scan = [&](uint32_t v, uint32_t* total) -> uint32_t {
    uint32_t wt;
    const uint32_t pre = warp_excl_scan(v, lane, &wt);
    uint32_t* sl = cnt + 40;
    uint32_t* wpre = cnt + 40 + 32 + (red_phase & 1u) * (C::NW + 1);
    ++red_phase;
    if (lane == 31) sl[warp] = pre + v;
    __syncthreads();
    if (warp == 0) {
      const uint32_t x = lane < static_cast<uint32_t>(C::NW) ? sl[lane] : 0u;
      uint32_t tot;
      const uint32_t ex = warp_excl_scan(x, lane, &tot);
      if (lane < static_cast<uint32_t>(C::NW)) wpre[lane] = ex;
      if (lane == 0) wpre[C::NW] = tot;
    }
    __syncthreads();
    *total = wpre[C::NW];
    return wpre[warp] + pre;
  };
  // Range-histogram selection.  select(hb, count, key_of, use, kth, &thr,
  // &rem, exact): the kth largest key among the entries i < count with use(i)
  // (at least kth of them).  The keys' range [lo, hi] (a CTA min/max) is cut
  // into 4096 bins of 2^s keys, s chosen so that the range fits; one pass of
  // shared atomics fills the histogram hb[4096] and a CTA scan finds the bin
  // holding the kth entry; the window shrinks to that bin.  exact: repeat until
  // a bin is one key value (two passes for a range of up to 2^24 keys): thr is
  // then the kth largest key and *rem = kth - (entries > thr).  Otherwise one
  // pass: thr is the start of the bin, a lower bound of the kth largest key
  // with at least kth entries >= thr.  Bins follow the data, so a narrow
  // distribution does not pile into a few bins.  Called by every thread.
  auto select = [&](uint32_t* hb, uint32_t count, auto&& key_of, auto&& use, uint32_t kth, uint32_t* out_thr,
                    uint32_t* out_rem, bool exact) {
    uint32_t mn = 0xFFFFFFFFu, mx = 0u;
    for (uint32_t i = tid; i < count; i += C::NT)
      if (use(i)) {
        const uint32_t k = key_of(i);
        mn = min(mn, k);
        mx = max(mx, k);
      }
    mn = __reduce_min_sync(0xFFFFFFFFu, mn);
    mx = __reduce_max_sync(0xFFFFFFFFu, mx);
    if (lane == 0) {
      wtot[warp] = mn;
      wtot[C::NW + warp] = mx;
    }
    __syncthreads();
    uint32_t lo = 0xFFFFFFFFu, hi = 0u;
#pragma unroll
    for (int w = 0; w < C::NW; ++w) {
      lo = min(lo, wtot[w]);
      hi = max(hi, wtot[C::NW + w]);
    }
    __syncthreads();   // wtot is reused below
    uint32_t need = kth;
    constexpr int HB_BITS = 12, HB_BINS = 1 << HB_BITS, PER_T = HB_BINS / C::NT;
    static_assert(HB_BINS % C::NT == 0, "bins per thread");
    for (;;) {
      const uint32_t span = hi - lo;
      const int bits = span == 0u ? 0 : 32 - __clz(span);
      const int sh = bits > HB_BITS ? bits - HB_BITS : 0;
      for (int i = tid; i < HB_BINS; i += C::NT) hb[i] = 0u;
      __syncthreads();
      for (uint32_t i = tid; i < count; i += C::NT)
        if (use(i)) {
          const uint32_t k = key_of(i);
          if (k >= lo && k <= hi) atomicAdd(&hb[(k - lo) >> sh], 1u);
        }
      __syncthreads();
      // thread t owns bins HB_BINS-1-PER_T t .. down (descending); a CTA scan
      // gives the entries above them
      const int top = HB_BINS - 1 - PER_T * static_cast<int>(tid);
      uint32_t c8[PER_T], sum = 0;
#pragma unroll
      for (int j = 0; j < PER_T; ++j) {
        c8[j] = hb[top - j];
        sum += c8[j];
      }
      uint32_t unused_total;
      const uint32_t excl = block_scan(sum, &unused_total);
      if (excl < need && need <= excl + sum) {
        uint32_t acc = excl;
#pragma unroll
        for (int j = 0; j < PER_T; ++j) {
          if (acc + c8[j] >= need) {
            misc[4] = static_cast<uint32_t>(top - j);
            misc[5] = acc;
            break;
          }
          acc += c8[j];
        }
      }
      __syncthreads();
      const uint32_t bin = misc[4];
      need -= misc[5];
      __syncthreads();   // every thread has read misc[4..5]
      lo += bin << sh;
      if (sh > 0) hi = min(hi, lo + ((1u << sh) - 1u));
      else hi = lo;
      if (sh == 0 || !exact) break;
    }
    *out_thr = lo;
    *out_rem = need;
  };
  // Exact selection among candidates ckey/cidx[0, nc) that hold every key
  // >= some bound b with at least topk keys >= b: the topk largest keys, ties
  // to the lowest index.  ordered: the candidates sit in an order that does
  // not depend on timing, and the chosen ones are written in that order;
  // otherwise (candidates placed by atomics) they are written in increasing
  // index order through a bitmap of the row (n <= BITMAP_BITS), so repeated
  // runs agree either way.  Called by every thread.
  auto finish_candidates = [&](uint32_t nc, bool ordered) {
    uint32_t* bitmap = reinterpret_cast<uint32_t*>(smem + C::OFF_BITMAP);
    uint32_t thr, need_eq;
    uint32_t* hb = reinterpret_cast<uint32_t*>(smem + C::OFF_WHIST);   // free once the candidates exist
    select(hb, nc, [&](uint32_t i) { return ckey[i]; }, [&](uint32_t) { return true; },
           static_cast<uint32_t>(topk), &thr, &need_eq, true);
    // ties at the threshold: the need_eq lowest indices (largest ~index)
    uint32_t ties_mine = 0, n_ties;
    for (uint32_t i = tid; i < nc; i += C::NT) ties_mine += ckey[i] == thr ? 1u : 0u;
    block_scan(ties_mine, &n_ties);
    uint32_t inv_idx_thr = 0u;   // select every tie
    if (n_ties > need_eq) {
      uint32_t rem2;
      select(hb, nc, [&](uint32_t i) { return ~static_cast<uint32_t>(cidx[i]); },
             [&](uint32_t i) { return ckey[i] == thr; }, need_eq, &inv_idx_thr, &rem2, true);
    }
    auto chosen = [&](uint32_t i) {
      const uint32_t key = ckey[i];
      return key > thr || (key == thr && ~static_cast<uint32_t>(cidx[i]) >= inv_idx_thr);
    };
    if (ordered) {
      // candidates in a deterministic order: compact the chosen ones in that order
      uint32_t mine = 0, unused_total;
      for (uint32_t i = tid; i < nc; i += C::NT) mine += chosen(i) ? 1u : 0u;
      uint32_t pos_out = block_scan(mine, &unused_total);
      for (uint32_t i = tid; i < nc; i += C::NT)
        if (chosen(i)) {
          if (in_bounds(pos_out < static_cast<uint32_t>(topk), 88)) out[pos_out] = cidx[i];
          ++pos_out;
        }
      return;
    }
    // ---- selection -> bitmap -> indices in increasing order
    const int nwords = (n + 31) / 32;
    for (int i = tid; i < nwords; i += C::NT) bitmap[i] = 0u;
    __syncthreads();
    for (uint32_t i = tid; i < nc; i += C::NT)
      if (chosen(i)) atomicOr(&bitmap[cidx[i] >> 5], 1u << (cidx[i] & 31));
    __syncthreads();
    const int per = (nwords + C::NT - 1) / C::NT;
    const int w0 = min(nwords, static_cast<int>(tid) * per), w1 = min(nwords, w0 + per);
    uint32_t bits_mine = 0, unused_total;
    for (int wdx = w0; wdx < w1; ++wdx) bits_mine += __popc(bitmap[wdx]);
    uint32_t pos_out = block_scan(bits_mine, &unused_total);
    for (int wdx = w0; wdx < w1; ++wdx) {
      uint32_t bits = bitmap[wdx];
      while (bits) {
        const int bpos = __ffs(bits) - 1;
        bits &= bits - 1;
        if (in_bounds(pos_out < static_cast<uint32_t>(topk), 90)) out[pos_out] = wdx * 32 + bpos;
        ++pos_out;
      }
    }
  };

  // ================================================================== part-maxima path
  // The indexer's epilogue wrote, beside the scores, the maximum of every
  // part of PART consecutive keys (-inf past the query's position).  Parts are
  // grouped G2 at a time (G2 a power of two: about 2 k to 4 k groups, at most
  // PM_CAP).  At least k scores are >= the k-th largest part maximum b (each
  // of the k parts above it holds one), so every selected score is >= b and
  // only the parts whose maximum is >= b (about k of them) can hold one:
  // those parts are read from the row, their scores >= b become the
  // candidates, and the exact selection runs among them.  The row itself is
  // read only where it matters.  Rows with fewer than 1.25 k groups, rows past
  // the bitmap, or candidate overflows (massive ties) take the paths below.
  if (part_max != nullptr && n <= C::BITMAP_BITS) {
    const int P = (n + PART - 1) / PART;
    // Groups of G2 parts (a power of two): about 2 k to 4 k groups keep the
    // selection over the group maxima short while the candidates stay near k.
    int G2 = 1;
    while ((P + 2 * G2 - 1) / (2 * G2) >= 2 * topk || (P + G2 - 1) / G2 > C::PM_CAP) G2 <<= 1;
    const int Pg = (P + G2 - 1) / G2;
    // With few groups per selected key the bound b is low and the candidates
    // would overflow; 1.25 k groups keep them at ~2.5 k for continuous scores.
    if (4 * static_cast<int64_t>(Pg) >= 5 * static_cast<int64_t>(topk)) {
      uint32_t* pk = reinterpret_cast<uint32_t*>(smem + C::OFF_RING);    // group maxima as keys
      int32_t* plist = reinterpret_cast<int32_t*>(smem + C::OFF_WHIST);  // groups that can hold a selection
      const float4* __restrict__ pm4 = reinterpret_cast<const float4*>(part_max + r * ld_pm);
      // Group maxima from 16-byte loads of 4 part maxima (rows of ld_pm, a
      // multiple of 4 that covers P, so a load that starts below P stays in
      // the row); parts past P count as the smallest key.
      const int nf4 = (P + 3) / 4;
      auto keys4 = [&](int f, uint32_t* k) {
        const float4 v = pm4[f];
        const float vals[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) k[e] = 4 * f + e < P ? order_key(vals[e]) : 0u;
      };
      if (G2 >= 4) {
        const int f4g = G2 / 4;
#pragma unroll 4
        for (int i = tid; i < Pg; i += C::NT) {
          uint32_t m = 0u;
          for (int j = 0; j < f4g; ++j) {
            const int f = i * f4g + j;
            if (f < nf4) {
              uint32_t k[4];
              keys4(f, k);
              m = max(m, max(max(k[0], k[1]), max(k[2], k[3])));
            }
          }
          pk[i] = m;
        }
      } else {
#pragma unroll 4
        for (int f = tid; f < nf4; f += C::NT) {
          uint32_t k[4];
          keys4(f, k);
          if (G2 == 1) {
#pragma unroll
            for (int e = 0; e < 4; ++e)
              if (4 * f + e < Pg) pk[4 * f + e] = k[e];
          } else {
            if (2 * f < Pg) pk[2 * f] = max(k[0], k[1]);
            if (2 * f + 1 < Pg) pk[2 * f + 1] = max(k[2], k[3]);
          }
        }
      }
      __syncthreads();
      phase(48);
      // A lower bound of the k-th largest group maximum (its top 16 bits):
      // at least k groups, hence k scores, are >= b.
      uint32_t b, unused_rem;
      select(reinterpret_cast<uint32_t*>(smem + C::OFF_WHIST), static_cast<uint32_t>(Pg),
             [&](uint32_t i) { return pk[i]; }, [&](uint32_t) { return true; }, static_cast<uint32_t>(topk), &b,
             &unused_rem, false);
      phase(50);
      // the groups whose maximum is >= b, in order (contiguous ranges per thread, one block scan)
      const int per = (Pg + C::NT - 1) / C::NT;
      const int g_lo = min(Pg, static_cast<int>(tid) * per), g_hi = min(Pg, g_lo + per);
      uint32_t mine = 0;
      for (int i = g_lo; i < g_hi; ++i) mine += pk[i] >= b ? 1u : 0u;
      uint32_t ng;
      uint32_t at = block_scan(mine, &ng);
      for (int i = g_lo; i < g_hi; ++i)
        if (pk[i] >= b) {
          if (at < static_cast<uint32_t>(C::PLIST_CAP)) plist[at] = i;
          ++at;
        }
      __syncthreads();
      if (ng <= static_cast<uint32_t>(C::PLIST_CAP)) {
        // Candidates: the scores >= b of those groups (below: one pass into
        // per-warp slices; if a slice overflows, counted in a first pass and
        // written in a second at offsets from a block scan, no atomics).  16-byte loads; a load starts below n, and n <= ld with ld
        // a multiple of 4, so it stays inside the row.
        const int f4_per_group = G2 * PART / 4;
        const uint32_t items = ng * static_cast<uint32_t>(f4_per_group);
        // Items (16-byte loads) in batches of IB per thread, every load of a
        // batch issued before any is used, so that the L2 latency overlaps
        // (decode128k: IB = 4 measured 33.4 us, 8 35.5 us, 2 35.4 us, 16 37.5 us).
        constexpr int IB = 4;
        auto batch = [&](uint32_t base, uint32_t* k, int* k0) {
          float4 v[IB];
#pragma unroll
          for (int u = 0; u < IB; ++u) {
            const uint32_t it = base + static_cast<uint32_t>(u) * C::NT;
            k0[u] = n;
            v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (it < items) {
              k0[u] = plist[it / f4_per_group] * G2 * PART + static_cast<int>(it % f4_per_group) * 4;
              if (k0[u] < n) v[u] = *reinterpret_cast<const float4*>(row + k0[u]);
            }
          }
#pragma unroll
          for (int u = 0; u < IB; ++u) {
            k[4 * u + 0] = order_key(v[u].x);
            k[4 * u + 1] = order_key(v[u].y);
            k[4 * u + 2] = order_key(v[u].z);
            k[4 * u + 3] = order_key(v[u].w);
          }
        };
        // One pass: every warp appends its candidates (in ballot order) to
        // its own slice of the ring -- free now, the group maxima are no
        // longer read -- and the slices are then packed into ckey / cidx in
        // warp order (a timing-independent order).  A slice that overflows,
        // or more than CAP candidates in all, falls back to the counted
        // two-pass placement below.
        {
          constexpr uint32_t WCAP = C::STAGES * C::CHUNK / (2 * C::NW);   // per warp: keys, then indices
          uint32_t* wkey = reinterpret_cast<uint32_t*>(smem + C::OFF_RING) + warp * WCAP;
          int32_t* widx = reinterpret_cast<int32_t*>(smem + C::OFF_RING) + (C::NW + warp) * WCAP;
          const uint32_t lt = (1u << lane) - 1u;
          uint32_t wcnt = 0;   // warp-uniform
          for (uint32_t b0 = 0; b0 < items; b0 += IB * C::NT) {   // the same trip count in every thread
            uint32_t k[4 * IB];
            int k0[IB];
            batch(b0 + tid, k, k0);
#pragma unroll
            for (int u = 0; u < IB; ++u)
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const bool cand = k0[u] + e < n && k[4 * u + e] >= b;
                const uint32_t bal = __ballot_sync(0xFFFFFFFFu, cand);
                const uint32_t pos = wcnt + __popc(bal & lt);
                if (cand && pos < WCAP) {
                  wkey[pos] = k[4 * u + e];
                  widx[pos] = k0[u] + e;
                }
                wcnt += __popc(bal);
              }
          }
          if (lane == 0) cnt[warp] = wcnt;
          __syncthreads();
          uint32_t off = 0, total = 0;
          bool fits = true;
          for (int w2 = 0; w2 < C::NW; ++w2) {
            const uint32_t c2 = cnt[w2];
            if (w2 < static_cast<int>(warp)) off += c2;
            total += c2;
            fits = fits && c2 <= WCAP;
          }
          if (fits && total <= static_cast<uint32_t>(C::CAP)) {
            for (uint32_t i = lane; i < wcnt; i += 32) {
              ckey[off + i] = wkey[i];
              cidx[off + i] = widx[i];
            }
            __syncthreads();
            phase(49);
            finish_candidates(total, true);
            phase(45);
            DSA_PROF_END();
            return;
          }
          __syncthreads();   // every thread has read cnt before the passes below reuse it
        }
        uint32_t count = 0;
        for (uint32_t base = tid; base < items; base += IB * C::NT) {
          uint32_t k[4 * IB];
          int k0[IB];
          batch(base, k, k0);
#pragma unroll
          for (int u = 0; u < IB; ++u)
#pragma unroll
            for (int e = 0; e < 4; ++e) count += (k0[u] + e < n && k[4 * u + e] >= b) ? 1u : 0u;
        }
        uint32_t nc;
        uint32_t w_at = block_scan(count, &nc);
        if (nc <= static_cast<uint32_t>(C::CAP)) {
          for (uint32_t base = tid; base < items; base += IB * C::NT) {
            uint32_t k[4 * IB];
            int k0[IB];
            batch(base, k, k0);
#pragma unroll
            for (int u = 0; u < IB; ++u)
#pragma unroll
              for (int e = 0; e < 4; ++e)
                if (k0[u] + e < n && k[4 * u + e] >= b) {
                  ckey[w_at] = k[4 * u + e];
                  cidx[w_at] = k0[u] + e;
                  ++w_at;
                }
          }
          __syncthreads();
          phase(49);
          finish_candidates(nc, true);
          phase(45);
          DSA_PROF_END();
          return;
        }
      }
      __syncthreads();   // overflow: the paths below
    }
  }

  // ================================================================== fast path
  // Split the row into parts of PS scores (part = PS consecutive scores of one
  // thread's 16 per chunk, or one thread's scores over G chunks).  At least k
  // scores are >= the k-th largest part maximum, so the lowest key b of the
  // 11-bit bin holding that part maximum is a safe lower bound on the k-th
  // largest score.  One pass keeps the scores >= b (typically ~1.2-2 k of
  // them), the exact selection runs among those in shared memory, and the
  // selected indices are written in increasing order through a bitmap.
  // Rows where this cannot apply or the candidates overflow fall through to
  // the exact path below.
  {
    int PS = 16;
    while (PS > 1 && n / PS < 2 * topk) PS >>= 1;
    const int parts_per_thread = 16 / PS;
    const int G = max(1, (nchunks * C::NT * parts_per_thread + C::PMAX_CAP - 1) / C::PMAX_CAP);
    const int P = ((nchunks + G - 1) / G) * C::NT * parts_per_thread;
    const bool eligible = n <= C::BITMAP_BITS && n > topk && P <= C::PMAX_CAP && (G == 1 || PS == 16);
    if (eligible) {
      uint32_t* pmax = reinterpret_cast<uint32_t*>(smem + C::OFF_PMAX);
      for (int i = tid; i < P; i += C::NT) pmax[i] = 0u;
      for (int i = tid; i < C::BINS1; i += C::NT) hist[i] = 0u;
      __syncthreads();
      // ---- part maxima
      uint32_t run = 0u;     // G > 1: running max of this thread's part over a chunk group
      bool ok = stream([&](int c, const float* buf) {
        uint32_t l0[16];      // keys of this thread's 16 scores, then pairwise maxima
#pragma unroll
        for (int rr = 0; rr < 4; ++rr) {
          const int off = static_cast<int>(warp) * C::PER_WARP + (static_cast<int>(lane) + 32 * rr) * 4;
          const float4 v = *reinterpret_cast<const float4*>(buf + off);
          const float vals[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int e = 0; e < 4; ++e)
            l0[rr * 4 + e] = c * C::CHUNK + off + e < n ? order_key(vals[e]) : 0u;
        }
        uint32_t l1[8], l2[4], l3[2];
#pragma unroll
        for (int j = 0; j < 8; ++j) l1[j] = max(l0[2 * j], l0[2 * j + 1]);
#pragma unroll
        for (int j = 0; j < 4; ++j) l2[j] = max(l1[2 * j], l1[2 * j + 1]);
#pragma unroll
        for (int j = 0; j < 2; ++j) l3[j] = max(l2[2 * j], l2[2 * j + 1]);
        const uint32_t l4 = max(l3[0], l3[1]);
        const int pbase = (c * C::NT + static_cast<int>(tid)) * parts_per_thread;
        switch (PS) {
          case 1:
#pragma unroll
            for (int q = 0; q < 16; ++q) pmax[pbase + q] = l0[q];
            break;
          case 2:
#pragma unroll
            for (int q = 0; q < 8; ++q) pmax[pbase + q] = l1[q];
            break;
          case 4:
#pragma unroll
            for (int q = 0; q < 4; ++q) pmax[pbase + q] = l2[q];
            break;
          case 8:
            pmax[pbase] = l3[0];
            pmax[pbase + 1] = l3[1];
            break;
          default:
            if (G == 1) {
              pmax[pbase] = l4;
            } else {
              run = max(run, l4);
              if ((c + 1) % G == 0 || c + 1 == nchunks) {
                pmax[(c / G) * C::NT + static_cast<int>(tid)] = run;
                run = 0u;
              }
            }
        }
      });
      phase(41);
      if (!ok) { DSA_PROF_END(); return; }
      // ---- lower bound b of the k-th largest part maximum (its top 16 bits)
      uint32_t b_lo, unused_rem;
      // (the histogram goes into the ring, free between the two streaming passes)
      select(reinterpret_cast<uint32_t*>(smem + C::OFF_RING), static_cast<uint32_t>(P),
             [&](uint32_t i) { return pmax[i]; }, [&](uint32_t) { return true; }, static_cast<uint32_t>(topk), &b_lo,
             &unused_rem, false);
      if (tid == 0) misc[4] = 0u;   // candidate count
      __syncthreads();
      phase(42);
      // ---- keep every score >= b_lo
      uint32_t* cand_n = &misc[4];
      ok = stream([&](int c, const float* buf) {
        // one ballot per element slot, one atomic per warp and chunk
        uint32_t keys[16], bal[16];
        uint32_t wsum = 0;
        const uint32_t lt = (1u << lane) - 1u;
#pragma unroll
        for (int rr = 0; rr < 4; ++rr) {
          const int off = static_cast<int>(warp) * C::PER_WARP + (static_cast<int>(lane) + 32 * rr) * 4;
          const float4 v = *reinterpret_cast<const float4*>(buf + off);
          const float vals[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            keys[rr * 4 + e] = order_key(vals[e]);
            const bool keep = c * C::CHUNK + off + e < n && keys[rr * 4 + e] >= b_lo;
            bal[rr * 4 + e] = __ballot_sync(0xFFFFFFFFu, keep);
            wsum += __popc(bal[rr * 4 + e]);
          }
        }
        if (wsum) {
          uint32_t base = 0;
          if (lane == 0) base = atomicAdd(cand_n, wsum);
          base = __shfl_sync(0xFFFFFFFFu, base, 0);
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            if ((bal[j] >> lane) & 1u) {
              const uint32_t at = base + __popc(bal[j] & lt);
              if (at < static_cast<uint32_t>(C::CAP)) {
                ckey[at] = keys[j];
                cidx[at] = c * C::CHUNK + static_cast<int>(warp) * C::PER_WARP +
                           (static_cast<int>(lane) + 32 * (j >> 2)) * 4 + (j & 3);
              }
            }
            base += __popc(bal[j]);
          }
        }
      });
      phase(43);
      if (!ok) { DSA_PROF_END(); return; }
      const uint32_t nc = *cand_n;
      if (nc <= static_cast<uint32_t>(C::CAP)) {
        finish_candidates(nc, false);
        phase(45);
        DSA_PROF_END();
        return;
      }
      __syncthreads();   // candidates overflowed: the exact path below
      phase(46);
    }
  }
  for (int i = tid; i < C::NW * (C::BINS1 / 2); i += C::NT) reinterpret_cast<uint32_t*>(smem + C::OFF_WHIST)[i] = 0u;
  for (int i = tid; i < C::BINS1; i += C::NT) hist[i] = 0u;
  __syncthreads();

  // ------------------------------------------------------------------ pass 1
  bool ok = stream([&](int c, const float* buf) {
#pragma unroll
    for (int rr = 0; rr < 4; ++rr) {
      const int off = static_cast<int>(warp) * C::PER_WARP + (static_cast<int>(lane) + 32 * rr) * 4;
      const float4 v = *reinterpret_cast<const float4*>(buf + off);
      const int gi = c * C::CHUNK + off;
      whist_add(order_key(v.x) >> C::SHIFT1, gi < n);
      whist_add(order_key(v.y) >> C::SHIFT1, gi + 1 < n);
      whist_add(order_key(v.z) >> C::SHIFT1, gi + 2 < n);
      whist_add(order_key(v.w) >> C::SHIFT1, gi + 3 < n);
    }
  });
  if (!ok) { DSA_PROF_END(); return; }
  // merge the per-warp counts
  for (int bin = tid; bin < C::BINS1; bin += C::NT) {
    uint32_t sum = 0;
#pragma unroll
    for (int w = 0; w < C::NW; ++w)
      sum += (reinterpret_cast<const uint32_t*>(smem + C::OFF_WHIST)[w * (C::BINS1 / 2) + (bin >> 1)] >>
              (16 * (bin & 1))) & 0xFFFFu;
    hist[bin] = sum;
  }
  __syncthreads();

  find_digit_fn(hist, C::BINS1, static_cast<uint32_t>(topk), &misc[0], &misc[1]);
  __syncthreads();
  const uint32_t bin_b = misc[0];
  const uint32_t above = misc[1];
  const uint32_t need = static_cast<uint32_t>(topk) - above;

  // ------------------------------------------------------------------ pass 2
  ok = stream([&](int c, const float* buf) {
    scan_chunk(
        c, buf,
        [&](uint32_t key, bool& gt, bool& eq) {
          const uint32_t b = key >> C::SHIFT1;
          gt = b > bin_b;
          eq = b == bin_b;
        },
        [&](uint32_t rank, int gi, uint32_t) {
          if (in_bounds(rank < static_cast<uint32_t>(topk), 89)) out[rank] = gi;
        },
        [&](uint32_t rank, int gi, uint32_t key) {
          if (rank < static_cast<uint32_t>(C::CAP)) {
            ckey[rank] = key;
            cidx[rank] = gi;
          }
        });
  });
  if (!ok) { DSA_PROF_END(); return; }
  const uint32_t n_eq = eq_base;          // keys in bin B (all of them, even past CAP)

  // ------------------------------------------------------------------ refine inside bin B
  // 21 remaining key bits as digits of 8, 8 and 5 bits.
  uint32_t prefix = bin_b << C::SHIFT1;
  uint32_t remaining = need;
  const bool in_smem = n_eq <= static_cast<uint32_t>(C::CAP);
  const int shifts[3] = {13, 5, 0};
  const int widths[3] = {8, 8, 5};
  for (int d = 0; d < 3; ++d) {
    const int shift = shifts[d], bits = widths[d];
    const uint32_t dmask = (1u << bits) - 1u;
    const int hi = shift + bits;                  // bits at or above `hi` are fixed by prefix
    for (int i = tid; i < 256; i += C::NT) hist[i] = 0u;
    __syncthreads();
    auto count_key = [&](uint32_t key, bool valid) {
      const bool m = valid && ((key >> hi) == (prefix >> hi));
      hist_add(hist, (key >> shift) & dmask, m);
    };
    if (in_smem) {
      for (uint32_t base = 0; base < n_eq; base += C::NT) {
        const uint32_t i = base + tid;
        count_key(i < n_eq ? ckey[i] : 0u, i < n_eq);
      }
    } else {
      ok = stream([&](int c, const float* buf) {
#pragma unroll
        for (int rr = 0; rr < 4; ++rr) {
          const int off = static_cast<int>(warp) * C::PER_WARP + (static_cast<int>(lane) + 32 * rr) * 4;
          const float4 v = *reinterpret_cast<const float4*>(buf + off);
          const int gi = c * C::CHUNK + off;
          count_key(order_key(v.x), gi < n);
          count_key(order_key(v.y), gi + 1 < n);
          count_key(order_key(v.z), gi + 2 < n);
          count_key(order_key(v.w), gi + 3 < n);
        }
      });
      if (!ok) { DSA_PROF_END(); return; }
    }
    __syncthreads();
    find_digit_fn(hist, 1 << bits, remaining, &misc[2], &misc[3]);
    __syncthreads();
    prefix |= misc[2] << shift;
    remaining -= misc[3];
    __syncthreads();
  }
  const uint32_t thr = prefix;            // the k-th largest key
  const uint32_t need_eq = remaining;     // how many keys equal to it are taken
  const uint32_t n_gt = need - need_eq;   // keys of bin B above it
  int32_t* out_b = out + above;

  // ------------------------------------------------------------------ emit bin B's selection
  gt_base = 0;
  eq_base = 0;
  if (in_smem) {
    for (uint32_t base = 0; base < n_eq; base += C::NT) {
      const uint32_t i = base + tid;
      const uint32_t key = i < n_eq ? ckey[i] : 0u;
      const bool gt = i < n_eq && key > thr;
      const bool eq = i < n_eq && key == thr;
      const uint32_t lt = (1u << lane) - 1u;
      const uint32_t bg = __ballot_sync(0xFFFFFFFFu, gt), be = __ballot_sync(0xFFFFFFFFu, eq);
      if (lane == 0) wtot[warp] = (static_cast<uint32_t>(__popc(bg))) | (static_cast<uint32_t>(__popc(be)) << 16);
      __syncthreads();
      uint32_t wpre = 0, ctot = 0;
#pragma unroll
      for (int w = 0; w < C::NW; ++w) {
        const uint32_t v = wtot[w];
        wpre += static_cast<uint32_t>(w) < warp ? v : 0u;
        ctot += v;
      }
      if (gt) out_b[gt_base + (wpre & 0xFFFFu) + __popc(bg & lt)] = cidx[i];
      if (eq) {
        const uint32_t rk = eq_base + (wpre >> 16) + __popc(be & lt);
        if (rk < need_eq) out_b[n_gt + rk] = cidx[i];
      }
      gt_base += ctot & 0xFFFFu;
      eq_base += ctot >> 16;
      __syncthreads();
    }
  } else {
    stream([&](int c, const float* buf) {
      scan_chunk(
          c, buf,
          [&](uint32_t key, bool& gt, bool& eq) {
            const bool inb = (key >> C::SHIFT1) == bin_b;
            gt = inb && key > thr;
            eq = inb && key == thr;
          },
          [&](uint32_t rank, int gi, uint32_t) { out_b[rank] = gi; },
          [&](uint32_t rank, int gi, uint32_t) {
            if (rank < need_eq) out_b[n_gt + rank] = gi;
          });
    });
  }
  phase(47);
  DSA_PROF_END();
}

}  // namespace dsa
