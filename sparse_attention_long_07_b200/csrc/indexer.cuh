// indexer.cuh -- lightning-indexer scores on the tcgen05 tensor cores.
//
// "DeepSeek-V3.2" (transformers model doc), "DeepSeek Sparse Attention
// (DSA)", item 1: a light module with few index heads scores each query
// against every preceding key.  With index heads j, per-query head weights w
// and a single-head index key per token:
//     I[t,s] = sum_j w[t,j] * max(0, q_I[t,j,:] . k_I[s,:]),   s <= pos(t).
//
// GEMM view: A = a tile of 128 index keys (M = 128, one key per TMEM lane),
// B = the index queries of NQ consecutive query tokens (N = NQ * H_I rows,
// K = d_I), D = [128 keys x NQ*H_I logits] in fp32 tensor memory.  The
// epilogue reads one key row per thread, so the ReLU, the head weights and the
// sum over heads stay inside one thread and the [T x L x H_I] logits never
// leave the SM; only the fp32 score per (query, key) is written.
//
// Roles (query-block grid): one TMA warp streams key tiles through a
// shared-memory ring; one thread issues the MMAs into two TMEM accumulators;
// one epilogue warpgroup (four, one per query, for four-query blocks) drains
// them.  For an e4m3 index-key cache, four more warps widen each raw tile to
// bf16 in the shared-memory UMMA layout (exact: every e4m3 value is a bf16
// value), and the per-key fp32 scale multiplies the head-reduced score (a
// positive scale commutes with ReLU).  The persistent decode schedule (below)
// widens keys to f16 into tensor memory instead, multiplies f16 operands,
// issues MMAs from two threads and drains four accumulators with four
// epilogue warpgroups.
#pragma once

#include "common.cuh"
#include "fp8.cuh"
#include "sm100.cuh"

namespace dsa {

__host__ __device__ constexpr int pow2_at_least(int v, int lo) {
  int p = lo;
  while (p < v) p <<= 1;
  return p;
}

template <int H_I_, int D_I_, int NQ_, bool KFP8_, bool PERSIST_ = false, bool QFP8_ = false>
struct IndexerCfg {
  static constexpr int H_I = H_I_, D_I = D_I_, NQ = NQ_;
  static constexpr bool KFP8 = KFP8_;
  // FP8 indexer: e4m3 queries and keys (Hadamard-rotated, power-of-two scales)
  // multiplied as they are by kind::f8f6f4 MMAs; otherwise bf16 MMAs, with
  // e4m3 keys widened to bf16 first (CONVERT)
  static constexpr bool QFP8 = QFP8_;
  static constexpr bool CONVERT = KFP8 && !QFP8;
  static constexpr bool PERSIST = PERSIST_;                 // one CTA per SM over a flat unit list
  static constexpr int MAX_SEQ = 2048;                    // persistent: sequences per call
  static constexpr int BK = 128;                          // keys per tile (MMA M)
  static constexpr int N = NQ * H_I;                      // MMA N
  static constexpr int ELEM = QFP8 ? 1 : 2;               // bytes per MMA operand element
  static constexpr int ROWB = D_I * ELEM;                 // bytes of one operand row
  static constexpr int SWB = ROWB >= 128 ? 128 : ROWB;    // swizzle span (128 or 64 bytes)
  static constexpr uint32_t SWZ = SWB == 128 ? 2u : 4u;   // descriptor swizzle code
  static constexpr int NATOM = ROWB / SWB;                // swizzle-atom columns per row
  static constexpr int ATOM_ELEMS = SWB / ELEM;
  static constexpr int KSTEPS = ROWB / 32;                // 32 bytes of K per MMA (16 bf16 or 32 e4m3)
  // Persistent schedule with bf16 queries: the widened bf16 key tile is
  // written to tensor memory and read from there as the A operand (TS-form
  // MMA), so shared memory holds only the raw e4m3 ring; otherwise the key
  // tile ring (bf16, or e4m3 as loaded for the FP8 indexer) is in shared
  // memory, twelve deep for the persistent FP8 schedule.
  static constexpr bool K_IN_TMEM = PERSIST && CONVERT;
  // ... and there the MMAs take f16 operands: e4m3 keys widen to f16 in one
  // conversion instruction per pair, and each sequence's bf16 query tile is
  // rewritten in place as f16, scaled by a power of two 2^sq that puts its
  // largest magnitude in [2^14, 2^15); the epilogue multiplies by 2^-sq.
  static constexpr bool QF16 = K_IN_TMEM;
  static constexpr int STAGES = K_IN_TMEM ? 4 : (PERSIST ? 12 : (CONVERT ? 2 : 4));  // key-tile ring (MMA operand)
  static constexpr int RSTAGES = CONVERT ? (PERSIST ? 11 : 4) : 0;  // raw e4m3 ring (to widen)
  static constexpr int A_TILE = BK * ROWB;
  static constexpr int B_TILE = N * ROWB;
  static constexpr int RAW_ROWB = D_I;                    // bytes of one e4m3 key row
  static constexpr int RAW_TILE = BK * RAW_ROWB;
  // epilogue warpgroups: four split the four queries of a wide tile (one
  // each), or (persistent schedule) four take every fourth tile, each owning
  // one TMEM accumulator.  The epilogue's per-tile chain (tensor-memory
  // loads, 64 ReLU-FMAs, the score and part-maximum stores) bounded both
  // schedules; measured with four warpgroups instead of two: decode128k
  // 0.154 -> 0.131 ms (bf16 queries), 0.119 -> 0.102 ms (FP8); prefill32k
  // 8.7 -> 8.0 ms.
  static constexpr int EPI_WG = (PERSIST || N >= 256) ? 4 : 1;
  static constexpr int QW = PERSIST ? NQ : NQ / EPI_WG;   // queries per epilogue warpgroup
  static constexpr int COLS_PER_THREAD = QW * H_I;
  static constexpr int LD_CHUNK = COLS_PER_THREAD >= 32 ? 32 : 16;
  // fp32 accumulators: the persistent schedule keeps four in flight so that
  // the MMAs of the next tiles never wait for the epilogue of the last one
  static constexpr int NACC = PERSIST ? 4 : 2;
  static constexpr int ACC_COLS = NACC * N;
  static constexpr int A_COLS = D_I / 2;                  // one bf16 key tile in tensor memory
  static constexpr int TMEM_COLS = pow2_at_least(ACC_COLS + (K_IN_TMEM ? STAGES * A_COLS : 0), 32);
  static constexpr int EPI_THREADS = 128 * EPI_WG;
  static constexpr int PRODUCER_WARP = 4 * EPI_WG;
  static constexpr int MMA_WARP = PRODUCER_WARP + 1;
  // persistent schedule: two MMA-issuing threads (one per warp) take alternate
  // tiles, so one's barrier waits and commits overlap the other's MMAs
  static constexpr int MMA_THREADS = PERSIST ? 2 : 1;
  static constexpr int CONVERT_WARP0 = MMA_WARP + MMA_THREADS;
  static constexpr int CONV_TEAMS = PERSIST ? 2 : 1;      // e4m3 converter teams (alternate tiles)
  static constexpr int NWARPS = MMA_WARP + MMA_THREADS + (CONVERT ? 4 * CONV_TEAMS : 0);
  static constexpr int NT = NWARPS * 32;
  static constexpr uint32_t IDESC =
      QFP8 ? idesc_e4m3_f32(128, N) : (QF16 ? idesc_f16_f32(128, N) : idesc_bf16_f32(128, N, false, false));
  // shared memory layout (offsets from a 1024-byte aligned base)
  static constexpr int QBUF = PERSIST ? 2 : 1;            // query tiles (double buffer when persistent)
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + QBUF * B_TILE;
  static constexpr int OFF_RAW = OFF_K + (K_IN_TMEM ? 0 : STAGES * A_TILE);
  static constexpr int OFF_W = OFF_RAW + RSTAGES * RAW_TILE;
  static constexpr int OFF_BAR = OFF_W + NQ * H_I * 4;
  // barriers: grid schedule 2 + 2 STAGES + 2 RSTAGES + 2 NACC; persistent
  // schedule 7 + STAGES (ready) + 2 RSTAGES + NACC (acc_full) + 2 STAGES
  // (k_full, k_empty) + NACC (acc_empty) + 2 (q_conv) + 2 (q_max), every
  // array reserved in both forms
  static constexpr int NBAR = 11 + 3 * STAGES + 2 * RSTAGES + 2 * NACC;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  // f16 queries: descale 2^-sq per query buffer and per accumulator, and the
  // converter teams' partial maxima (team, buffer, warp)
  static constexpr int OFF_QCONV = OFF_MISC + 16;
  static constexpr int OFF_UPRE = OFF_QCONV + 128;        // persistent: unit prefix per sequence
  // persistent: per-warp head weights, read as float4 (16-byte aligned)
  static constexpr int OFF_WEPI = (OFF_UPRE + (PERSIST ? (MAX_SEQ + 1) * 4 : 0) + 15) / 16 * 16;
  static constexpr int SMEM_BYTES = OFF_WEPI + (PERSIST ? 4 * EPI_WG * H_I * 4 : 0) + 1024;  // + alignment slack
  static_assert(N % 16 == 0 && N >= 16 && N <= 256, "MMA N");
  static_assert(B_TILE % 1024 == 0 && A_TILE % 1024 == 0, "atom alignment");
  static_assert(COLS_PER_THREAD % LD_CHUNK == 0, "TMEM load chunking");
  static_assert(!KFP8 || D_I == 128, "e4m3 keys: 128-byte rows");
  static_assert(!QFP8 || (KFP8 && D_I == 128), "FP8 indexer: e4m3 keys, 128-byte rows");
  static_assert(TMEM_COLS <= 512, "tensor memory columns");
  static_assert(!K_IN_TMEM || (KFP8 && STAGES % CONV_TEAMS == 0), "converter teams own alternate stages");
  static_assert(!PERSIST || NACC % EPI_WG == 0, "each accumulator is drained by one epilogue warpgroup");
  static_assert(2 + 2 * STAGES + 2 * RSTAGES + 2 * NACC <= NBAR, "grid barrier layout");
  static_assert(!PERSIST || 11 + 3 * STAGES + 2 * RSTAGES + 2 * NACC <= NBAR, "persistent barrier layout");
  static_assert(!PERSIST || CONV_TEAMS <= 2, "query-maximum barriers");
  static_assert(4 * (2 + NACC) + 4 * 2 * CONV_TEAMS * 4 <= 128, "query-conversion scratch");
  static_assert(!QF16 || (B_TILE / 16) % 128 == 0, "query tile in 16-byte pieces per converter thread");
  static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
  static_assert(!K_IN_TMEM || STAGES == NACC, "key stage and accumulator of a tile share one barrier");
  static_assert(!PERSIST || NQ == 1, "persistent schedule: one query per sequence block");
  static_assert(OFF_K % 1024 == 0 && OFF_RAW % 1024 == 0, "swizzled tiles on 1024-byte boundaries");
  static_assert(OFF_WEPI % 16 == 0 && OFF_W % 16 == 0, "16-byte vector accesses");
  static_assert(OFF_BAR % 8 == 0 && OFF_UPRE % 4 == 0, "barrier / prefix alignment");
};

// Four e4m3 bytes -> four bf16 values (two bf16x2 words, lower element in the
// low half), with integer and bf16 arithmetic only.  PRMT puts each byte in
// the low byte of a 16-bit half and fills the high byte with copies of its
// sign bit; shifting left by 4 and masking leaves the sign in bit 15 and the
// byte's 4 exponent and 3 mantissa bits in bits 10..4.  Read as bf16 that is
// 2^(e-127)(1 + m/8), or 2^-126 (m/8) when e = 0, and one multiplication by
// 2^120 (exact; bf16 arithmetic keeps subnormal operands) gives the e4m3 value
// 2^(e-7)(1 + m/8), or 2^-6 (m/8).  The two NaN codes (0x7F, 0xFF) are not
// special-cased: key caches hold finite values.
__device__ __forceinline__ void e4m3x4_to_bf16x4(uint32_t src, uint32_t& lo, uint32_t& hi) {
  uint32_t a, b;
  // selector nibbles, low byte first: byte 0, sign of byte 0, byte 1, sign of byte 1
  asm("prmt.b32 %0, %1, 0, 0x9180;" : "=r"(a) : "r"(src));
  asm("prmt.b32 %0, %1, 0, 0xB3A2;" : "=r"(b) : "r"(src));   // the same for bytes 2 and 3
  a = (a << 4) & 0x87F087F0u;
  b = (b << 4) & 0x87F087F0u;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(lo) : "r"(a), "r"(0x7B807B80u));   // 0x7B80 = bf16 2^120
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(hi) : "r"(b), "r"(0x7B807B80u));
}

// One key row of a raw e4m3 tile (128 bytes, 128-byte TMA swizzle) -> the
// same row of the bf16 UMMA tile (two 128-byte swizzle atoms).  Exact: every
// e4m3 value is a bf16 value (e4m3x4_to_bf16x4).
template <int BK>
__device__ __forceinline__ void e4m3_row_to_bf16(const uint8_t* raw_row, uint8_t* dst_tile, int row) {
  uint4 chunk[8];
#pragma unroll
  for (int j = 0; j < 8; ++j)  // 128-byte swizzle: logical chunk j sits at j ^ (row & 7)
    chunk[j] = *reinterpret_cast<const uint4*>(raw_row + ((j ^ (row & 7)) << 4));
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const uint32_t src[4] = {chunk[j].x, chunk[j].y, chunk[j].z, chunk[j].w};
    uint32_t outw[8];
#pragma unroll
    for (int e = 0; e < 4; ++e) e4m3x4_to_bf16x4(src[e], outw[2 * e], outw[2 * e + 1]);
    // 16 bf16 = logical chunks 2j, 2j+1 of the row; 64 elements per atom
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int lc = 2 * j + h;
      uint8_t* dst = dst_tile + (lc >> 3) * (BK * 128) + row * 128 + (((lc & 7) ^ (row & 7)) << 4);
      *reinterpret_cast<uint4*>(dst) = make_uint4(outw[4 * h], outw[4 * h + 1], outw[4 * h + 2], outw[4 * h + 3]);
    }
  }
}

// Four e4m3 bytes -> four f16 values (two f16x2 words, lower element in the
// low half), exact: one hardware conversion per pair.
__device__ __forceinline__ void e4m3x4_to_f16x4(uint32_t src, uint32_t& lo, uint32_t& hi) {
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, l;\n\tcvt.rn.f16x2.e4m3x2 %1, h;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(src));
}

struct IndexerParams {
  const float* w;            // [T, H_I]
  const float* q_scale;      // [T, H_I] (FP8 indexer) or null
  const float* k_scale;      // [cache rows] (e4m3 keys) or null
  PageMap pages;             // where the caches keep each entry
  int cache_rows;            // rows of the index-key cache (checked builds)
  const int32_t* cu_q;
  const int32_t* cu_k;
  int B;
  int64_t q_begin, q_end;    // global query rows of this call
  float* scores;             // [q_end - q_begin, ld]
  int64_t ld;
  float* part_max;           // [q_end - q_begin, ld_pm] or null: max over each part of PART keys
  int64_t ld_pm;
  int chunk_tiles;           // key tiles per CTA
};

// Max over the PART consecutive lanes of `v` (lanes 8i .. 8i+7); every lane
// of the warp takes part.  Lane 8i gets the maximum of its part.
__device__ __forceinline__ float part_max8(float v) {
  v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, 1));
  v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, 2));
  v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, 4));
  return v;
}

template <class C>
__global__ void __launch_bounds__(C::NT, 1)
    indexer_scores_kernel(const __grid_constant__ CUtensorMap tm_q,
                          const __grid_constant__ CUtensorMap tm_k, const IndexerParams p) {
  // ---------------------------------------------------------------- work unit
  const int b = blockIdx.z;
  const int qb = gridDim.y - 1 - blockIdx.y;  // heaviest query blocks first
  const int cq0 = p.cu_q[b], cq1 = p.cu_q[b + 1];
  const int k_base = p.cu_k[b];
  const int kv_len = p.cu_k[b + 1] - k_base;
  const int64_t lo = cq0 > p.q_begin ? cq0 : p.q_begin;
  const int64_t hi = cq1 < p.q_end ? cq1 : p.q_end;
  const int64_t q0 = lo + static_cast<int64_t>(qb) * C::NQ;
  if (q0 >= hi) return;
  const int nq = static_cast<int>(hi - q0 < C::NQ ? hi - q0 : C::NQ);
  const int pos0 = kv_len - (cq1 - cq0) + static_cast<int>(q0 - cq0);  // position of query q0
  const int ntiles = (pos0 + nq - 1) / C::BK + 1;
  const int t_begin = blockIdx.x * p.chunk_tiles;
  const int t_end = min(ntiles, t_begin + p.chunk_tiles);
  grid_launch_dependents();   // the top-k may be scheduled as SMs free up (it waits for this grid)
  if (t_begin >= t_end || device_error_pending()) return;
  const int n_iter = t_end - t_begin;

  // ---------------------------------------------------------------- shared memory
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t s_q = sbase + C::OFF_Q;
  const uint32_t s_k = sbase + C::OFF_K;
  const uint32_t s_raw = sbase + C::OFF_RAW;
  float* w_s = reinterpret_cast<float*>(smem + C::OFF_W);
  const uint32_t bar0 = sbase + C::OFF_BAR;
  const uint32_t bar_q_full = bar0;
  const uint32_t bar_drain = bar0 + 8;
  auto bar_k_full = [&](int s) { return bar0 + 16 + 8 * s; };
  auto bar_k_empty = [&](int s) { return bar0 + 16 + 8 * (C::STAGES + s); };
  auto bar_raw_full = [&](int s) { return bar0 + 16 + 8 * (2 * C::STAGES + s); };
  auto bar_raw_empty = [&](int s) { return bar0 + 16 + 8 * (2 * C::STAGES + C::RSTAGES + s); };
  auto bar_acc_full = [&](int a) { return bar0 + 16 + 8 * (2 * C::STAGES + 2 * C::RSTAGES + a); };
  auto bar_acc_empty = [&](int a) { return bar0 + 16 + 8 * (2 * C::STAGES + 2 * C::RSTAGES + 2 + a); };
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(bar_q_full, 1);
    mbar_init(bar_drain, 1);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(bar_k_full(s), C::CONVERT ? 128 : 1);
      mbar_init(bar_k_empty(s), 1);
    }
    for (int s = 0; s < C::RSTAGES; ++s) {
      mbar_init(bar_raw_full(s), 1);
      mbar_init(bar_raw_empty(s), 128);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(bar_acc_full(a), 1);
      mbar_init(bar_acc_empty(a), C::EPI_THREADS);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == C::MMA_WARP) {
    tmem_alloc(smem_u32(tmem_holder), C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == C::PRODUCER_WARP && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
  }
  // head weights of this block's queries (rows past the block are zero); the
  // FP8 indexer folds in each query head's scale and the 2^-7 of the rotation
  for (int i = threadIdx.x; i < C::NQ * C::H_I; i += C::NT) {
    const int qi = i / C::H_I;
    float wv = 0.f;
    if (qi < nq) {
      const int64_t g = (q0 + qi) * C::H_I + (i % C::H_I);
      wv = p.w[g];
      if (C::QFP8) wv *= ldexpf(p.q_scale[g], -FP8_HADAMARD_LOG2);
    }
    w_s[i] = wv;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == C::PRODUCER_WARP) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int armed_q = 0;
      mbar_arrive_expect_tx(bar_q_full, C::B_TILE);
      for (int a = 0; a < C::NATOM; ++a)
        tma_load_2d(s_q + a * C::N * C::SWB, &tm_q, bar_q_full, a * C::ATOM_ELEMS,
                    static_cast<int32_t>(q0 * C::H_I));
      armed_q = 1;
      int it = 0;
      for (; it < n_iter; ++it) {
        // Key tile: one box of BK rows (packed), or BK / 64 boxes of 64 rows,
        // each inside one page (paged; a missing page loads as zeros from a
        // row coordinate outside the cache).
        const int s0 = (t_begin + it) * C::BK;
        int y[C::BK / 64];
#pragma unroll
        for (int h = 0; h < C::BK / 64; ++h) {
          // (a box that starts past the sequence is never read: its scores are masked)
          int r = p.pages.row(b, k_base, s0 + 64 * h);
          if (r >= 0 && s0 + 64 * h < kv_len && !in_bounds(r < p.cache_rows, 81)) r = -1;
          y[h] = r >= 0 ? r : -64;
        }
        const int nbox = p.pages.paged() ? C::BK / 64 : 1;
        if constexpr (C::CONVERT) {
          const int r = it % C::RSTAGES;
          if (!mbar_wait(bar_raw_empty(r), ((it / C::RSTAGES) & 1) ^ 1, abort_flag, 11)) break;
          mbar_arrive_expect_tx(bar_raw_full(r), C::RAW_TILE);
          for (int h = 0; h < nbox; ++h)
            tma_load_2d(s_raw + r * C::RAW_TILE + h * 64 * C::RAW_ROWB, &tm_k, bar_raw_full(r), 0, y[h]);
        } else {
          const int s = it % C::STAGES;
          if (!mbar_wait(bar_k_empty(s), ((it / C::STAGES) & 1) ^ 1, abort_flag, 12)) break;
          mbar_arrive_expect_tx(bar_k_full(s), C::A_TILE);
          for (int a = 0; a < C::NATOM; ++a)
            for (int h = 0; h < nbox; ++h)
              tma_load_2d(s_k + s * C::A_TILE + a * C::BK * C::SWB + h * 64 * C::SWB, &tm_k, bar_k_full(s),
                          a * C::ATOM_ELEMS, y[h]);
        }
      }
      if (*abort_flag) {
        // let copies already in flight land before the CTA's memory is released
        long long t0 = clock64();
        constexpr int ring = C::CONVERT ? C::RSTAGES : C::STAGES;
        for (int j = (it > ring ? it - ring : 0); j < it; ++j) {
          const uint32_t bar = C::CONVERT ? bar_raw_full(j % ring) : bar_k_full(j % ring);
          while (!mbar_try_wait(bar, (j / ring) & 1) && clock64() - t0 < kWaitLimitCycles) {
          }
        }
        if (armed_q)
          while (!mbar_try_wait(bar_q_full, 0) && clock64() - t0 < kWaitLimitCycles) {
          }
      }
    }
  } else if (warp == C::MMA_WARP) {
    // ------------------------------------------------------------ MMA issuer
    const uint64_t a_desc0 = smem_desc(s_k, 16, 8 * C::SWB, C::SWZ);
    const uint64_t b_desc0 = smem_desc(s_q, 16, 8 * C::SWB, C::SWZ);
    if (lane == 0) {
      if (mbar_wait(bar_q_full, 0, abort_flag, 13)) {
        tc_fence_after();
        for (int it = 0; it < n_iter; ++it) {
          const int s = it % C::STAGES;
          const int a = it & 1;
          if (!mbar_wait(bar_k_full(s), (it / C::STAGES) & 1, abort_flag, 14)) break;
          if (!mbar_wait(bar_acc_empty(a), ((it >> 1) & 1) ^ 1, abort_flag, 15)) break;
          tc_fence_after();
          const uint64_t a_stage = a_desc0 + static_cast<uint64_t>((s * C::A_TILE) >> 4);
#pragma unroll
          for (int kk = 0; kk < C::KSTEPS; ++kk) {
            const int atom = (kk * 32) / C::SWB;
            const int off = (kk * 32) % C::SWB;
            const uint64_t ad = a_stage + static_cast<uint64_t>((atom * C::BK * C::SWB + off) >> 4);
            const uint64_t bd = b_desc0 + static_cast<uint64_t>((atom * C::N * C::SWB + off) >> 4);
            if constexpr (C::QFP8) umma_ss_e4m3(tmem + a * C::N, ad, bd, C::IDESC, kk > 0 ? 1u : 0u);
            else umma_ss(tmem + a * C::N, ad, bd, C::IDESC, kk > 0 ? 1u : 0u);
          }
          umma_commit(bar_k_empty(s));
          umma_commit(bar_acc_full(a));
        }
      }
      // every MMA issued above has completed once this arrives
      umma_commit(bar_drain);
      long long t0 = clock64();
      while (!mbar_try_wait(bar_drain, 0) && clock64() - t0 < kWaitLimitCycles) {
      }
    }
  } else if (warp >= C::CONVERT_WARP0) {
    // ------------------------------------------------------------ e4m3 -> bf16
    // (bf16 queries only: the FP8 schedule has no converter warps)
    if constexpr (C::CONVERT) {
    const int row = threadIdx.x - C::CONVERT_WARP0 * 32;  // key row of the tile
    for (int it = 0; it < n_iter; ++it) {
      const int r = it % C::RSTAGES;
      const int s = it % C::STAGES;
      if (!mbar_wait(bar_raw_full(r), (it / C::RSTAGES) & 1, abort_flag, 16)) break;
      const uint8_t* raw_row = smem + C::OFF_RAW + r * C::RAW_TILE + row * 128;
      // the raw stage is read into registers inside the conversion; release it after
      if (!mbar_wait(bar_k_empty(s), ((it / C::STAGES) & 1) ^ 1, abort_flag, 17)) break;
      e4m3_row_to_bf16<C::BK>(raw_row, smem + C::OFF_K + s * C::A_TILE, row);
      mbar_arrive(bar_raw_empty(r));
      fence_proxy_async_smem();
      mbar_arrive(bar_k_full(s));
    }
    }
  } else if (warp < C::PRODUCER_WARP) {
    // ------------------------------------------------------------ epilogue
    const int g = warp >> 2;        // epilogue warpgroup
    const int sub = warp & 3;       // TMEM sub-partition = lanes 32*sub ..
    const int key_in_tile = sub * 32 + lane;
    for (int it = 0; it < n_iter; ++it) {
      const int a = it & 1;
      if (!mbar_wait_warp(bar_acc_full(a), (it >> 1) & 1, abort_flag, 18)) break;
      tc_fence_after();
      float acc[C::QW];
#pragma unroll
      for (int q = 0; q < C::QW; ++q) acc[q] = 0.f;
      const uint32_t t_row = tmem + (static_cast<uint32_t>(sub * 32) << 16) + a * C::N + g * C::COLS_PER_THREAD;
#pragma unroll
      for (int c0 = 0; c0 < C::COLS_PER_THREAD; c0 += C::LD_CHUNK) {
        uint32_t v[32];
        if (C::LD_CHUNK == 32) tmem_ld32(t_row + c0, v); else tmem_ld16(t_row + c0, v);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < C::LD_CHUNK; ++j) {
          const int c = c0 + j;
          const int q = c / C::H_I;
          const float wv = w_s[(g * C::QW + q) * C::H_I + (c % C::H_I)];
          acc[q] = fmaf(wv, fmaxf(__uint_as_float(v[j]), 0.f), acc[q]);
        }
      }
      tc_fence_before();
      mbar_arrive(bar_acc_empty(a));
      const int s = (t_begin + it) * C::BK + key_in_tile;
      const bool in_seq = s < kv_len;
      float kscale = 1.f;
      if (C::KFP8 && in_seq) {
        if (!p.pages.paged()) {
          kscale = p.k_scale[k_base + s];
        } else {
          const int r = p.pages.row(b, k_base, s);
          kscale = (r >= 0 && in_bounds(r < p.cache_rows, 85)) ? p.k_scale[r] : 0.f;
        }
      }
#pragma unroll
      for (int q = 0; q < C::QW; ++q) {
        const int qi = g * C::QW + q;          // the same for the whole warp
        if (qi < nq) {
          // keys past the query's position (and past the cache) score -inf
          const float val = s <= pos0 + qi ? acc[q] * kscale : -INFINITY;
          const int64_t row = q0 + qi - p.q_begin;
          if (in_seq && in_bounds(s < p.ld, 83)) p.scores[row * p.ld + s] = val;
          if (p.part_max != nullptr) {
            const float m = part_max8(val);
            if ((lane & (PART - 1)) == 0 && in_seq) p.part_max[row * p.ld_pm + s / PART] = m;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// Persistent schedule for decode-like calls (at most one query row per
// sequence in the call).  The work units are the (sequence, 128-key tile)
// pairs of the call, flattened in sequence order; CTA c of G (G = number of
// SMs) takes units [c U / G, (c+1) U / G), so every SM streams the same
// number of key tiles.  Consecutive units of one sequence share its query tile,
// which is reloaded only when the sequence changes.
template <class C>
__global__ void __launch_bounds__(C::NT, 1)
    indexer_persistent_kernel(const __grid_constant__ CUtensorMap tm_q,
                              const __grid_constant__ CUtensorMap tm_k, const IndexerParams p) {
  static_assert(C::PERSIST && C::KFP8 && C::NQ == 1, "persistent path: e4m3 keys, one query per block");
  // bf16 queries: e4m3 key tiles are widened into tensor memory by converter
  // warps.  FP8 indexer (QFP8): the e4m3 key tiles go from the TMA ring
  // straight into kind::f8f6f4 MMAs; no converter warps.
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  int* upre = reinterpret_cast<int*>(smem + C::OFF_UPRE);      // upre[b] = first unit of sequence b
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  grid_launch_dependents();   // the top-k may be scheduled as SMs free up (it waits for this grid)
  if (device_error_pending()) return;

  // ---------------------------------------------------------------- unit list
  for (int b = threadIdx.x; b < p.B; b += C::NT) {
    const int cq0 = p.cu_q[b], cq1 = p.cu_q[b + 1];
    const int64_t lo = cq0 > p.q_begin ? cq0 : p.q_begin;
    const int64_t hi = cq1 < p.q_end ? cq1 : p.q_end;
    int cnt = 0;
    if (lo < hi) {
      const int kv = p.cu_k[b + 1] - p.cu_k[b];
      const int pos = kv - (cq1 - cq0) + static_cast<int>(lo - cq0);
      cnt = pos / C::BK + 1;
    }
    upre[b + 1] = cnt;
  }
  DSA_PROF_BEGIN();
  __syncthreads();
  if (threadIdx.x == 0) {
    upre[0] = 0;
    for (int b = 0; b < p.B; ++b) upre[b + 1] += upre[b];
  }
  __syncthreads();
  const int64_t U = upre[p.B];
  const int u0 = static_cast<int>(U * blockIdx.x / gridDim.x);
  const int u1 = static_cast<int>(U * (blockIdx.x + 1) / gridDim.x);
  if (u0 >= u1) return;
  const int n_iter = u1 - u0;
  int b_first = 0;
  {
    int lo = 0, hi = p.B - 1;     // largest b with upre[b] <= u0
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (upre[mid] <= u0) lo = mid; else hi = mid - 1;
    }
    b_first = lo;
  }
  // per-sequence facts of unit u (walks b forward as u increases)
  struct Seq {
    int b, q0, pos, k_base, kv_len;
  };
  auto seq_of = [&](int b) {
    Seq q;
    q.b = b;
    const int cq0 = p.cu_q[b], cq1 = p.cu_q[b + 1];
    q.q0 = static_cast<int>(cq0 > p.q_begin ? cq0 : p.q_begin);
    q.k_base = p.cu_k[b];
    q.kv_len = p.cu_k[b + 1] - q.k_base;
    q.pos = q.kv_len - (cq1 - cq0) + (q.q0 - cq0);
    return q;
  };

  // ---------------------------------------------------------------- shared memory
  const uint32_t sbase = smem_u32(smem);
  const uint32_t s_q = sbase + C::OFF_Q;
  const uint32_t s_raw = sbase + C::OFF_RAW;
  const uint32_t s_k = sbase + C::OFF_K;
  const uint32_t bar0 = sbase + C::OFF_BAR;
  const uint32_t bar_drain = bar0;
  // query tile of segment g (the g-th sequence of this CTA) in buffer g & 1:
  // q_full(buf) from the TMA, q_empty(t, buf) from MMA thread t, once per
  // segment, after its last MMA that reads the tile
  auto bar_q_full = [&](int buf) { return bar0 + 8 + 8 * buf; };
  auto bar_q_empty = [&](int t, int buf) { return bar0 + 24 + 8 * (2 * t + buf); };
  // ready(s): tile it (s = it % STAGES) is widened in TMEM and its accumulator
  // (the same index) has been drained: 128 converter + 128 epilogue arrivals
  auto bar_ready = [&](int s) { return bar0 + 56 + 8 * s; };
  auto bar_raw_full = [&](int s) { return bar0 + 56 + 8 * (C::STAGES + s); };
  auto bar_raw_empty = [&](int s) { return bar0 + 56 + 8 * (C::STAGES + C::RSTAGES + s); };
  auto bar_acc_full = [&](int a) { return bar0 + 56 + 8 * (C::STAGES + 2 * C::RSTAGES + a); };
  // FP8 indexer: key ring full / empty, accumulator drained by the epilogue
  auto bar_k_full = [&](int s) { return bar0 + 56 + 8 * (C::STAGES + 2 * C::RSTAGES + C::NACC + s); };
  auto bar_k_empty = [&](int s) { return bar0 + 56 + 8 * (2 * C::STAGES + 2 * C::RSTAGES + C::NACC + s); };
  auto bar_acc_empty = [&](int a) { return bar0 + 56 + 8 * (3 * C::STAGES + 2 * C::RSTAGES + C::NACC + a); };
  // f16 queries: q_conv(buf) once the converter team of the segment's first
  // tile has rewritten the query tile as f16 (128 arrivals)
  auto bar_q_conv = [&](int buf) { return bar0 + 56 + 8 * (3 * C::STAGES + 2 * C::RSTAGES + 2 * C::NACC + buf); };
  // q_max(team): the team's four partial maxima of a query tile are stored
  // (128 arrivals; one phase per query tile the team rewrites)
  auto bar_q_max = [&](int team) {
    return bar0 + 56 + 8 * (3 * C::STAGES + 2 * C::RSTAGES + 2 * C::NACC + 2 + team);
  };
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  float* qfac_buf = reinterpret_cast<float*>(smem + C::OFF_QCONV);        // [2]: 2^-sq of each query buffer
  float* qfac_acc = qfac_buf + 2;                                         // [NACC]: 2^-sq of each accumulator
  uint32_t* qmax_part = reinterpret_cast<uint32_t*>(qfac_acc + C::NACC);  // [team][parity][warp]

  if (threadIdx.x == 0) {
    mbar_init(bar_drain, C::MMA_THREADS);
    for (int buf = 0; buf < 2; ++buf) {
      mbar_init(bar_q_full(buf), 1);
      for (int t = 0; t < C::MMA_THREADS; ++t) mbar_init(bar_q_empty(t, buf), 1);
    }
    if constexpr (C::CONVERT) {
      for (int s = 0; s < C::STAGES; ++s) mbar_init(bar_ready(s), 256);
      for (int s = 0; s < C::RSTAGES; ++s) {
        mbar_init(bar_raw_full(s), 1);
        mbar_init(bar_raw_empty(s), 128);
      }
      for (int buf = 0; buf < 2; ++buf) mbar_init(bar_q_conv(buf), 128);
      for (int team = 0; team < C::CONV_TEAMS; ++team) mbar_init(bar_q_max(team), 128);
    } else {
      for (int s = 0; s < C::STAGES; ++s) {
        mbar_init(bar_k_full(s), 1);
        mbar_init(bar_k_empty(s), 1);
      }
      for (int a = 0; a < C::NACC; ++a) mbar_init(bar_acc_empty(a), 128);
    }
    // f16 queries: the MMA thread's arrival (after it stored the descale of
    // the accumulator) joins the commit's
    for (int a = 0; a < C::NACC; ++a) mbar_init(bar_acc_full(a), C::QF16 ? 2 : 1);
    *abort_flag = 0;
    fence_mbar_init();
    // every accumulator starts drained: the epilogue's share of the first phase
    if constexpr (C::CONVERT)
      for (int s = 0; s < C::STAGES; ++s) mbar_arrive_count(bar_ready(s), 128);
  }
  if (warp == C::MMA_WARP) {
    tmem_alloc(smem_u32(tmem_holder), C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == C::PRODUCER_WARP && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  // Launched as a dependent of the previous kernel in the stream (the previous
  // step's attention): the set-up above overlaps its end; the scores and part
  // maxima this kernel writes may still be read by that step's kernels until
  // it completes, so wait for it here.
  grid_dependency_wait();
  const long long t_role = clock64();

  if (warp == C::PRODUCER_WARP) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int b = b_first, seg = -1, loaded_q = 0, it = 0;
      // the key cache is streamed once per call: first out of L2, so that the
      // scores and part maxima the top-k reads next stay there (decode128k
      // step 0.2552 -> 0.2523 ms; marking those stores evict_last as well
      // measured no better)
      const uint64_t stream_policy = l2_policy_evict_first();
      Seq q{};
      for (; it < n_iter; ++it) {
        const int u = u0 + it;
        while (u >= upre[b + 1]) ++b;
        if (b != q.b || seg < 0) {
          ++seg;
          const int buf = seg & 1;
          if (seg >= 2) {   // both MMA threads are done with segment seg - 2
            bool free_ = true;
            for (int t = 0; t < C::MMA_THREADS && free_; ++t)
              free_ = mbar_wait(bar_q_empty(t, buf), ((seg - 2) >> 1) & 1, abort_flag, 50);
            if (!free_) break;
          }
          q = seq_of(b);
          mbar_arrive_expect_tx(bar_q_full(buf), C::B_TILE);
          for (int at = 0; at < C::NATOM; ++at)
            tma_load_2d(s_q + buf * C::B_TILE + at * C::N * C::SWB, &tm_q, bar_q_full(buf), at * C::ATOM_ELEMS,
                        q.q0 * C::H_I);
          loaded_q = seg + 1;
        }
        const int tile = u - upre[b];
        // the raw ring (widened by the converters) or the key ring (FP8 MMA operand)
        constexpr int ring = C::CONVERT ? C::RSTAGES : C::STAGES;
        const int r = it % ring;
        const uint32_t full = C::CONVERT ? bar_raw_full(r) : bar_k_full(r);
        const uint32_t empty = C::CONVERT ? bar_raw_empty(r) : bar_k_empty(r);
        const uint32_t dst = C::CONVERT ? s_raw + r * C::RAW_TILE : s_k + r * C::A_TILE;
        if (!mbar_wait(empty, ((it / ring) & 1) ^ 1, abort_flag, 51)) break;
        mbar_arrive_expect_tx(full, C::RAW_TILE);
        if (!p.pages.paged()) {
          tma_load_2d_hint(dst, &tm_k, full, 0, q.k_base + tile * C::BK, stream_policy);
        } else {
          for (int h = 0; h < C::BK / 64; ++h) {   // 64-row boxes, each inside one page
            int y = p.pages.row(q.b, q.k_base, tile * C::BK + 64 * h);
            if (y >= 0 && tile * C::BK + 64 * h < q.kv_len && !in_bounds(y < p.cache_rows, 82)) y = -1;
            tma_load_2d_hint(dst + h * 64 * C::RAW_ROWB, &tm_k, full, 0, y >= 0 ? y : -64, stream_policy);
          }
        }
      }
      if (*abort_flag) {
        long long t0 = clock64();
        constexpr int ring = C::CONVERT ? C::RSTAGES : C::STAGES;
        for (int j = (it > ring ? it - ring : 0); j < it; ++j)
          while (!mbar_try_wait(C::CONVERT ? bar_raw_full(j % ring) : bar_k_full(j % ring), (j / ring) & 1) &&
                 clock64() - t0 < kWaitLimitCycles) {
          }
        for (int g = (loaded_q > 2 ? loaded_q - 2 : 0); g < loaded_q; ++g)
          while (!mbar_try_wait(bar_q_full(g & 1), (g >> 1) & 1) && clock64() - t0 < kWaitLimitCycles) {
          }
      }
    }
    if (lane == 0) DSA_PROF_SPAN(61, t_role);
  } else if (warp >= C::MMA_WARP && warp < C::CONVERT_WARP0) {
    // ------------------------------------------------------------ MMA issuers
    // Thread t (lane 0 of warp MMA_WARP + t) issues tiles it = t, t + 2, ...
    // It walks the CTA's segments in order and, for every segment, waits for
    // its query tile and commits q_empty(t, .) once, also for a segment in
    // which it has no tile, so that the producer can count on both threads.
    const int mt = warp - C::MMA_WARP;
    const uint64_t b_desc0 = smem_desc(s_q, 16, 8 * C::SWB, C::SWZ);
    if (lane == 0) {
      int b = b_first, seg = 0, seq_end = upre[b_first + 1];
      bool have_q = false, ok = true;
      uint64_t b_desc = b_desc0;
      auto next_segment = [&]() {
        ++seg;
        do {
          ++b;
        } while (upre[b + 1] == upre[b]);   // sequences without units in the call
        seq_end = upre[b + 1];
      };
      // the query tile as the MMAs read it: loaded, and (f16 queries) rewritten
      auto q_ready = [&](int sg) { return C::QF16 ? bar_q_conv(sg & 1) : bar_q_full(sg & 1); };
      float qfac = 1.f;
      auto release_segment = [&]() -> bool {   // done with segment seg
        if (!have_q && !mbar_wait(q_ready(seg), (seg >> 1) & 1, abort_flag, 52)) return false;
        umma_commit(bar_q_empty(mt, seg & 1));
        have_q = false;
        return true;
      };
      for (int it = mt; it < n_iter; it += C::MMA_THREADS) {
        const int u = u0 + it;
        while (ok && u >= seq_end) {
          ok = release_segment();
          next_segment();
        }
        if (!ok) break;
        if (!have_q) {
          if (!mbar_wait(q_ready(seg), (seg >> 1) & 1, abort_flag, 52)) { ok = false; break; }
          have_q = true;
          b_desc = b_desc0 + static_cast<uint64_t>(((seg & 1) * C::B_TILE) >> 4);
          if constexpr (C::QF16) qfac = qfac_buf[seg & 1];
        }
        if constexpr (C::CONVERT) {
          const int s = it % C::STAGES;
          const int a = s;
          if (!mbar_wait(bar_ready(s), (it / C::STAGES) & 1, abort_flag, 53)) { ok = false; break; }
          tc_fence_after();
          // A: the key tile in tensor memory, 8 columns (16 bf16) per k-step.
          // B: the query descriptor's start-address field (16-byte units, low
          // bits) advances by the k-step offset; it never carries.
          const uint32_t a_tile = tmem + C::ACC_COLS + s * C::A_COLS;
#pragma unroll
          for (int kk = 0; kk < C::KSTEPS; ++kk) {
            const int atom = (kk * 32) / C::SWB;
            const int off = (kk * 32) % C::SWB;
            const uint64_t bd = b_desc + static_cast<uint64_t>((atom * C::N * C::SWB + off) >> 4);
            umma_ts(tmem + a * C::N, a_tile + kk * 8, bd, C::IDESC, kk > 0 ? 1u : 0u);
          }
          umma_commit(bar_acc_full(a));   // also frees key stage s (== a)
          // the epilogue of tile it reads this after acc_full(a); it was last
          // read by the epilogue of tile it - NACC, before its ready(a) arrival
          qfac_acc[a] = qfac;
          mbar_arrive(bar_acc_full(a));
        } else {
          // FP8 indexer: A = the e4m3 key tile as loaded (128 rows of 128
          // bytes, 128-byte swizzle), B = the e4m3 query tile; 32 bytes of K
          // per MMA, the start addresses advance inside the swizzle atom.
          const int s = it % C::STAGES;
          const int a = it % C::NACC;
          if (!mbar_wait(bar_k_full(s), (it / C::STAGES) & 1, abort_flag, 53)) { ok = false; break; }
          if (!mbar_wait(bar_acc_empty(a), ((it / C::NACC) & 1) ^ 1, abort_flag, 54)) { ok = false; break; }
          tc_fence_after();
          const uint64_t a_desc = smem_desc(s_k + s * C::A_TILE, 16, 8 * C::SWB, C::SWZ);
#pragma unroll
          for (int kk = 0; kk < C::KSTEPS; ++kk)
            umma_ss_e4m3(tmem + a * C::N, a_desc + static_cast<uint64_t>((kk * 32) >> 4),
                         b_desc + static_cast<uint64_t>((kk * 32) >> 4), C::IDESC, kk > 0 ? 1u : 0u);
          umma_commit(bar_k_empty(s));
          umma_commit(bar_acc_full(a));
        }
      }
      // release the current segment and every later one of the CTA
      while (ok && !*abort_flag) {
        ok = release_segment();
        if (seq_end >= u1) break;
        next_segment();
      }
      DSA_PROF_SPAN(62, t_role);
      umma_commit(bar_drain);
      long long t0 = clock64();
      while (!mbar_try_wait(bar_drain, 0) && clock64() - t0 < kWaitLimitCycles) {
      }
    }
  } else if (warp >= C::CONVERT_WARP0) {
    // ------------------------------------------------------------ e4m3 -> bf16
    // (bf16 queries only: the FP8 schedule has no converter warps)
    if constexpr (C::CONVERT) {
    // Each thread widens one key row into its own TMEM lane: a warp reaches
    // lanes 32 (warp % 4) .. +31, so the row is fixed by the warp's position.
    const int team = (warp - C::CONVERT_WARP0) / 4;
    const int row = (warp & 3) * 32 + lane;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16) + C::ACC_COLS;
    // The query tile of segment sg (buffer sg & 1), bf16 as loaded, rewritten
    // in place as f16 x 2^sq (same 16-bit element positions, so the swizzled
    // layout holds).  sq = 14 - E for the largest magnitude 2^E (1 + f): that
    // value becomes < 2^15, every element of magnitude >= 2^(E-31) stays
    // exact (f16 keeps 11 significant bits down to 2^-14 and whole multiples
    // of 2^-24 below), and smaller ones move by at most 2^(E-39).  A zero or
    // non-finite maximum keeps sq = 0; sq <= 126 keeps 2^-sq a normal float.
    int n_widened = 0;   // query tiles this team has rewritten
    auto widen_query = [&](int sg) -> bool {
      const int buf = sg & 1;
      if (!mbar_wait(bar_q_full(buf), (sg >> 1) & 1, abort_flag, 58)) return false;
      uint4* qv = reinterpret_cast<uint4*>(smem + C::OFF_Q + buf * C::B_TILE);
      constexpr int PER = C::B_TILE / 16 / 128;
      const int tt = row;   // 0..127 across the team
      uint32_t m2 = 0;      // the largest magnitude (bf16 bit patterns order as magnitudes)
#pragma unroll
      for (int i = 0; i < PER; ++i) {
        const uint4 x = qv[tt + 128 * i];
        m2 = __vmaxu2(m2, __vmaxu2(__vmaxu2(x.x & 0x7FFF7FFFu, x.y & 0x7FFF7FFFu),
                                   __vmaxu2(x.z & 0x7FFF7FFFu, x.w & 0x7FFF7FFFu)));
      }
      uint32_t m = __reduce_max_sync(0xFFFFFFFFu, max(m2 & 0xFFFFu, m2 >> 16));
      // the team's four warps meet: slot n_widened & 1 is rewritten only after
      // every warp has passed this phase of q_max and read it
      const int par = n_widened & 1;
      ++n_widened;
      uint32_t* part = qmax_part + (team * 2 + par) * 4;
      if (lane == 0) part[warp & 3] = m;
      mbar_arrive_warp(bar_q_max(team));
      if (!mbar_wait_warp(bar_q_max(team), par, abort_flag, 59)) return false;
      m = max(max(part[0], part[1]), max(part[2], part[3]));
      const int ef = static_cast<int>(m >> 7);   // biased exponent of the maximum
      int sq = 0;
      if (m != 0 && ef < 255) sq = min(141 - ef, 126);
      const float up = __int_as_float((127 + sq) << 23);
#pragma unroll
      for (int i = 0; i < PER; ++i) {   // read again: the same thread's own 16-byte pieces
        const uint4 x = qv[tt + 128 * i];
        uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float lo = __uint_as_float(w[e] << 16) * up;
          const float hi = __uint_as_float(w[e] & 0xFFFF0000u) * up;
          asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(w[e]) : "f"(hi), "f"(lo));
        }
        qv[tt + 128 * i] = make_uint4(w[0], w[1], w[2], w[3]);
      }
      fence_proxy_async_smem();   // the MMAs read the tile through the async proxy
      if (tt == 0) qfac_buf[buf] = __int_as_float((127 - sq) << 23);
      mbar_arrive(bar_q_conv(buf));
      return true;
    };
    int b = b_first, seg = 0;
    for (int it = team; it < n_iter; it += C::CONV_TEAMS) {
      const int r = it % C::RSTAGES;
      const int s = it % C::STAGES;
      const int u = u0 + it;
      while (u >= upre[b + 1]) {
        ++b;
        if (upre[b + 1] > upre[b]) ++seg;   // sequences with units in the call
      }
      if (u == max(upre[b], u0) && !widen_query(seg)) break;   // the segment's first tile
      if (!mbar_wait(bar_raw_full(r), (it / C::RSTAGES) & 1, abort_flag, 55)) break;
      const uint8_t* raw_row = smem + C::OFF_RAW + r * C::RAW_TILE + row * 128;
      uint4 chunk[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)  // 128-byte swizzle: logical chunk j sits at j ^ (row & 7)
        chunk[j] = *reinterpret_cast<const uint4*>(raw_row + ((j ^ (row & 7)) << 4));
      mbar_arrive(bar_raw_empty(r));
      // stage s is free once the MMAs of tile it - STAGES completed: the phase
      // before the one the epilogue of tile it waits for on the same barrier
      // (warp-uniform outcome: the tensor-memory stores below are warp-collective)
      if (!mbar_wait_warp(bar_acc_full(s), ((it / C::STAGES) & 1) ^ 1, abort_flag, 56)) break;
      tc_fence_after();
#pragma unroll
      for (int h = 0; h < 2; ++h) {   // 64 elements (32 columns) per store
        uint32_t cols[32];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint4 c = chunk[4 * h + j];
          e4m3x4_to_f16x4(c.x, cols[8 * j + 0], cols[8 * j + 1]);
          e4m3x4_to_f16x4(c.y, cols[8 * j + 2], cols[8 * j + 3]);
          e4m3x4_to_f16x4(c.z, cols[8 * j + 4], cols[8 * j + 5]);
          e4m3x4_to_f16x4(c.w, cols[8 * j + 6], cols[8 * j + 7]);
        }
        tmem_st32(t_lane + s * C::A_COLS + 32 * h, cols);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar_ready(s));
    }
    }
    if (lane == 0) DSA_PROF_SPAN(63, t_role);
  } else {
    // ------------------------------------------------------------ epilogue
    // Warpgroup g drains tiles it = g, g + EPI_WG, ... (accumulator it % NACC);
    // the key scales of its next tile are loaded one iteration ahead.
    const int g = warp >> 2;
    const int sub = warp & 3;
    const int key_in_tile = sub * 32 + lane;
    int b = b_first, cur = -1, bp = b_first;
    Seq q{};
    float* wsm = reinterpret_cast<float*>(smem + C::OFF_WEPI) + warp * C::H_I;   // this warp's copy
    auto fetch_scale = [&](int itx) -> float {
      if (itx >= n_iter) return 0.f;
      const int u = u0 + itx;
      while (u >= upre[bp + 1]) ++bp;
      const int kb = p.cu_k[bp];
      const int s_key = (u - upre[bp]) * C::BK + key_in_tile;
      if (s_key >= p.cu_k[bp + 1] - kb) return 0.f;
      const int r = p.pages.row(bp, kb, s_key);
      return (r >= 0 && in_bounds(r < p.cache_rows, 86)) ? p.k_scale[r] : 0.f;
    };
    float ks = fetch_scale(g);
    for (int it = g; it < n_iter; it += C::EPI_WG) {
      const float ks_next = fetch_scale(it + C::EPI_WG);
      const int a = it % C::NACC;
      const int u = u0 + it;
      while (u >= upre[b + 1]) ++b;
      if (b != cur) {
        cur = b;
        q = seq_of(b);
        __syncwarp();
        const float4* w4 = reinterpret_cast<const float4*>(p.w + static_cast<int64_t>(q.q0) * C::H_I);
        if (lane < C::H_I / 4) {
          float4 wv = w4[lane];
          if constexpr (C::QFP8) {   // fold in each query head's scale and the 2^-7 of the rotation
            const float* qs = p.q_scale + static_cast<int64_t>(q.q0) * C::H_I + 4 * lane;
            wv.x *= ldexpf(qs[0], -FP8_HADAMARD_LOG2);
            wv.y *= ldexpf(qs[1], -FP8_HADAMARD_LOG2);
            wv.z *= ldexpf(qs[2], -FP8_HADAMARD_LOG2);
            wv.w *= ldexpf(qs[3], -FP8_HADAMARD_LOG2);
          }
          reinterpret_cast<float4*>(wsm)[lane] = wv;
        }
        __syncwarp();
      }
      if (!mbar_wait_warp(bar_acc_full(a), (it / C::NACC) & 1, abort_flag, 57)) break;
      tc_fence_after();
      const float qfac = C::QF16 ? qfac_acc[a] : 1.f;
      const uint32_t t_row = tmem + (static_cast<uint32_t>(sub * 32) << 16) + a * C::N;
      float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
      for (int half = 0; half < C::H_I / 32; ++half) {
        uint32_t v[32];
        tmem_ld32(t_row + 32 * half, v);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
          const float4 wv = reinterpret_cast<const float4*>(wsm)[(32 * half + j) / 4];
          acc0 = fmaf(wv.x, fmaxf(__uint_as_float(v[j]), 0.f), acc0);
          acc1 = fmaf(wv.y, fmaxf(__uint_as_float(v[j + 1]), 0.f), acc1);
          acc0 = fmaf(wv.z, fmaxf(__uint_as_float(v[j + 2]), 0.f), acc0);
          acc1 = fmaf(wv.w, fmaxf(__uint_as_float(v[j + 3]), 0.f), acc1);
        }
      }
      tc_fence_before();
      // per-thread arrivals: measured faster here than one warp-aggregated arrive
      if constexpr (C::CONVERT) mbar_arrive(bar_ready(a));   // accumulator a is free for tile it + NACC
      else mbar_arrive_warp(bar_acc_empty(a));
      const int s_key = (u - upre[b]) * C::BK + key_in_tile;
      // keys past the query's position (and past the cache) score -inf
      const float val = s_key <= q.pos ? (acc0 + acc1) * qfac * ks : -INFINITY;
      const int64_t row = static_cast<int64_t>(q.q0) - p.q_begin;
      if (s_key < q.kv_len && in_bounds(s_key < p.ld, 84)) p.scores[row * p.ld + s_key] = val;
      if (p.part_max != nullptr) {
        const float m = part_max8(val);
        if ((lane & (PART - 1)) == 0 && s_key < q.kv_len) p.part_max[row * p.ld_pm + s_key / PART] = m;
      }
      ks = ks_next;
    }
    if (lane == 0) DSA_PROF_SPAN(60, t_role);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
  DSA_PROF_END();
}

}  // namespace dsa
