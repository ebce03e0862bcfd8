// sparse_mla.cuh -- MLA attention in absorbed MQA form over the selected rows.
//
// "DeepSeek-V3.2" (transformers model doc), "DeepSeek Sparse Attention
// (DSA)", item 2: main MLA attention runs only over the top-k tokens of each
// query.  "DeepSeek-V3.2 - Experimental Exp Version" (altools), "Technical
// Principles": MLA with MQA, so one cached entry per token serves every query
// head; the entry is the compressed latent (512) plus the RoPE key (64)
// (released config: kv_lora_rank 512, qk_rope_head_dim 64, 128 heads).
//
// Per query t: S = q[t] (128 heads x 576) . C_sel^T (576 x k),
// out = softmax(scale * S) . C_sel[:, :512], lse = log-sum-exp per head.
//
// sm_100a mapping.  The 128 heads are the MMA M dimension and the selected
// rows stream through in tiles of BN = 32, gathered straight from the latent
// cache by TMA tile::gather4 (four arbitrary rows per instruction) into
// swizzled K-major atoms (128-byte atoms for the released shape; narrower atoms
// for narrow test shapes, so that every TMA box lies inside the row).  The fp32
// output accumulator O[128 x 512] alone fills all 512 columns of an SM's
// tensor memory, so the released shape runs on a cluster of two CTAs (two
// SMs): CTA r owns output columns [256 r, 256 r + 256).  QK is split along K
// in halves -- CTA 0 multiplies columns [0, 288), CTA 1 columns [288, 576),
// 18 k-steps each, since a CTA's tile time is its QK issue -- so each CTA
// gathers 320 columns of every selected row (CTA 0 [0, 320), CTA 1
// [256, 576): its values and its QK half, one 64-column atom shared) and no
// MMA is duplicated.  Random-row gathers are bound by
// the rate at which an SM can have rows requested and in flight, so eight
// warps issue them (warp w the four rows 4w .. 4w+3 of a tile, one gather4
// per atom) into a six-deep ring.  The two partial score tiles are
// exchanged through distributed shared memory (each CTA stages its part in its
// own shared memory and bulk copies, one per softmax warp, move it into the
// peer's buffer, completing on the peer's mbarrier); both CTAs add them in the same
// commutative way, so both hold bit-identical scores and take the same
// softmax decisions.  Tensor memory holds O, three score buffers (a tile's P,
// in bf16, overwrites its scores once they are in registers) and this CTA's
// slice of the query, the A operand of every QK MMA, so shared memory is left
// to the ring of gathered rows and the score exchange.  The online
// softmax keeps a per-head running max and only rescales O (in TMEM) when the
// max grows by more than 2^8, which is exact arithmetic with the same final
// normalisation.
//
// Roles per CTA: warps 0-7 query load, softmax and epilogue (two teams of
// four warps taking alternate tiles, a head row and all of a tile's columns
// per thread), warps 8 and 9 MMA issuers (QK and PV; warp 8 owns the TMEM),
// warps 10.. gather (eight with two CTAs, one with one CTA).  The query slice
// is loaded while the other warps scan the selection; the kernel may start
// while the top-k before it finishes (a programmatic dependent launch), and
// only the warps that read the selection wait for it.
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace dsa {

template <int H_, int DQK_, int DV_, int SPLIT_, int SWB_>
struct MlaCfg {
  static constexpr int H = H_, DQK = DQK_, DV = DV_, SPLIT = SPLIT_;
  static constexpr int SWB = SWB_;                        // swizzle-atom row bytes (128, 64 or 32)
  static constexpr uint32_t SWZ = SWB == 128 ? 2u : (SWB == 64 ? 4u : 6u);
  static constexpr int BN = 32;                           // selected rows per tile
  static constexpr int ATOM = SWB / 2;                    // bf16 columns per swizzle atom
  static constexpr int KPA = SWB / 32;                    // 16-wide k-steps per atom
  static constexpr int NATOM_ALL = DQK / ATOM;
  static constexpr int DVS = DV / SPLIT;                  // output columns per CTA
  static constexpr int NV = DVS / ATOM;                   // value atoms per CTA
  // QK reduction: CTA r multiplies query / latent elements [r QKH, r QKH + QKH)
  static constexpr int QKH = DQK / SPLIT;
  static constexpr int KSTEPS = QKH / 16;                 // QK k-steps per tile and CTA
  // atoms gathered: rank 0 from atom 0, rank 1 from atom A0_R1 (its first
  // value column), each through the last atom its values or QK elements reach
  static constexpr int A0_R1 = SPLIT == 1 ? 0 : DVS / ATOM;
  static constexpr int cdiv(int a, int b) { return (a + b - 1) / b; }
  static constexpr int NA0 = SPLIT == 1 ? NATOM_ALL : (NV > cdiv(QKH, ATOM) ? NV : cdiv(QKH, ATOM));
  static constexpr int NA1 = SPLIT == 1 ? 0 : NATOM_ALL - A0_R1;
  static constexpr int NA_MAX = NA0 > NA1 ? NA0 : NA1;
  static constexpr int KF1 = SPLIT == 1 ? 0 : (QKH - A0_R1 * ATOM) / 16;   // rank 1's first local k-step
  static constexpr int NS = SPLIT == 1 ? 4 : 6;           // gather ring depth
  static constexpr int C_ATOM_BYTES = BN * SWB;
  static constexpr int C_STAGE = NA_MAX * C_ATOM_BYTES;
  static constexpr int X_BYTES = SPLIT == 2 ? 128 * BN * 4 : 0;   // one partial-score tile
  static constexpr int OFF_C = 0;
  // Received partial-score tiles: tile j lands in buffer j % XR.  With four
  // buffers a CTA never has to be told that the peer is done with one: the
  // peer sent tile j - 2 (which this CTA waited for before it sends tile j)
  // only after it had consumed tile j - 4, the buffer's previous content.
  static constexpr int XR = 4;
  static constexpr int OFF_X = OFF_C + NS * C_STAGE;
  static constexpr int XS = 2;                             // outgoing tiles staged (one per softmax team)
  static constexpr int OFF_XS = OFF_X + XR * X_BYTES;
  // softmax warps: two teams of four (one warp per TMEM lane quarter) taking
  // alternate tiles, each thread one head row and all of a tile's columns;
  // the teams pass the softmax reference max along through shared memory and
  // add their row sums at the end
  static constexpr int NSM = 8;
  static constexpr int OFF_MX = OFF_XS + XS * X_BYTES;     // [2 teams][128] published, [2 teams][128] final
  static constexpr int OFF_LS = OFF_MX + 2 * 2 * 128 * 4;  // [2 teams][128] fp32
  static constexpr int OFF_MASK = OFF_LS + 2 * 128 * 4;
  static constexpr int OFF_BAR = (OFF_MASK + NS * 4 + 7) / 8 * 8;
  static constexpr int NSB = 3;                            // S buffers (each later holds its P)
  // q_ready, c_full/c_empty per stage, 3 per S buffer, x_full per receive
  // buffer, drain, m_pub per team, and per lane quarter the row-sum exchange
  static constexpr int NBAR = 1 + 2 * NS + 3 * NSB + XR + 1 + 2 + 4;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  // tensor memory columns: O [0, DVS); S[NSB] (fp32, BN each; P of the same
  // tile, bf16 pairs, overwrites the first BN/2 columns once S is read); the
  // query slice this CTA multiplies, bf16 pairs (the A operand of QK)
  static constexpr int TMEM_S = DVS;
  static constexpr int TMEM_Q = DVS + NSB * BN;
  static constexpr int QCOLS = QKH / 2;
  static constexpr int TMEM_USED = TMEM_Q + QCOLS;
  static constexpr int TMEM_COLS = TMEM_USED <= 128 ? 128 : (TMEM_USED <= 256 ? 256 : 512);
  // roles: warps 0 .. NSM-1 softmax and epilogue, MMA_WARP the QK issuer (and
  // TMEM owner), MMA_WARP + 1 the PV issuer, then NPROD gather warps: more
  // warps issuing TMA gathers raise the rate at which one SM requests rows
  static constexpr int MMA_WARP = NSM;
  static constexpr int NPROD = SPLIT == 2 ? BN / 4 : 1;   // one per four-row group of a tile
  static constexpr int PROD_WARP0 = NSM + 2;
  static constexpr int NT = (PROD_WARP0 + NPROD) * 32;
  static constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, BN, false, false);
  static constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, DVS, false, true);
  static constexpr float kRescaleThreshold = 8.0f;        // log2 units
  static_assert(H <= 128, "heads = MMA M rows");
  static_assert(DQK % ATOM == 0, "every TMA box stays inside the row: no partial atoms");
  static_assert(DVS % ATOM == 0 && DVS <= 256 && DVS % 16 == 0, "PV N");
  static_assert(SPLIT == 1 || NV <= NA1, "rank 1 must gather its value columns");
  static_assert(QKH % 16 == 0 && (SPLIT == 1 || (A0_R1 * ATOM <= QKH && 2 * DVS <= DQK)),
                "QK halves in whole k-steps, rank 1's half inside its atoms");
  static_assert(SPLIT == 1 || (QKH * 2) % 16 == 0, "16-byte query loads from the half's first element");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
  static_assert(NSB <= NS, "the rows of every score tile in flight stay resident");
  static_assert(QCOLS % 8 == 0, "query columns are stored eight at a time");
  static_assert(TMEM_USED <= 512, "tensor memory");
  static_assert(OFF_C % 1024 == 0 && C_STAGE % 1024 == 0 && C_ATOM_BYTES % 1024 == 0, "swizzle atoms");
  static_assert(SPLIT == 1 || NA_MAX <= 32, "one lane per atom");
  static_assert(BN == 32 && (DVS / 2) % 16 == 0 && QCOLS % 8 == 0, "softmax rows (32 columns) and column halves");
  static_assert(OFF_XS % 16 == 0 && OFF_MX % 16 == 0, "bulk-copy / vector alignment");
  static_assert(OFF_X % 16 == 0 && OFF_XS % 16 == 0 && OFF_BAR % 8 == 0, "vector / bulk-copy / barrier alignment");
};

struct MlaParams {
  const __nv_bfloat16* q;    // [T, H, DQK]
  const int32_t* idx;        // [q_end - q_begin, topk]
  const int32_t* cu_q;
  const int32_t* cu_k;
  PageMap pages;             // where the latent cache keeps each entry
  int cache_rows;            // rows of the latent cache (checked builds)
  int B;
  int64_t q_begin;
  int topk;
  float scale_log2;          // softmax scale * log2(e)
  const float2* rope;        // null, or [max_pos, (DQK - DV) / 2] (cos, sin): RoPE on q's rope columns
  __nv_bfloat16* out;        // [T, H, DV]
  float* lse;                // [T, H] or null
};

// Cache row of selected entry sel of query row ri, or -1 when the entry is
// skipped: outside 0 .. pos (the -1 padding included), or (paged caches) on
// a missing page, which is also recorded in the device error word.  Skipped
// entries are gathered from row 0 and masked.
__device__ __forceinline__ int gather_row(const PageMap& pages, const RowInfo& ri, int sel, int cache_rows) {
  if (sel < 0 || sel > ri.pos) return -1;
  const int r = pages.row(ri.b, ri.k_base, sel);
  if (r < 0) record_device_error(kErrMissingPage | (23 << 8));
  if (r >= 0 && !in_bounds(r < cache_rows, 80)) return -1;
  return r;
}

template <class C>
__global__ void __launch_bounds__(C::NT, 1)
    sparse_mla_kernel(const __grid_constant__ CUtensorMap tm_lat, const MlaParams p) {
  grid_launch_dependents();   // the next step's indexer may be scheduled as SMs free up (it waits for this grid)
  const uint32_t rank = C::SPLIT == 2 ? cluster_ctarank() : 0u;
  const uint32_t peer = rank ^ 1u;
  const int64_t r_local = blockIdx.x / C::SPLIT;          // chunk-relative query row
  const int64_t t = p.q_begin + r_local;
  const RowInfo ri = locate_row_block(p.cu_q, p.cu_k, p.B, t);
  const int32_t* __restrict__ idx_row = p.idx + r_local * p.topk;
  const int a0 = rank == 0 ? 0 : C::A0_R1;                // first atom of this CTA's columns (global)
  const int na = rank == 0 ? C::NA0 : C::NA1;             // atoms of this CTA's columns
  const int kf = rank == 0 ? 0 : C::KF1;                  // first QK k-step (local to the gathered atoms)
  const int qk_lo = static_cast<int>(rank) * C::QKH;      // first query / latent element of this CTA's QK

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t s_c = sbase + C::OFF_C;
  float* xbuf = reinterpret_cast<float*>(smem + C::OFF_X);
  float* xs = reinterpret_cast<float*>(smem + C::OFF_XS);
  float* mx_s = reinterpret_cast<float*>(smem + C::OFF_MX);
  float* l_s = reinterpret_cast<float*>(smem + C::OFF_LS);
  uint32_t* mask_s = reinterpret_cast<uint32_t*>(smem + C::OFF_MASK);
  const uint32_t bar0 = sbase + C::OFF_BAR;
  const uint32_t bar_q_ready = bar0;                     // query slice stored in TMEM (128 arrivals)
  auto bar_c_full = [&](int s) { return bar0 + 8 * (1 + s); };
  auto bar_c_empty = [&](int s) { return bar0 + 8 * (1 + C::NS + s); };
  constexpr int SB0 = 1 + 2 * C::NS;                     // first S barrier
  auto bar_s_full = [&](int a) { return bar0 + 8 * (SB0 + a); };
  auto bar_pv_done = [&](int a) { return bar0 + 8 * (SB0 + C::NSB + a); };   // PV of the P in S buffer a
  // p_full(a): P of tile j (a = j % NSB) stored; one per S buffer, so the
  // softmax can never complete a phase twice ahead of the MMA thread's wait
  auto bar_p_full = [&](int a) { return bar0 + 8 * (SB0 + 2 * C::NSB + a); };
  constexpr int XB0 = SB0 + 3 * C::NSB;
  auto bar_x_full = [&](int b) { return bar0 + 8 * (XB0 + b); };          // b < XR
  const uint32_t bar_drain = bar0 + 8 * (XB0 + C::XR);
  // m_pub(c): softmax team c published the reference max of its latest tile
  // (128 arrivals, one phase per tile of the team but its last)
  auto bar_m_pub = [&](int team) { return bar0 + 8 * (XB0 + C::XR + 1 + team); };
  // the two softmax warps of lane quarter q (one per team) meet here (64
  // arrivals) with their row sums at the end
  auto bar_pair_l = [&](int q) { return bar0 + 8 * (XB0 + C::XR + 3 + q); };
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  int* ntiles_s = reinterpret_cast<int*>(smem + C::OFF_MISC + 8);
  uint32_t* pending_s = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC + 12);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(bar_q_ready, C::NSM * 32);
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(bar_c_full(s), C::NPROD);   // every gather warp arrives with its bytes
      mbar_init(bar_c_empty(s), 1);
    }
    for (int a = 0; a < C::NSB; ++a) {
      mbar_init(bar_s_full(a), 1);
      mbar_init(bar_pv_done(a), 1);
      mbar_init(bar_p_full(a), C::NSM * 16);   // the four warps of the tile's team
    }
    for (int b = 0; b < C::XR; ++b) mbar_init(bar_x_full(b), 1);   // armed locally; filled by the peer's copy
    mbar_init(bar_drain, 2);   // both MMA threads
    for (int team = 0; team < 2; ++team) mbar_init(bar_m_pub(team), C::NSM * 16);
    for (int q = 0; q < 4; ++q) mbar_init(bar_pair_l(q), 64);
    *abort_flag = 0;
    *ntiles_s = 0;
    // an error recorded earlier by any CTA of this library: skip the work
    *pending_s = device_error_pending() ? 1u : 0u;
    fence_mbar_init();
  }
  if (warp == C::MMA_WARP) {
    tmem_alloc(smem_u32(tmem_holder), C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp >= C::PROD_WARP0 && lane == 0) tma_prefetch_desc(&tm_lat);
  DSA_PROF_BEGIN();
  tc_fence_before();
  __syncthreads();   // barriers initialised, tensor memory allocated
  if (warp < C::NSM) {
    // The softmax warps load the query slice (the A operand of every QK MMA)
    // into tensor memory while the other warps scan the selection and start
    // gathering: it is on every cluster's critical path.  This CTA's barriers
    // are initialised, so its arrival at the cluster barrier goes first; the
    // wait (for the peer's) comes before any access to the peer.
    if (C::SPLIT == 2) cluster_arrive();
    tc_fence_after();
    const uint32_t tmem_q = *tmem_holder;
    const int c = warp >> 2;
    const int h = (warp & 3) * 32 + lane;                // head row = TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    // Query elements [qk_lo, qk_lo + QKH) of head row h into TMEM lane h; rows
    // h >= H hold zeros.  (Loaded whatever the selection holds.)
    {
      const bool row_ok = h < C::H;
      const uint4* qrow = reinterpret_cast<const uint4*>(p.q + (static_cast<int64_t>(t) * C::H + (row_ok ? h : 0)) * C::DQK +
                                                         qk_lo);
#pragma unroll 1
      for (int c0 = 8 * c; c0 < C::QCOLS; c0 += 16) {   // 8 columns = 16 bf16 = two 16-byte loads
        uint4 v0 = make_uint4(0u, 0u, 0u, 0u), v1 = v0;
        if (row_ok) {
          v0 = __ldg(qrow + c0 / 4);
          v1 = __ldg(qrow + c0 / 4 + 1);
        }
        uint32_t w8[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
        const int g0 = qk_lo + 2 * c0;   // first query element of this chunk
        if (p.rope != nullptr && g0 >= C::DV) {
          // RoPE of the rope columns at this row's position: element pair
          // (2i, 2i + 1) of the rope part times (cos, sin) of pair i.
          const float2* cs = p.rope + static_cast<int64_t>(ri.pos) * ((C::DQK - C::DV) / 2) + (g0 - C::DV) / 2;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float re = __uint_as_float(w8[j] << 16), im = __uint_as_float(w8[j] & 0xFFFF0000u);
            const float2 r = __ldg(cs + j);
            const __nv_bfloat162 b2 = __floats2bfloat162_rn(fmaf(re, r.x, -im * r.y), fmaf(re, r.y, im * r.x));
            w8[j] = *reinterpret_cast<const uint32_t*>(&b2);
          }
        }
        tmem_st8(tmem_q + lane_base + C::TMEM_Q + c0, w8);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive_warp(bar_q_ready);
    }
    if (C::SPLIT == 2) cluster_wait(); else __syncthreads();
  } else {
    // The selection comes from the previous kernel (the top-k): when this
    // kernel is launched as its dependent it may start early, so wait for it
    // here (the query slice above is an input of the call, not its output).
    grid_dependency_wait();
    // Tiles up to the last one holding a valid entry (trailing -1 padding is skipped).
    int last = -1;
    for (int e = static_cast<int>(threadIdx.x) - C::NSM * 32; e < p.topk; e += C::NT - C::NSM * 32) {
      const int s = idx_row[e];
      if (s >= 0 && s <= ri.pos) last = e;
    }
    for (int off = 16; off > 0; off >>= 1) last = max(last, __shfl_xor_sync(0xFFFFFFFFu, last, off));
    if (lane == 0 && last >= 0) atomicMax(ntiles_s, last / C::BN + 1);
    tc_fence_before();
    if (C::SPLIT == 2) cluster_sync(); else __syncthreads();   // peer barriers initialised
  }
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  // Both CTAs of a cluster take the same skip decision (own flag OR the peer's),
  // so neither leaves the other waiting at a cluster barrier.
  bool skip = *pending_s != 0u;
  if (C::SPLIT == 2) skip = skip || ld_cluster_u32(mapa_shared(smem_u32(pending_s), peer)) != 0u;
  const int n_tiles = skip ? 0 : *ntiles_s;

  const long long t_role = clock64();
  if (C::SPLIT == 1 && warp >= C::PROD_WARP0) {
    // ------------------------------------------------------------ gather producer (one CTA)
    int it = 0;
    if (n_tiles > 0) {
      for (; it < n_tiles; ++it) {
        const int s = it % C::NS;
        int ok = 1;
        if (lane == 0) ok = mbar_wait(bar_c_empty(s), ((it / C::NS) & 1) ^ 1, abort_flag, 21);
        ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
        if (!ok) break;
        const int e = it * C::BN + lane;
        const int sel = e < p.topk ? idx_row[e] : -1;
        const int grow = gather_row(p.pages, ri, sel, p.cache_rows);
        const bool valid = grow >= 0;
        const uint32_t vmask = __ballot_sync(0xFFFFFFFFu, valid);
        int y[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) y[j] = __shfl_sync(0xFFFFFFFFu, valid ? grow : 0, (4 * lane + j) & 31);
        if (lane == 0) {
          mask_s[s] = vmask;
          mbar_arrive_expect_tx(bar_c_full(s), na * C::C_ATOM_BYTES);
        }
        __syncwarp();
        if (lane < C::BN / 4) {
          const uint32_t dst = s_c + s * C::C_STAGE + lane * 4 * C::SWB;
          for (int a = 0; a < na; ++a)
            tma_gather4(dst + a * C::C_ATOM_BYTES, &tm_lat, bar_c_full(s), (a0 + a) * C::ATOM, y[0],
                        y[1], y[2], y[3]);
        }
      }
      if (lane == 0 && *abort_flag) {
        long long t0 = clock64();
        for (int j = (it > C::NS ? it - C::NS : 0); j < it; ++j)
          while (!mbar_try_wait(bar_c_full(j % C::NS), (j / C::NS) & 1) &&
                 clock64() - t0 < kWaitLimitCycles) {
          }
      }
    }
    if (lane == 0) DSA_PROF_SPAN(61, t_role);
  } else if (C::SPLIT == 2 && warp >= C::PROD_WARP0) {
    // ------------------------------------------------------------ gather warps (2-CTA split)
    // Gather warp w fetches the four rows 4w .. 4w+3 of every tile, lane a
    // the 64-column atom a of this CTA's columns (one gather4 each).
    const int w = warp - C::PROD_WARP0;
    int it = 0;
    if (n_tiles > 0) {
      for (; it < n_tiles; ++it) {
        const int s = it % C::NS;
        int ok = 1;
        if (lane == 0) ok = mbar_wait(bar_c_empty(s), ((it / C::NS) & 1) ^ 1, abort_flag, 21);
        ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
        if (!ok) break;
        const int e = it * C::BN + lane;
        const int sel = e < p.topk ? idx_row[e] : -1;
        const int grow = gather_row(p.pages, ri, sel, p.cache_rows);
        const bool valid = grow >= 0;
        int y[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) y[j] = __shfl_sync(0xFFFFFFFFu, valid ? grow : 0, 4 * w + j);
        if (w == 0) {
          const uint32_t vmask = __ballot_sync(0xFFFFFFFFu, valid);   // validity of the tile's rows
          if (lane == 0) mask_s[s] = vmask;
        }
        if (lane == 0) mbar_arrive_expect_tx(bar_c_full(s), na * 4 * C::SWB);
        __syncwarp();
        if (lane < na)
          tma_gather4(s_c + s * C::C_STAGE + lane * C::C_ATOM_BYTES + w * 4 * C::SWB, &tm_lat, bar_c_full(s),
                      (a0 + lane) * C::ATOM, y[0], y[1], y[2], y[3]);
      }
      if (lane == 0 && *abort_flag) {
        // let this warp's copies in flight land before the CTA leaves
        long long t0 = clock64();
        for (int j = (it > C::NS ? it - C::NS : 0); j < it; ++j)
          while (!mbar_try_wait(bar_c_full(j % C::NS), (j / C::NS) & 1) && clock64() - t0 < kWaitLimitCycles) {
          }
      }
    }
    if (lane == 0 && w == 0) DSA_PROF_SPAN(61, t_role);
  } else if (warp == C::MMA_WARP || warp == C::MMA_WARP + 1) {
    // ------------------------------------------------------------ MMA issuers
    // Lane 0 of MMA_WARP issues every QK, lane 0 of MMA_WARP + 1 every PV, so
    // that a PV goes out as soon as its P is stored instead of waiting behind
    // the (much longer) issue of a QK.  Each thread's commits track its own
    // MMAs.  QK(j) waits for the gathered rows of tile j and for PV(j - NSB),
    // the last reader of S buffer j % NSB; PV(j) waits for P(j), which the
    // softmax stores only after QK(j) completed, so its commit of c_empty also
    // covers QK(j)'s reads of the stage.
    const bool qk_thread = warp == C::MMA_WARP;
    if (lane == 0 && n_tiles > 0) {
      bool ok = true;
      if (qk_thread) {
        ok = mbar_wait(bar_q_ready, 0, abort_flag, 23);
        tc_fence_after();
        for (int j = 0; ok && j < n_tiles; ++j) {
          const int s = j % C::NS;
          const int sb = j % C::NSB;
          if (!mbar_wait(bar_c_full(s), (j / C::NS) & 1, abort_flag, 24)) break;
          // S buffer sb last held P(j - NSB): its PV must have read it
          if (!mbar_wait(bar_pv_done(sb), ((j / C::NSB) & 1) ^ 1, abort_flag, 25)) break;
          tc_fence_after();
          const uint32_t c_base = s_c + s * C::C_STAGE;
          for (int ks = 0; ks < C::KSTEPS; ++ks) {
            // A = the query slice in tensor memory (8 columns per 16-wide k-step);
            // B = k-step kf + ks of the gathered atoms
            const int kk = kf + ks;
            const int atom = kk / C::KPA;
            const int off = (kk % C::KPA) * 32;
            const uint64_t bd = smem_desc(c_base + atom * C::C_ATOM_BYTES + off, 16, 8 * C::SWB, C::SWZ);
            umma_ts(tmem + C::TMEM_S + sb * C::BN, tmem + C::TMEM_Q + ks * 8, bd, C::IDESC_QK, ks > 0 ? 1u : 0u);
          }
          umma_commit(bar_s_full(sb));
        }
      } else {
        for (int j = 0; ok && j < n_tiles; ++j) {
          const int sb = j % C::NSB;
          if (!mbar_wait(bar_p_full(sb), (j / C::NSB) & 1, abort_flag, 22)) break;
          tc_fence_after();
          const uint32_t v_base = s_c + (j % C::NS) * C::C_STAGE;
#pragma unroll
          for (int kk = 0; kk < C::BN / 16; ++kk) {
            // A = P (bf16 pairs in S buffer sb): 16 k-elements = 8 columns per step
            const uint32_t a_tmem = tmem + C::TMEM_S + sb * C::BN + kk * 8;
            const uint64_t bd = smem_desc(v_base + kk * 16 * C::SWB, C::C_ATOM_BYTES, 8 * C::SWB, C::SWZ);
            umma_ts(tmem, a_tmem, bd, C::IDESC_PV, (j > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(bar_c_empty(j % C::NS));
          umma_commit(bar_pv_done(sb));
        }
      }
    }
    if (lane == 0) {
      DSA_PROF_SPAN(qk_thread ? 62 : 20, t_role);
      umma_commit(bar_drain);
      long long t0 = clock64();
      while (!mbar_try_wait(bar_drain, 0) && clock64() - t0 < kWaitLimitCycles) {
      }
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    // Thread (head row h, team c): warps q4 and q4 + 4 share the TMEM lanes
    // 32 q4 .. 32 q4 + 31; warp q4 + 4c takes the tiles of team c (all their
    // columns), columns [c DVS/2, ...) of O in the epilogue, and the 8-column
    // chunks c, c + 2, ... of the query slice.
    const int q4 = warp & 3, c = warp >> 2;
    const int h = q4 * 32 + lane;                          // head row = TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
    const uint32_t x_peer = C::SPLIT == 2 ? mapa_shared(smem_u32(xbuf), peer) : 0u;
    const uint32_t bar_x_full_peer0 = C::SPLIT == 2 ? mapa_shared(bar_x_full(0), peer) : 0u;
    float m_used = -INFINITY;    // reference max (log2 units) of this team's latest tile
    float l_run = 0.f;           // this team's tiles, against m_used; the teams add at the end
    bool ok = true;
    // Team c takes tiles j = c, c + 2, ...; a thread owns head row h of its
    // team's tiles, all BN columns, so a tile's row maximum needs no partner.
    // The reference max the exponentials are taken against is one sequence
    // over the tiles (O accumulates every tile's P against it): team c reads
    // the decision of tile j - 1 (the other team's) from m_pub and publishes
    // its own for tile j + 1.  Each team sums its own tiles' probabilities
    // against the reference it last used; the epilogue brings both sums to the
    // final reference.
    //
    // 2-CTA split: a tile's partial scores go to the peer as four bulk copies,
    // one per warp (its 32 rows of the team's staging buffer), completing on
    // the peer's x_full(j % XR); team c's first warp arms that phase with the
    // bytes to expect.  A tile is sent when its team starts on it, after the
    // team took tile j - 2 from the peer, which the peer sent only once it had
    // finished tile j - 4 -- the previous content of receive buffer j % XR.
    // Staging row h holds BN / 4 16-byte chunks, chunk k at slot (k + h) mod
    // (BN / 4) (no bank conflicts); the receiver reads with the same rotation.
    float* m_pub = mx_s;                                   // [2 teams][128]: reference after the team's last tile
    float sv[C::BN];
    for (int j = c; ok && j < n_tiles; j += 2) {
      const int sb = j % C::NSB;   // S buffer of this tile; its P goes there too
      if (!mbar_wait_warp(bar_s_full(sb), (j / C::NSB) & 1, abort_flag, 26)) { ok = false; break; }
      tc_fence_after();
      {
        uint32_t raw[C::BN];
        tmem_ld32(tmem + lane_base + C::TMEM_S + sb * C::BN, raw);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < C::BN; ++k) sv[k] = __uint_as_float(raw[k]);
      }
      if (C::SPLIT == 2) {
        const int xr = j % C::XR;
        if (q4 == 0 && lane == 0) mbar_arrive_expect_tx(bar_x_full(xr), C::X_BYTES);
        // this warp's rows of the staging buffer were last read by its copy of tile j - 2
        if (lane == 0) bulk_wait_group_read<0>();
        __syncwarp();
        float* row = xs + c * (C::X_BYTES / 4) + h * C::BN;
#pragma unroll
        for (int k = 0; k < C::BN / 4; ++k) {
          const int slot = (k + h) & (C::BN / 4 - 1);
          *reinterpret_cast<float4*>(row + slot * 4) = make_float4(sv[4 * k], sv[4 * k + 1], sv[4 * k + 2],
                                                                   sv[4 * k + 3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          constexpr uint32_t kWarpBytes = 32 * C::BN * 4;
          bulk_copy_to_peer(x_peer + xr * C::X_BYTES + q4 * kWarpBytes,
                            smem_u32(xs + c * (C::X_BYTES / 4)) + q4 * kWarpBytes, kWarpBytes,
                            bar_x_full_peer0 + 8 * xr);
          bulk_commit_group();
        }
        // the copy completes on this CTA's own barrier: CTA-scope acquire, as for a TMA load
        if (!mbar_wait_warp(bar_x_full(xr), (j / C::XR) & 1, abort_flag, 28)) { ok = false; break; }
        const float* xrow = xbuf + xr * (C::X_BYTES / 4) + h * C::BN;
#pragma unroll
        for (int k = 0; k < C::BN / 4; ++k) {
          const int slot = (k + h) & (C::BN / 4 - 1);
          const float4 v = *reinterpret_cast<const float4*>(xrow + slot * 4);
          sv[4 * k] += v.x;
          sv[4 * k + 1] += v.y;
          sv[4 * k + 2] += v.z;
          sv[4 * k + 3] += v.w;
        }
      }
      // validity of the tile's entries (written by the producer before it armed c_full)
      if (!mbar_wait_warp(bar_c_full(j % C::NS), (j / C::NS) & 1, abort_flag, 29)) { ok = false; break; }
      const uint32_t vmask = mask_s[j % C::NS];
      float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int k = 0; k < C::BN; ++k) {
        sv[k] = ((vmask >> k) & 1u) ? sv[k] * p.scale_log2 : -INFINITY;
        mx[k & 3] = fmaxf(mx[k & 3], sv[k]);
      }
      const float mt = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
      // the reference after tile j - 1 (the other team's decision)
      float m_prev = -INFINITY;
      if (j > 0) {
        if (!mbar_wait_warp(bar_m_pub(c ^ 1), ((j - 1) >> 1) & 1, abort_flag, 38)) { ok = false; break; }
        m_prev = m_pub[(c ^ 1) * 128 + h];
      }
      const float m_new = mt > m_prev + C::kRescaleThreshold ? mt : m_prev;
      if (j + 1 < n_tiles) {
        m_pub[c * 128 + h] = m_new;
        mbar_arrive_warp(bar_m_pub(c));
      }
      const float corr_o = m_new > m_prev ? exp2f(m_prev - m_new) : 1.f;   // 0 on the first valid tile
      const float corr_l = m_new > m_used ? exp2f(m_used - m_new) : 1.f;
      m_used = m_new;
      uint32_t pk[C::BN / 2];
      float ps[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int k = 0; k < C::BN; k += 2) {
        const float e0 = sv[k] == -INFINITY ? 0.f : ex2_approx(sv[k] - m_used);
        const float e1 = sv[k + 1] == -INFINITY ? 0.f : ex2_approx(sv[k + 1] - m_used);
        const __nv_bfloat162 b2 = __floats2bfloat162_rn(e0, e1);
        const float2 back = __bfloat1622float2(b2);
        ps[(k >> 1) & 3] += back.x + back.y;
        pk[k / 2] = *reinterpret_cast<const uint32_t*>(&b2);
      }
      l_run = l_run * corr_l + ((ps[0] + ps[1]) + (ps[2] + ps[3]));
      // O holds the PVs of tiles < j against m_prev.  The rescale decision is
      // per head row, but the TMEM accesses below are warp-collective
      // (.sync.aligned): the warp rescales if any lane needs it, and lanes
      // that do not multiply by 1.
      if (__any_sync(0xFFFFFFFFu, corr_o != 1.f && j > 0)) {
        // O must hold every earlier PV before it is rescaled in place
        if (!mbar_wait_warp(bar_pv_done((j - 1) % C::NSB), ((j - 1) / C::NSB) & 1, abort_flag, 31)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll 1
        for (int c0 = 0; c0 < C::DVS; c0 += 16) {
          uint32_t o[16];
          tmem_ld16(tmem + lane_base + c0, o);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 16; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * corr_o);
          tmem_st16(tmem + lane_base + c0, o);
        }
        tmem_wait_st();
      }
      // P row h (bf16 pairs) over the first BN / 2 columns of the S buffer; the PV MMA reads it from there
      tmem_st16(tmem + lane_base + C::TMEM_S + sb * C::BN, pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive_warp(bar_p_full(sb));
    }
    if (C::SPLIT == 2 && lane == 0) bulk_wait_group<0>();   // this warp's outgoing copies have completed
    if (lane == 0) DSA_PROF_SPAN(63, t_role);
    // ------------------------------------------------------------ epilogue
    // the row sum over both teams, against the final reference (the larger
    // of the two teams' last ones: the reference never decreases)
    l_s[c * 128 + h] = l_run;
    m_pub[256 + c * 128 + h] = m_used;
    mbar_arrive_warp(bar_pair_l(q4));
    if (!mbar_wait_warp(bar_pair_l(q4), 0, abort_flag, 39)) ok = false;
    {
      const float m0 = m_pub[256 + h], m1 = m_pub[256 + 128 + h];
      const float l0 = l_s[h], l1 = l_s[128 + h];
      m_used = fmaxf(m0, m1);
      l_run = (l0 > 0.f ? l0 * exp2f(m0 - m_used) : 0.f) + (l1 > 0.f ? l1 * exp2f(m1 - m_used) : 0.f);
    }
    const int t_out = static_cast<int>(t);
    if (ok && n_tiles > 0) {
      const int j = n_tiles - 1;
      ok = mbar_wait_warp(bar_pv_done(j % C::NSB), (j / C::NSB) & 1, abort_flag, 32);
      tc_fence_after();
    }
    // every lane takes part in the warp-collective TMEM loads; only rows h < H are stored
    if (ok && !skip) {
      const bool store = h < C::H;
      __nv_bfloat16* orow = p.out + (static_cast<int64_t>(t_out) * C::H + (store ? h : 0)) * C::DV + rank * C::DVS;
      const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
#pragma unroll 1
      for (int c0 = c * (C::DVS / 2); c0 < (c + 1) * (C::DVS / 2); c0 += 16) {
        uint32_t o[16];
        if (n_tiles > 0) {
          tmem_ld16(tmem + lane_base + c0, o);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) o[jj] = 0u;
        }
        uint32_t pk[8];
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          const __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(o[2 * jj]) * inv_l,
                                                         __uint_as_float(o[2 * jj + 1]) * inv_l);
          pk[jj] = *reinterpret_cast<const uint32_t*>(&b2);
        }
        if (store) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c0);
          dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        }
      }
      if (store && c == 0 && rank == 0 && p.lse != nullptr)
        p.lse[static_cast<int64_t>(t_out) * C::H + h] =
            l_run > 0.f ? (m_used + log2f(l_run)) * 0.69314718055994531f : -INFINITY;
    }
  }

  if (lane == 0 && warp < C::NSM) DSA_PROF_SPAN(60, t_role);
  tc_fence_before();
  __syncthreads();
  if (C::SPLIT == 2) cluster_sync();   // no remote access into this CTA after this point
  DSA_PROF_END();
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace dsa
