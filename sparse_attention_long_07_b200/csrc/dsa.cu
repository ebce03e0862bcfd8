// dsa.cu -- C ABI of the DSA hot path (declarations and contracts in include/dsa.h).
//
// Host side: argument validation (all of it before the first CUDA call, so an
// invalid call touches no device state), TMA descriptor encoding, launch
// configuration, and the chunked forward.  Device side: the kernels in
// indexer.cuh, topk.cuh and sparse_mla.cuh.

#include <cuda.h>
#include <cuda_bf16.h>
#include <nvtx3/nvToolsExt.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "dsa.h"
#include "cache.cuh"
#include "fp8.cuh"
#include "indexer.cuh"
#include "sparse_mla.cuh"
#include "topk.cuh"
#include "up_proj.cuh"

namespace {

using dsa::IndexerCfg;
using dsa::MlaCfg;

// ----------------------------------------------------------------------------
// Validation of the sequence and cache layout (host copies only)
// ----------------------------------------------------------------------------
struct Layout {
  int B = 0;
  int64_t T = 0;         // total query rows
  int64_t S = 0;         // cache rows (packed: cu_k[B]; paged: n_pages * page_size)
  int max_kv = 0;        // longest kv_len over sequences with a row in [q_begin, q_end)
  int max_q_rows = 0;    // most rows of one sequence inside [q_begin, q_end)
  int max_tiles = 0;     // most 128-key tiles one query row of the range needs
};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// NVTX range around each stage's launches and each entry point (visible in
// Nsight timelines; a no-op unless a tool is attached).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

dsa::PageMap page_map(const dsa_varlen& v) {
  dsa::PageMap m;
  m.block_table = v.block_table;
  m.page_shift = 0;
  while (v.block_table && (1 << m.page_shift) < v.page_size) ++m.page_shift;
  m.pages_per_seq = v.block_table ? v.pages_per_seq : 0;
  m.n_pages = v.block_table ? static_cast<int>(v.n_pages) : 0;
  return m;
}

dsa_status check_varlen(const dsa_varlen& v, int64_t q_begin, int64_t q_end, Layout* out) {
  if (v.batch < 1 || !v.cu_q || !v.cu_k || !v.cu_q_host || !v.cu_k_host) return DSA_ERR_INVALID_ARG;
  if (v.cu_q_host[0] != 0 || v.cu_k_host[0] != 0) return DSA_ERR_INVALID_ARG;
  Layout L;
  L.B = v.batch;
  for (int b = 0; b < v.batch; ++b) {
    const int64_t ql = static_cast<int64_t>(v.cu_q_host[b + 1]) - v.cu_q_host[b];
    const int64_t kl = static_cast<int64_t>(v.cu_k_host[b + 1]) - v.cu_k_host[b];
    if (ql < 0 || kl < ql) return DSA_ERR_INVALID_ARG;
  }
  L.T = v.cu_q_host[v.batch];
  L.S = v.cu_k_host[v.batch];
  if (v.block_table) {
    if ((reinterpret_cast<uintptr_t>(v.block_table) & 3u) || v.page_size < 64 || (v.page_size & (v.page_size - 1)) ||
        v.pages_per_seq < 1 || v.n_pages < 1 || v.n_pages > 0x7FFFFFFF / v.page_size)
      return DSA_ERR_INVALID_ARG;
    for (int b = 0; b < v.batch; ++b) {
      const int64_t kl = static_cast<int64_t>(v.cu_k_host[b + 1]) - v.cu_k_host[b];
      if (kl > static_cast<int64_t>(v.pages_per_seq) * v.page_size) return DSA_ERR_INVALID_ARG;
    }
    L.S = v.n_pages * v.page_size;
  }
  if (q_begin < 0 || q_end < q_begin || q_end > L.T) return DSA_ERR_INVALID_ARG;
  for (int b = 0; b < v.batch; ++b) {
    const int64_t lo = std::max<int64_t>(v.cu_q_host[b], q_begin);
    const int64_t hi = std::min<int64_t>(v.cu_q_host[b + 1], q_end);
    if (lo >= hi) continue;
    const int kl = v.cu_k_host[b + 1] - v.cu_k_host[b];
    const int ql = v.cu_q_host[b + 1] - v.cu_q_host[b];
    const int pos_last = kl - ql + static_cast<int>(hi - 1 - v.cu_q_host[b]);
    L.max_kv = std::max(L.max_kv, kl);
    L.max_q_rows = std::max(L.max_q_rows, static_cast<int>(hi - lo));
    L.max_tiles = std::max(L.max_tiles, pos_last / 128 + 1);
  }
  *out = L;
  return DSA_OK;
}

// Optional host-side fault injection for tests of the error paths:
// DSA_INJECT_FAULT=cuda | timeout makes the next entry point report that
// failure without launching anything.
dsa_status injected_fault() {
  const char* f = std::getenv("DSA_INJECT_FAULT");
  if (!f) return DSA_OK;
  if (!std::strcmp(f, "cuda")) return DSA_ERR_CUDA;
  if (!std::strcmp(f, "timeout")) return DSA_ERR_DEVICE_TIMEOUT;
  return DSA_OK;
}

// ----------------------------------------------------------------------------
// TMA descriptors (cuTensorMapEncodeTiled through the runtime's entry point)
// ----------------------------------------------------------------------------
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Row-major 2D tensor [rows, cols] with a row stride in bytes; box
// {box_cols, box_rows}; out-of-bounds elements read as zero.
bool make_map(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t cols,
              uint64_t rows, uint64_t row_stride_bytes, uint32_t box_cols, uint32_t box_rows,
              CUtensorMapSwizzle swz) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {row_stride_bytes};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3D tiled map: dims (d0, d1, d2) innermost first, byte strides of dims 1 and 2.
bool make_map_3d(CUtensorMap* map, CUtensorMapDataType dt, const void* base, const uint64_t dims[3],
                 const uint64_t strides[2], const uint32_t box[3], CUtensorMapSwizzle swz) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t d[3] = {dims[0], dims[1], dims[2]};
  const cuuint64_t st[2] = {strides[0], strides[1]};
  const cuuint32_t bx[3] = {box[0], box[1], box[2]};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, dt, 3, const_cast<void*>(base), d, st, bx, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Per-device state.  Kernel attributes (the dynamic shared-memory limit) and
// the SM count belong to a device, so they are kept per device ordinal and set
// up the first time a kernel runs on that device.
constexpr int kMaxDevices = 64;

int current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
  return dev;
}

// Raise Kernel's dynamic shared-memory limit to `bytes` on the current device
// (once per device).
template <auto Kernel>
cudaError_t ensure_smem(int bytes) {
  static std::once_flag once[kMaxDevices];
  static cudaError_t err[kMaxDevices];
  const int dev = current_device();
  if (dev < 0) return cudaErrorInvalidDevice;
  std::call_once(once[dev], [dev, bytes] {
    err[dev] = cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  });
  return err[dev];
}

int num_sms() {
  static std::once_flag once[kMaxDevices];
  static int n[kMaxDevices];
  const int dev = current_device();
  if (dev < 0) return 0;
  std::call_once(once[dev], [dev] {
    if (cudaDeviceGetAttribute(&n[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) n[dev] = 0;
  });
  return n[dev];
}

bool is_released_indexer(int h, int d) { return h == 64 && d == 128; }
bool is_tiny_indexer(int h, int d) { return h == 4 && d == 32; }
bool is_released_mla(int h, int dqk, int dv) { return h == 128 && dqk == 576 && dv == 512; }
bool is_tiny_mla(int h, int dqk, int dv) { return h == 4 && dqk == 80 && dv == 64; }

// ----------------------------------------------------------------------------
// Launchers (arguments already validated)
// ----------------------------------------------------------------------------
template <class C>
dsa_status launch_indexer(const void* q_idx, const float* q_scale, const float* w, const void* k_idx,
                          const float* k_scale, const dsa_varlen& v, const Layout& L,
                          int64_t q_begin, int64_t q_end, float* scores, int64_t ld,
                          float* part_max, int64_t ld_pm, cudaStream_t stream) {
  CUtensorMap tm_q, tm_k;
  if (!make_map(&tm_q, C::QFP8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, q_idx, C::D_I,
                static_cast<uint64_t>(L.T) * C::H_I, C::D_I * C::ELEM, C::ATOM_ELEMS, C::N,
                C::SWB == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B))
    return DSA_ERR_CUDA;
  const uint32_t box_rows = v.block_table ? 64u : static_cast<uint32_t>(C::BK);   // paged: 64-row boxes
  if (C::KFP8) {
    if (!make_map(&tm_k, CU_TENSOR_MAP_DATA_TYPE_UINT8, k_idx, C::D_I, static_cast<uint64_t>(L.S),
                  C::D_I, C::D_I, box_rows, CU_TENSOR_MAP_SWIZZLE_128B))
      return DSA_ERR_CUDA;
  } else {
    if (!make_map(&tm_k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, k_idx, C::D_I,
                  static_cast<uint64_t>(L.S), C::D_I * 2, C::ATOM_ELEMS, box_rows,
                  C::SWB == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B))
      return DSA_ERR_CUDA;
  }
  if (ensure_smem<dsa::indexer_scores_kernel<C>>(C::SMEM_BYTES) != cudaSuccess) return DSA_ERR_CUDA;

  dsa::IndexerParams p;
  p.w = w;
  p.q_scale = q_scale;
  p.k_scale = k_scale;
  p.pages = page_map(v);
  p.cache_rows = static_cast<int>(L.S);
  p.cu_q = v.cu_q;
  p.cu_k = v.cu_k;
  p.B = v.batch;
  p.q_begin = q_begin;
  p.q_end = q_end;
  p.scores = scores;
  p.ld = ld;
  p.part_max = part_max;
  p.ld_pm = ld_pm;
  p.chunk_tiles = C::NQ == 1 ? 32 : 64;
  const int qblocks = (L.max_q_rows + C::NQ - 1) / C::NQ;
  const int chunks = (L.max_tiles + p.chunk_tiles - 1) / p.chunk_tiles;
  if (qblocks == 0 || chunks == 0) return DSA_OK;
  if (qblocks > 65535 || v.batch > 65535) return DSA_ERR_UNSUPPORTED;   // checked by indexer_limits first
  dim3 grid(chunks, qblocks, v.batch);
  dsa::indexer_scores_kernel<C><<<grid, C::NT, C::SMEM_BYTES, stream>>>(tm_q, tm_k, p);
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

// Decode-like calls: one persistent CTA per SM over the flat (sequence, key tile) list.
template <class C>
dsa_status launch_indexer_persistent(const void* q_idx, const float* q_scale, const float* w, const void* k_idx,
                                     const float* k_scale, const dsa_varlen& v, const Layout& L,
                                     int64_t q_begin, int64_t q_end, float* scores, int64_t ld,
                                     float* part_max, int64_t ld_pm, cudaStream_t stream) {
  int64_t units = 0;
  for (int b = 0; b < v.batch; ++b) {
    const int64_t lo = std::max<int64_t>(v.cu_q_host[b], q_begin);
    const int64_t hi = std::min<int64_t>(v.cu_q_host[b + 1], q_end);
    if (lo >= hi) continue;
    const int kv = v.cu_k_host[b + 1] - v.cu_k_host[b];
    const int ql = v.cu_q_host[b + 1] - v.cu_q_host[b];
    units += (kv - ql + static_cast<int>(lo - v.cu_q_host[b])) / C::BK + 1;
  }
  const int sms = num_sms();
  if (units == 0) return DSA_OK;
  if (sms <= 0) return DSA_ERR_CUDA;
  CUtensorMap tm_q, tm_k;
  if (!make_map(&tm_q, C::QFP8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, q_idx, C::D_I,
                static_cast<uint64_t>(L.T) * C::H_I, C::D_I * C::ELEM, C::ATOM_ELEMS, C::N, CU_TENSOR_MAP_SWIZZLE_128B))
    return DSA_ERR_CUDA;
  if (!make_map(&tm_k, CU_TENSOR_MAP_DATA_TYPE_UINT8, k_idx, C::D_I, static_cast<uint64_t>(L.S), C::D_I, C::D_I,
                v.block_table ? 64u : static_cast<uint32_t>(C::BK), CU_TENSOR_MAP_SWIZZLE_128B))
    return DSA_ERR_CUDA;
  if (ensure_smem<dsa::indexer_persistent_kernel<C>>(C::SMEM_BYTES) != cudaSuccess) return DSA_ERR_CUDA;
  dsa::IndexerParams p;
  p.w = w;
  p.q_scale = q_scale;
  p.k_scale = k_scale;
  p.pages = page_map(v);
  p.cache_rows = static_cast<int>(L.S);
  p.cu_q = v.cu_q;
  p.cu_k = v.cu_k;
  p.B = v.batch;
  p.q_begin = q_begin;
  p.q_end = q_end;
  p.scores = scores;
  p.ld = ld;
  p.part_max = part_max;
  p.ld_pm = ld_pm;
  p.chunk_tiles = 0;
  const unsigned grid = static_cast<unsigned>(std::min<int64_t>(units, sms));
  // a dependent of the previous kernel in the stream (see run_mla)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(C::NT, 1, 1);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, dsa::indexer_persistent_kernel<C>, tm_q, tm_k, p) != cudaSuccess) return DSA_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

template <class C>
dsa_status launch_mla(const void* q, const void* latent, const int32_t* idx, const dsa_varlen& v,
                      const Layout& L, int64_t q_begin, int64_t q_end, int topk, float scale,
                      const float* rope, void* out, float* lse, cudaStream_t stream) {
  CUtensorMap tm_lat;
  const CUtensorMapSwizzle swz = C::SWB == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                 : (C::SWB == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
  if (!make_map(&tm_lat, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, latent, C::DQK, static_cast<uint64_t>(L.S),
                C::DQK * 2, C::ATOM, 1, swz))
    return DSA_ERR_CUDA;
  if (ensure_smem<dsa::sparse_mla_kernel<C>>(C::SMEM_BYTES) != cudaSuccess) return DSA_ERR_CUDA;

  dsa::MlaParams p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.idx = idx;
  p.cu_q = v.cu_q;
  p.cu_k = v.cu_k;
  p.pages = page_map(v);
  p.cache_rows = static_cast<int>(L.S);
  p.B = v.batch;
  p.q_begin = q_begin;
  p.topk = topk;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.rope = reinterpret_cast<const float2*>(rope);
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  const int64_t rows = q_end - q_begin;
  if (rows == 0) return DSA_OK;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(rows * C::SPLIT), 1, 1);
  cfg.blockDim = dim3(C::NT, 1, 1);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C::SPLIT;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  // a dependent of the previous kernel in the stream: it may start while that
  // kernel finishes (the top-k frees most SMs early) and waits for it before
  // it reads the selection
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaError_t e = cudaLaunchKernelEx(&cfg, dsa::sparse_mla_kernel<C>, tm_lat, p);
  return e == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

dsa_status check_indexer_args(const void* q_idx, const float* q_scale, const float* w, const void* k_idx,
                              const float* k_scale, dsa_kidx_dtype kd, int h, int d,
                              const float* scores, int64_t ld, const Layout& L) {
  // FP8 indexer (q_scale given): e4m3 queries and keys, released shape only
  if (q_scale) {
    if (reinterpret_cast<uintptr_t>(q_scale) & 3u) return DSA_ERR_INVALID_ARG;
    if (kd != DSA_KIDX_FP8_E4M3) return DSA_ERR_INVALID_ARG;
    if (!is_released_indexer(h, d)) return DSA_ERR_UNSUPPORTED;
  }
  // scores == nullptr: the score buffer is validated by the caller (dsa_forward's workspace)
  if (!q_idx || !w || !k_idx) return DSA_ERR_INVALID_ARG;
  if (!aligned16(q_idx) || !aligned16(w) || !aligned16(k_idx) || (scores && !aligned16(scores)))
    return DSA_ERR_INVALID_ARG;
  if (kd != DSA_KIDX_BF16 && kd != DSA_KIDX_FP8_E4M3) return DSA_ERR_INVALID_ARG;
  if (kd == DSA_KIDX_FP8_E4M3 && !k_scale) return DSA_ERR_INVALID_ARG;
  if (ld < L.max_kv || ld % 4 != 0) return DSA_ERR_INVALID_ARG;
  if (is_released_indexer(h, d)) return DSA_OK;
  if (is_tiny_indexer(h, d) && kd == DSA_KIDX_BF16) return DSA_OK;
  return DSA_ERR_UNSUPPORTED;
}

dsa_status check_mla_args(const void* q, const void* latent, const int32_t* idx, int topk, int h,
                          int dqk, int dv, float scale, const void* out, const float* lse) {
  // idx == nullptr: the selections are validated by the caller (dsa_forward)
  if (!q || !latent || !out) return DSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(latent) || (idx && !aligned16(idx)) || !aligned16(out) ||
      (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return DSA_ERR_INVALID_ARG;
  if (topk < 1 || topk > 2048) return DSA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return DSA_ERR_INVALID_ARG;
  if (is_released_mla(h, dqk, dv) || is_tiny_mla(h, dqk, dv)) return DSA_OK;
  return DSA_ERR_UNSUPPORTED;
}

// Which indexer kernel a pass uses.  Decode-like passes (at most one query row
// per sequence) over an e4m3 cache take the persistent kernel; otherwise the
// query-block grid kernel with 1 or 4 queries per CTA.
enum class IndexerKind {
  kTiny, kPersistent, kGridFp8x1, kGridFp8x4, kGridBf16x1, kGridBf16x4, kFp8Fp8Persistent, kFp8Fp8x1, kFp8Fp8x4
};

IndexerKind choose_indexer(bool q_fp8, dsa_kidx_dtype kd, int h, int d, const dsa_varlen& v, const Layout& L) {
  if (is_tiny_indexer(h, d)) return IndexerKind::kTiny;
  const bool decode_like = L.max_q_rows <= 2;
  if (q_fp8) {
    if (L.max_q_rows <= 1 && v.batch <= IndexerCfg<64, 128, 1, true, true, true>::MAX_SEQ)
      return IndexerKind::kFp8Fp8Persistent;
    return decode_like ? IndexerKind::kFp8Fp8x1 : IndexerKind::kFp8Fp8x4;
  }
  if (kd == DSA_KIDX_FP8_E4M3) {
    if (L.max_q_rows <= 1 && v.batch <= IndexerCfg<64, 128, 1, true, true>::MAX_SEQ) return IndexerKind::kPersistent;
    return decode_like ? IndexerKind::kGridFp8x1 : IndexerKind::kGridFp8x4;
  }
  return decode_like ? IndexerKind::kGridBf16x1 : IndexerKind::kGridBf16x4;
}

// Launch limits of one indexer pass, checked before anything is launched.
dsa_status indexer_limits(bool q_fp8, dsa_kidx_dtype kd, int h, int d, const dsa_varlen& v, const Layout& L) {
  if (L.max_q_rows == 0) return DSA_OK;
  const IndexerKind k = choose_indexer(q_fp8, kd, h, d, v, L);
  if (k == IndexerKind::kPersistent || k == IndexerKind::kFp8Fp8Persistent) return DSA_OK;
  const int nq = (k == IndexerKind::kGridFp8x1 || k == IndexerKind::kGridBf16x1 || k == IndexerKind::kFp8Fp8x1) ? 1 : 4;
  const int64_t qblocks = (L.max_q_rows + nq - 1) / nq;
  if (qblocks > 65535 || v.batch > 65535) return DSA_ERR_UNSUPPORTED;   // gridDim.y / gridDim.z
  return DSA_OK;
}

dsa_status run_indexer(const void* q_idx, const float* q_scale, const float* w, const void* k_idx,
                       const float* k_scale, dsa_kidx_dtype kd, const dsa_varlen& v, const Layout& L, int h, int d,
                       int64_t q_begin, int64_t q_end, float* scores, int64_t ld, float* part_max,
                       int64_t ld_pm, cudaStream_t stream) {
  if (q_end == q_begin) return DSA_OK;
  NvtxRange range("dsa.indexer");
  switch (choose_indexer(q_scale != nullptr, kd, h, d, v, L)) {
    case IndexerKind::kFp8Fp8Persistent:
      return launch_indexer_persistent<IndexerCfg<64, 128, 1, true, true, true>>(q_idx, q_scale, w, k_idx, k_scale,
                                                                                 v, L, q_begin, q_end, scores, ld,
                                                                                 part_max, ld_pm, stream);
    case IndexerKind::kFp8Fp8x1:
      return launch_indexer<IndexerCfg<64, 128, 1, true, false, true>>(q_idx, q_scale, w, k_idx, k_scale, v, L,
                                                                        q_begin, q_end, scores, ld, part_max, ld_pm,
                                                                        stream);
    case IndexerKind::kFp8Fp8x4:
      return launch_indexer<IndexerCfg<64, 128, 4, true, false, true>>(q_idx, q_scale, w, k_idx, k_scale, v, L,
                                                                        q_begin, q_end, scores, ld, part_max, ld_pm,
                                                                        stream);
    case IndexerKind::kTiny:
      return launch_indexer<IndexerCfg<4, 32, 4, false>>(q_idx, nullptr, w, k_idx, k_scale, v, L, q_begin, q_end,
                                                          scores, ld, part_max, ld_pm, stream);
    case IndexerKind::kPersistent:
      return launch_indexer_persistent<IndexerCfg<64, 128, 1, true, true>>(q_idx, nullptr, w, k_idx, k_scale, v, L,
                                                                           q_begin, q_end, scores, ld, part_max, ld_pm, stream);
    case IndexerKind::kGridFp8x1:
      return launch_indexer<IndexerCfg<64, 128, 1, true>>(q_idx, nullptr, w, k_idx, k_scale, v, L, q_begin, q_end,
                                                           scores, ld, part_max, ld_pm, stream);
    case IndexerKind::kGridFp8x4:
      return launch_indexer<IndexerCfg<64, 128, 4, true>>(q_idx, nullptr, w, k_idx, k_scale, v, L, q_begin, q_end,
                                                           scores, ld, part_max, ld_pm, stream);
    case IndexerKind::kGridBf16x1:
      return launch_indexer<IndexerCfg<64, 128, 1, false>>(q_idx, nullptr, w, k_idx, k_scale, v, L, q_begin, q_end,
                                                            scores, ld, part_max, ld_pm, stream);
    case IndexerKind::kGridBf16x4:
      return launch_indexer<IndexerCfg<64, 128, 4, false>>(q_idx, nullptr, w, k_idx, k_scale, v, L, q_begin, q_end,
                                                            scores, ld, part_max, ld_pm, stream);
  }
  return DSA_ERR_UNSUPPORTED;
}

// Launch limits of one top-k pass: one CTA per row; rows up to MAX_N keys.
dsa_status topk_limits(const Layout& L, int64_t rows) {
  if (rows > 0x7FFFFFFF) return DSA_ERR_UNSUPPORTED;
  if (L.max_kv > dsa::TopkCfg::MAX_N) return DSA_ERR_UNSUPPORTED;   // 16-bit pass-1 counters
  return DSA_OK;
}

// Launch limits of one attention pass: one cluster of SPLIT CTAs per row.
dsa_status mla_limits(int64_t rows) { return rows * 2 > 0x7FFFFFFF ? DSA_ERR_UNSUPPORTED : DSA_OK; }

dsa_status run_topk(const float* scores, int64_t ld, const float* part_max, int64_t ld_pm, const dsa_varlen& v,
                    const Layout& L, int64_t q_begin, int64_t q_end, int topk, int32_t* idx, cudaStream_t stream) {
  const int64_t rows = q_end - q_begin;
  if (rows == 0) return DSA_OK;
  NvtxRange range("dsa.topk");
  if (topk_limits(L, rows) != DSA_OK) return DSA_ERR_UNSUPPORTED;
  if (ensure_smem<dsa::topk_kernel>(dsa::TopkCfg::SMEM_BYTES) != cudaSuccess) return DSA_ERR_CUDA;
  // a dependent of the previous kernel in the stream (see run_mla): its
  // launch overlaps that kernel's end; it waits for it before reading scores
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(rows), 1, 1);
  cfg.blockDim = dim3(dsa::TopkCfg::NT, 1, 1);
  cfg.dynamicSmemBytes = dsa::TopkCfg::SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, dsa::topk_kernel, scores, ld, part_max, ld_pm, v.cu_q, v.cu_k,
                                           v.batch, q_begin, topk, idx);
  return e == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

dsa_status run_mla(const void* q, const void* latent, const int32_t* idx, const dsa_varlen& v,
                   const Layout& L, int64_t q_begin, int64_t q_end, int topk, int h, int dqk, int dv,
                   float scale, const float* rope, void* out, float* lse, cudaStream_t stream) {
  NvtxRange range("dsa.sparse_mla");
  if (is_tiny_mla(h, dqk, dv))
    return launch_mla<MlaCfg<4, 80, 64, 1, 32>>(q, latent, idx, v, L, q_begin, q_end, topk, scale, rope, out,
                                                lse, stream);
  return launch_mla<MlaCfg<128, 576, 512, 2, 128>>(q, latent, idx, v, L, q_begin, q_end, topk, scale, rope, out,
                                                   lse, stream);
}

constexpr size_t kWsAlign = 256;
size_t align_up(size_t x) { return (x + kWsAlign - 1) / kWsAlign * kWsAlign; }

int64_t scores_ld(const Layout& L) { return std::max<int64_t>(4, (L.max_kv + 3) / 4 * 4); }

// Row stride of the part maxima: one per PART keys, rounded up to 4 (16-byte rows).
int64_t part_max_ld(int64_t ld_scores) { return std::max<int64_t>(4, ((ld_scores + dsa::PART - 1) / dsa::PART + 3) / 4 * 4); }

// part_max (nullable) must cover every part of the longest row, 16-byte rows.
dsa_status check_part_max(const float* part_max, int64_t ld_pm, const Layout& L) {
  if (!part_max) return DSA_OK;
  if (!aligned16(part_max) || ld_pm % 4 != 0 || ld_pm < (L.max_kv + dsa::PART - 1) / dsa::PART)
    return DSA_ERR_INVALID_ARG;
  return DSA_OK;
}

}  // namespace

extern "C" {

dsa_status dsa_indexer_scores(const void* q_idx, const float* q_scale, const float* w, const void* k_idx,
                              const float* k_scale, dsa_kidx_dtype k_dtype, dsa_varlen v,
                              int32_t n_idx_heads, int32_t idx_dim, int64_t q_begin,
                              int64_t q_end, float* scores, int64_t ld_scores, float* part_max,
                              int64_t ld_part_max, cudaStream_t stream) {
  Layout L;
  dsa_status st = check_varlen(v, q_begin, q_end, &L);
  if (st != DSA_OK) return st;
  if (!scores) return DSA_ERR_INVALID_ARG;
  st = check_indexer_args(q_idx, q_scale, w, k_idx, k_scale, k_dtype, n_idx_heads, idx_dim, scores, ld_scores, L);
  if (st != DSA_OK) return st;
  if ((st = check_part_max(part_max, ld_part_max, L)) != DSA_OK) return st;
  if ((st = indexer_limits(q_scale != nullptr, k_dtype, n_idx_heads, idx_dim, v, L)) != DSA_OK) return st;
  if ((st = injected_fault()) != DSA_OK) return st;
  return run_indexer(q_idx, q_scale, w, k_idx, k_scale, k_dtype, v, L, n_idx_heads, idx_dim, q_begin, q_end,
                     scores, ld_scores, part_max, ld_part_max, stream);
}

dsa_status dsa_topk(const float* scores, int64_t ld_scores, const float* part_max, int64_t ld_part_max,
                    dsa_varlen v, int64_t q_begin, int64_t q_end, int32_t topk, int32_t* idx,
                    cudaStream_t stream) {
  Layout L;
  dsa_status st = check_varlen(v, q_begin, q_end, &L);
  if (st != DSA_OK) return st;
  if (!scores || !idx || !aligned16(scores) || (reinterpret_cast<uintptr_t>(idx) & 3u))
    return DSA_ERR_INVALID_ARG;
  if (topk < 1 || topk > 2048 || ld_scores < L.max_kv || ld_scores % 4 != 0) return DSA_ERR_INVALID_ARG;
  if ((st = check_part_max(part_max, ld_part_max, L)) != DSA_OK) return st;
  if ((st = topk_limits(L, q_end - q_begin)) != DSA_OK) return st;
  if ((st = injected_fault()) != DSA_OK) return st;
  return run_topk(scores, ld_scores, part_max, ld_part_max, v, L, q_begin, q_end, topk, idx, stream);
}

dsa_status dsa_sparse_mla_attn(const void* q, const void* latent, const int32_t* idx,
                               dsa_varlen v, int64_t q_begin, int64_t q_end, int32_t topk,
                               int32_t n_heads, int32_t d_qk, int32_t d_v, float scale,
                               const float* rope_cs, int64_t rope_max_pos,
                               void* out, float* lse, cudaStream_t stream) {
  Layout L;
  dsa_status st = check_varlen(v, q_begin, q_end, &L);
  if (st != DSA_OK) return st;
  if (!idx) return DSA_ERR_INVALID_ARG;
  st = check_mla_args(q, latent, idx, topk, n_heads, d_qk, d_v, scale, out, lse);
  if (st != DSA_OK) return st;
  // every row's position is below its sequence's kv length
  if (rope_cs && ((reinterpret_cast<uintptr_t>(rope_cs) & 7u) || rope_max_pos < L.max_kv))
    return DSA_ERR_INVALID_ARG;
  if ((st = mla_limits(q_end - q_begin)) != DSA_OK) return st;
  if ((st = injected_fault()) != DSA_OK) return st;
  return run_mla(q, latent, idx, v, L, q_begin, q_end, topk, n_heads, d_qk, d_v, scale, rope_cs, out, lse,
                 stream);
}

size_t dsa_forward_workspace_size(dsa_varlen v, int32_t topk, int64_t q_chunk) {
  Layout full;
  if (v.batch < 1 || !v.cu_q_host || topk < 1 || topk > 2048) return 0;
  if (check_varlen(v, 0, v.cu_q_host[v.batch], &full) != DSA_OK) return 0;
  const int64_t rows = std::max<int64_t>(1, q_chunk > 0 ? std::min<int64_t>(q_chunk, full.T) : full.T);
  const int64_t ld = scores_ld(full);
  return align_up(static_cast<size_t>(rows) * ld * sizeof(float)) +
         align_up(static_cast<size_t>(rows) * part_max_ld(ld) * sizeof(float)) +
         align_up(static_cast<size_t>(rows) * topk * sizeof(int32_t));
}

}  // extern "C"

namespace {

// Every check of a dsa_forward call that does not involve the workspace:
// arguments, supported shapes and each pass's launch limits.  Host arithmetic
// only (no CUDA call).
dsa_status forward_checks(const void* q_idx, const float* q_scale, const float* w, const void* k_idx,
                          const float* k_scale,
                          dsa_kidx_dtype k_dtype, const void* q, const void* latent, const dsa_varlen& v,
                          int32_t n_idx_heads, int32_t idx_dim, int32_t topk, int32_t n_heads, int32_t d_qk,
                          int32_t d_v, float scale, int64_t q_chunk, const void* out, const float* lse,
                          const int32_t* idx_out) {
  if (v.batch < 1 || !v.cu_q_host) return DSA_ERR_INVALID_ARG;
  Layout full;
  dsa_status st = check_varlen(v, 0, v.cu_q_host[v.batch], &full);
  if (st != DSA_OK) return st;
  const int64_t ld = scores_ld(full);
  // the score buffer is the (256-byte aligned) workspace: checked by the caller
  st = check_indexer_args(q_idx, q_scale, w, k_idx, k_scale, k_dtype, n_idx_heads, idx_dim, nullptr, ld, full);
  if (st != DSA_OK) return st;
  if (idx_out && (reinterpret_cast<uintptr_t>(idx_out) & 15u)) return DSA_ERR_INVALID_ARG;
  st = check_mla_args(q, latent, nullptr, topk, n_heads, d_qk, d_v, scale, out, lse);
  if (st != DSA_OK) return st;
  const int64_t T = full.T;
  const int64_t rows = q_chunk > 0 ? std::min<int64_t>(q_chunk, T) : T;
  for (int64_t q0 = 0; q0 < T; q0 += rows) {
    const int64_t q1 = std::min(T, q0 + rows);
    Layout L;
    if ((st = check_varlen(v, q0, q1, &L)) != DSA_OK) return st;
    if ((st = indexer_limits(q_scale != nullptr, k_dtype, n_idx_heads, idx_dim, v, L)) != DSA_OK) return st;
    if ((st = topk_limits(L, q1 - q0)) != DSA_OK) return st;
    if ((st = mla_limits(q1 - q0)) != DSA_OK) return st;
  }
  return DSA_OK;
}

}  // namespace

extern "C" {

dsa_status dsa_forward(const void* q_idx, const float* q_scale, const float* w, const void* k_idx,
                       const float* k_scale, dsa_kidx_dtype k_dtype, const void* q,
                       const void* latent, dsa_varlen v, int32_t n_idx_heads,
                       int32_t idx_dim, int32_t topk, int32_t n_heads, int32_t d_qk,
                       int32_t d_v, float scale, int64_t q_chunk, void* out, float* lse,
                       int32_t* idx_out, void* workspace, size_t workspace_bytes,
                       cudaStream_t stream) {
  dsa_status st = forward_checks(q_idx, q_scale, w, k_idx, k_scale, k_dtype, q, latent, v, n_idx_heads, idx_dim,
                                 topk, n_heads, d_qk, d_v, scale, q_chunk, out, lse, idx_out);
  if (st != DSA_OK) return st;
  if (!workspace) return DSA_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) % kWsAlign) return DSA_ERR_INVALID_ARG;
  const size_t need = dsa_forward_workspace_size(v, topk, q_chunk);
  if (need == 0) return DSA_ERR_INVALID_ARG;
  if (workspace_bytes < need) return DSA_ERR_WORKSPACE;
  if ((st = injected_fault()) != DSA_OK) return st;
  NvtxRange range("dsa.forward");

  Layout full;
  check_varlen(v, 0, v.cu_q_host[v.batch], &full);
  const int64_t ld = scores_ld(full);
  const int64_t T = full.T;
  const int64_t rows = q_chunk > 0 ? std::min<int64_t>(q_chunk, T) : T;
  // workspace: one pass's scores | part maxima | selections
  const int64_t ld_pm = part_max_ld(ld);
  const size_t rows_ws = static_cast<size_t>(std::max<int64_t>(rows, 1));
  float* scores = static_cast<float*>(workspace);
  float* part_max = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + align_up(rows_ws * ld * sizeof(float)));
  int32_t* idx_ws = reinterpret_cast<int32_t*>(reinterpret_cast<uint8_t*>(part_max) +
                                               align_up(rows_ws * ld_pm * sizeof(float)));
  for (int64_t q0 = 0; q0 < T; q0 += rows) {
    const int64_t q1 = std::min(T, q0 + rows);
    Layout L;
    if ((st = check_varlen(v, q0, q1, &L)) != DSA_OK) return st;
    int32_t* idx = idx_out ? idx_out + q0 * topk : idx_ws;
    if ((st = run_indexer(q_idx, q_scale, w, k_idx, k_scale, k_dtype, v, L, n_idx_heads, idx_dim, q0, q1, scores,
                          ld, part_max, ld_pm, stream)) != DSA_OK)
      return st;
    if ((st = run_topk(scores, ld, part_max, ld_pm, v, L, q0, q1, topk, idx, stream)) != DSA_OK) return st;
    if ((st = run_mla(q, latent, idx, v, L, q0, q1, topk, n_heads, d_qk, d_v, scale, nullptr, out, lse,
                      stream)) != DSA_OK)
      return st;
  }
  return DSA_OK;
}

// ---------------------------------------------------------------------------
// Forward for callers that cannot allocate: the workspace is a file-scope
// device array instead of caller memory (contract in include/dsa.h).
// ---------------------------------------------------------------------------
static __device__ __align__(256) uint8_t g_dsa_static_scratch[DSA_STATIC_SCRATCH_BYTES];

namespace {
std::once_flag g_scratch_once[kMaxDevices];
void* g_scratch_ptr[kMaxDevices];
cudaError_t g_scratch_err[kMaxDevices];
}  // namespace

dsa_status dsa_forward_static_scratch(const void* q_idx, const float* q_scale, const float* w, const void* k_idx,
                                      const float* k_scale, dsa_kidx_dtype k_dtype,
                                      const void* q, const void* latent, dsa_varlen v,
                                      int32_t n_idx_heads, int32_t idx_dim, int32_t topk,
                                      int32_t n_heads, int32_t d_qk, int32_t d_v, float scale,
                                      void* out, float* lse, int32_t* idx_out,
                                      cudaStream_t stream) {
  if (v.batch < 1 || !v.cu_q_host) return DSA_ERR_INVALID_ARG;
  // largest pass (query rows) whose scores + selections fit the array
  const size_t per_pass_one = dsa_forward_workspace_size(v, topk, 1);
  if (per_pass_one == 0) return DSA_ERR_INVALID_ARG;
  if (per_pass_one > DSA_STATIC_SCRATCH_BYTES) return DSA_ERR_WORKSPACE;
  const int64_t T = v.cu_q_host[v.batch];
  int64_t lo = 1, hi = T > 1 ? T : 1;     // dsa_forward_workspace_size is monotone in the pass size
  while (lo < hi) {
    const int64_t mid = lo + (hi - lo + 1) / 2;
    if (dsa_forward_workspace_size(v, topk, mid) <= DSA_STATIC_SCRATCH_BYTES) lo = mid; else hi = mid - 1;
  }
  const int64_t q_chunk = lo;
  dsa_status st = forward_checks(q_idx, q_scale, w, k_idx, k_scale, k_dtype, q, latent, v, n_idx_heads, idx_dim,
                                 topk, n_heads, d_qk, d_v, scale, q_chunk, out, lse, idx_out);
  if (st != DSA_OK) return st;
  // the array's device address, looked up once per device with that device current
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DSA_ERR_CUDA;
  std::call_once(g_scratch_once[dev], [dev] {
    g_scratch_err[dev] = cudaGetSymbolAddress(&g_scratch_ptr[dev], g_dsa_static_scratch);
  });
  if (g_scratch_err[dev] != cudaSuccess || g_scratch_ptr[dev] == nullptr) return DSA_ERR_CUDA;
  return dsa_forward(q_idx, q_scale, w, k_idx, k_scale, k_dtype, q, latent, v, n_idx_heads, idx_dim, topk, n_heads,
                     d_qk, d_v, scale, q_chunk, out, lse, idx_out, g_scratch_ptr[dev], DSA_STATIC_SCRATCH_BYTES,
                     stream);
}

dsa_status dsa_device_error(int32_t* code, cudaStream_t stream) {
  if (!code) return DSA_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return DSA_ERR_CUDA;
  int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, dsa::g_device_error, sizeof(int)) != cudaSuccess) return DSA_ERR_CUDA;
  if (cudaMemcpyToSymbol(dsa::g_device_error, &zero, sizeof(int)) != cudaSuccess) return DSA_ERR_CUDA;
  *code = v;
  return v == 0 ? DSA_OK : DSA_ERR_DEVICE_TIMEOUT;
}

dsa_status dsa_hadamard_quantize_fp8(const void* x, int64_t n, void* q, float* scale, cudaStream_t stream) {
  if (n < 0) return DSA_ERR_INVALID_ARG;
  if (n == 0) return DSA_OK;
  if (!x || !q || !scale || !aligned16(x) || !aligned16(q) || (reinterpret_cast<uintptr_t>(scale) & 3u))
    return DSA_ERR_INVALID_ARG;
  if ((n + 7) / 8 > 0x7FFFFFFF) return DSA_ERR_UNSUPPORTED;
  dsa_status st;
  if ((st = injected_fault()) != DSA_OK) return st;
  dsa::hadamard_quantize_kernel<<<static_cast<unsigned>((n + 7) / 8), 256, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(x), n, static_cast<uint8_t*>(q), scale);
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

dsa_status dsa_cache_append(const void* latent_new, const void* kidx_new, dsa_varlen v, int32_t d_qk, int32_t d_v,
                            int32_t idx_dim, const float* rope_cs, int64_t rope_max_pos, dsa_kidx_quant k_quant,
                            void* latent_cache, void* k_cache, float* k_scale, cudaStream_t stream) {
  if (v.batch < 1 || !v.cu_q_host) return DSA_ERR_INVALID_ARG;
  Layout L;
  dsa_status st = check_varlen(v, 0, v.cu_q_host[v.batch], &L);
  if (st != DSA_OK) return st;
  if ((latent_new == nullptr) != (latent_cache == nullptr) || (kidx_new == nullptr) != (k_cache == nullptr))
    return DSA_ERR_INVALID_ARG;
  if ((latent_new && (!aligned16(latent_new) || !aligned16(latent_cache))) ||
      (kidx_new && (!aligned16(kidx_new) || !aligned16(k_cache))))
    return DSA_ERR_INVALID_ARG;
  if (latent_new && !is_released_mla(128, d_qk, d_v) && !is_tiny_mla(4, d_qk, d_v)) return DSA_ERR_UNSUPPORTED;
  if (rope_cs && (!latent_new || (reinterpret_cast<uintptr_t>(rope_cs) & 7u) || rope_max_pos < L.max_kv))
    return DSA_ERR_INVALID_ARG;
  if (kidx_new) {
    if (k_quant != DSA_KQ_BF16 && k_quant != DSA_KQ_E4M3_AMAX && k_quant != DSA_KQ_E4M3_HADAMARD)
      return DSA_ERR_INVALID_ARG;
    if (k_quant == DSA_KQ_BF16) {
      if (!is_released_indexer(64, idx_dim) && !is_tiny_indexer(4, idx_dim)) return DSA_ERR_UNSUPPORTED;
    } else {
      if (!k_scale || (reinterpret_cast<uintptr_t>(k_scale) & 3u)) return DSA_ERR_INVALID_ARG;
      if (idx_dim != dsa::FP8_DIM) return DSA_ERR_UNSUPPORTED;
    }
  }
  if ((L.T + 7) / 8 > 0x7FFFFFFF) return DSA_ERR_UNSUPPORTED;
  if (L.T == 0 || (!latent_new && !kidx_new)) return DSA_OK;
  if ((st = injected_fault()) != DSA_OK) return st;
  NvtxRange range("dsa.cache_append");
  dsa::AppendParams p;
  p.latent_new = static_cast<const __nv_bfloat16*>(latent_new);
  p.kidx_new = static_cast<const __nv_bfloat16*>(kidx_new);
  p.cu_q = v.cu_q;
  p.cu_k = v.cu_k;
  p.B = v.batch;
  p.T = L.T;
  p.pages = page_map(v);
  p.cache_rows = static_cast<int>(L.S);
  p.rope = reinterpret_cast<const float2*>(rope_cs);
  p.dqk = d_qk;
  p.dv = d_v;
  p.di = idx_dim;
  p.k_quant = static_cast<int>(k_quant);
  p.latent_cache = static_cast<__nv_bfloat16*>(latent_cache);
  p.k_cache = k_cache;
  p.k_scale = k_scale;
  dsa::cache_append_kernel<<<static_cast<unsigned>((L.T + 7) / 8), 256, 0, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

dsa_status dsa_mla_up_proj(const void* o, const void* w_uv, int64_t n_rows, int32_t n_heads, int32_t d_c,
                           int32_t d_v, void* y, cudaStream_t stream) {
  using C = dsa::UpProjCfg;
  if (n_rows < 0) return DSA_ERR_INVALID_ARG;
  if (!o || !w_uv || !y || !aligned16(o) || !aligned16(w_uv) || !aligned16(y)) return DSA_ERR_INVALID_ARG;
  if (n_heads != C::H || d_c != C::DC || d_v != C::DV) return DSA_ERR_UNSUPPORTED;
  if ((n_rows + C::BM - 1) / C::BM > 65535) return DSA_ERR_UNSUPPORTED;
  if (n_rows == 0) return DSA_OK;
  dsa_status st;
  if ((st = injected_fault()) != DSA_OK) return st;
  CUtensorMap tm_o, tm_w;
  {
    const uint64_t dims[3] = {C::DC, C::H, static_cast<uint64_t>(n_rows)};
    const uint64_t strides[2] = {C::DC * 2ull, static_cast<uint64_t>(C::H) * C::DC * 2ull};
    const uint32_t box[3] = {C::BKC, 1, C::BM};
    if (!make_map_3d(&tm_o, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, o, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return DSA_ERR_CUDA;
  }
  {
    const uint64_t dims[3] = {C::DV, C::DC, C::H};
    const uint64_t strides[2] = {C::DV * 2ull, static_cast<uint64_t>(C::DC) * C::DV * 2ull};
    const uint32_t box[3] = {64, C::BKC, 1};
    if (!make_map_3d(&tm_w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w_uv, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return DSA_ERR_CUDA;
  }
  if (ensure_smem<dsa::up_proj_kernel>(C::SMEM_BYTES) != cudaSuccess) return DSA_ERR_CUDA;
  NvtxRange range("dsa.up_proj");
  const dim3 grid(C::H, static_cast<unsigned>((n_rows + C::BM - 1) / C::BM));
  dsa::up_proj_kernel<<<grid, C::NT, C::SMEM_BYTES, stream>>>(tm_o, tm_w, static_cast<__nv_bfloat16*>(y), n_rows);
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

}  // extern "C"

namespace dsa {
// One bounded wait on an mbarrier that nothing arrives on: it gives up after
// limit_cycles, records the timeout (site kSelftestSite) in the device error
// word and returns, exactly as the waits of the DSA kernels do.  No copy or
// MMA is in flight, so the CTA can leave at once.
constexpr int kSelftestSite = 99;
__global__ void wait_selftest_kernel(long long limit_cycles) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(smem_u32(&bar), 0, &abort_flag, kSelftestSite, limit_cycles);
}
}  // namespace dsa

extern "C" {

dsa_status dsa_debug_wait_selftest(int64_t limit_cycles, cudaStream_t stream) {
  if (limit_cycles < 1 || limit_cycles > 2000000000LL) return DSA_ERR_INVALID_ARG;
  if (injected_fault() != DSA_OK) return injected_fault();
  dsa::wait_selftest_kernel<<<1, 32, 0, stream>>>(static_cast<long long>(limit_cycles));
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

dsa_status dsa_debug_wait_profile(uint64_t* cycles, uint64_t* counts, int32_t n, int32_t reset) {
#ifdef DSA_PROFILE_WAITS
  if (!cycles || !counts || n < 1) return DSA_ERR_INVALID_ARG;
  const int m = n < dsa::kWaitSites ? n : dsa::kWaitSites;
  if (cudaDeviceSynchronize() != cudaSuccess) return DSA_ERR_CUDA;
  if (cudaMemcpyFromSymbol(cycles, dsa::g_wait_cycles, m * sizeof(uint64_t)) != cudaSuccess ||
      cudaMemcpyFromSymbol(counts, dsa::g_wait_count, m * sizeof(uint64_t)) != cudaSuccess)
    return DSA_ERR_CUDA;
  if (reset) {
    static const unsigned long long zeros[dsa::kWaitSites] = {};
    if (cudaMemcpyToSymbol(dsa::g_wait_cycles, zeros, sizeof(zeros)) != cudaSuccess ||
        cudaMemcpyToSymbol(dsa::g_wait_count, zeros, sizeof(zeros)) != cudaSuccess)
      return DSA_ERR_CUDA;
  }
  return DSA_OK;
#else
  (void)cycles;
  (void)counts;
  (void)n;
  (void)reset;
  return DSA_ERR_UNSUPPORTED;
#endif
}

const char* dsa_status_string(dsa_status s) {
  switch (s) {
    case DSA_OK: return "ok";
    case DSA_ERR_INVALID_ARG: return "invalid argument";
    case DSA_ERR_UNSUPPORTED: return "unsupported shape";
    case DSA_ERR_CUDA: return "CUDA error";
    case DSA_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    case DSA_ERR_WORKSPACE: return "workspace missing or too small";
  }
  return "unknown status";
}

const char* dsa_version(void) { return "0.1.0"; }

}  // extern "C"
