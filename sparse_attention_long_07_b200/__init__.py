"""B200 (sm_100a) DeepSeek Sparse Attention hot path -- Python binding.

A thin ctypes layer over ``libdsa.so`` whose functions carry the names of the
C ABI in ``include/dsa.h``: ``dsa_indexer_scores``, ``dsa_topk``,
``dsa_sparse_mla_attn``, ``dsa_forward_workspace_size``, ``dsa_forward``,
``dsa_device_error``, ``dsa_status_string``.  It only marshals arguments:
every step of the computation runs in the library's CUDA kernels.  Tensors are
torch tensors in device memory (PyTorch provides memory and streams); the
packed sequence layout is described by :class:`Varlen`.

There is no fallback: if ``libdsa.so`` is missing or cannot be loaded, the
import of this package fails.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# DSA_LIBRARY_VARIANT=checked loads the build with device-side bounds checks
# (libdsa_checked.so, build.py --checked); the default is the release build.
LIB_PATH = os.path.join(_HERE, "libdsa_checked.so" if os.environ.get("DSA_LIBRARY_VARIANT") == "checked"
                        else "libdsa.so")

DSA_OK, DSA_ERR_INVALID_ARG, DSA_ERR_UNSUPPORTED, DSA_ERR_CUDA, DSA_ERR_DEVICE_TIMEOUT, DSA_ERR_WORKSPACE = range(6)
DSA_KIDX_BF16, DSA_KIDX_FP8_E4M3 = 0, 1


class DSAError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {dsa_status_string(status)} (status {status})")
        self.status = status


class dsa_varlen(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32),
        ("cu_q", ctypes.c_void_p),
        ("cu_k", ctypes.c_void_p),
        ("cu_q_host", ctypes.POINTER(ctypes.c_int32)),
        ("cu_k_host", ctypes.POINTER(ctypes.c_int32)),
        ("block_table", ctypes.c_void_p),
        ("page_size", ctypes.c_int32),
        ("pages_per_seq", ctypes.c_int32),
        ("n_pages", ctypes.c_int64),
    ]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python sparse_attention_long_07_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    for name in EXPORTED:
        if not hasattr(lib, name):
            raise ImportError(f"{LIB_PATH} predates the binding (no symbol {name}): rebuild it with "
                              "`python sparse_attention_long_07_b200/build.py --force`")
    vp, i32, i64, f32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float
    lib.dsa_indexer_scores.argtypes = [vp, vp, vp, vp, vp, ctypes.c_int, dsa_varlen, i32, i32, i64, i64, vp, i64,
                                       vp, i64, vp]
    lib.dsa_topk.argtypes = [vp, i64, vp, i64, dsa_varlen, i64, i64, i32, vp, vp]
    lib.dsa_sparse_mla_attn.argtypes = [vp, vp, vp, dsa_varlen, i64, i64, i32, i32, i32, i32, f32, vp, i64, vp, vp,
                                        vp]
    lib.dsa_forward_workspace_size.argtypes = [dsa_varlen, i32, i64]
    lib.dsa_forward_workspace_size.restype = ctypes.c_size_t
    lib.dsa_forward.argtypes = [vp, vp, vp, vp, vp, ctypes.c_int, vp, vp, dsa_varlen, i32, i32, i32, i32, i32, i32,
                                f32, i64, vp, vp, vp, vp, ctypes.c_size_t, vp]
    lib.dsa_device_error.argtypes = [ctypes.POINTER(ctypes.c_int32), vp]
    lib.dsa_status_string.argtypes = [ctypes.c_int]
    lib.dsa_status_string.restype = ctypes.c_char_p
    lib.dsa_version.restype = ctypes.c_char_p
    lib.dsa_debug_wait_profile.argtypes = [ctypes.POINTER(ctypes.c_uint64), ctypes.POINTER(ctypes.c_uint64),
                                           ctypes.c_int32, ctypes.c_int32]
    lib.dsa_debug_wait_profile.restype = ctypes.c_int
    lib.dsa_forward_static_scratch.argtypes = [vp, vp, vp, vp, vp, ctypes.c_int, vp, vp, dsa_varlen, i32, i32, i32,
                                               i32, i32, i32, f32, vp, vp, vp, vp]
    lib.dsa_forward_static_scratch.restype = ctypes.c_int
    lib.dsa_hadamard_quantize_fp8.argtypes = [vp, i64, vp, vp, vp]
    lib.dsa_hadamard_quantize_fp8.restype = ctypes.c_int
    lib.dsa_mla_up_proj.argtypes = [vp, vp, i64, i32, i32, i32, vp, vp]
    lib.dsa_cache_append.argtypes = [vp, vp, dsa_varlen, i32, i32, i32, vp, i64, ctypes.c_int, vp, vp, vp, vp]
    lib.dsa_cache_append.restype = ctypes.c_int
    lib.dsa_mla_up_proj.restype = ctypes.c_int
    lib.dsa_debug_wait_selftest.argtypes = [i64, vp]
    lib.dsa_debug_wait_selftest.restype = ctypes.c_int
    for fn in ("dsa_indexer_scores", "dsa_topk", "dsa_sparse_mla_attn", "dsa_forward", "dsa_device_error"):
        getattr(lib, fn).restype = ctypes.c_int
    return lib


EXPORTED = ("dsa_indexer_scores", "dsa_topk", "dsa_sparse_mla_attn", "dsa_forward_workspace_size",
            "dsa_forward", "dsa_device_error", "dsa_status_string", "dsa_version", "dsa_debug_wait_profile",
            "dsa_forward_static_scratch", "dsa_debug_wait_selftest", "dsa_hadamard_quantize_fp8",
            "dsa_mla_up_proj", "dsa_cache_append")

# bytes of the library's static scratch array (DSA_STATIC_SCRATCH_BYTES in include/dsa.h)
DSA_STATIC_SCRATCH_BYTES = 32 << 20

_lib = _load()


def library():
    """The loaded ctypes library (for symbol checks)."""
    return _lib


class Varlen:
    """Sequence layout: cumulative query-row and cache-entry offsets, and
    (optionally) the page table of paged caches.

    Keeps both the device copies the kernels read and the host copies the
    library validates and plans launches with.  block_table: int32 [B,
    pages_per_seq] device tensor of page ids (None: packed caches, entry s of
    sequence b at row cu_k[b] + s); page_size a power of two >= 64; n_pages
    the pages of the pool the caches hold.
    """

    def __init__(self, cu_q, cu_k, device=None, block_table=None, page_size=0, n_pages=0):
        cu_q = torch.as_tensor(cu_q, dtype=torch.int32).cpu().contiguous()
        cu_k = torch.as_tensor(cu_k, dtype=torch.int32).cpu().contiguous()
        self.cu_q_host, self.cu_k_host = cu_q, cu_k
        if device is None:
            self.cu_q, self.cu_k = cu_q, cu_k
        else:
            self.cu_q, self.cu_k = cu_q.to(device), cu_k.to(device)
        self.batch = cu_q.numel() - 1
        self.T = int(cu_q[-1])
        self.S = int(cu_k[-1])
        kv = (cu_k[1:] - cu_k[:-1])
        self.max_kv = int(kv.max()) if kv.numel() else 0
        self.block_table = None if block_table is None else block_table.contiguous()
        self.page_size, self.n_pages = int(page_size), int(n_pages)
        self.pages_per_seq = 0 if block_table is None else int(self.block_table.shape[1])

    def c(self) -> dsa_varlen:
        return dsa_varlen(self.batch, self.cu_q.data_ptr(), self.cu_k.data_ptr(),
                          ctypes.cast(self.cu_q_host.data_ptr(), ctypes.POINTER(ctypes.c_int32)),
                          ctypes.cast(self.cu_k_host.data_ptr(), ctypes.POINTER(ctypes.c_int32)),
                          _ptr(self.block_table), self.page_size, self.pages_per_seq, self.n_pages)


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _check(status: int, what: str):
    if status != DSA_OK:
        raise DSAError(status, what)


def _kdtype(k_idx):
    return DSA_KIDX_FP8_E4M3 if k_idx.dtype in (torch.float8_e4m3fn, torch.uint8) else DSA_KIDX_BF16


def dsa_status_string(status: int) -> str:
    return _lib.dsa_status_string(int(status)).decode()


def dsa_version() -> str:
    return _lib.dsa_version().decode()


PART = 8  # keys per part maximum


def part_max_ld(ld_scores: int) -> int:
    """Row stride of the part maxima for score rows of stride ld_scores."""
    return max(4, ((ld_scores + PART - 1) // PART + 3) // 4 * 4)


def dsa_indexer_scores(q_idx, w, k_idx, k_scale, v: Varlen, q_begin, q_end, scores, stream=None, part_max=None,
                       q_scale=None):
    """Lightning-indexer scores for global query rows [q_begin, q_end) into
    ``scores`` [q_end - q_begin, ld] fp32 (chunk-relative rows), and, when
    ``part_max`` is given, the maximum of every 8 consecutive keys of each row.
    With ``q_scale`` the FP8 indexer: q_idx and k_idx are e4m3 from
    dsa_hadamard_quantize_fp8, q_scale / k_scale their scales."""
    T, H_I, d_I = q_idx.shape
    _check(_lib.dsa_indexer_scores(_ptr(q_idx), _ptr(q_scale), _ptr(w), _ptr(k_idx), _ptr(k_scale), _kdtype(k_idx),
                                   v.c(),
                                   H_I, d_I, q_begin, q_end, _ptr(scores), scores.stride(0), _ptr(part_max),
                                   0 if part_max is None else part_max.stride(0), _stream(stream)),
           "dsa_indexer_scores")
    return scores


def dsa_topk(scores, v: Varlen, q_begin, q_end, topk, idx, stream=None, part_max=None):
    """Top-k selection of chunk-relative score rows into ``idx`` [rows, topk]
    int32 (with the indexer's part maxima when ``part_max`` is given)."""
    _check(_lib.dsa_topk(_ptr(scores), scores.stride(0), _ptr(part_max),
                         0 if part_max is None else part_max.stride(0), v.c(), q_begin, q_end, topk, _ptr(idx),
                         _stream(stream)), "dsa_topk")
    return idx


def dsa_sparse_mla_attn(q, latent, idx, v: Varlen, q_begin, q_end, scale, out, lse=None, d_v=None,
                        stream=None, rope=None):
    """MLA attention (absorbed MQA) over the selected rows; writes out/lse for
    global rows [q_begin, q_end).  rope (optional): fp32 [max_pos, (d_qk -
    d_v) / 2, 2] (cos, sin) table; the kernel then rotates q's RoPE part at
    each row's position."""
    T, H, d_qk = q.shape
    d_v = out.shape[-1] if d_v is None else d_v
    max_pos = 0 if rope is None else rope.shape[0]
    _check(_lib.dsa_sparse_mla_attn(_ptr(q), _ptr(latent), _ptr(idx), v.c(), q_begin, q_end, idx.shape[1], H,
                                    d_qk, d_v, float(scale), _ptr(rope), max_pos, _ptr(out), _ptr(lse),
                                    _stream(stream)),
           "dsa_sparse_mla_attn")
    return out, lse


def dsa_hadamard_quantize_fp8(x, q=None, scale=None, stream=None):
    """Hadamard rotation and e4m3 quantization of the 128-value vectors of x
    (bf16 [..., 128]); returns (q e4m3 [..., 128], scale fp32 [...])."""
    n = x.numel() // 128
    if q is None:
        q = torch.empty(x.shape, dtype=torch.float8_e4m3fn, device=x.device)
    if scale is None:
        scale = torch.empty(x.shape[:-1], dtype=torch.float32, device=x.device)
    _check(_lib.dsa_hadamard_quantize_fp8(_ptr(x), n, _ptr(q), _ptr(scale), _stream(stream)),
           "dsa_hadamard_quantize_fp8")
    return q, scale


DSA_KQ_BF16, DSA_KQ_E4M3_AMAX, DSA_KQ_E4M3_HADAMARD = 0, 1, 2


def dsa_cache_append(v: Varlen, latent_new=None, latent_cache=None, kidx_new=None, k_cache=None, k_scale=None,
                     k_quant=DSA_KQ_BF16, rope=None, d_v=None, stream=None):
    """Write the step's new tokens (its query rows, at positions pos(t)) into
    the latent cache (optionally rotating its RoPE columns with the (cos, sin)
    table `rope`) and the index-key cache (bf16 copy or one of the e4m3 forms)."""
    d_qk = 0 if latent_new is None else latent_new.shape[-1]
    if d_v is None:
        d_v = {576: 512, 80: 64}.get(d_qk, 0)
    idx_dim = 0 if kidx_new is None else kidx_new.shape[-1]
    max_pos = 0 if rope is None else rope.shape[0]
    _check(_lib.dsa_cache_append(_ptr(latent_new), _ptr(kidx_new), v.c(), d_qk, d_v, idx_dim, _ptr(rope), max_pos,
                                 int(k_quant), _ptr(latent_cache), _ptr(k_cache), _ptr(k_scale), _stream(stream)),
           "dsa_cache_append")


def dsa_mla_up_proj(o, w_uv, y=None, stream=None):
    """Per-head up-projection y[r, h, :] = o[r, h, :] @ w_uv[h] (o bf16
    [n, H, d_c], w_uv bf16 [H, d_c, d_v]); returns y bf16 [n, H, d_v]."""
    n, H, d_c = o.shape
    d_v = w_uv.shape[-1]
    if y is None:
        y = torch.empty((n, H, d_v), dtype=torch.bfloat16, device=o.device)
    _check(_lib.dsa_mla_up_proj(_ptr(o), _ptr(w_uv), n, H, d_c, d_v, _ptr(y), _stream(stream)), "dsa_mla_up_proj")
    return y


def dsa_forward_workspace_size(v: Varlen, topk: int, q_chunk: int = 0) -> int:
    return int(_lib.dsa_forward_workspace_size(v.c(), topk, q_chunk))


def dsa_forward(q_idx, w, k_idx, k_scale, q, latent, v: Varlen, topk, scale, out, lse, workspace,
                idx_out=None, q_chunk: int = 0, stream=None, q_scale=None):
    """Indexer -> top-k -> sparse MLA for every query row (see include/dsa.h)."""
    T, H_I, d_I = q_idx.shape
    _, H, d_qk = q.shape
    d_v = out.shape[-1]
    _check(_lib.dsa_forward(_ptr(q_idx), _ptr(q_scale), _ptr(w), _ptr(k_idx), _ptr(k_scale), _kdtype(k_idx), _ptr(q),
                            _ptr(latent), v.c(), H_I, d_I, topk, H, d_qk, d_v, float(scale), q_chunk,
                            _ptr(out), _ptr(lse), _ptr(idx_out), _ptr(workspace),
                            0 if workspace is None else workspace.numel() * workspace.element_size(),
                            _stream(stream)), "dsa_forward")
    return out, lse


def dsa_forward_static_scratch(q_idx, w, k_idx, k_scale, q, latent, v: Varlen, topk, scale, out, lse,
                               idx_out=None, stream=None, q_scale=None):
    """dsa_forward for callers that cannot allocate device memory: the scratch
    is the library's own static device array (see include/dsa.h for who needs
    this, the size limit, and why overlapping calls must be serialised)."""
    T, H_I, d_I = q_idx.shape
    _, H, d_qk = q.shape
    d_v = out.shape[-1]
    _check(_lib.dsa_forward_static_scratch(_ptr(q_idx), _ptr(q_scale), _ptr(w), _ptr(k_idx), _ptr(k_scale),
                                           _kdtype(k_idx),
                                           _ptr(q), _ptr(latent), v.c(), H_I, d_I, topk, H, d_qk, d_v,
                                           float(scale), _ptr(out), _ptr(lse), _ptr(idx_out), _stream(stream)),
           "dsa_forward_static_scratch")
    return out, lse


def dsa_device_error(stream=None) -> int:
    """Read and clear the library's device error word (0 = no device wait gave up)."""
    code = ctypes.c_int32(0)
    st = _lib.dsa_device_error(ctypes.byref(code), _stream(stream))
    if st not in (DSA_OK, DSA_ERR_DEVICE_TIMEOUT):
        raise DSAError(st, "dsa_device_error")
    return int(code.value)


def dsa_debug_wait_selftest(limit_cycles: int, stream=None):
    """Launch the one-wait self-test kernel whose wait gives up after
    ``limit_cycles`` device cycles (read the result with dsa_device_error)."""
    _check(_lib.dsa_debug_wait_selftest(int(limit_cycles), _stream(stream)), "dsa_debug_wait_selftest")


def dsa_debug_wait_profile(reset: bool = True):
    """Per wait site (cycles, completed waits) from a profiling build, or None."""
    n = 64
    cyc = (ctypes.c_uint64 * n)()
    cnt = (ctypes.c_uint64 * n)()
    st = _lib.dsa_debug_wait_profile(cyc, cnt, n, 1 if reset else 0)
    if st == DSA_ERR_UNSUPPORTED:
        return None
    _check(st, "dsa_debug_wait_profile")
    return {i: (int(cyc[i]), int(cnt[i])) for i in range(n) if cnt[i]}
