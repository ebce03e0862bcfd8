"""CPU oracle for the DSA hot path -- TEST INFRASTRUCTURE ONLY.

A ctypes front end over ``dsa_oracle.c``: a literal, double-precision
restatement of the lightning-indexer scores, the per-query top-k selection and
the absorbed-MQA MLA attention over the selected tokens ("DeepSeek-V3.2",
transformers model doc, section "DeepSeek Sparse Attention (DSA)", items 1 and
2; "DeepSeek-V3.2-Exp" token-ids page, released config and causal mask).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It shares no code with the CUDA library
and never imports it.  Inputs are CPU torch tensors or numpy arrays: bf16
tensors are handed over as raw bit patterns and decoded by the C code, fp8
index keys as raw bytes plus one float32 scale per key row.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dsa_oracle.c")
_DEFAULT_LIB = os.path.join(_HERE, "liboracle.so")
_LIB = _DEFAULT_LIB
_lock = threading.Lock()
_lib = None

BF16, E4M3, F64 = 0, 1, 2

_I32P = ctypes.POINTER(ctypes.c_int32)
_F64P = ctypes.POINTER(ctypes.c_double)
_F32P = ctypes.POINTER(ctypes.c_float)


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, OpenMP) into ``oracle/liboracle.so``."""
    return compile_source(_SRC, _DEFAULT_LIB, force)


def compile_source(src: str, out: str, force: bool = False) -> str:
    """gcc -O2 -fopenmp build of one oracle source file into a shared library."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", src, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, out)
    return out


def _load():
    global _lib
    with _lock:
        if _lib is None:
            if _LIB == _DEFAULT_LIB:
                build()
            lib = ctypes.CDLL(_LIB)
            lib.oracle_bf16_to_double.restype = ctypes.c_double
            lib.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
            lib.oracle_e4m3_to_double.restype = ctypes.c_double
            lib.oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
            lib.oracle_num_threads.restype = ctypes.c_int
            vp = ctypes.c_void_p
            lib.oracle_indexer_scores.restype = ctypes.c_int
            lib.oracle_indexer_scores.argtypes = [
                ctypes.c_int, _I32P, _I32P, ctypes.c_int, ctypes.c_int,
                ctypes.c_int, vp, _F64P, ctypes.c_int, vp, _F32P,
                ctypes.c_int64, _I32P, _F64P, ctypes.c_int64]
            lib.oracle_topk.restype = ctypes.c_int
            lib.oracle_topk.argtypes = [
                ctypes.c_int, _I32P, _I32P, ctypes.c_int64, _I32P, _F64P, ctypes.c_int64,
                ctypes.c_int, _I32P]
            lib.oracle_hadamard.restype = ctypes.c_int
            lib.oracle_hadamard.argtypes = [ctypes.c_int64, ctypes.c_int, _F64P, _F64P, ctypes.c_int]
            lib.oracle_double_to_e4m3.restype = ctypes.c_uint8
            lib.oracle_double_to_e4m3.argtypes = [ctypes.c_double]
            lib.oracle_quant_e4m3_pow2.restype = ctypes.c_int
            lib.oracle_quant_e4m3_pow2.argtypes = [ctypes.c_int64, ctypes.c_int, _F64P, vp, _F32P]
            lib.oracle_indexer_scores_fp8.restype = ctypes.c_int
            lib.oracle_indexer_scores_fp8.argtypes = [
                ctypes.c_int, _I32P, _I32P, ctypes.c_int, ctypes.c_int, vp, _F32P, _F64P, vp, _F32P,
                ctypes.c_int64, _I32P, _F64P, ctypes.c_int64]
            lib.oracle_rope.restype = ctypes.c_int
            lib.oracle_rope.argtypes = [ctypes.c_int64, ctypes.c_int, _F64P, _I32P, _F64P, ctypes.c_int64, _F64P]
            lib.oracle_up_proj.restype = ctypes.c_int
            lib.oracle_up_proj.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int, _F64P,
                                           ctypes.c_int, vp, _F64P]
            lib.oracle_paged_rows.restype = ctypes.c_int
            lib.oracle_paged_rows.argtypes = [ctypes.c_int, _I32P, _I32P, ctypes.c_int, ctypes.c_int,
                                              ctypes.c_int64, ctypes.POINTER(ctypes.c_int64)]
            lib.oracle_quant_e4m3_amax.restype = ctypes.c_int
            lib.oracle_quant_e4m3_amax.argtypes = [ctypes.c_int64, ctypes.c_int, _F64P, vp, _F32P]
            for name in ("oracle_sparse_mla", "oracle_dense_mla_masked"):
                fn = getattr(lib, name)
                fn.restype = ctypes.c_int
                fn.argtypes = [
                    ctypes.c_int, _I32P, _I32P, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                    ctypes.c_int, vp, ctypes.c_int, vp, ctypes.c_int64, _I32P, _I32P,
                    ctypes.c_int, ctypes.c_double, _F64P, _F64P]
            _lib = lib
    return _lib


def num_threads() -> int:
    """Host threads the oracle's OpenMP loops use."""
    return int(_load().oracle_num_threads())


def _np(x):
    """CPU numpy view of a torch tensor or array (no copy when contiguous)."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous()
            if x.dtype == torch.bfloat16:
                return x.view(torch.int16).numpy().view(np.uint16), BF16
            if x.dtype == torch.float8_e4m3fn:
                return x.view(torch.uint8).numpy(), E4M3
            x = x.numpy()
    except ImportError:  # pragma: no cover
        pass
    x = np.ascontiguousarray(x)
    if x.dtype == np.uint16:
        return x, BF16
    if x.dtype == np.uint8:
        return x, E4M3
    return np.ascontiguousarray(x, dtype=np.float64), F64


def _ptr(a, typ):
    return a.ctypes.data_as(typ)


def _i32(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def _rows(rows, T):
    if rows is None:
        return None, T
    r = _i32(rows)
    return r, int(r.size)


def bf16_to_double(bits: int) -> float:
    return float(_load().oracle_bf16_to_double(int(bits)))


def e4m3_to_double(byte: int) -> float:
    return float(_load().oracle_e4m3_to_double(int(byte)))


def indexer_scores(cu_q, cu_k, q_idx, w, k_idx, k_scale=None, rows=None, ld=None):
    """Lightning-indexer scores, [n_rows, ld] float64 (-inf above the diagonal).

    q_idx [T, H_I, d_I] (bf16 or float64); w [T, H_I]; k_idx [sum kv, d_I]
    (bf16, float64, or float8_e4m3fn/uint8 bytes with ``k_scale`` [sum kv]).
    """
    lib = _load()
    cu_q, cu_k = _i32(cu_q), _i32(cu_k)
    B = cu_q.size - 1
    T = int(cu_q[-1])
    qa, qk = _np(q_idx)
    ka, kk = _np(k_idx)
    T_, H_I, d_I = qa.shape
    assert T_ == T, (T_, T)
    wa = np.ascontiguousarray(np.asarray(_np(w)[0], dtype=np.float64)).reshape(T, H_I)
    sa = None
    if kk == E4M3:
        assert k_scale is not None
        sa = np.ascontiguousarray(np.asarray(_np(k_scale)[0], dtype=np.float32))
    kv_lens = np.diff(cu_k)
    if ld is None:
        ld = int(kv_lens.max()) if kv_lens.size else 1
    r, n = _rows(rows, T)
    out = np.full((n, ld), -np.inf, dtype=np.float64)   # columns past kv_len stay -inf
    rc = lib.oracle_indexer_scores(
        B, _ptr(cu_q, _I32P), _ptr(cu_k, _I32P), H_I, d_I, qk, qa.ctypes.data_as(ctypes.c_void_p),
        _ptr(wa, _F64P), kk, ka.ctypes.data_as(ctypes.c_void_p),
        None if sa is None else _ptr(sa, _F32P), n, None if r is None else _ptr(r, _I32P),
        _ptr(out, _F64P), ld)
    if rc != 0:
        raise ValueError("oracle_indexer_scores rejected its arguments")
    return out


def topk(cu_q, cu_k, scores, k, rows=None):
    """Top-k selection, [n_rows, k] int32 in (score desc, index asc) order, -1 padded."""
    lib = _load()
    cu_q, cu_k = _i32(cu_q), _i32(cu_k)
    B = cu_q.size - 1
    T = int(cu_q[-1])
    sc = np.ascontiguousarray(np.asarray(scores, dtype=np.float64))
    r, n = _rows(rows, T)
    assert sc.shape[0] == n
    out = np.empty((n, k), dtype=np.int32)
    rc = lib.oracle_topk(B, _ptr(cu_q, _I32P), _ptr(cu_k, _I32P), n,
                         None if r is None else _ptr(r, _I32P), _ptr(sc, _F64P), sc.shape[1], k,
                         _ptr(out, _I32P))
    if rc != 0:
        raise ValueError("oracle_topk rejected its arguments")
    return out


def _mla(fn_name, cu_q, cu_k, q, latent, idx, scale, d_v, rows):
    lib = _load()
    cu_q, cu_k = _i32(cu_q), _i32(cu_k)
    B = cu_q.size - 1
    T = int(cu_q[-1])
    qa, qk = _np(q)
    ca, ck = _np(latent)
    _, H, d_qk = qa.shape
    ix = _i32(idx)
    r, n = _rows(rows, T)
    assert ix.shape[0] == n
    k = ix.shape[1]
    out = np.empty((n, H, d_v), dtype=np.float64)
    lse = np.empty((n, H), dtype=np.float64)
    rc = getattr(lib, fn_name)(
        B, _ptr(cu_q, _I32P), _ptr(cu_k, _I32P), H, d_qk, d_v, qk,
        qa.ctypes.data_as(ctypes.c_void_p), ck, ca.ctypes.data_as(ctypes.c_void_p), n,
        None if r is None else _ptr(r, _I32P), _ptr(ix, _I32P), k, float(scale),
        _ptr(out, _F64P), _ptr(lse, _F64P))
    if rc != 0:
        raise ValueError(f"{fn_name} rejected its arguments")
    return out, lse


def sparse_mla(cu_q, cu_k, q, latent, idx, scale, d_v, rows=None):
    """Absorbed-MQA MLA attention over the selected rows: (out [n,H,Dv], lse [n,H])."""
    return _mla("oracle_sparse_mla", cu_q, cu_k, q, latent, idx, scale, d_v, rows)


def dense_mla_masked(cu_q, cu_k, q, latent, idx, scale, d_v, rows=None):
    """Dense MLA attention with the additive selection mask (same result as sparse_mla)."""
    return _mla("oracle_dense_mla_masked", cu_q, cu_k, q, latent, idx, scale, d_v, rows)


def forward(cu_q, cu_k, q_idx, w, k_idx, k_scale, q, latent, k, scale, d_v, rows=None):
    """All three steps for the requested rows: (scores, idx, out, lse)."""
    sc = indexer_scores(cu_q, cu_k, q_idx, w, k_idx, k_scale, rows=rows)
    ix = topk(cu_q, cu_k, sc, k, rows=rows)
    out, lse = sparse_mla(cu_q, cu_k, q, latent, ix, scale, d_v, rows=rows)
    return sc, ix, out, lse


def _f64(x):
    a, kind = _np(x)
    if kind == BF16:
        import torch
        a = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).double().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def hadamard(x, normalize=True):
    """Sylvester-Hadamard rotation of the last axis (a power of two):
    orthonormal (H / sqrt(d)) by default, the +-1 matrix H itself otherwise."""
    xa = _f64(x)
    d = xa.shape[-1]
    y = np.empty_like(xa)
    if _load().oracle_hadamard(xa.size // d, d, _ptr(xa, _F64P), _ptr(y, _F64P), 1 if normalize else 0) != 0:
        raise ValueError("oracle_hadamard: the length must be a power of two")
    return y


def double_to_e4m3(v: float) -> int:
    """The e4m3 byte nearest to v (ties to even, saturating at +-448)."""
    return int(_load().oracle_double_to_e4m3(float(v)))


def quant_e4m3_pow2(x):
    """Per-vector (last axis) e4m3 quantization with power-of-two scales:
    (bytes uint8 [..., d], scale float32 [...])."""
    xa = _f64(x)
    d = xa.shape[-1]
    n = xa.size // d
    q = np.empty(xa.shape, dtype=np.uint8)
    sc = np.empty(xa.shape[:-1], dtype=np.float32)
    if _load().oracle_quant_e4m3_pow2(n, d, _ptr(xa, _F64P), q.ctypes.data_as(ctypes.c_void_p),
                                      _ptr(sc, _F32P)) != 0:
        raise ValueError("oracle_quant_e4m3_pow2 rejected its arguments")
    return q, sc


def indexer_scores_fp8(cu_q, cu_k, q_bytes, q_scale, w, k_bytes, k_scale, rows=None, ld=None):
    """Indexer scores with e4m3 index queries [T, H_I, d_I] (scales [T, H_I])
    and e4m3 index keys [sum kv, d_I] (scales [sum kv]): [n_rows, ld] float64."""
    lib = _load()
    cu_q, cu_k = _i32(cu_q), _i32(cu_k)
    B = cu_q.size - 1
    T = int(cu_q[-1])
    qa, _ = _np(q_bytes)
    ka, _ = _np(k_bytes)
    T_, H_I, d_I = qa.shape
    assert T_ == T
    qs = np.ascontiguousarray(np.asarray(_np(q_scale)[0], dtype=np.float32)).reshape(T, H_I)
    ks = np.ascontiguousarray(np.asarray(_np(k_scale)[0], dtype=np.float32))
    wa = np.ascontiguousarray(np.asarray(_np(w)[0], dtype=np.float64)).reshape(T, H_I)
    kv_lens = np.diff(cu_k)
    if ld is None:
        ld = int(kv_lens.max()) if kv_lens.size else 1
    r, n = _rows(rows, T)
    out = np.full((n, ld), -np.inf, dtype=np.float64)
    rc = lib.oracle_indexer_scores_fp8(
        B, _ptr(cu_q, _I32P), _ptr(cu_k, _I32P), H_I, d_I, qa.ctypes.data_as(ctypes.c_void_p), _ptr(qs, _F32P),
        _ptr(wa, _F64P), ka.ctypes.data_as(ctypes.c_void_p), _ptr(ks, _F32P), n,
        None if r is None else _ptr(r, _I32P), _ptr(out, _F64P), ld)
    if rc != 0:
        raise ValueError("oracle_indexer_scores_fp8 rejected its arguments")
    return out


def rope(x, pos, freqs):
    """Rotary embedding of the last axis (consecutive pairs as complex numbers)
    by the table freqs [max_pos, d/2, 2] = (cos, sin) at each vector's position."""
    xa = _f64(x)
    d = xa.shape[-1]
    n = xa.size // d
    pa = _i32(np.broadcast_to(np.asarray(pos), xa.shape[:-1]).reshape(-1))
    fa = np.ascontiguousarray(np.asarray(freqs, dtype=np.float64))
    y = np.empty_like(xa)
    if _load().oracle_rope(n, d, _ptr(xa, _F64P), _ptr(pa, _I32P), _ptr(fa, _F64P), fa.shape[0],
                           _ptr(y, _F64P)) != 0:
        raise ValueError("oracle_rope rejected its arguments")
    return y


def up_proj(o, w_uv):
    """Per-head up-projection y[r, h, :] = o[r, h, :] @ w_uv[h] ([n, H, d_c] x [H, d_c, d_v])."""
    oa = _f64(o)
    wa, wk = _np(w_uv)
    n, H, d_c = oa.shape
    H_, d_c_, d_v = wa.shape
    assert (H_, d_c_) == (H, d_c)
    y = np.empty((n, H, d_v), dtype=np.float64)
    if _load().oracle_up_proj(n, H, d_c, d_v, _ptr(oa, _F64P), wk, wa.ctypes.data_as(ctypes.c_void_p),
                              _ptr(y, _F64P)) != 0:
        raise ValueError("oracle_up_proj rejected its arguments")
    return y


def paged_rows(cu_k, block_table=None, page_size=0, n_pages=0):
    """Cache row of every entry, in packed order: rows[cu_k[b] + s] for entry s
    of sequence b (int64; -1 where the block table has no valid page).
    block_table: None (packed caches) or int32 [B, pages_per_seq]."""
    ck = _i32(cu_k)
    B = ck.shape[0] - 1
    rows = np.empty(int(ck[-1]), dtype=np.int64)
    bt = None if block_table is None else _i32(block_table)
    pps = 0 if bt is None else bt.shape[1]
    if _load().oracle_paged_rows(B, _ptr(ck, _I32P), None if bt is None else _ptr(bt, _I32P), page_size, pps,
                                 n_pages, rows.ctypes.data_as(ctypes.POINTER(ctypes.c_int64))) != 0:
        raise ValueError("oracle_paged_rows rejected its arguments")
    return rows


def quant_e4m3_amax(x):
    """Per-vector (last axis) e4m3 quantization with scale amax / 448 in
    float32: (bytes uint8 [..., d], scale float32 [...])."""
    xa = _f64(x)
    d = xa.shape[-1]
    n = xa.size // d
    q = np.empty(xa.shape, dtype=np.uint8)
    sc = np.empty(xa.shape[:-1], dtype=np.float32)
    if _load().oracle_quant_e4m3_amax(n, d, _ptr(xa, _F64P), q.ctypes.data_as(ctypes.c_void_p),
                                      _ptr(sc, _F32P)) != 0:
        raise ValueError("oracle_quant_e4m3_amax rejected its arguments")
    return q, sc


KQ_BF16, KQ_E4M3_AMAX, KQ_E4M3_HADAMARD = 0, 1, 2


def cache_append(cu_q, cu_k, latent_new=None, kidx_new=None, k_quant=KQ_BF16, rope_freqs=None, d_v=None,
                 block_table=None, page_size=0, n_pages=0):
    """What appending a step's new tokens writes into the caches.

    The new tokens are the step's query rows: row t is entry pos(t) of its
    sequence (the lengths in cu_k already count it).  Returns a dict with
    rows (int64 [T], the cache row of each new token, -1 if unmapped),
    latent (float64 [T, d_qk]: the latent row, its columns from d_v on
    rotated by rope_freqs at pos(t) when a table is given), and the index-key
    row: k (float64 [T, d_I] values, k_quant KQ_BF16) or k (uint8 bytes) with
    k_scale (float32 [T]) for the two e4m3 forms (amax / 448 scale, or the
    Hadamard rotation with a power-of-two scale)."""
    cq, ck = _i32(cu_q), _i32(cu_k)
    T = int(cq[-1])
    pos = np.empty(T, dtype=np.int64)
    packed = np.empty(T, dtype=np.int64)
    for b in range(cq.shape[0] - 1):
        q_len, kv_len = int(cq[b + 1] - cq[b]), int(ck[b + 1] - ck[b])
        for i in range(q_len):
            pos[cq[b] + i] = kv_len - q_len + i
            packed[cq[b] + i] = ck[b] + kv_len - q_len + i
    out = dict(rows=paged_rows(ck, block_table, page_size, n_pages)[packed], pos=pos)
    if latent_new is not None:
        lat = _f64(latent_new).copy()
        if rope_freqs is not None:
            lat[:, d_v:] = rope(lat[:, d_v:], pos.astype(np.int32), rope_freqs)
        out["latent"] = lat
    if kidx_new is not None:
        k = _f64(kidx_new)
        if k_quant == KQ_BF16:
            out["k"], out["k_scale"] = k.copy(), None
        elif k_quant == KQ_E4M3_AMAX:
            out["k"], out["k_scale"] = quant_e4m3_amax(k)
        elif k_quant == KQ_E4M3_HADAMARD:
            out["k"], out["k_scale"] = quant_e4m3_pow2(hadamard(k, normalize=False))
        else:
            raise ValueError("k_quant")
    return out


class use_library:
    """Context manager that points this module at another build of dsa_oracle.c.

    Used by the mutation tests, which compile copies of the source with one
    planted mistake and check that the pins reject each copy.
    """

    def __init__(self, so_path: str):
        self.so_path = so_path

    def __enter__(self):
        global _lib, _LIB
        with _lock:
            self._saved = (_lib, _LIB)
            _lib, _LIB = None, self.so_path
        _load()
        return self

    def __exit__(self, *exc):
        global _lib, _LIB
        with _lock:
            _lib, _LIB = self._saved
        return False
