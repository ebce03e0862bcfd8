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
