"""Seeded synthetic inputs for the DSA hot path.

This module only draws numbers; it holds none of the method's arithmetic.  It
serves both the CUDA library's tests/benchmark and the CPU oracle.

Every value is a pure function of (seed, tensor id, flat element index), so any
slice of a tensor can be regenerated on its own and the same tensor comes out
on the CPU and on a GPU.  The counter hash is SplitMix64 (Steele, Lea and
Flood, "Fast splittable pseudorandom number generators", OOPSLA 2014; the
64-bit finaliser constants published with it):

    stream key  K = mix(mix(seed) ^ tensor_id)
    element i   h = mix(K + i)          (all arithmetic mod 2^64)

Integer draws use the top 53 bits; normals use the Box-Muller transform of the
two 32-bit halves of h, evaluated in float64 and rounded once (RNE) to the
storage type.  Transcendentals may differ in the last float64 ulp between the
host and the device libm, so tests that need bit-identical inputs on both
sides generate on one device and copy.

Workload specs follow the shapes of the released DeepSeek-V3.2 layer
("DeepSeek-V3.2-Exp" token-ids page, released config: 128 heads, index_n_heads
64, index_head_dim 128, index_topk 2048, kv_lora_rank 512, qk_rope_head_dim
64) and a tiny integer-valued case whose scores are exact in fp32.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import torch

_M64 = (1 << 64) - 1


def _s64(v: int) -> int:
    v &= _M64
    return v - (1 << 64) if v >= (1 << 63) else v


_GOLDEN = _s64(0x9E3779B97F4A7C15)
_MIX1 = _s64(0xBF58476D1CE4E5B9)
_MIX2 = _s64(0x94D049BB133111EB)


def mix64_int(x: int) -> int:
    """SplitMix64 finaliser on a Python int (mod 2^64), returned unsigned."""
    z = (x + 0x9E3779B97F4A7C15) & _M64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _M64
    return z ^ (z >> 31)


def _lsr(z: torch.Tensor, s: int) -> torch.Tensor:
    """Logical right shift of int64 lanes holding uint64 bit patterns."""
    return (z >> s) & ((1 << (64 - s)) - 1)


def mix64(z: torch.Tensor) -> torch.Tensor:
    """SplitMix64 finaliser on int64 tensors (two's-complement wrap = mod 2^64)."""
    z = z + _GOLDEN
    z = (z ^ _lsr(z, 30)) * _MIX1
    z = (z ^ _lsr(z, 27)) * _MIX2
    return z ^ _lsr(z, 31)


def stream_key(seed: int, tensor_id: int) -> int:
    return mix64_int(mix64_int(seed) ^ tensor_id)


def hashes(seed: int, tensor_id: int, start: int, count: int, device) -> torch.Tensor:
    """h[i] for flat indices start .. start+count-1, int64 bit patterns."""
    key = _s64(stream_key(seed, tensor_id))
    i = torch.arange(start, start + count, dtype=torch.int64, device=device)
    return mix64(i + key)


def uniform_int(h: torch.Tensor, lo: int, hi: int) -> torch.Tensor:
    """Integers in [lo, hi] from the top 53 bits (bias < 2^-40 for small ranges)."""
    return _lsr(h, 11) % (hi - lo + 1) + lo


def normal(h: torch.Tensor) -> torch.Tensor:
    """Standard normal float64 by Box-Muller on the two 32-bit halves of h."""
    u1 = (_lsr(h, 32) + 1).to(torch.float64) * (2.0 ** -32)          # (0, 1]
    u2 = (h & 0xFFFFFFFF).to(torch.float64) * (2.0 ** -32)            # [0, 1)
    return torch.sqrt(-2.0 * torch.log(u1)) * torch.cos((2.0 * math.pi) * u2)


# tensor ids of the streams
T_QIDX, T_W, T_KIDX, T_Q, T_LAT, T_LEN, T_DUP, T_DUPSRC, T_WUV, T_O = range(1, 11)

_CHUNK = 1 << 25  # elements per generation chunk (bounded temporaries)


def _fill(out: torch.Tensor, seed: int, tid: int, start: int, kind: str, std: float = 1.0):
    """Fill a contiguous tensor whose element e has flat stream index start+e."""
    flat = out.view(-1)
    n = flat.numel()
    for c0 in range(0, n, _CHUNK):
        c1 = min(n, c0 + _CHUNK)
        h = hashes(seed, tid, start + c0, c1 - c0, out.device)
        if kind == "int3":
            v = uniform_int(h, -3, 3).to(torch.float64)
        else:
            v = normal(h) * std
        flat[c0:c1] = v.to(out.dtype)
        del h, v


def _fill_rows(out, seed, tid, row_ranges, row_width, kind, std=1.0):
    """Fill rows of `out` from global row ranges [(global_row0, n_rows, local_row0), ...]."""
    for g0, n, l0 in row_ranges:
        if n:
            _fill(out[l0:l0 + n], seed, tid, g0 * row_width, kind, std)


@dataclass(frozen=True)
class Spec:
    """One synthetic workload: dims, lengths and value distributions."""
    name: str
    q_lens: tuple
    kv_lens: tuple
    H_I: int = 64
    d_I: int = 128
    topk: int = 2048
    H: int = 128
    d_qk: int = 576
    d_v: int = 512
    dist: str = "normal"          # "normal" or "int3" (integers -3..3)
    seed: int = 0
    kfp8: bool = False            # index-key cache as e4m3 + one fp32 scale per key
    dup_frac: float = 0.0         # fraction of key positions copied from another position
    scale: float = field(default=0.0)

    @property
    def B(self):
        return len(self.q_lens)

    @property
    def softmax_scale(self):
        return self.scale if self.scale else 1.0 / math.sqrt(self.d_qk)

    @property
    def T(self):
        return sum(self.q_lens)

    @property
    def total_kv(self):
        return sum(self.kv_lens)


def decode_lengths(seed: int, B: int, lo: int, hi: int):
    h = hashes(seed, T_LEN, 0, B, "cpu")
    return tuple(int(v) for v in uniform_int(h, lo, hi))


RELEASED = dict(H_I=64, d_I=128, topk=2048, H=128, d_qk=576, d_v=512, scale=1.0 / math.sqrt(192.0))


def config(name: str) -> Spec:
    """The named workloads (shapes and distributions of the released layer)."""
    if name == "tiny":
        return Spec("tiny", (256,), (256,), H_I=4, d_I=32, topk=32, H=4, d_qk=80, d_v=64,
                    dist="int3", seed=0, scale=1.0 / math.sqrt(80.0))
    if name == "prefill4k":
        return Spec("prefill4k", (4096,), (4096,), seed=1, **RELEASED)
    if name == "prefill32k":
        return Spec("prefill32k", (32768,), (32768,), seed=2, **RELEASED)
    if name == "prefill64k":
        return Spec("prefill64k", (65536,), (65536,), seed=2, **RELEASED)
    if name == "decode128k":
        kv = decode_lengths(3, 64, 16384, 131072)
        return Spec("decode128k", (1,) * 64, kv, seed=3, kfp8=True, **RELEASED)
    if name == "ragged128k":
        prefix = (0, 4096, 8192, 16384, 32768, 65536, 98304, 131072)
        return Spec("ragged128k", (2048,) * 8, tuple(p + 2048 for p in prefix), seed=4,
                    dup_frac=0.01, **RELEASED)
    raise KeyError(name)


CONFIG_NAMES = ("tiny", "prefill4k", "prefill32k", "prefill64k", "decode128k", "ragged128k")


def cu_seqlens(lens):
    out = [0]
    for n in lens:
        out.append(out[-1] + int(n))
    return torch.tensor(out, dtype=torch.int32)


def _dup_map(spec: Spec, b: int, kv_len: int):
    """Positions of sequence b that copy another position: (targets, sources)."""
    if spec.dup_frac <= 0.0 or kv_len < 2:
        return None
    per = int(round(1.0 / spec.dup_frac))
    base = sum(spec.kv_lens[:b])
    h = hashes(spec.seed, T_DUP, base, kv_len, "cpu")
    tgt = torch.nonzero(uniform_int(h, 0, per - 1) == 0).view(-1)
    if tgt.numel() == 0:
        return None
    hs = hashes(spec.seed, T_DUPSRC, base, kv_len, "cpu")[tgt]
    src = uniform_int(hs, 0, kv_len - 1)
    keep = src != tgt
    return tgt[keep], src[keep]


ALL_TENSORS = ("q_idx", "w", "q", "latent", "k_idx")


def make_inputs(spec: Spec, device="cpu", seqs=None, tensors=ALL_TENSORS):
    """Generate the workload's tensors on `device`.

    seqs: optional list of sequence indices; only those sequences are built
    (their values are identical to the same rows of the full workload).
    tensors: which of q_idx, w, q, latent, k_idx (with k_scale) to build; the
    others are None (a tensor's values do not depend on which others are built).

    Returns a dict with cu_q/cu_k (int32, CPU), q_idx [T,H_I,d_I] bf16,
    w [T,H_I] fp32, k_idx [sum kv,d_I] (bf16, or float8_e4m3fn with
    k_scale [sum kv] fp32), q [T,H,d_qk] bf16, latent [sum kv,d_qk] bf16.
    """
    if seqs is None:
        seqs = list(range(spec.B))
    cu_q_full = cu_seqlens(spec.q_lens).tolist()
    cu_k_full = cu_seqlens(spec.kv_lens).tolist()
    q_lens = [spec.q_lens[b] for b in seqs]
    kv_lens = [spec.kv_lens[b] for b in seqs]
    cu_q, cu_k = cu_seqlens(q_lens), cu_seqlens(kv_lens)
    T, S = int(cu_q[-1]), int(cu_k[-1])
    qrows = [(cu_q_full[b], spec.q_lens[b], int(cu_q[i])) for i, b in enumerate(seqs)]
    krows = [(cu_k_full[b], spec.kv_lens[b], int(cu_k[i])) for i, b in enumerate(seqs)]
    d = dict(spec=spec, cu_q=cu_q, cu_k=cu_k, seqs=list(seqs))
    bf = torch.bfloat16
    kind = spec.dist
    d.update(q_idx=None, w=None, q=None, latent=None, k_idx=None, k_scale=None)
    if "q_idx" in tensors:
        d["q_idx"] = torch.empty((T, spec.H_I, spec.d_I), dtype=bf, device=device)
        _fill_rows(d["q_idx"], spec.seed, T_QIDX, qrows, spec.H_I * spec.d_I, kind)
    if "w" in tensors:
        d["w"] = torch.empty((T, spec.H_I), dtype=torch.float32, device=device)
        _fill_rows(d["w"], spec.seed, T_W, qrows, spec.H_I, kind, std=1.0 / 8.0)
    if "q" in tensors:
        d["q"] = torch.empty((T, spec.H, spec.d_qk), dtype=bf, device=device)
        _fill_rows(d["q"], spec.seed, T_Q, qrows, spec.H * spec.d_qk, kind)
    if "latent" in tensors:
        d["latent"] = torch.empty((S, spec.d_qk), dtype=bf, device=device)
        _fill_rows(d["latent"], spec.seed, T_LAT, krows, spec.d_qk, kind)
    if "k_idx" not in tensors:
        pass
    elif spec.kfp8:
        kf = torch.empty((S, spec.d_I), dtype=torch.float64, device=device)
        _fill_rows(kf, spec.seed, T_KIDX, krows, spec.d_I, kind)
        # Quantised index-key cache: one fp32 scale per key = amax / 448 (the
        # largest finite e4m3 magnitude); bytes = e4m3 (RNE) of x / scale
        # after rounding that quotient to fp32.
        amax = kf.abs().amax(dim=1).clamp_min(1e-30)
        k_scale = (amax / 448.0).to(torch.float32)
        kq = (kf / k_scale.to(torch.float64)[:, None]).clamp(-448.0, 448.0)
        d["k_idx"] = kq.to(torch.float32).to(torch.float8_e4m3fn)
        d["k_scale"] = k_scale
        del kf, kq
    else:
        d["k_idx"] = torch.empty((S, spec.d_I), dtype=bf, device=device)
        _fill_rows(d["k_idx"], spec.seed, T_KIDX, krows, spec.d_I, kind)
        d["k_scale"] = None
    for i, b in enumerate(seqs):
        m = _dup_map(spec, b, spec.kv_lens[b])
        if m is None:
            continue
        tgt, src = (m[0] + int(cu_k[i])).to(device), (m[1] + int(cu_k[i])).to(device)
        for name in ("k_idx", "latent") + (("k_scale",) if spec.kfp8 else ()):
            t = d[name]
            if t is None:
                continue
            vals = t[src].clone()          # read every source before any write
            t[tgt] = vals
    return d


def with_lengths(spec: Spec, q_lens, kv_lens, **kw) -> Spec:
    """A copy of `spec` with other sequence lengths (and optional overrides)."""
    return replace(spec, q_lens=tuple(q_lens), kv_lens=tuple(kv_lens), **kw)


def make_w_uv(seed: int, H: int = 128, d_c: int = 512, d_v: int = 128, device="cpu"):
    """Per-head value up-projection weights W_UV [H, d_c, d_v] bf16, normal
    with standard deviation 1/sqrt(d_c) (random init: no trained weights)."""
    w = torch.empty((H, d_c, d_v), dtype=torch.bfloat16, device=device)
    _fill(w, seed, T_WUV, 0, "normal", std=1.0 / math.sqrt(d_c))
    return w


def make_latent_out(seed: int, n: int, H: int = 128, d_c: int = 512, device="cpu"):
    """An attention output in latent space, o [n, H, d_c] bf16 (standard normal)."""
    o = torch.empty((n, H, d_c), dtype=torch.bfloat16, device=device)
    _fill(o, seed, T_O, 0, "normal")
    return o
