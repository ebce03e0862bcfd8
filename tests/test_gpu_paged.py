"""Paged caches and the in-kernel cache append ("DeepSeek-V3.2",
transformers doc, DSA: the indexer's per-token key cache beside the main
cache, growing or preallocated, updated every step by update_indexer).

  - append: every written row against the oracle's cache_append (bf16 copies
    and amax/448 e4m3 bit-exact; the RoPE columns within one bf16 rounding of
    the oracle's exact rotation; the Hadamard form by the rule of the FP8
    quantization test), every other row untouched;
  - paged forward: the same workload through a shuffled page pool whose free
    rows hold garbage (NaN codes included) gives bit-identical selections,
    out and lse to the packed layout, for every indexer kernel kind;
  - a missing page records device error code 2 and nothing faults."""
import math

import numpy as np
import pytest
import torch

import dsa_inputs as di
from tests import parity as P

pytestmark = pytest.mark.gpu

RELEASED = dict(H_I=64, d_I=128, topk=2048, H=128, d_qk=576, d_v=512, scale=1.0 / math.sqrt(192.0))


@pytest.fixture(scope="module")
def dsa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import sparse_attention_long_07_b200 as m
    return m


def rope_table(max_pos, d_rope, base=10000.0):
    i = np.arange(d_rope // 2, dtype=np.float64)
    ang = np.arange(max_pos, dtype=np.float64)[:, None] * base ** (-2.0 * i / d_rope)[None, :]
    return np.stack([np.cos(ang), np.sin(ang)], axis=-1).astype(np.float32)


def page_pool(kv_lens, page_size, seed, spare=3):
    """A shuffled block table with room for every sequence, and the pool size."""
    g = np.random.default_rng(seed)
    pps = max(1, max((n + page_size - 1) // page_size for n in kv_lens)) + 1
    n_pages = len(kv_lens) * pps + spare
    bt = g.permutation(n_pages)[:len(kv_lens) * pps].reshape(len(kv_lens), pps).astype(np.int32)
    return bt, n_pages


def _bf16_near(gpu_bits, ref):
    """gpu bf16 values are the bf16 rounding of ref, or its neighbour when ref
    lies within 2^-20 (relative) of the midpoint between two bf16 values."""
    g = gpu_bits.astype(np.float64)
    want = torch.from_numpy(ref).to(torch.bfloat16).double().numpy()
    diff = g != want
    if diff.any():
        mid = (want[diff] + g[diff]) / 2           # the midpoint of the two neighbours
        assert np.all(np.abs(ref[diff] - mid) <= 2.0 ** -20 * np.abs(ref[diff])), "not a rounding tie"
        assert diff.sum() <= 8, f"{int(diff.sum())} elements rounded differently"


@pytest.mark.parametrize("paged", [False, True], ids=["packed", "paged"])
@pytest.mark.parametrize("shape", ["released", "tiny"])
@pytest.mark.parametrize("k_quant", [0, 1, 2], ids=["bf16", "e4m3-amax", "e4m3-hadamard"])
def test_cache_append_matches_the_oracle(dsa, oracle_lib, paged, shape, k_quant):
    if shape == "tiny" and k_quant != 0:
        pytest.skip("the e4m3 forms have the released key width only")
    d_qk, d_v, d_i = (576, 512, 128) if shape == "released" else (80, 64, 32)
    q_lens, kv_lens = (3, 1, 5, 1), (3, 70, 200, 129)          # a prefill from empty, decode steps, a prefill
    cu_q = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)
    cu_k = np.concatenate([[0], np.cumsum(kv_lens)]).astype(np.int32)
    T = int(cu_q[-1])
    g = torch.Generator().manual_seed(61)
    lat = (torch.randn(T, d_qk, generator=g) * 2).to(torch.bfloat16)
    kid = (torch.randn(T, d_i, generator=g) * torch.exp(torch.randn(T, 1, generator=g))).to(torch.bfloat16)
    if paged:
        bt, n_pages = page_pool(kv_lens, 64, seed=62)
        rows_total, paging = n_pages * 64, dict(block_table=bt, page_size=64, n_pages=n_pages)
        v = dsa.Varlen(cu_q, cu_k, "cuda", block_table=torch.from_numpy(bt).cuda(), page_size=64, n_pages=n_pages)
    else:
        rows_total, paging = int(cu_k[-1]), {}
        v = dsa.Varlen(cu_q, cu_k, "cuda")
    table = rope_table(int(max(kv_lens)), d_qk - d_v)
    lat_cache = torch.full((rows_total, d_qk), -7.0, dtype=torch.bfloat16, device="cuda")
    if k_quant == 0:
        k_cache = torch.full((rows_total, d_i), -7.0, dtype=torch.bfloat16, device="cuda")
        k_scale = None
    else:
        k_cache = torch.full((rows_total, d_i), 0x55, dtype=torch.uint8, device="cuda")
        k_scale = torch.full((rows_total,), -1.0, dtype=torch.float32, device="cuda")
    dsa.dsa_cache_append(v, lat.cuda(), lat_cache, kid.cuda(), k_cache, k_scale, k_quant=k_quant,
                         rope=torch.from_numpy(table).cuda())
    torch.cuda.synchronize()
    assert dsa.dsa_device_error() == 0
    ref = oracle_lib.cache_append(cu_q, cu_k, lat, kid, k_quant, table, d_v, **paging)
    rows = ref["rows"]
    assert np.all(rows >= 0)
    got_lat = lat_cache.cpu()
    # latent: the first d_v columns are bit copies, the RoPE columns one rounding of the exact rotation
    assert torch.equal(got_lat[rows][:, :d_v], lat[:, :d_v])
    _bf16_near(got_lat[rows][:, d_v:].double().numpy(), ref["latent"][:, d_v:])
    others = np.setdiff1d(np.arange(rows_total), rows)
    assert torch.all(got_lat[others] == -7.0)
    got_k = k_cache.cpu()
    if k_quant == 0:
        assert torch.equal(got_k[rows], kid)
        assert torch.all(got_k[others] == -7.0)
        return
    gk, gs = got_k[rows].numpy(), k_scale.cpu().numpy()[rows]
    assert np.all(got_k[others].numpy() == 0x55) and np.all(k_scale.cpu().numpy()[others] == -1.0)
    if k_quant == 1:
        assert np.array_equal(gs, ref["k_scale"]) and np.array_equal(gk, ref["k"])
    else:
        hx = oracle_lib.hadamard(kid, normalize=False)
        vals = np.array([oracle_lib.e4m3_to_double(c) for c in range(256)])
        assert np.array_equal(gs, ref["k_scale"])
        for v_, i in zip(*np.nonzero(gk != ref["k"])):
            y = hx[v_, i] / gs[v_]
            mid = (vals[gk[v_, i]] + vals[ref["k"][v_, i]]) / 2.0
            assert abs(y - mid) <= 2.0 ** -20 * abs(y)


def _paged_copy(oracle_lib, d, page_size, seed):
    """The workload's caches moved into a shuffled page pool whose other rows hold garbage."""
    kv_lens = [int(d["cu_k"][b + 1] - d["cu_k"][b]) for b in range(len(d["cu_k"]) - 1)]
    bt, n_pages = page_pool(kv_lens, page_size, seed)
    rows = torch.from_numpy(oracle_lib.paged_rows(d["cu_k"], bt, page_size, n_pages))
    n = n_pages * page_size
    g = torch.Generator().manual_seed(seed)
    out = {}
    lat = torch.randn(n, d["latent"].shape[1], generator=g).to(torch.bfloat16)
    lat[rows] = d["latent"]
    out["latent"] = lat
    if d["k_idx"].dtype == torch.float8_e4m3fn:
        k = torch.randint(0, 256, (n, d["k_idx"].shape[1]), generator=g, dtype=torch.uint8)   # NaN codes too
        k[rows] = d["k_idx"].view(torch.uint8)
        out["k_idx"] = k.view(torch.float8_e4m3fn)
        ks = torch.full((n,), float("nan"))
        ks[rows] = d["k_scale"]
        out["k_scale"] = ks
    else:
        k = torch.randn(n, d["k_idx"].shape[1], generator=g).to(torch.bfloat16)
        k[0] = float("nan")
        k[rows] = d["k_idx"]
        out["k_idx"], out["k_scale"] = k, None
    return out, torch.from_numpy(bt), n_pages


def _fwd(dsa, spec, dd, v, q_scale=None, q_idx=None, k_idx=None, k_scale=None):
    ws = torch.empty(dsa.dsa_forward_workspace_size(v, spec.topk), dtype=torch.uint8, device="cuda")
    out = torch.full((spec.T, spec.H, spec.d_v), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((spec.T, spec.H), float("nan"), dtype=torch.float32, device="cuda")
    idx = torch.full((spec.T, spec.topk), -2, dtype=torch.int32, device="cuda")
    dsa.dsa_forward(dd["q_idx"] if q_idx is None else q_idx, dd["w"], dd["k_idx"] if k_idx is None else k_idx,
                    dd["k_scale"] if k_scale is None else k_scale, dd["q"], dd["latent"], v, spec.topk,
                    spec.softmax_scale, out, lse, ws, idx_out=idx, q_scale=q_scale)
    torch.cuda.synchronize()
    assert dsa.dsa_device_error() == 0
    return out, lse, idx


CASES = [
    ("decode-e4m3", (1, 1, 1), (300, 5000, 2049), True, False),       # persistent indexer
    ("prefill-e4m3", (40, 3), (700, 2600), True, False),             # grid indexer, 4 queries per CTA
    ("prefill-bf16", (1, 30), (3000, 900), False, False),            # bf16 keys
    ("fp8-indexer", (1, 9), (2500, 1300), True, True),               # e4m3 queries and keys
    ("fp8-decode", (1, 1, 1), (300, 5000, 2049), True, True),        # persistent FP8 indexer
]


@pytest.mark.parametrize("page_size", [64, 128])
@pytest.mark.parametrize("name,q_lens,kv_lens,kfp8,qfp8", CASES, ids=[c[0] for c in CASES])
def test_paged_forward_is_bit_identical_to_packed(dsa, oracle_lib, page_size, name, q_lens, kv_lens, kfp8, qfp8):
    spec = di.Spec(name, q_lens, kv_lens, seed=63, kfp8=kfp8 and not qfp8, **RELEASED)
    d = di.make_inputs(spec)
    qs = None
    if qfp8:
        dd0 = P.to_device(d)
        qq, qs = dsa.dsa_hadamard_quantize_fp8(dd0["q_idx"])
        kq, ks = dsa.dsa_hadamard_quantize_fp8(dd0["k_idx"])
        d["q_idx"], d["k_idx"], d["k_scale"] = qq.cpu(), kq.cpu(), ks.cpu()
    dd = P.to_device(d)
    v = dsa.Varlen(d["cu_q"], d["cu_k"], "cuda")
    ref = _fwd(dsa, spec, dd, v, q_scale=qs)
    pg, bt, n_pages = _paged_copy(oracle_lib, d, page_size, seed=64)
    pgd = P.to_device(pg)
    vp = dsa.Varlen(d["cu_q"], d["cu_k"], "cuda", block_table=bt.cuda(), page_size=page_size, n_pages=n_pages)
    dd_p = dict(dd, latent=pgd["latent"])
    got = _fwd(dsa, spec, dd_p, vp, q_scale=qs, k_idx=pgd["k_idx"], k_scale=pgd["k_scale"])
    for a, b, what in zip(ref, got, ("out", "lse", "idx")):
        assert torch.equal(a, b), what


def test_tiny_shape_paged_forward_is_bit_identical(dsa, oracle_lib):
    spec = di.with_lengths(di.config("tiny"), (9, 1), (140, 300))
    d = di.make_inputs(spec)
    dd = P.to_device(d)
    v = dsa.Varlen(d["cu_q"], d["cu_k"], "cuda")
    ref = _fwd(dsa, spec, dd, v)
    pg, bt, n_pages = _paged_copy(oracle_lib, d, 64, seed=65)
    pgd = P.to_device(pg)
    vp = dsa.Varlen(d["cu_q"], d["cu_k"], "cuda", block_table=bt.cuda(), page_size=64, n_pages=n_pages)
    got = _fwd(dsa, spec, dict(dd, latent=pgd["latent"]), vp, k_idx=pgd["k_idx"], k_scale=pgd["k_scale"])
    for a, b in zip(ref, got):
        assert torch.equal(a, b)


def test_missing_page_is_recorded_and_skipped(dsa):
    spec = di.Spec("hole", (1,), (300,), seed=66, kfp8=True, **RELEASED)
    d = di.make_inputs(spec)
    dd = P.to_device(d)
    bt = torch.tensor([[0, 1, -1, 2, 3]], dtype=torch.int32)     # entries 128 .. 191 have no page
    n_pages = 4
    vp = dsa.Varlen(d["cu_q"], d["cu_k"], "cuda", block_table=bt.cuda(), page_size=64, n_pages=n_pages)
    lat = torch.zeros(n_pages * 64, spec.d_qk, dtype=torch.bfloat16)
    k = torch.zeros(n_pages * 64, spec.d_I, dtype=torch.uint8)
    ks = torch.zeros(n_pages * 64)
    for s in range(300):
        page = int(bt[0, s // 64])
        if page >= 0:
            r = page * 64 + s % 64
            lat[r], k[r], ks[r] = d["latent"][s], d["k_idx"][s].view(torch.uint8), d["k_scale"][s]
    out, lse, idx = _fwd(dsa, spec, dd, dsa.Varlen(d["cu_q"], d["cu_k"], "cuda"))   # clean reference run
    ws = torch.empty(dsa.dsa_forward_workspace_size(vp, spec.topk), dtype=torch.uint8, device="cuda")
    out_p = torch.empty_like(out)
    lse_p = torch.empty_like(lse)
    dsa.dsa_forward(dd["q_idx"], dd["w"], k.cuda().view(torch.float8_e4m3fn), ks.cuda(), dd["q"], lat.cuda(), vp,
                    spec.topk, spec.softmax_scale, out_p, lse_p, ws)
    torch.cuda.synchronize()
    code = dsa.dsa_device_error()
    assert code & 0xFF == 2, hex(code)                          # the attention met the hole
    assert torch.isfinite(lse_p).all() and torch.isfinite(out_p.float()).all()
    # the append skips a token whose page is missing
    v1 = dsa.Varlen([0, 1], [0, 150], "cuda", block_table=bt.cuda(), page_size=64, n_pages=n_pages)
    lat_new = torch.ones(1, spec.d_qk, dtype=torch.bfloat16, device="cuda")
    lat_c = lat.cuda()
    dsa.dsa_cache_append(v1, lat_new, lat_c)
    torch.cuda.synchronize()
    assert dsa.dsa_device_error() == 2 | (24 << 8)
    assert torch.equal(lat_c.cpu(), lat)
