"""GPU parity: every step of the CUDA path, called through the C ABI, against
the CPU oracle on the same seeded inputs.  Tolerances live in tests/parity.py.

Small cases run the oracle on every row (several tiles and ragged tails);
the full-size workloads run in the launch configuration the benchmark times
and compare a seeded sample of rows that the oracle computes one by one."""
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


def released(name, q_lens, kv_lens, seed, **kw):
    return di.Spec(name, tuple(q_lens), tuple(kv_lens), seed=seed, **{**RELEASED, **kw})


def gpu_scores(dsa, d, v, q_begin, q_end, ld):
    sc = torch.full((q_end - q_begin, ld), float("nan"), dtype=torch.float32, device="cuda")
    dsa.dsa_indexer_scores(d["q_idx"], d["w"], d["k_idx"], d["k_scale"], v, q_begin, q_end, sc)
    torch.cuda.synchronize()
    code = dsa.dsa_device_error()
    assert code == 0, f"device error word {code:#x} (a bounded wait gave up at site {code >> 8})"
    return sc


def ld_for(spec):
    return (max(spec.kv_lens) + 3) // 4 * 4


# ------------------------------------------------------------------ top-k

TOPK_CASES = [
    # q_lens, kv_lens, k, levels (None = continuous normal scores)
    ((1,) * 8, (1, 31, 32, 33, 2047, 2048, 2049, 5000), 2048, 3),
    ((1,) * 4, (3000, 20000, 65, 131072), 2048, None),
    ((6, 1), (70, 40), 32, 1),
    ((3,), (9000,), 2048, 0),           # every score equal: the lowest indices win
    ((1, 1), (200000, 300000), 2048, None),   # grouped part maxima; a row past the bitmap
    ((2,), (100000,), 64, 40),          # small k on a long row, ties
    ((1, 1), (40000, 16390), 2048, 0),  # all equal on rows with >= k parts: candidate overflow
    ((1, 1, 1), (20472, 20480, 20489), 2048, None),   # just below and at 1.25 k parts; a ragged last part
    ((1,), (262144,), 2048, 2),         # the longest row of the bitmap, heavy ties; parts grouped by 2
]


def host_part_max(sc, pos, ld_pm):
    """Part maxima as the indexer writes them: max over keys 8p .. 8p+7 that are <= pos."""
    pm = np.full((sc.shape[0], ld_pm), np.nan, dtype=np.float32)
    for r, p_ in enumerate(pos):
        n = p_ + 1
        P = (n + 7) // 8
        row = np.full(P * 8, -np.inf, dtype=np.float32)
        row[:n] = sc[r, :n]
        pm[r, :P] = row.reshape(P, 8).max(axis=1)
    return pm


@pytest.mark.parametrize("use_pm", [False, True], ids=["scores", "part-max"])
@pytest.mark.parametrize("case", TOPK_CASES, ids=[f"case{i}" for i in range(len(TOPK_CASES))])
def test_topk_bit_exact_against_oracle(dsa, oracle_lib, case, use_pm):
    q_lens, kv_lens, k, levels = case
    cu_q, cu_k = di.cu_seqlens(q_lens), di.cu_seqlens(kv_lens)
    T = sum(q_lens)
    ld = (max(kv_lens) + 3) // 4 * 4
    g = np.random.default_rng(len(q_lens) * 7 + k)
    if levels is None:
        sc = g.standard_normal((T, ld)).astype(np.float32)
    else:
        sc = g.integers(-levels, levels + 1, size=(T, ld)).astype(np.float32)
    sc[g.random(sc.shape) < 0.02] = -0.0
    pos = P.row_positions(cu_q, cu_k)
    for r, p_ in enumerate(pos):
        sc[r, p_ + 1:] = 1e30                        # never read: beyond the diagonal
    v = dsa.Varlen(cu_q, cu_k, "cuda")
    sc_gpu = torch.from_numpy(sc).cuda()
    pm = None
    if use_pm:
        pm = torch.from_numpy(host_part_max(sc, pos, dsa.part_max_ld(ld))).cuda()
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    dsa.dsa_topk(sc_gpu, v, 0, T, k, idx, part_max=pm)
    idx2 = torch.empty_like(idx)
    dsa.dsa_topk(sc_gpu, v, 0, T, k, idx2, part_max=pm)
    torch.cuda.synchronize()
    assert dsa.dsa_device_error() == 0
    assert torch.equal(idx, idx2), "top-k must be deterministic"
    o_rows = sc.astype(np.float64)
    for r, p_ in enumerate(pos):
        o_rows[r, p_ + 1:] = -np.inf
    ref = oracle_lib.topk(cu_q, cu_k, o_rows, k)
    got = idx.cpu().numpy()
    P.assert_index_sets(got, ref, o_rows, pos, exact=True)
    # rows with at most k candidates list them in index order; all rows end in -1 padding
    for r, p_ in enumerate(pos):
        n = min(k, p_ + 1)
        if p_ + 1 <= k:
            assert np.array_equal(got[r, :n], np.arange(n))
        assert np.all(got[r, n:] == -1)


def test_topk_on_a_chunk_of_rows(dsa, oracle_lib):
    q_lens, kv_lens, k = (5, 9), (300, 2600), 64
    cu_q, cu_k = di.cu_seqlens(q_lens), di.cu_seqlens(kv_lens)
    ld = 2600
    g = np.random.default_rng(1)
    sc = g.standard_normal((14, ld)).astype(np.float32)
    v = dsa.Varlen(cu_q, cu_k, "cuda")
    q0, q1 = 3, 11
    idx = torch.empty((q1 - q0, k), dtype=torch.int32, device="cuda")
    dsa.dsa_topk(torch.from_numpy(sc[q0:q1]).cuda(), v, q0, q1, k, idx)
    pos = P.row_positions(cu_q, cu_k)[q0:q1]
    o = sc[q0:q1].astype(np.float64)
    ref = oracle_lib.topk(cu_q, cu_k, o, k, rows=list(range(q0, q1)))
    P.assert_index_sets(idx.cpu().numpy(), ref, o, pos, exact=True)


# ------------------------------------------------------------------ indexer

def test_indexer_tiny_integer_scores_are_exact(dsa, oracle_lib):
    spec = di.config("tiny")
    d = di.make_inputs(spec)
    dd = P.to_device(d)
    v = dsa.Varlen(d["cu_q"], d["cu_k"], "cuda")
    got = gpu_scores(dsa, dd, v, 0, spec.T, 256).cpu().numpy()
    ref = oracle_lib.indexer_scores(d["cu_q"], d["cu_k"], d["q_idx"], d["w"], d["k_idx"])
    pos = P.row_positions(d["cu_q"], d["cu_k"])
    P.assert_scores_close(got, ref, pos, exact=True)
    for r, p_ in enumerate(pos):           # -inf after the diagonal inside its 128-key tile
        end = min((p_ // 128 + 1) * 128, 256)
        assert np.all(np.isneginf(got[r, p_ + 1:end]))


@pytest.mark.parametrize("kfp8,q_lens,kv_lens", [
    (False, (5, 130, 1, 7), (5, 700, 333, 2000)),
    (False, (64,), (64,)),
    (True, (1, 1, 1, 1, 2), (1, 129, 1000, 4097, 300)),
    (True, (1, 1, 1, 1, 1, 1), (1, 129, 1000, 4097, 300, 20000)),   # persistent decode schedule
    (True, (37, 3), (600, 128)),
], ids=["bf16-ragged", "bf16-square", "e4m3-decode2", "e4m3-decode1", "e4m3-prefill"])
def test_indexer_released_shape(dsa, oracle_lib, kfp8, q_lens, kv_lens):
    spec = released("idx", q_lens, kv_lens, seed=5, kfp8=kfp8)
    d = di.make_inputs(spec)
    dd = P.to_device(d)
    v = dsa.Varlen(d["cu_q"], d["cu_k"], "cuda")
    ld = ld_for(spec)
    got = gpu_scores(dsa, dd, v, 0, spec.T, ld).cpu().numpy()
    ref = oracle_lib.indexer_scores(d["cu_q"], d["cu_k"], d["q_idx"], d["w"], d["k_idx"], d["k_scale"], ld=ld)
    pos = P.row_positions(d["cu_q"], d["cu_k"])
    P.assert_scores_close(got, ref, pos)
    # the part maxima written beside the scores: exact maxima of the GPU's own scores
    pm = torch.full((spec.T, dsa.part_max_ld(ld)), float("nan"), dtype=torch.float32, device="cuda")
    again = torch.full((spec.T, ld), float("nan"), dtype=torch.float32, device="cuda")
    dsa.dsa_indexer_scores(dd["q_idx"], dd["w"], dd["k_idx"], dd["k_scale"], v, 0, spec.T, again, part_max=pm)
    torch.cuda.synchronize()
    assert dsa.dsa_device_error() == 0
    again = again.cpu().numpy()
    want = host_part_max(again, pos, pm.shape[1])
    got_pm = pm.cpu().numpy()
    for r, p_ in enumerate(pos):
        assert np.array_equal(again[r, : p_ + 1], got[r, : p_ + 1]), "scores must not depend on part_max"
        n_parts = (p_ + 1 + 7) // 8
        assert np.array_equal(got_pm[r, :n_parts], want[r, :n_parts]), f"row {r}: part maxima"
    # a sub-range of rows (chunk-relative output) gives the same values
    q0, q1 = spec.T // 3, spec.T
    part = gpu_scores(dsa, dd, v, q0, q1, ld).cpu().numpy()
    for r in range(q1 - q0):
        p_ = pos[q0 + r]
        assert np.array_equal(part[r, : p_ + 1], got[q0 + r, : p_ + 1])


def _all_e4m3_codes_case(q_lens, kv_lens):
    """Index keys whose bytes run through every finite e4m3 code (key s, dim d
    holds code (s + 7 d) mod 256, the two NaN codes replaced by zeros), scale
    1; query row t is a one-hot vector at dim d_t with sign +1 or -1 in index
    head 0, and only head 0 has weight.  Score[t, s] = ReLU(sign_t *
    decode(code)), one product per score, so the widened keys are checked
    code by code and must match the oracle exactly."""
    B = len(q_lens)
    cu_q = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)
    cu_k = np.concatenate([[0], np.cumsum(kv_lens)]).astype(np.int32)
    T, S = int(cu_q[-1]), int(cu_k[-1])
    codes = np.zeros((S, 128), dtype=np.uint8)
    for b in range(B):
        s = np.arange(kv_lens[b])[:, None]
        codes[cu_k[b]:cu_k[b + 1]] = (s + 7 * np.arange(128)[None, :]) % 256
    codes[codes == 0x7F] = 0x00
    codes[codes == 0xFF] = 0x80
    q = torch.zeros((T, 64, 128), dtype=torch.float32)
    for t in range(T):
        q[t, 0, (5 * t) % 128] = 1.0 if t % 2 == 0 else -1.0
    w = torch.zeros((T, 64), dtype=torch.float32)
    w[:, 0] = 1.0
    return {"cu_q": cu_q, "cu_k": cu_k, "q_idx": q.to(torch.bfloat16), "w": w,
            "k_idx": torch.from_numpy(codes).view(torch.float8_e4m3fn), "k_scale": torch.ones(S, dtype=torch.float32)}


@pytest.mark.parametrize("q_lens,kv_lens", [
    ((1,) * 128, tuple(256 + b for b in range(128))),   # persistent decode schedule
    ((5, 5, 5, 3), (300, 260, 400, 257)),                # query-block schedule
], ids=["decode", "prefill"])
def test_indexer_widens_every_e4m3_code_exactly(dsa, oracle_lib, q_lens, kv_lens):
    d = _all_e4m3_codes_case(q_lens, kv_lens)
    dd = P.to_device(d)
    v = dsa.Varlen(d["cu_q"], d["cu_k"], "cuda")
    ld = (max(kv_lens) + 3) // 4 * 4
    got = gpu_scores(dsa, dd, v, 0, sum(q_lens), ld).cpu().numpy()
    ref = oracle_lib.indexer_scores(d["cu_q"], d["cu_k"], d["q_idx"], d["w"], d["k_idx"], d["k_scale"], ld=ld)
    pos = P.row_positions(d["cu_q"], d["cu_k"])
    P.assert_scores_close(got, ref, pos, exact=True)


# Query tiles of very different magnitudes, one per sequence: the decode
# schedule rewrites each sequence's bf16 query tile as f16 times a power of
# two chosen from the tile's largest magnitude, so the scores must follow the
# oracle whatever that magnitude is (the tolerance is relative to the row).
# Sequence 0 holds an all-zero query (exact zeros); the last spreads its heads
# over 2^0 .. 2^-126, so most of its elements fall below f16's normal range
# once the tile is scaled and only the largest heads decide the scores.
QUERY_EXPONENTS = (None, -100, -60, -24, -10, 0, 8, 20, 60, 100, "spread")


@pytest.mark.parametrize("q_lens", [(1,) * len(QUERY_EXPONENTS), (2,) * len(QUERY_EXPONENTS)],
                         ids=["decode", "prefill"])
def test_indexer_query_magnitudes(dsa, oracle_lib, q_lens):
    kv_lens = tuple(300 + 97 * b for b in range(len(QUERY_EXPONENTS)))
    spec = released("idx", q_lens, kv_lens, seed=11, kfp8=True)
    d = di.make_inputs(spec)
    q = d["q_idx"].float()
    cu_q = d["cu_q"]
    for b, e in enumerate(QUERY_EXPONENTS):
        rows = slice(int(cu_q[b]), int(cu_q[b + 1]))
        if e is None:
            q[rows] = 0.0
        elif e == "spread":
            q[rows] = q[rows] * torch.exp2(-2.0 * torch.arange(64, dtype=torch.float32))[None, :, None]
        else:
            q[rows] = q[rows] * 2.0 ** e
    d["q_idx"] = q.to(torch.bfloat16)    # powers of two: the bf16 values scale exactly
    dd = P.to_device(d)
    v = dsa.Varlen(d["cu_q"], d["cu_k"], "cuda")
    ld = ld_for(spec)
    got = gpu_scores(dsa, dd, v, 0, spec.T, ld).cpu().numpy()
    ref = oracle_lib.indexer_scores(d["cu_q"], d["cu_k"], d["q_idx"], d["w"], d["k_idx"], d["k_scale"], ld=ld)
    pos = P.row_positions(d["cu_q"], d["cu_k"])
    P.assert_scores_close(got, ref, pos)
    for r in range(int(cu_q[1])):          # the all-zero query
        assert np.all(got[r, : pos[r] + 1] == 0.0)


# ------------------------------------------------------------------ sparse MLA

def _attention_case(dsa, oracle_lib, spec, idx=None):
    d = di.make_inputs(spec)
    dd = P.to_device(d)
    v = dsa.Varlen(d["cu_q"], d["cu_k"], "cuda")
    if idx is None:
        sc = oracle_lib.indexer_scores(d["cu_q"], d["cu_k"], d["q_idx"], d["w"], d["k_idx"], d["k_scale"])
        idx = oracle_lib.topk(d["cu_q"], d["cu_k"], sc, spec.topk)
    out = torch.full((spec.T, spec.H, spec.d_v), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((spec.T, spec.H), float("nan"), dtype=torch.float32, device="cuda")
    dsa.dsa_sparse_mla_attn(dd["q"], dd["latent"], torch.from_numpy(np.ascontiguousarray(idx)).cuda(), v, 0,
                            spec.T, spec.softmax_scale, out, lse)
    torch.cuda.synchronize()
    code = dsa.dsa_device_error()
    assert code == 0, f"device error word {code:#x} (a bounded wait gave up at site {code >> 8})"
    o_out, o_lse = oracle_lib.sparse_mla(d["cu_q"], d["cu_k"], d["q"], d["latent"], idx, spec.softmax_scale,
                                         spec.d_v)
    return out.float().cpu().numpy(), lse.cpu().numpy(), o_out, o_lse


def test_sparse_mla_tiny(dsa, oracle_lib):
    g_out, g_lse, o_out, o_lse = _attention_case(dsa, oracle_lib, di.config("tiny"))
    P.assert_attention_close(g_out, g_lse, o_out, o_lse, "tiny")


def test_sparse_mla_released_shape(dsa, oracle_lib):
    spec = released("mla", (3, 2, 1), (3000, 70, 2500), seed=6)
    g_out, g_lse, o_out, o_lse = _attention_case(dsa, oracle_lib, spec)
    P.assert_attention_close(g_out, g_lse, o_out, o_lse, "released")


def test_sparse_mla_ignores_invalid_entries_and_empty_rows(dsa, oracle_lib):
    spec = released("mla-edge", (4,), (300,), seed=7, topk=128)
    g = np.random.default_rng(2)
    idx = np.full((4, 128), -1, np.int32)
    idx[0, :50] = g.permutation(297)[:50]
    idx[0, 50:55] = [298, 299, 5000, -7, 297]      # 298, 299 beyond pos 297; 5000 beyond the cache
    idx[1, 60:70] = np.arange(10)                  # valid entries only in the second tile
    idx[3, :] = g.permutation(300)[:128]
    # row 2 keeps no valid entry
    g_out, g_lse, o_out, o_lse = _attention_case(dsa, oracle_lib, spec, idx=idx)
    P.assert_attention_close(g_out, g_lse, o_out, o_lse, "edges")
    assert np.all(g_out[2] == 0) and np.all(np.isneginf(g_lse[2]))


# ------------------------------------------------------------------ fused forward

def _forward(dsa, dd, spec, v, q_chunk=0):
    ws = torch.empty(dsa.dsa_forward_workspace_size(v, spec.topk, q_chunk), dtype=torch.uint8, device="cuda")
    out = torch.full((spec.T, spec.H, spec.d_v), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((spec.T, spec.H), float("nan"), dtype=torch.float32, device="cuda")
    idx = torch.full((spec.T, spec.topk), -2, dtype=torch.int32, device="cuda")
    dsa.dsa_forward(dd["q_idx"], dd["w"], dd["k_idx"], dd["k_scale"], dd["q"], dd["latent"], v, spec.topk,
                    spec.softmax_scale, out, lse, ws, idx_out=idx, q_chunk=q_chunk)
    torch.cuda.synchronize()
    code = dsa.dsa_device_error()
    assert code == 0, f"device error word {code:#x} (a bounded wait gave up at site {code >> 8})"
    return out, lse, idx


def test_forward_tiny_end_to_end_bit_exact_sets(dsa, oracle_lib):
    spec = di.config("tiny")
    d = di.make_inputs(spec)
    dd = P.to_device(d)
    v = dsa.Varlen(d["cu_q"], d["cu_k"], "cuda")
    out, lse, idx = _forward(dsa, dd, spec, v)
    sc, o_idx, o_out, o_lse = oracle_lib.forward(d["cu_q"], d["cu_k"], d["q_idx"], d["w"], d["k_idx"], None,
                                                 d["q"], d["latent"], spec.topk, spec.softmax_scale, spec.d_v)
    pos = P.row_positions(d["cu_q"], d["cu_k"])
    P.assert_index_sets(idx.cpu().numpy(), o_idx, sc, pos, exact=True)
    P.assert_attention_close(out.float().cpu().numpy(), lse.cpu().numpy(), o_out, o_lse, "tiny e2e")
    assert dsa.dsa_device_error() == 0


def test_forward_chunking_does_not_change_results(dsa):
    spec = released("chunk", (70, 9), (400, 3000), seed=8)
    d = di.make_inputs(spec)
    dd = P.to_device(d)
    v = dsa.Varlen(d["cu_q"], d["cu_k"], "cuda")
    a = _forward(dsa, dd, spec, v, q_chunk=0)
    b = _forward(dsa, dd, spec, v, q_chunk=17)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_back_to_back_forwards_match_separate_calls(dsa):
    """The decode indexer, the top-k and the attention start while the kernel
    before them finishes (programmatic dependent launch) and wait for it
    before touching its data.  Forwards of two batches issued back to back
    through one workspace, with nothing between them, must give exactly what
    the same calls give with the device synchronised after each."""
    specs = [released("b2b", (1,) * 12, tuple(3000 + 700 * b for b in range(12)), seed=s, kfp8=True)
             for s in (31, 32)]
    ds = [P.to_device(di.make_inputs(sp)) for sp in specs]
    vs = [dsa.Varlen(sp_d["cu_q"], sp_d["cu_k"], "cuda") for sp_d in ds]
    sp = specs[0]
    ws = torch.empty(dsa.dsa_forward_workspace_size(vs[0], sp.topk), dtype=torch.uint8, device="cuda")

    def fwd(i, out, lse, idx):
        dsa.dsa_forward(ds[i]["q_idx"], ds[i]["w"], ds[i]["k_idx"], ds[i]["k_scale"], ds[i]["q"], ds[i]["latent"],
                        vs[i], sp.topk, sp.softmax_scale, out, lse, ws, idx_out=idx)

    def bufs():
        return (torch.empty((sp.T, sp.H, sp.d_v), dtype=torch.bfloat16, device="cuda"),
                torch.empty((sp.T, sp.H), dtype=torch.float32, device="cuda"),
                torch.empty((sp.T, sp.topk), dtype=torch.int32, device="cuda"))

    ref = [bufs(), bufs()]
    for i in (0, 1):
        fwd(i, *ref[i])
        torch.cuda.synchronize()
    got = [[bufs(), bufs()] for _ in range(3)]
    for r in range(3):
        for i in (0, 1):
            fwd(i, *got[r][i])
    torch.cuda.synchronize()
    assert dsa.dsa_device_error() == 0
    for r in range(3):
        for i in (0, 1):
            for a, b in zip(got[r][i], ref[i]):
                assert torch.equal(a, b), f"round {r}, batch {i}"


def test_forward_many_sequences(dsa, oracle_lib):
    """700 decode sequences: more than the threads of a top-k (512) or an
    attention CTA (576), so the kernels' parallel count over cu_q that finds a
    row's sequence takes several rounds; rows sampled around those counts.
    Most caches are shorter than k (every key selected); three are longer."""
    g = np.random.default_rng(21)
    kv = [int(x) for x in g.integers(1, 401, size=700)]
    for b in (300, 520, 600):
        kv[b] = 5000
    spec = released("many", (1,) * 700, tuple(kv), seed=21, kfp8=True)
    d = di.make_inputs(spec)
    dd = P.to_device(d)
    v = dsa.Varlen(d["cu_q"], d["cu_k"], "cuda")
    out, lse, idx = _forward(dsa, dd, spec, v)
    rows = [0, 1, 255, 256, 300, 511, 512, 513, 520, 575, 576, 577, 600, 698, 699]
    _check_sampled(dsa, oracle_lib, spec, dd, d["cu_q"], d["cu_k"], out, lse, idx, rows)


def _check_sampled(dsa, oracle_lib, spec, dd, cu_q, cu_k, out, lse, idx, rows):
    """Oracle on sampled rows of a (possibly huge) GPU-resident workload."""
    cu_q_l, cu_k_l = list(map(int, cu_q)), list(map(int, cu_k))
    by_seq = {}
    for t in rows:
        b = max(i for i in range(len(cu_q_l) - 1) if cu_q_l[i] <= t < cu_q_l[i + 1])
        by_seq.setdefault(b, []).append(t)
    for b, ts in by_seq.items():
        q0, q1, k0, k1 = cu_q_l[b], cu_q_l[b + 1], cu_k_l[b], cu_k_l[b + 1]
        scq, sck = [0, q1 - q0], [0, k1 - k0]
        sub = {n: dd[n][q0:q1].cpu() for n in ("q_idx", "w", "q")}
        sub["k_idx"] = dd["k_idx"][k0:k1].cpu()
        sub["k_scale"] = None if dd["k_scale"] is None else dd["k_scale"][k0:k1].cpu()
        sub["latent"] = dd["latent"][k0:k1].cpu()
        local = [t - q0 for t in ts]
        sc = oracle_lib.indexer_scores(scq, sck, sub["q_idx"], sub["w"], sub["k_idx"], sub["k_scale"], rows=local)
        o_idx = oracle_lib.topk(scq, sck, sc, spec.topk, rows=local)
        pos = [(k1 - k0) - (q1 - q0) + i for i in local]
        g_idx = idx[ts].cpu().numpy()
        P.assert_index_sets(g_idx, o_idx, sc, pos)
        g_out = out[ts].float().cpu().numpy()
        g_lse = lse[ts].cpu().numpy()
        # attention on the GPU's own selection isolates the attention kernel ...
        a_out, a_lse = oracle_lib.sparse_mla(scq, sck, sub["q"], sub["latent"], g_idx, spec.softmax_scale,
                                             spec.d_v, rows=local)
        P.assert_attention_close(g_out, g_lse, a_out, a_lse, f"seq {b} (gpu idx)")
        # ... and on the oracle's selection it is the end-to-end check
        e_out, e_lse = oracle_lib.sparse_mla(scq, sck, sub["q"], sub["latent"], o_idx, spec.softmax_scale,
                                             spec.d_v, rows=local)
        P.assert_attention_close(g_out, g_lse, e_out, e_lse, f"seq {b} (oracle idx)")


def _full_size(dsa, oracle_lib, name, n_per_seq, q_chunk=0, max_seqs=None):
    spec = di.config(name)
    dd = di.make_inputs(spec, device="cuda")
    v = dsa.Varlen(dd["cu_q"], dd["cu_k"], "cuda")
    out, lse, idx = _forward(dsa, dd, spec, v, q_chunk=q_chunk)
    assert dsa.dsa_device_error() == 0
    rows = P.sample_rows(dd["cu_q"], n_per_seq, seed=spec.seed)
    if max_seqs is not None:
        # a seeded sample of sequences, always with the longest and the shortest cache
        g = np.random.default_rng(spec.seed)
        keep = set(int(b) for b in g.choice(spec.B, size=max_seqs, replace=False))
        keep |= {int(np.argmax(spec.kv_lens)), int(np.argmin(spec.kv_lens))}
        cu_q_l = list(map(int, dd["cu_q"]))
        rows = [t for t in rows if any(cu_q_l[b] <= t < cu_q_l[b + 1] for b in keep)]
    _check_sampled(dsa, oracle_lib, spec, dd, dd["cu_q"], dd["cu_k"], out, lse, idx, rows)
    del dd, out, lse, idx
    torch.cuda.empty_cache()


def test_full_prefill4k(dsa, oracle_lib):
    _full_size(dsa, oracle_lib, "prefill4k", n_per_seq=24)


def test_full_decode128k(dsa, oracle_lib):
    _full_size(dsa, oracle_lib, "decode128k", n_per_seq=1, max_seqs=8)


def test_full_ragged128k(dsa, oracle_lib):
    _full_size(dsa, oracle_lib, "ragged128k", n_per_seq=3)


def test_full_prefill32k(dsa, oracle_lib):
    _full_size(dsa, oracle_lib, "prefill32k", n_per_seq=8, q_chunk=8192)


def test_full_prefill64k(dsa, oracle_lib):
    _full_size(dsa, oracle_lib, "prefill64k", n_per_seq=8, q_chunk=8192)
