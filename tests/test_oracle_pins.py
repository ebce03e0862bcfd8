"""Pins of the CPU oracle against things other than itself.

Each check ties one step of the oracle to the format definitions (through
torch's own dtypes), to an independent library routine (numpy einsum, numpy
lexsort, torch scaled_dot_product_attention), to exact integer arithmetic, to
the Hadamard identity Hq.Hk = q.k named on the transformers page ("DeepSeek
Sparse Attention (DSA)", item 1), or to closed forms of softmax attention.
"""
import math

import numpy as np
import pytest
import torch

import dsa_inputs as di

pytestmark = pytest.mark.filterwarnings("ignore::UserWarning")


def _f64(t):
    if t.dtype == torch.float8_e4m3fn:
        return t.to(torch.float64)
    return t.to(torch.float64)


def _spec(q_lens=(5, 1, 7), kv_lens=(9, 20, 7), **kw):
    base = dict(H_I=4, d_I=32, topk=8, H=4, d_qk=80, d_v=64, seed=11)
    base.update(kw)
    return di.Spec("small", tuple(q_lens), tuple(kv_lens), **base)


def positions(spec):
    out = []
    for b in range(spec.B):
        for i in range(spec.q_lens[b]):
            out.append((b, spec.kv_lens[b] - spec.q_lens[b] + i))
    return out


# ---------------------------------------------------------------- formats

def test_e4m3_decode_exhaustive(oracle_lib):
    """All 256 byte patterns against torch.float8_e4m3fn (OCP E4M3, NaN at S.1111.111)."""
    ref = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn)
    ref = ref.to(torch.float64).numpy()
    for b in range(256):
        got = oracle_lib.e4m3_to_double(b)
        if math.isnan(ref[b]):
            assert math.isnan(got), b
        else:
            assert got == ref[b], (b, got, ref[b])
    assert oracle_lib.e4m3_to_double(0x7E) == 448.0
    assert oracle_lib.e4m3_to_double(0x01) == 2.0 ** -9


def test_bf16_decode_random_patterns(oracle_lib):
    g = np.random.default_rng(0)
    bits = g.integers(0, 1 << 16, size=4000, dtype=np.int64)
    bits = bits[((bits >> 7) & 0xFF) != 0xFF]       # finite patterns only
    ref = torch.from_numpy(bits.astype(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([oracle_lib.bf16_to_double(int(b)) for b in bits])
    assert np.array_equal(got, ref)


# ---------------------------------------------------------------- indexer

def _einsum_scores(d, spec):
    """Brute force with numpy einsum over torch-decoded float64 inputs."""
    q = _f64(d["q_idx"]).numpy()
    w = d["w"].to(torch.float64).numpy()
    k = _f64(d["k_idx"]).numpy()
    if d["k_scale"] is not None:
        k = k * d["k_scale"].to(torch.float64).numpy()[:, None]
    cu_k = d["cu_k"].tolist()
    ld = max(spec.kv_lens)
    out = np.full((spec.T, ld), -np.inf)
    for t, (b, pos) in enumerate(positions(spec)):
        keys = k[cu_k[b]:cu_k[b] + pos + 1]
        logits = np.einsum("jd,sd->sj", q[t], keys)
        out[t, :pos + 1] = np.einsum("sj,j->s", np.maximum(logits, 0.0), w[t])
    return out


@pytest.mark.parametrize("kfp8", [False, True])
def test_scores_match_einsum(oracle_lib, kfp8):
    spec = _spec(kfp8=kfp8)
    d = di.make_inputs(spec)
    got = oracle_lib.indexer_scores(d["cu_q"], d["cu_k"], d["q_idx"], d["w"], d["k_idx"], d["k_scale"])
    ref = _einsum_scores(d, spec)
    fin = np.isfinite(ref)
    assert np.array_equal(fin, np.isfinite(got))
    np.testing.assert_allclose(got[fin], ref[fin], rtol=1e-12, atol=1e-12)


def test_scores_exact_on_integer_inputs(oracle_lib):
    """Tiny integer workload: the score is an integer; int64 arithmetic gives it exactly."""
    spec = di.config("tiny")
    d = di.make_inputs(spec)
    got = oracle_lib.indexer_scores(d["cu_q"], d["cu_k"], d["q_idx"], d["w"], d["k_idx"])
    q = d["q_idx"].to(torch.int64).numpy()
    w = d["w"].to(torch.int64).numpy()
    k = d["k_idx"].to(torch.int64).numpy()
    assert np.array_equal(d["w"].to(torch.int64).to(torch.float32), d["w"])
    for t in range(spec.T):
        logits = q[t] @ k[: t + 1].T                     # [H_I, t+1] int64
        ref = (np.maximum(logits, 0) * w[t][:, None]).sum(0)
        assert np.array_equal(got[t, : t + 1], ref.astype(np.float64)), t
        assert np.all(np.isneginf(got[t, t + 1:]))
    assert np.abs(got[np.isfinite(got)]).max() <= 4 * 3 * 32 * 9


def _sylvester(n):
    H = np.array([[1.0]])
    while H.shape[0] < n:
        H = np.block([[H, H], [H, -H]])
    return H


def test_hadamard_rotation_leaves_scores_unchanged(oracle_lib):
    """Orthogonal H: I(Hq, Hk) = I(q, k) (the transformers page's identity Hq.Hk = q.k)."""
    spec = _spec(d_I=32)
    d = di.make_inputs(spec)
    H = _sylvester(32) / math.sqrt(32)
    q = _f64(d["q_idx"]).numpy() @ H.T
    k = _f64(d["k_idx"]).numpy() @ H.T
    base = oracle_lib.indexer_scores(d["cu_q"], d["cu_k"], d["q_idx"], d["w"], d["k_idx"])
    rot = oracle_lib.indexer_scores(d["cu_q"], d["cu_k"], q, d["w"], k)
    fin = np.isfinite(base)
    np.testing.assert_allclose(rot[fin], base[fin], rtol=1e-12, atol=1e-10)


def test_unnormalised_hadamard_scales_integer_scores_exactly(oracle_lib):
    """Unnormalised Sylvester H on integer inputs: I' = d_I * I exactly, same top-k."""
    spec = di.config("tiny")
    d = di.make_inputs(spec)
    H = _sylvester(spec.d_I)
    q = _f64(d["q_idx"]).numpy() @ H.T
    k = _f64(d["k_idx"]).numpy() @ H.T
    base = oracle_lib.indexer_scores(d["cu_q"], d["cu_k"], d["q_idx"], d["w"], d["k_idx"])
    rot = oracle_lib.indexer_scores(d["cu_q"], d["cu_k"], q, d["w"], k)
    fin = np.isfinite(base)
    assert np.array_equal(rot[fin], spec.d_I * base[fin])
    a = oracle_lib.topk(d["cu_q"], d["cu_k"], base, spec.topk)
    b = oracle_lib.topk(d["cu_q"], d["cu_k"], rot, spec.topk)
    assert np.array_equal(a, b)


# ---------------------------------------------------------------- top-k

def _lexsort_topk(scores, spec, k):
    out = np.full((spec.T, k), -1, dtype=np.int32)
    for t, (b, pos) in enumerate(positions(spec)):
        s = scores[t, : pos + 1]
        order = np.lexsort((np.arange(pos + 1), -s))     # score desc, then index asc
        sel = order[:k]
        out[t, : sel.size] = sel
    return out


@pytest.mark.parametrize("levels", [3, 1000])
def test_topk_matches_lexsort_with_ties(oracle_lib, levels):
    spec = _spec(q_lens=(40, 3, 17), kv_lens=(64, 3, 90))
    g = np.random.default_rng(levels)
    ld = max(spec.kv_lens)
    scores = g.integers(-levels, levels + 1, size=(spec.T, ld)).astype(np.float64)
    scores[g.random(scores.shape) < 0.05] = -0.0                 # -0 ties +0
    for k in (1, 7, 16, 100):
        got = oracle_lib.topk(spec_cu(spec)[0], spec_cu(spec)[1], scores, k)
        assert np.array_equal(got, _lexsort_topk(scores, spec, k)), k


def spec_cu(spec):
    return di.cu_seqlens(spec.q_lens), di.cu_seqlens(spec.kv_lens)


def test_topk_invariants(oracle_lib):
    spec = di.config("tiny")
    d = di.make_inputs(spec)
    sc = oracle_lib.indexer_scores(d["cu_q"], d["cu_k"], d["q_idx"], d["w"], d["k_idx"])
    ix = oracle_lib.topk(d["cu_q"], d["cu_k"], sc, spec.topk)
    for t in range(spec.T):
        pos = t
        sel = ix[t][ix[t] >= 0]
        assert sel.size == min(spec.topk, pos + 1)
        assert np.all(ix[t][sel.size:] == -1)
        assert len(set(sel.tolist())) == sel.size and sel.max() <= pos
        rest = np.setdiff1d(np.arange(pos + 1), sel)
        if rest.size:
            worst = sc[t, sel].min()
            assert sc[t, rest].max() <= worst
            # among equal scores at the boundary the lower index wins
            tied = rest[sc[t, rest] == worst]
            assert tied.size == 0 or tied.min() > sel[sc[t, sel] == worst].max()


# ---------------------------------------------------------------- attention

def _sdpa_reference(d, spec, rows_pos):
    """torch SDPA in float64 with a causal (offset) mask, per sequence, MQA-expanded."""
    q = d["q"].to(torch.float64)
    c = d["latent"].to(torch.float64)
    cu_q, cu_k = d["cu_q"].tolist(), d["cu_k"].tolist()
    outs, lses = [], []
    for b in range(spec.B):
        qb = q[cu_q[b]:cu_q[b + 1]].transpose(0, 1)[None]            # [1,H,Lq,Dqk]
        kb = c[cu_k[b]:cu_k[b + 1]]
        Lq, Lk = qb.shape[2], kb.shape[0]
        k4 = kb[None, None].expand(1, spec.H, Lk, spec.d_qk)
        v4 = kb[None, None, :, : spec.d_v].expand(1, spec.H, Lk, spec.d_v)
        pos = torch.arange(Lq)[:, None] + (Lk - Lq)
        mask = torch.arange(Lk)[None, :] <= pos
        o = torch.nn.functional.scaled_dot_product_attention(qb, k4, v4, attn_mask=mask,
                                                             scale=spec.softmax_scale)
        logits = (qb @ k4.transpose(-1, -2)) * spec.softmax_scale
        lse = torch.logsumexp(logits.masked_fill(~mask, -math.inf), dim=-1)
        outs.append(o[0].transpose(0, 1))
        lses.append(lse[0].transpose(0, 1))
    return torch.cat(outs).numpy(), torch.cat(lses).numpy()


def test_sparse_equals_dense_causal_when_topk_covers_everything(oracle_lib):
    spec = _spec(q_lens=(6, 1, 9), kv_lens=(10, 33, 9), topk=64)
    d = di.make_inputs(spec)
    sc = oracle_lib.indexer_scores(d["cu_q"], d["cu_k"], d["q_idx"], d["w"], d["k_idx"])
    ix = oracle_lib.topk(d["cu_q"], d["cu_k"], sc, spec.topk)
    out, lse = oracle_lib.sparse_mla(d["cu_q"], d["cu_k"], d["q"], d["latent"], ix,
                                     spec.softmax_scale, spec.d_v)
    ref_o, ref_l = _sdpa_reference(d, spec, None)
    np.testing.assert_allclose(out, ref_o, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(lse, ref_l, rtol=1e-12, atol=1e-12)


def test_sparse_equals_additive_mask_formulation(oracle_lib):
    spec = _spec(q_lens=(12, 4), kv_lens=(30, 50), topk=8)
    d = di.make_inputs(spec)
    sc = oracle_lib.indexer_scores(d["cu_q"], d["cu_k"], d["q_idx"], d["w"], d["k_idx"])
    ix = oracle_lib.topk(d["cu_q"], d["cu_k"], sc, spec.topk)
    a = oracle_lib.sparse_mla(d["cu_q"], d["cu_k"], d["q"], d["latent"], ix, spec.softmax_scale, spec.d_v)
    b = oracle_lib.dense_mla_masked(d["cu_q"], d["cu_k"], d["q"], d["latent"], ix,
                                    spec.softmax_scale, spec.d_v)
    np.testing.assert_allclose(a[0], b[0], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(a[1], b[1], rtol=1e-13, atol=1e-13)


def test_attention_closed_forms(oracle_lib):
    spec = _spec(q_lens=(3,), kv_lens=(40,), topk=16)
    d = di.make_inputs(spec)
    cu_q, cu_k = d["cu_q"], d["cu_k"]
    c = d["latent"].to(torch.float64).numpy()
    q = d["q"].to(torch.float64).numpy()
    # a single selected row: out is that row's value part, lse its logit
    ix = np.full((spec.T, spec.topk), -1, np.int32)
    ix[:, 0] = [0, 5, 39]
    out, lse = oracle_lib.sparse_mla(cu_q, cu_k, d["q"], d["latent"], ix, spec.softmax_scale, spec.d_v)
    for t, s in enumerate([0, 5, 39]):
        np.testing.assert_array_equal(out[t], np.broadcast_to(c[s, : spec.d_v], out[t].shape))
        np.testing.assert_allclose(lse[t], spec.softmax_scale * (q[t] @ c[s]), rtol=1e-13)
    # q = 0: uniform weights, out = mean of the selected rows, lse = log(count)
    zero_q = torch.zeros_like(d["q"])
    ix = np.full((spec.T, spec.topk), -1, np.int32)
    ix[:, :5] = [[1, 2, 3, 4, 7]] * spec.T
    ix[2, 5] = 38
    out, lse = oracle_lib.sparse_mla(cu_q, cu_k, zero_q, d["latent"], ix, spec.softmax_scale, spec.d_v)
    for t in range(spec.T):
        sel = ix[t][ix[t] >= 0]
        np.testing.assert_allclose(out[t], np.broadcast_to(c[sel, : spec.d_v].mean(0), out[t].shape),
                                   rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(lse[t], math.log(sel.size), rtol=1e-14)


def test_attention_ignores_order_padding_and_invalid_entries(oracle_lib):
    spec = _spec(q_lens=(4,), kv_lens=(64,), topk=16)
    d = di.make_inputs(spec)
    g = np.random.default_rng(3)
    ix = np.stack([g.permutation(61 + t)[:12] for t in range(4)]).astype(np.int32)
    ix = np.concatenate([ix, np.full((4, 4), -1, np.int32)], 1)
    a = oracle_lib.sparse_mla(d["cu_q"], d["cu_k"], d["q"], d["latent"], ix, spec.softmax_scale, spec.d_v)
    perm = ix[:, g.permutation(16)]
    b = oracle_lib.sparse_mla(d["cu_q"], d["cu_k"], d["q"], d["latent"], perm, spec.softmax_scale, spec.d_v)
    np.testing.assert_allclose(a[0], b[0], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(a[1], b[1], rtol=1e-13)
    bad = ix.copy()
    bad[:, 12] = 63          # beyond pos for rows 0..2 (causal), valid for row 3 (pos 63)
    bad[:, 13] = 9999        # beyond the sequence
    c = oracle_lib.sparse_mla(d["cu_q"], d["cu_k"], d["q"], d["latent"], bad, spec.softmax_scale, spec.d_v)
    np.testing.assert_allclose(c[0][:3], a[0][:3], rtol=1e-12, atol=1e-13)
    assert not np.allclose(c[0][3], a[0][3])


def test_no_valid_entry_gives_zero_output_and_neg_inf_lse(oracle_lib):
    spec = _spec(q_lens=(2,), kv_lens=(5,), topk=4)
    d = di.make_inputs(spec)
    ix = np.full((2, 4), -1, np.int32)
    out, lse = oracle_lib.sparse_mla(d["cu_q"], d["cu_k"], d["q"], d["latent"], ix,
                                     spec.softmax_scale, spec.d_v)
    assert np.all(out == 0) and np.all(np.isneginf(lse))
