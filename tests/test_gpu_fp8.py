"""GPU parity of the FP8 indexer ("DeepSeek-V3.2", transformers doc, DSA item 1:
FP8 with a Hadamard transform; released config: ue8m0 scales) against the
oracle: the rotation and quantization kernel, and the kind::f8f6f4 indexer on
the quantized operands.

Quantization compares bytes exactly, except where the oracle's own quotient
(Hx)/s lies within 2^-20 (relative) of the midpoint between two e4m3 values:
there the kernel's fp32 rotation may legitimately round to the other
neighbour, and the two codes must then be adjacent.  Scales must match
exactly unless max|Hx| / 448 sits within 2^-20 of a power of two."""
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


def _e4m3_values(oracle_lib):
    return np.array([oracle_lib.e4m3_to_double(c) for c in range(256)])


def test_hadamard_quantize_matches_the_oracle(dsa, oracle_lib):
    g = torch.Generator().manual_seed(7)
    x = (torch.randn(4096, 128, generator=g) * torch.exp(torch.randn(4096, 1, generator=g) * 2)).to(torch.bfloat16)
    x[5] = 0                                   # a zero vector: scale 1, zero bytes
    x[6, :] = 0
    x[6, 3] = 1.0                              # one-hot: every rotated value is +-1
    q, s = dsa.dsa_hadamard_quantize_fp8(x.cuda())
    torch.cuda.synchronize()
    gq = q.view(torch.uint8).cpu().numpy()
    gs = s.cpu().numpy()
    hx = oracle_lib.hadamard(x, normalize=False)
    oq, os_ = oracle_lib.quant_e4m3_pow2(hx)
    amax = np.abs(hx).max(axis=1)
    ratio = np.where(amax > 0, amax / 448.0, 1.0)
    near_pow2 = np.abs(np.log2(ratio) - np.round(np.log2(ratio))) < 2.0 ** -20
    assert np.all((gs == os_) | near_pow2), "scales"
    vals = _e4m3_values(oracle_lib)
    bad = 0
    for v in np.unique(np.nonzero(gq != oq)[0]):
        if gs[v] != os_[v]:
            continue                           # a scale at a power-of-two boundary (checked above)
        for i in np.nonzero(gq[v] != oq[v])[0]:
            y = hx[v, i] / os_[v]
            a, b = vals[gq[v, i]], vals[oq[v, i]]
            mid = (a + b) / 2.0
            assert abs(y - mid) <= 2.0 ** -20 * abs(y), (v, i, y, a, b)
            bad += 1
    assert bad <= 8, f"{bad} codes decided differently"
    assert np.all(gq[5] & 0x7F == 0) and gs[5] == 1.0
    assert gs[6] == 2.0 ** -8 and np.all(np.abs(vals[gq[6]]) == 256.0)   # 1 = 256 * 2^-8


@pytest.mark.parametrize("q_lens,kv_lens", [
    ((1, 1, 1, 1, 1), (1, 129, 1000, 4097, 20000)),     # decode: the persistent schedule
    ((1,) * 8, (20000, 130, 65536, 1, 7000, 128, 129, 30000)),   # decode: sequences split across CTAs
    ((2, 1), (3000, 500)),                              # decode-like blocks of one query (grid)
    ((37, 3, 130), (600, 128, 2200)),                   # prefill blocks of four queries, ragged tails
], ids=["decode", "decode-long", "decode-grid", "prefill"])
def test_fp8_indexer_scores_match_the_oracle(dsa, oracle_lib, q_lens, kv_lens):
    spec = di.Spec("fp8", tuple(q_lens), tuple(kv_lens), seed=31, **RELEASED)
    d = di.make_inputs(spec, tensors=("q_idx", "w", "k_idx"))
    v = dsa.Varlen(d["cu_q"], d["cu_k"], "cuda")
    qq, qs = dsa.dsa_hadamard_quantize_fp8(d["q_idx"].cuda())
    kq, ks = dsa.dsa_hadamard_quantize_fp8(d["k_idx"].cuda())
    ld = (max(kv_lens) + 3) // 4 * 4
    sc = torch.full((spec.T, ld), float("nan"), dtype=torch.float32, device="cuda")
    pm = torch.full((spec.T, dsa.part_max_ld(ld)), float("nan"), dtype=torch.float32, device="cuda")
    dsa.dsa_indexer_scores(qq, d["w"].cuda(), kq, ks, v, 0, spec.T, sc, part_max=pm, q_scale=qs)
    torch.cuda.synchronize()
    assert dsa.dsa_device_error() == 0
    # the oracle's FP8 score of the same bytes; the unnormalised rotation's 128 divided out
    ref = oracle_lib.indexer_scores_fp8(d["cu_q"], d["cu_k"], qq.cpu(), qs.cpu(), d["w"], kq.cpu(), ks.cpu(), ld=ld)
    ref = ref / 128.0
    pos = P.row_positions(d["cu_q"], d["cu_k"])
    got = sc.cpu().numpy()
    P.assert_scores_close(got, ref, pos)
    got_pm = pm.cpu().numpy()
    for r, p_ in enumerate(pos):
        n = p_ + 1
        P_ = (n + 7) // 8
        row = np.full(P_ * 8, -np.inf, dtype=np.float32)
        row[:n] = got[r, :n]
        assert np.array_equal(got_pm[r, :P_], row.reshape(P_, 8).max(axis=1))


def test_fp8_forward_end_to_end(dsa, oracle_lib):
    """dsa_forward in FP8 mode: the selections agree with the oracle's top-k
    over the oracle's FP8 scores (within the score tolerance), and the
    attention matches the oracle on the GPU's selection."""
    spec = di.Spec("fp8fwd", (3, 1), (2600, 5000), seed=32, **RELEASED)
    d = di.make_inputs(spec)
    dd = P.to_device(d)
    v = dsa.Varlen(d["cu_q"], d["cu_k"], "cuda")
    qq, qs = dsa.dsa_hadamard_quantize_fp8(dd["q_idx"])
    kq, ks = dsa.dsa_hadamard_quantize_fp8(dd["k_idx"])
    ws = torch.empty(dsa.dsa_forward_workspace_size(v, spec.topk), dtype=torch.uint8, device="cuda")
    out = torch.empty((spec.T, spec.H, spec.d_v), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((spec.T, spec.H), dtype=torch.float32, device="cuda")
    idx = torch.empty((spec.T, spec.topk), dtype=torch.int32, device="cuda")
    dsa.dsa_forward(qq, dd["w"], kq, ks, dd["q"], dd["latent"], v, spec.topk, spec.softmax_scale, out, lse, ws,
                    idx_out=idx, q_scale=qs)
    torch.cuda.synchronize()
    assert dsa.dsa_device_error() == 0
    sc = oracle_lib.indexer_scores_fp8(d["cu_q"], d["cu_k"], qq.cpu(), qs.cpu(), d["w"], kq.cpu(), ks.cpu()) / 128.0
    o_idx = oracle_lib.topk(d["cu_q"], d["cu_k"], sc, spec.topk)
    pos = P.row_positions(d["cu_q"], d["cu_k"])
    g_idx = idx.cpu().numpy()
    P.assert_index_sets(g_idx, o_idx, sc, pos)
    a_out, a_lse = oracle_lib.sparse_mla(d["cu_q"], d["cu_k"], d["q"], d["latent"], g_idx, spec.softmax_scale, spec.d_v)
    P.assert_attention_close(out.float().cpu().numpy(), lse.cpu().numpy(), a_out, a_lse, "fp8 forward")
