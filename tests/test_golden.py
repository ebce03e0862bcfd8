"""Stored fixtures under tests/golden/: the released layer dims as printed on
the pages, and the tiny workload's expected values written by
tests/golden/make_golden.py from the oracle alone."""
import json
import math
import os

import numpy as np

import dsa_inputs as di

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_released_dims_follow_the_printed_config():
    """The released-shape workloads take their dims from the config excerpt on
    the DeepSeek-V3.2-Exp token-ids page."""
    cfg = json.load(open(os.path.join(GOLDEN, "released_config.json")))
    spec = di.config("prefill4k")
    assert spec.H == cfg["n_heads"]
    assert spec.H_I == cfg["index_n_heads"]
    assert spec.d_I == cfg["index_head_dim"]
    assert spec.topk == cfg["index_topk"]
    # absorbed MQA: one latent row (kv_lora_rank) plus the shared RoPE key per token
    assert spec.d_qk == cfg["kv_lora_rank"] + cfg["qk_rope_head_dim"]
    assert spec.d_v == cfg["kv_lora_rank"]
    # softmax scale of the un-absorbed head dim: 1/sqrt(qk_nope + qk_rope)
    assert math.isclose(spec.softmax_scale, 1.0 / math.sqrt(cfg["qk_nope_head_dim"] + cfg["qk_rope_head_dim"]))
    for name in ("decode128k", "ragged128k", "prefill32k", "prefill64k"):
        s = di.config(name)
        assert (s.H, s.H_I, s.d_I, s.topk, s.d_qk, s.d_v) == (spec.H, spec.H_I, spec.d_I, spec.topk, spec.d_qk, spec.d_v)


def test_oracle_reproduces_tiny_golden(oracle_lib):
    g = json.load(open(os.path.join(GOLDEN, "tiny_expected.json")))
    spec = di.config("tiny")
    d = di.make_inputs(spec)
    sc = oracle_lib.indexer_scores(d["cu_q"], d["cu_k"], d["q_idx"], d["w"], d["k_idx"])
    ix = oracle_lib.topk(d["cu_q"], d["cu_k"], sc, spec.topk)
    out, lse = oracle_lib.sparse_mla(d["cu_q"], d["cu_k"], d["q"], d["latent"], ix, spec.softmax_scale, spec.d_v)
    assert [sorted(int(v) for v in r if v >= 0) for r in ix] == g["topk_sets"]
    for t, row in g["score_rows"].items():
        assert sc[int(t), : int(t) + 1].tolist() == row
    assert int(np.where(np.isfinite(sc), sc, 0.0).sum()) == g["score_sum"]
    for t, row in g["lse_rows"].items():
        np.testing.assert_allclose(lse[int(t)], row, rtol=1e-13)
    np.testing.assert_allclose(out[0, 0], g["out_row0_head0"], rtol=1e-13)


def test_decode_lengths_in_range():
    s = di.config("decode128k")
    assert s.B == 64 and all(16384 <= n <= 131072 for n in s.kv_lens)
    assert s.q_lens == (1,) * 64 and s.kfp8


def test_ragged_has_duplicated_keys():
    s = di.with_lengths(di.config("ragged128k"), (16, 16), (400, 1200))
    d = di.make_inputs(s)
    k = d["k_idx"].view(-1, s.d_I)
    cu = d["cu_k"].tolist()
    for b in range(2):
        seg = k[cu[b]:cu[b + 1]].float().numpy()
        uniq = np.unique(seg, axis=0).shape[0]
        assert uniq < seg.shape[0]          # some rows are copies of others
