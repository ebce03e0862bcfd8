"""Host-side pieces of bench.py that the reported numbers rest on: the
algorithmic work model (bytes and flops per stage, the roofline numerators) and
the reference arm's cut-cache sample."""
import math

import pytest
import torch

import bench
import dsa_inputs as di


def test_work_model_counts_the_definitions():
    spec = di.config("decode128k")
    w = bench.work_model(spec, True)
    kv = sum(spec.kv_lens)
    # one query per sequence at position kv_len - 1: it scores every key of its cache
    assert w["indexer"]["flops"] == kv * 2 * spec.H_I * spec.d_I
    # e4m3 key (128 B) + fp32 scale per key, the query block and weights, one fp32 score per pair
    assert w["indexer"]["bytes"] == kv * (spec.d_I + 4) + spec.T * (spec.H_I * spec.d_I * 2 + spec.H_I * 4) + kv * 4
    # every decode row here is longer than k: k selected rows per query
    assert all(n > spec.topk for n in spec.kv_lens)
    rows = spec.T * spec.topk
    assert w["attention"]["flops"] == rows * 2 * spec.H * (spec.d_qk + spec.d_v)
    assert w["attention"]["bytes"] == (rows * spec.d_qk * 2 + spec.T * (spec.H * spec.d_qk * 2 + spec.H * spec.d_v * 2
                                       + spec.H * 4) + spec.T * spec.topk * 4)
    assert w["topk"]["bytes"] == kv * 4 + spec.T * spec.topk * 4


def test_work_model_prefill_counts_causal_pairs():
    spec = di.config("tiny")
    w = bench.work_model(spec, False)
    pairs = sum(sum(kl - ql + i + 1 for i in range(ql)) for ql, kl in zip(spec.q_lens, spec.kv_lens))
    sel = sum(sum(min(spec.topk, kl - ql + i + 1) for i in range(ql)) for ql, kl in zip(spec.q_lens, spec.kv_lens))
    assert w["indexer"]["flops"] == pairs * 2 * spec.H_I * spec.d_I
    assert w["attention"]["flops"] == sel * 2 * spec.H * (spec.d_qk + spec.d_v)


def test_cut_cache_sample_keeps_each_rows_query_and_its_first_keys():
    spec = di.Spec("cut", (1, 1, 1), (40, 7, 100), H_I=4, d_I=32, topk=32, H=4, d_qk=80, d_v=64,
                   scale=1.0 / math.sqrt(80.0), seed=3)
    d = di.make_inputs(spec)
    seqs = [0, 1, 2]
    cut, lens = bench._truncated_rows(spec, d, seqs, 16)
    assert lens == [16, 7, 16]
    assert [int(x) for x in cut["cu_k"]] == [0, 16, 23, 39]
    assert [int(x) for x in cut["cu_q"]] == [0, 1, 2, 3]
    cu_k = [int(x) for x in d["cu_k"]]
    for i, b in enumerate(seqs):
        assert torch.equal(cut["q_idx"][i], d["q_idx"][b])          # one query row per sequence
        a = int(cut["cu_k"][i])
        assert torch.equal(cut["latent"][a:a + lens[i]], d["latent"][cu_k[b]:cu_k[b] + lens[i]])
