"""GPU parity of the RoPE the attention applies to its queries while loading
them ("DeepSeek-V3.2-Exp" token-ids page, released config: qk_rope_head_dim
64; "DeepSeek-V3.2" transformers doc: MLA) against the oracle's rotation
followed by the oracle's attention.

The kernel rotates in fp32 and rounds the rotated query to bf16 before its
MMAs; the oracle's rotation is exact (double) and is rounded to bf16 here
before its attention, so the two sides can differ by a rounding decision on
a few query elements, which the attention tolerance covers."""
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
    """The usual RoPE angles pos * base^(-2i/d) as a (cos, sin) table, fp32."""
    i = np.arange(d_rope // 2, dtype=np.float64)
    ang = np.arange(max_pos, dtype=np.float64)[:, None] * base ** (-2.0 * i / d_rope)[None, :]
    return np.stack([np.cos(ang), np.sin(ang)], axis=-1).astype(np.float32)


def random_selection(cu_q, cu_k, topk, seed):
    g = np.random.default_rng(seed)
    pos = P.row_positions(cu_q, cu_k)
    idx = np.full((len(pos), topk), -1, np.int32)
    for r, p in enumerate(pos):
        n = min(topk, p + 1)
        idx[r, :n] = g.permutation(p + 1)[:n]
    return idx


@pytest.mark.parametrize("kind", ["tiny", "released"])
def test_attention_rope_matches_the_oracle(dsa, oracle_lib, kind):
    if kind == "tiny":
        spec = di.with_lengths(di.config("tiny"), (5, 2), (40, 90), dist="normal", seed=51)
    else:
        spec = di.Spec("rope", (3, 1), (3000, 2600), seed=52, **RELEASED)
    d = di.make_inputs(spec, tensors=("q", "latent"))
    v = dsa.Varlen(d["cu_q"], d["cu_k"], "cuda")
    idx = random_selection(d["cu_q"], d["cu_k"], spec.topk, seed=53)
    d_rope = spec.d_qk - spec.d_v
    table = rope_table(max(spec.kv_lens), d_rope)
    out = torch.full((spec.T, spec.H, spec.d_v), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((spec.T, spec.H), float("nan"), dtype=torch.float32, device="cuda")
    idx_d = torch.from_numpy(idx).cuda()
    dsa.dsa_sparse_mla_attn(d["q"].cuda(), d["latent"].cuda(), idx_d, v, 0, spec.T, spec.softmax_scale, out, lse,
                            rope=torch.from_numpy(table).cuda())
    torch.cuda.synchronize()
    assert dsa.dsa_device_error() == 0
    pos = P.row_positions(d["cu_q"], d["cu_k"])
    q_rot = d["q"].clone()
    pe = oracle_lib.rope(d["q"][:, :, spec.d_v:], np.repeat(np.asarray(pos)[:, None], spec.H, axis=1), table)
    q_rot[:, :, spec.d_v:] = torch.from_numpy(pe).to(torch.bfloat16)
    o_out, o_lse = oracle_lib.sparse_mla(d["cu_q"], d["cu_k"], q_rot, d["latent"], idx, spec.softmax_scale,
                                         spec.d_v)
    P.assert_attention_close(out.float().cpu().numpy(), lse.cpu().numpy(), o_out, o_lse, f"rope {kind}")
    # the table was applied: without it the result is far from the rotated one
    out0 = torch.empty_like(out)
    dsa.dsa_sparse_mla_attn(d["q"].cuda(), d["latent"].cuda(), idx_d, v, 0, spec.T, spec.softmax_scale, out0)
    torch.cuda.synchronize()
    assert (out0.float() - out.float()).abs().max().item() > 1e-2


def test_attention_rope_table_too_short_is_rejected(dsa):
    spec = di.Spec("rope-short", (1,), (300,), seed=54, **RELEASED)
    d = di.make_inputs(spec, tensors=("q", "latent"))
    v = dsa.Varlen(d["cu_q"], d["cu_k"], "cuda")
    idx = torch.zeros((1, spec.topk), dtype=torch.int32, device="cuda")
    out = torch.empty((1, spec.H, spec.d_v), dtype=torch.bfloat16, device="cuda")
    short = torch.zeros((299, 32, 2), dtype=torch.float32, device="cuda")
    with pytest.raises(RuntimeError):
        dsa.dsa_sparse_mla_attn(d["q"].cuda(), d["latent"].cuda(), idx, v, 0, 1, spec.softmax_scale, out,
                                rope=short)
