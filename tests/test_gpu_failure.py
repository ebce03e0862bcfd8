"""Failure detection on the GPU without a fault: a bounded device wait runs
out (an mbarrier that nothing arrives on, with a short limit), the kernel
records the timeout in the library's device error word and returns, the host
reads the status, kernels launched while the word is set skip their work, and
after the word is cleared the next real call passes parity."""
import numpy as np
import pytest
import torch

import dsa_inputs as di
from tests import parity as P

pytestmark = pytest.mark.gpu

SELFTEST_SITE = 99


@pytest.fixture(scope="module")
def dsa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import sparse_attention_long_07_b200 as m
    return m


def _tiny_forward(dsa, spec, d, v):
    ws = torch.empty(dsa.dsa_forward_workspace_size(v, spec.topk), dtype=torch.uint8, device="cuda")
    out = torch.full((spec.T, spec.H, spec.d_v), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((spec.T, spec.H), float("nan"), dtype=torch.float32, device="cuda")
    idx = torch.full((spec.T, spec.topk), -2, dtype=torch.int32, device="cuda")
    dsa.dsa_forward(d["q_idx"], d["w"], d["k_idx"], None, d["q"], d["latent"], v, spec.topk, spec.softmax_scale,
                    out, lse, ws, idx_out=idx)
    torch.cuda.synchronize()
    return out, lse, idx


def test_bounded_wait_gives_up_reports_and_the_next_call_is_correct(dsa, oracle_lib):
    assert dsa.dsa_device_error() == 0
    dsa.dsa_debug_wait_selftest(200_000)             # ~0.1 ms at the boost clock
    code = dsa.dsa_device_error()
    assert code == 1 | (SELFTEST_SITE << 8), f"device error word {code:#x}"
    assert dsa.dsa_device_error() == 0, "dsa_device_error clears the word"

    spec = di.config("tiny")
    h = di.make_inputs(spec)
    d = P.to_device(h)
    v = dsa.Varlen(h["cu_q"], h["cu_k"], "cuda")

    # while the word is set, kernels that start skip their work: the outputs stay untouched
    dsa.dsa_debug_wait_selftest(200_000)
    torch.cuda.synchronize()
    out, lse, idx = _tiny_forward(dsa, spec, d, v)
    assert torch.isnan(out.float()).all() and torch.isnan(lse).all()
    assert dsa.dsa_device_error() == 1 | (SELFTEST_SITE << 8)

    # cleared: the next call runs and matches the oracle
    out, lse, idx = _tiny_forward(dsa, spec, d, v)
    assert dsa.dsa_device_error() == 0
    sc, o_idx, o_out, o_lse = oracle_lib.forward(h["cu_q"], h["cu_k"], h["q_idx"], h["w"], h["k_idx"], None, h["q"],
                                                 h["latent"], spec.topk, spec.softmax_scale, spec.d_v)
    pos = P.row_positions(h["cu_q"], h["cu_k"])
    P.assert_index_sets(idx.cpu().numpy(), o_idx, sc, pos, exact=True)
    P.assert_attention_close(out.float().cpu().numpy(), lse.cpu().numpy(), o_out, o_lse, "after the timeout")
