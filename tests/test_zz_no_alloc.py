"""dsa_forward_static_scratch: the forward for callers that cannot allocate
device memory (their memory belongs to a host framework or a preallocated pool
that forbids cudaMalloc once serving has started, or they cannot afford the
device-wide synchronisation of cudaMalloc/cudaFree).  It takes no workspace:
its scratch is the library's static device array.

Each case calls it twice in a row (the array keeps the previous call's
contents) and compares both results with dsa_forward given a caller
workspace, within the parity tolerances of the other GPU tests.  The file is
named so that pytest collects it last."""
import numpy as np
import pytest
import torch

import dsa_inputs as di
from tests import parity as P

pytestmark = pytest.mark.gpu

RELEASED = di.RELEASED
TINY = dict(H_I=4, d_I=32, topk=32, H=4, d_qk=80, d_v=64)


@pytest.fixture(scope="module")
def dsa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from tests.conftest import build_library
    build_library()
    import sparse_attention_long_07_b200 as m
    return m


CASES = {
    "tiny-prefill": di.config("tiny"),
    "decode-e4m3": di.Spec("decode", (1,) * 5, (1, 700, 5000, 20000, 70000), seed=21, kfp8=True, **RELEASED),
    "ragged-bf16": di.Spec("ragged", (3, 40, 1), (3, 900, 4097), seed=22, **RELEASED),
    # rows of 250K keys: one row's scores take 1 MB, so the static array holds ~31
    # rows and the 80 query rows run in three passes inside one call
    "multi-pass": di.Spec("long", (40, 40), (250000, 260000), seed=23, dist="normal", **TINY),
}


def _run(dsa, spec, static):
    dd = di.make_inputs(spec, device="cuda")
    v = dsa.Varlen(dd["cu_q"], dd["cu_k"], "cuda")
    T = spec.T
    out = torch.full((T, spec.H, spec.d_v), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((T, spec.H), float("nan"), dtype=torch.float32, device="cuda")
    idx = torch.full((T, spec.topk), -2, dtype=torch.int32, device="cuda")
    if static:
        dsa.dsa_forward_static_scratch(dd["q_idx"], dd["w"], dd["k_idx"], dd["k_scale"], dd["q"], dd["latent"], v,
                                       spec.topk, spec.softmax_scale, out, lse, idx_out=idx)
    else:
        ws = torch.empty(dsa.dsa_forward_workspace_size(v, spec.topk), dtype=torch.uint8, device="cuda")
        dsa.dsa_forward(dd["q_idx"], dd["w"], dd["k_idx"], dd["k_scale"], dd["q"], dd["latent"], v, spec.topk,
                        spec.softmax_scale, out, lse, ws, idx_out=idx)
    torch.cuda.synchronize()
    assert dsa.dsa_device_error() == 0
    return out.float().cpu().numpy(), lse.cpu().numpy(), idx.cpu().numpy()


@pytest.mark.parametrize("name", list(CASES))
def test_static_scratch_matches_workspace_forward_on_two_calls(dsa, name):
    spec = CASES[name]
    ref_out, ref_lse, ref_idx = _run(dsa, spec, static=False)
    for call in range(2):
        out, lse, idx = _run(dsa, spec, static=True)
        for r in range(spec.T):
            a = set(int(x) for x in idx[r] if x >= 0)
            b = set(int(x) for x in ref_idx[r] if x >= 0)
            assert a == b, f"call {call}, row {r}: selections differ"
            assert np.all(idx[r][len(a):] == -1)
        P.assert_attention_close(out, lse, ref_out.astype(np.float64), ref_lse.astype(np.float64),
                                 f"{name} call {call}")
