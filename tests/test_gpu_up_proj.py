"""GPU parity of the per-head value up-projection ("DeepSeek-V3.2",
transformers doc, DSA: MLA with latents shared by all heads; released config
kv_lora_rank 512, v_head_dim 128, n_heads 128) against the oracle.

Bound per element: the bf16 rounding of y (half an ulp: bf16 carries 8
significant bits, so at most 2^-8 relative) plus the
accumulation of 512 exact products in fp32 by the tensor core, which adds
products in groups aligned to the largest exponent and truncates: at most two
fp32 ulps (2^-22) of the running magnitude per addition, 512 * 2^-22 * sum_c
|o w| = 2^-13 * sum_c |o w| (the n*u bound on a dot product with u = 2^-22)."""
import numpy as np
import pytest
import torch

import dsa_inputs as di
from tests import parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import sparse_attention_long_07_b200 as m
    return m


@pytest.mark.parametrize("n", [1, 64, 300], ids=["one-row", "decode-batch", "ragged-tiles"])
def test_up_proj_matches_the_oracle(dsa, oracle_lib, n):
    o = di.make_latent_out(41, n)
    w = di.make_w_uv(42)
    guard = 7
    y_full = torch.full((n + guard, 128, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    dsa.dsa_mla_up_proj(o.cuda(), w.cuda(), y=y_full[:n])
    torch.cuda.synchronize()
    assert dsa.dsa_device_error() == 0
    got = y_full[:n].float().cpu().numpy().astype(np.float64)
    ref = oracle_lib.up_proj(o, w)
    mag = np.einsum("rhc,hce->rhe", np.abs(o.double().numpy()), np.abs(w.double().numpy()))
    bound = 2.0 ** -8 * np.abs(ref) + 2.0 ** -13 * mag + 1e-30
    err = np.abs(got - ref)
    P._margin("up-projection", float((err / bound).max()))
    assert np.all(err <= bound), f"worst {float((err / bound).max()):.3f} of the bound"
    assert torch.isnan(y_full[n:].float()).all(), "rows past n were written"


def test_up_proj_rejects_other_shapes(dsa):
    o = torch.zeros((2, 64, 512), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((64, 512, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(RuntimeError):
        dsa.dsa_mla_up_proj(o, w)
