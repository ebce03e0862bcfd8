"""Pins of the oracle functions for the FP8 indexer (Hadamard rotation and
e4m3 quantization with power-of-two scales), the rotary embedding and the
per-head up-projection, against things other than the oracle itself: the
e4m3 format through torch.float8_e4m3fn, numpy's Kronecker construction of
the Sylvester matrix, numpy einsum and complex multiplication, and closed
forms (orthogonality, involution, norm preservation, the relative-position
property of rotary embeddings, the bounds of a power-of-two scale)."""
import numpy as np
import pytest
import torch

import dsa_inputs as di

pytestmark = pytest.mark.filterwarnings("ignore::UserWarning")


def sylvester(d):
    h = np.array([[1.0]])
    while h.shape[0] < d:
        h = np.kron(np.array([[1.0, 1.0], [1.0, -1.0]]), h)
    return h


# ---------------------------------------------------------------- Hadamard rotation

@pytest.mark.parametrize("d", [32, 128])
def test_hadamard_is_the_normalised_sylvester_matrix(oracle_lib, d):
    g = np.random.default_rng(d)
    x = g.standard_normal((5, d))
    want = x @ sylvester(d).T / np.sqrt(d)
    np.testing.assert_allclose(oracle_lib.hadamard(x), want, rtol=0, atol=1e-12)
    # orthonormal and symmetric: applying it twice gives the input back
    np.testing.assert_allclose(oracle_lib.hadamard(oracle_lib.hadamard(x)), x, rtol=0, atol=1e-12)
    # the unit vectors map to the matrix columns
    np.testing.assert_allclose(oracle_lib.hadamard(np.eye(d)), sylvester(d).T / np.sqrt(d), atol=1e-15)
    # unnormalised: the +-1 matrix itself, exactly, and (Hq).(Hk) = d (q.k)
    assert np.array_equal(oracle_lib.hadamard(np.eye(d), normalize=False), sylvester(d).T)
    q, k = x[0], x[1]
    hq, hk = oracle_lib.hadamard(q[None], normalize=False)[0], oracle_lib.hadamard(k[None], normalize=False)[0]
    assert abs(hq @ hk - d * (q @ k)) <= 1e-11 * d * (np.abs(q) @ np.abs(k))


def test_hadamard_rejects_lengths_that_are_not_powers_of_two(oracle_lib):
    with pytest.raises(ValueError):
        oracle_lib.hadamard(np.zeros((2, 96)))


# ---------------------------------------------------------------- e4m3 encoding

def test_e4m3_encoding_round_trips_every_finite_code(oracle_lib):
    for code in range(256):
        if code & 0x7F == 0x7F:
            continue                                   # the two NaN patterns
        v = oracle_lib.e4m3_to_double(code)
        got = oracle_lib.double_to_e4m3(v)
        if v == 0.0:
            assert oracle_lib.e4m3_to_double(got) == 0.0
        else:
            assert got == code, (code, v, got)


def test_e4m3_encoding_matches_torch_round_to_nearest_even(oracle_lib):
    """torch's float32 -> float8_e4m3fn conversion rounds to nearest, ties to
    even; compared on random values, on every midpoint between neighbouring
    codes (the ties) and just beside them."""
    g = np.random.default_rng(3)
    vals = list(g.standard_normal(3000) * 30.0) + list(g.uniform(-1, 1, 500) * 2.0 ** -6)
    finite = [oracle_lib.e4m3_to_double(c) for c in range(0, 0x7F)]
    for a, b in zip(finite[:-1], finite[1:]):
        mid = (a + b) / 2.0
        vals += [mid, np.nextafter(mid, 0.0), np.nextafter(mid, 1e9), -mid]
    vals = np.array([v for v in vals if abs(v) <= 448.0], dtype=np.float32)
    ref = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    for v, r in zip(vals, ref):
        got = oracle_lib.double_to_e4m3(float(v))
        assert oracle_lib.e4m3_to_double(got) == oracle_lib.e4m3_to_double(int(r)), (float(v), got, int(r))


def test_e4m3_encoding_saturates(oracle_lib):
    assert oracle_lib.double_to_e4m3(1e6) == 0x7E
    assert oracle_lib.double_to_e4m3(-1e6) == 0xFE
    assert oracle_lib.double_to_e4m3(460.0) == 0x7E


# ---------------------------------------------------------------- power-of-two scaled quantization

def test_quantization_scale_is_the_smallest_power_of_two_that_fits(oracle_lib):
    g = np.random.default_rng(4)
    x = g.standard_normal((40, 128)) * np.exp(g.uniform(-8, 8, size=(40, 1)))
    x[3] = 0.0
    q, s = oracle_lib.quant_e4m3_pow2(x)
    amax = np.abs(x).max(axis=1)
    for i in range(x.shape[0]):
        m, e = np.frexp(s[i])
        assert m == 0.5, "the scale is a power of two"
        if amax[i] == 0:
            assert s[i] == 1.0 and np.all(q[i] & 0x7F == 0)
            continue
        assert amax[i] / s[i] <= 448.0 < 2 * amax[i] / s[i], (amax[i], s[i])
        # every value is the nearest e4m3 value of x / s (torch as the reference)
        ref = torch.from_numpy((x[i] / s[i]).astype(np.float32)).to(torch.float8_e4m3fn).to(torch.float64).numpy()
        got = np.array([oracle_lib.e4m3_to_double(int(b)) for b in q[i]])
        np.testing.assert_array_equal(got, ref)


# ---------------------------------------------------------------- FP8 indexer scores

def test_fp8_scores_match_einsum_of_the_dequantized_values(oracle_lib):
    spec = di.Spec("fp8", (5, 1, 7), (9, 20, 7), H_I=4, d_I=32, topk=8, H=4, d_qk=80, d_v=64, seed=12)
    d = di.make_inputs(spec)
    qx = oracle_lib.hadamard(d["q_idx"])
    kx = oracle_lib.hadamard(d["k_idx"])
    qb, qs = oracle_lib.quant_e4m3_pow2(qx)
    kb, ks = oracle_lib.quant_e4m3_pow2(kx)
    got = oracle_lib.indexer_scores_fp8(d["cu_q"], d["cu_k"], qb, qs, d["w"], kb, ks)
    deq = lambda b: torch.from_numpy(b).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    qv = deq(qb) * qs[..., None].astype(np.float64)
    kv = deq(kb) * ks[:, None].astype(np.float64)
    w = d["w"].double().numpy()
    cu_q, cu_k = d["cu_q"].tolist(), d["cu_k"].tolist()
    for b in range(spec.B):
        for i in range(spec.q_lens[b]):
            t = cu_q[b] + i
            pos = spec.kv_lens[b] - spec.q_lens[b] + i
            keys = kv[cu_k[b]:cu_k[b] + pos + 1]
            logits = np.einsum("jd,sd->js", qv[t], keys)
            want = np.einsum("j,js->s", w[t], np.maximum(logits, 0.0))
            np.testing.assert_allclose(got[t, :pos + 1], want, rtol=1e-12, atol=1e-12)
            assert np.all(np.isneginf(got[t, pos + 1:spec.kv_lens[b]]))


def test_fp8_scores_stay_within_the_e4m3_rounding_bound_of_the_definition(oracle_lib):
    """Quantization error only (H is orthonormal, so the rotation leaves the
    exact score unchanged): rounding to nearest e4m3 moves each rotated value
    x by at most max(2^-4 |x|, 2^-10 s) (half a unit in the last place of a
    3-bit mantissa, or half the subnormal spacing 2^-9 times the scale s), so
    each head's dot product moves by at most sum_i (dq_i |k_i| + |q_i| dk_i +
    dq_i dk_i), and the score (ReLU is 1-Lipschitz) by the |w|-weighted sum."""
    spec = di.Spec("fp8", (3,), (64,), H_I=4, d_I=32, topk=8, H=4, d_qk=80, d_v=64, seed=13)
    d = di.make_inputs(spec)
    ref = oracle_lib.indexer_scores(d["cu_q"], d["cu_k"], d["q_idx"], d["w"], d["k_idx"])
    qx, kx = oracle_lib.hadamard(d["q_idx"]), oracle_lib.hadamard(d["k_idx"])
    qb, qs = oracle_lib.quant_e4m3_pow2(qx)
    kb, ks = oracle_lib.quant_e4m3_pow2(kx)
    got = oracle_lib.indexer_scores_fp8(d["cu_q"], d["cu_k"], qb, qs, d["w"], kb, ks)
    dq = np.maximum(2.0 ** -4 * np.abs(qx), 2.0 ** -10 * qs[..., None])      # [T, H_I, d_I]
    dk = np.maximum(2.0 ** -4 * np.abs(kx), 2.0 ** -10 * ks[:, None])        # [S, d_I]
    dot_err = (np.einsum("tjd,sd->tjs", dq, np.abs(kx)) + np.einsum("tjd,sd->tjs", np.abs(qx), dk)
               + np.einsum("tjd,sd->tjs", dq, dk))
    bound = np.einsum("tj,tjs->ts", np.abs(d["w"].double().numpy()), dot_err)
    fin = np.isfinite(ref)
    assert np.all(np.abs(got[fin] - ref[fin]) <= bound[fin] * (1 + 1e-9))
    assert np.abs(got[fin] - ref[fin]).max() > 0        # the quantization does change the scores


# ---------------------------------------------------------------- rotary embedding

def rope_table(max_pos, d, theta=10000.0):
    f = theta ** (-np.arange(0, d, 2) / d)
    ang = np.arange(max_pos)[:, None] * f[None, :]
    return np.stack([np.cos(ang), np.sin(ang)], axis=-1)


def test_rope_is_complex_multiplication_by_the_table(oracle_lib):
    g = np.random.default_rng(5)
    x = g.standard_normal((7, 64))
    pos = g.integers(0, 500, size=7)
    tab = rope_table(512, 64)
    got = oracle_lib.rope(x, pos, tab)
    z = (x[:, 0::2] + 1j * x[:, 1::2]) * (tab[pos, :, 0] + 1j * tab[pos, :, 1])
    want = np.empty_like(x)
    want[:, 0::2], want[:, 1::2] = z.real, z.imag
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_rope_closed_forms(oracle_lib):
    g = np.random.default_rng(6)
    tab = rope_table(300, 64)
    q, k = g.standard_normal(64), g.standard_normal(64)
    # position 0 is the identity; norms are preserved
    np.testing.assert_allclose(oracle_lib.rope(q[None], [0], tab)[0], q, atol=1e-15)
    for p in (1, 17, 299):
        np.testing.assert_allclose(np.linalg.norm(oracle_lib.rope(q[None], [p], tab)), np.linalg.norm(q), rtol=1e-13)
    # relative positions: <R(p) q, R(s) k> = <R(p - s) q, k>
    for p, s in ((40, 7), (250, 250), (123, 0)):
        lhs = oracle_lib.rope(q[None], [p], tab)[0] @ oracle_lib.rope(k[None], [s], tab)[0]
        rhs = oracle_lib.rope(q[None], [p - s], tab)[0] @ k
        assert abs(lhs - rhs) < 1e-10 * (1 + abs(rhs))


# ---------------------------------------------------------------- up-projection

def test_up_projection_matches_einsum_and_selects_with_a_unit_matrix(oracle_lib):
    g = np.random.default_rng(7)
    o = g.standard_normal((3, 4, 64))
    w = torch.from_numpy(g.standard_normal((4, 64, 16))).to(torch.bfloat16)
    got = oracle_lib.up_proj(o, w)
    np.testing.assert_allclose(got, np.einsum("rhc,hce->rhe", o, w.double().numpy()), rtol=1e-12, atol=1e-12)
    # W = the first 16 rows of the identity, per head, picks latent columns 0..15
    eye = np.zeros((4, 64, 16))
    for h in range(4):
        eye[h, :16, :] = np.eye(16) * (h + 1)
    got = oracle_lib.up_proj(o, eye)
    for h in range(4):
        np.testing.assert_array_equal(got[:, h, :], o[:, h, :16] * (h + 1))
