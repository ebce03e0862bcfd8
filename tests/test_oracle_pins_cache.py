"""Pins of the oracle's cache functions (the paged layout of the index-key
and latent caches and what appending a step's tokens writes into them)
against things other than the oracle's own formulas: a worked example
enumerated by hand, a pool filled page by page with array slices, the packed
layout as the degenerate case, torch.float8_e4m3fn and numpy float32
division for the amax/448 quantization, and closed forms of the append
(decode rows are the last rows of their sequences; an identity and a
quarter-turn RoPE table)."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.filterwarnings("ignore::UserWarning")


# ---------------------------------------------------------------- paged layout

def test_paged_rows_worked_example(oracle_lib):
    # Two sequences of 5 and 3 entries, pages of 2 rows, 5 pages in the pool.
    # Sequence 0 uses pages 4, 0, 2: entries 0,1 -> rows 8,9; 2,3 -> 0,1; 4 -> 4.
    # Sequence 1 uses pages 1, 3: entries 0,1 -> rows 2,3; 2 -> 6.
    rows = oracle_lib.paged_rows([0, 5, 8], [[4, 0, 2], [1, 3, -1]], page_size=2, n_pages=5)
    assert rows.tolist() == [8, 9, 0, 1, 4, 2, 3, 6]


def test_packed_layout_is_the_identity(oracle_lib):
    assert oracle_lib.paged_rows([0, 3, 3, 10]).tolist() == list(range(10))


def test_paged_rows_agree_with_a_pool_filled_page_by_page(oracle_lib):
    g = np.random.default_rng(3)
    lens = [1, 64, 65, 200, 0, 130]
    P, pps = 64, 4
    n_pages = 40
    cu_k = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    bt = g.permutation(n_pages)[:len(lens) * pps].reshape(len(lens), pps).astype(np.int32)
    vals = g.standard_normal(int(cu_k[-1]))
    pool = np.full(n_pages * P, np.nan)
    for b, n in enumerate(lens):          # copy each sequence page by page with slices
        seq = vals[cu_k[b]:cu_k[b] + n]
        for j in range(0, n, P):
            chunk = seq[j:j + P]
            pool[bt[b, j // P] * P:bt[b, j // P] * P + len(chunk)] = chunk
    rows = oracle_lib.paged_rows(cu_k, bt, page_size=P, n_pages=n_pages)
    assert np.all(rows >= 0)
    assert np.array_equal(pool[rows], vals)
    assert len(set(rows.tolist())) == len(rows)      # no two entries share a row


def test_paged_rows_mark_missing_pages(oracle_lib):
    # entry 2 of sequence 0 needs a third page the table does not have; the
    # second page of sequence 1 is -1 and its first page is beyond the pool
    rows = oracle_lib.paged_rows([0, 3, 6], [[1, 0], [7, -1]], page_size=2, n_pages=4)
    assert rows.tolist() == [2, 3, 0, -1, -1, -1]


# ---------------------------------------------------------------- amax / 448 quantization

def test_amax_quantization_matches_float32_division_and_torch_cast(oracle_lib):
    g = torch.Generator().manual_seed(5)
    x = (torch.randn(300, 128, generator=g) * torch.exp(torch.randn(300, 1, generator=g) * 3)).to(torch.bfloat16)
    x[7] = 0
    x[8, :5] = torch.tensor([-0.0, 1e-30, -3.0, 2.5, 0.0])
    q, s = oracle_lib.quant_e4m3_amax(x)
    x32 = x.float().numpy()
    amax = np.abs(x32).max(axis=1)
    want_s = np.where(amax > 0, amax / np.float32(448.0), np.float32(1.0)).astype(np.float32)
    assert np.array_equal(s, want_s)
    quot = (x32 / want_s[:, None]).astype(np.float32)
    want_q = torch.from_numpy(quot).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(q, want_q)
    # the largest magnitude of each non-zero vector is the largest e4m3 code
    nz = amax > 0
    assert np.all((q[nz] & 0x7F).max(axis=1) == 0x7E)
    assert np.all(q[7] & 0x7F == 0) and s[7] == 1.0


# ---------------------------------------------------------------- append

def _angle_table(max_pos, pairs, angle):
    t = np.zeros((max_pos, pairs, 2))
    t[..., 0], t[..., 1] = np.cos(angle), np.sin(angle)
    return t


def test_append_decode_rows_are_the_last_rows_and_rope_closed_forms(oracle_lib):
    cu_q = [0, 1, 2, 3]
    cu_k = [0, 5, 6, 70]
    g = torch.Generator().manual_seed(9)
    lat = torch.randn(3, 80, generator=g).to(torch.bfloat16)
    kid = torch.randn(3, 32, generator=g).to(torch.bfloat16)
    d_v = 64
    ident = oracle_lib.cache_append(cu_q, cu_k, lat, kid, oracle_lib.KQ_BF16, _angle_table(70, 8, 0.0), d_v)
    assert ident["rows"].tolist() == [4, 5, 69] and ident["pos"].tolist() == [4, 0, 63]
    assert np.array_equal(ident["latent"], lat.double().numpy())
    assert np.array_equal(ident["k"], kid.double().numpy())
    quarter = oracle_lib.cache_append(cu_q, cu_k, lat, None, rope_freqs=_angle_table(70, 8, np.pi / 2), d_v=d_v)
    x = lat.double().numpy()
    got = quarter["latent"]
    assert np.array_equal(got[:, :d_v], x[:, :d_v])
    np.testing.assert_allclose(got[:, d_v::2], -x[:, d_v + 1::2], atol=1e-15)     # re' = -im
    np.testing.assert_allclose(got[:, d_v + 1::2], x[:, d_v::2], atol=1e-15)      # im' = re


def test_append_prefill_rows_and_paging(oracle_lib):
    # a prefill step of 3 new tokens at the end of a 6-entry sequence, pages of 4
    out = oracle_lib.cache_append([0, 3], [0, 6], None, None, block_table=[[2, 0]], page_size=4, n_pages=3)
    assert out["pos"].tolist() == [3, 4, 5]
    assert out["rows"].tolist() == [11, 0, 1]
