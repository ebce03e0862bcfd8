"""Host-side tests of the C-ABI library: it loads, exports every entry point
declared in include/dsa.h, and rejects invalid arguments on the host before
any CUDA call (so these run without a GPU).  The validation tests pass
invented, aligned "device" addresses that validation never dereferences; they
run only where no GPU is present, so that a regression in the order of the
checks can never launch a kernel on addresses that are not mapped.  Without a
GPU, a call that got as far as a CUDA call would return DSA_ERR_CUDA instead of
the expected status, so these tests also prove that nothing was launched."""
import ctypes
import os
import re

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def dsa():
    from tests.conftest import build_library
    build_library()
    import sparse_attention_long_07_b200 as m
    return m


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "dsa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(dsa_[a-z_0-9]+)\s*\(", src)))


def test_header_declares_the_boundary():
    syms = declared_symbols()
    for name in ("dsa_indexer_scores", "dsa_topk", "dsa_sparse_mla_attn", "dsa_forward",
                 "dsa_forward_workspace_size", "dsa_status_string"):
        assert name in syms


def test_library_exports_every_declared_symbol(dsa):
    lib = dsa.library()
    for name in declared_symbols():
        assert hasattr(lib, name), name
    assert dsa.dsa_version().count(".") == 2


def test_status_strings(dsa):
    for s in range(6):
        assert dsa.dsa_status_string(s) not in ("", "unknown status")
    assert dsa.dsa_status_string(99) == "unknown status"


FAKE = 1 << 20  # an aligned, never-dereferenced "device" address

host_only = pytest.mark.skipif(torch.cuda.is_available(),
                               reason="passes invented device addresses: runs only where no GPU is present")


def fake(n=1):
    return [FAKE * (i + 1) for i in range(n)]


def varlen(cu_q, cu_k):
    from sparse_attention_long_07_b200 import dsa_varlen
    qh = (ctypes.c_int32 * len(cu_q))(*cu_q)
    kh = (ctypes.c_int32 * len(cu_k))(*cu_k)
    v = dsa_varlen(len(cu_q) - 1, FAKE, FAKE, ctypes.cast(qh, ctypes.POINTER(ctypes.c_int32)),
                   ctypes.cast(kh, ctypes.POINTER(ctypes.c_int32)))
    v._keep = (qh, kh)
    return v


def scores_call(dsa, v, q_begin=0, q_end=None, ld=None, h=64, d=128, kd=0, ptrs=None, kscale=FAKE, pm=None,
                ld_pm=0, qscale=None):
    lib = dsa.library()
    q_end = v.cu_q_host[v.batch] if q_end is None else q_end
    ld = 1024 if ld is None else ld
    p = ptrs or fake(4)
    return lib.dsa_indexer_scores(p[0], qscale, p[1], p[2], kscale, kd, v, h, d, q_begin, q_end, p[3], ld, pm, ld_pm,
                                  None)


@host_only
def test_indexer_argument_validation(dsa):
    INV, UNS = dsa.DSA_ERR_INVALID_ARG, dsa.DSA_ERR_UNSUPPORTED
    ok = varlen([0, 3, 5], [0, 10, 300])
    assert scores_call(dsa, varlen([0, 3, 5], [0, 2, 300])) == INV            # q_len > kv_len
    assert scores_call(dsa, varlen([1, 3], [0, 10])) == INV                   # cu_q[0] != 0
    assert scores_call(dsa, varlen([0, 5, 3], [0, 10, 20])) == INV            # decreasing
    assert scores_call(dsa, ok, q_begin=-1) == INV
    assert scores_call(dsa, ok, q_begin=4, q_end=3) == INV
    assert scores_call(dsa, ok, q_end=6) == INV                               # past T
    assert scores_call(dsa, ok, ld=288) == INV                                # ld < longest kv (290)
    assert scores_call(dsa, ok, ld=302) == INV                                # ld % 4
    assert scores_call(dsa, ok, ptrs=[FAKE + 4, FAKE, FAKE, FAKE]) == INV     # misaligned q_idx
    assert scores_call(dsa, ok, ptrs=[0, FAKE, FAKE, FAKE]) == INV            # null
    assert scores_call(dsa, ok, kd=1, kscale=None) == INV                     # e4m3 without scales
    assert scores_call(dsa, ok, kd=7) == INV
    assert scores_call(dsa, ok, h=32) == UNS
    assert scores_call(dsa, ok, h=4, d=32, kd=1) == UNS                       # tiny shape is bf16 only
    assert scores_call(dsa, ok, pm=FAKE, ld_pm=36) == INV                     # part maxima: ld < ceil(290 / 8)
    assert scores_call(dsa, ok, pm=FAKE, ld_pm=38) == INV                     # ld % 4
    assert scores_call(dsa, ok, pm=FAKE + 8, ld_pm=40) == INV                 # misaligned
    assert scores_call(dsa, ok, qscale=FAKE, kd=0) == INV                      # FP8 queries need e4m3 keys
    assert scores_call(dsa, ok, qscale=FAKE + 2, kd=1) == INV                  # misaligned scales
    assert scores_call(dsa, ok, qscale=FAKE, kd=1, h=4, d=32) == UNS          # FP8 indexer: released shape only


@host_only
def test_topk_and_attention_validation(dsa):
    lib = dsa.library()
    INV, UNS = dsa.DSA_ERR_INVALID_ARG, dsa.DSA_ERR_UNSUPPORTED
    v = varlen([0, 4], [0, 100])
    assert lib.dsa_topk(FAKE, 100, None, 0, v, 0, 4, 0, FAKE, None) == INV
    assert lib.dsa_topk(FAKE, 100, None, 0, v, 0, 4, 2049, FAKE, None) == INV
    assert lib.dsa_topk(FAKE, 96, None, 0, v, 0, 4, 16, FAKE, None) == INV
    assert lib.dsa_topk(0, 100, None, 0, v, 0, 4, 16, FAKE, None) == INV
    args = dict(topk=64, h=128, dqk=576, dv=512, scale=0.07, rope=None, max_pos=0)

    def mla(**kw):
        a = dict(args)
        a.update(kw)
        return lib.dsa_sparse_mla_attn(FAKE, FAKE, FAKE, v, 0, 4, a["topk"], a["h"], a["dqk"], a["dv"],
                                       ctypes.c_float(a["scale"]), a["rope"], a["max_pos"], FAKE, FAKE, None)
    assert mla(rope=FAKE + 4, max_pos=100) == INV      # RoPE table not 8-byte aligned
    assert mla(rope=FAKE, max_pos=99) == INV           # positions reach 99: a table of 99 is short
    assert mla(topk=0) == INV
    assert mla(scale=0.0) == INV
    assert mla(scale=float("nan")) == INV
    assert mla(h=64) == UNS
    assert mla(dqk=512) == UNS


@host_only
def test_forward_workspace_contract(dsa):
    lib = dsa.library()
    v = varlen([0, 3, 5], [0, 10, 301])
    ld = 292                       # longest kv_len 291, rounded up to a multiple of 4
    need = lib.dsa_forward_workspace_size(v, 16, 0)
    al = lambda x: (x + 255) // 256 * 256
    ld_pm = (ld // 8 + 1 + 3) // 4 * 4         # one part maximum per 8 keys, rows of a multiple of 4
    assert ld_pm == dsa.part_max_ld(ld) == 40
    assert need == al(5 * ld * 4) + al(5 * ld_pm * 4) + al(5 * 16 * 4)
    assert lib.dsa_forward_workspace_size(v, 16, 2) == al(2 * ld * 4) + al(2 * ld_pm * 4) + al(2 * 16 * 4)
    assert lib.dsa_forward_workspace_size(v, 0, 0) == 0
    assert lib.dsa_forward_workspace_size(varlen([0, 3], [0, 2]), 16, 0) == 0

    def fwd(ws, ws_bytes, topk=16, h_i=64, d_i=128):
        return lib.dsa_forward(FAKE, None, FAKE, FAKE, None, 0, FAKE, FAKE, v, h_i, d_i, topk, 128, 576, 512,
                               ctypes.c_float(0.07), 0, FAKE, FAKE, None, ws, ws_bytes, None)
    assert fwd(None, 0) == dsa.DSA_ERR_WORKSPACE
    assert fwd(FAKE, need - 1) == dsa.DSA_ERR_WORKSPACE
    assert fwd(FAKE + 16, need) == dsa.DSA_ERR_INVALID_ARG              # not 256-byte aligned
    assert fwd(FAKE, need, h_i=8) == dsa.DSA_ERR_UNSUPPORTED


@host_only
def test_injected_faults_are_reported_without_launching(dsa, monkeypatch):
    lib = dsa.library()
    v = varlen([0, 3], [0, 10])
    monkeypatch.setenv("DSA_INJECT_FAULT", "cuda")
    assert scores_call(dsa, v) == dsa.DSA_ERR_CUDA
    assert lib.dsa_topk(FAKE, 16, None, 0, v, 0, 3, 4, FAKE, None) == dsa.DSA_ERR_CUDA
    monkeypatch.setenv("DSA_INJECT_FAULT", "timeout")
    assert scores_call(dsa, v) == dsa.DSA_ERR_DEVICE_TIMEOUT


def test_binding_raises_on_bad_status(dsa):
    v = dsa.Varlen([0, 2], [0, 1])     # q_len > kv_len
    q_idx = torch.zeros(2, 64, 128, dtype=torch.bfloat16)
    with pytest.raises(dsa.DSAError) as e:
        dsa.dsa_indexer_scores(q_idx, torch.zeros(2, 64), torch.zeros(1, 128, dtype=torch.bfloat16), None, v, 0,
                               2, torch.zeros(2, 4), stream=0)
    assert e.value.status == dsa.DSA_ERR_INVALID_ARG


@host_only
def test_layouts_beyond_the_launch_limits_are_rejected_before_any_launch(dsa):
    """Rows longer than the top-k supports: every entry point returns
    DSA_ERR_UNSUPPORTED before launching anything (the indexer of the first
    pass included), and the static-scratch forward returns DSA_ERR_WORKSPACE
    for a row whose scores alone exceed its array."""
    lib = dsa.library()
    f = ctypes.c_float(0.07)
    long_row = varlen([0, 1], [0, 2_000_000])           # past the top-k row limit
    assert lib.dsa_topk(FAKE, 2_000_000, None, 0, long_row, 0, 1, 2048, FAKE, None) == dsa.DSA_ERR_UNSUPPORTED
    need = lib.dsa_forward_workspace_size(long_row, 2048, 0)
    assert need > 0
    assert lib.dsa_forward(FAKE, None, FAKE, FAKE, None, 0, FAKE, FAKE, long_row, 64, 128, 2048, 128, 576, 512, f, 0,
                           FAKE, FAKE, None, FAKE, need, None) == dsa.DSA_ERR_UNSUPPORTED
    assert lib.dsa_forward_static_scratch(FAKE, None, FAKE, FAKE, None, 0, FAKE, FAKE, long_row, 64, 128, 2048, 128,
                                          576, 512, f, FAKE, FAKE, None, None) == dsa.DSA_ERR_UNSUPPORTED
    kv = (dsa.DSA_STATIC_SCRATCH_BYTES // 4) + 1000     # one row of scores alone exceeds the array
    huge = varlen([0, 1], [0, kv])
    assert lib.dsa_forward_static_scratch(FAKE, None, FAKE, FAKE, None, 0, FAKE, FAKE, huge, 64, 128, 2048, 128, 576,
                                          512, f, FAKE, FAKE, None, None) == dsa.DSA_ERR_WORKSPACE


@host_only
def test_self_test_arguments(dsa):
    lib = dsa.library()
    assert lib.dsa_debug_wait_selftest(0, None) == dsa.DSA_ERR_INVALID_ARG
    assert lib.dsa_debug_wait_selftest(3_000_000_000, None) == dsa.DSA_ERR_INVALID_ARG


@host_only
def test_fp8_quantize_arguments(dsa):
    lib = dsa.library()
    assert lib.dsa_hadamard_quantize_fp8(FAKE, -1, FAKE, FAKE, None) == dsa.DSA_ERR_INVALID_ARG
    assert lib.dsa_hadamard_quantize_fp8(FAKE, 0, FAKE, FAKE, None) == dsa.DSA_OK          # nothing to do
    assert lib.dsa_hadamard_quantize_fp8(FAKE + 8, 4, FAKE, FAKE, None) == dsa.DSA_ERR_INVALID_ARG
    assert lib.dsa_hadamard_quantize_fp8(FAKE, 4, FAKE, FAKE + 2, None) == dsa.DSA_ERR_INVALID_ARG


@host_only
def test_paged_layout_validation(dsa):
    lib = dsa.library()

    def paged(page_size, pages_per_seq, n_pages, table=FAKE):
        v = varlen([0, 1, 2], [0, 300, 370])
        v.block_table, v.page_size, v.pages_per_seq, v.n_pages = table, page_size, pages_per_seq, n_pages
        return lib.dsa_forward_workspace_size(v, 16, 0)
    assert paged(64, 5, 10) > 0                    # 5 pages of 64 hold the 300 entries
    assert paged(128, 3, 10) > 0
    assert paged(64, 4, 10) == 0                   # 4 pages of 64 < 300 entries
    assert paged(32, 10, 10) == 0                  # pages shorter than 64 rows
    assert paged(192, 2, 10) == 0                  # not a power of two
    assert paged(64, 5, 0) == 0                    # empty pool
    assert paged(1 << 20, 1, 1 << 11) == 0         # pool of 2^31 rows
    assert paged(64, 5, 10, table=FAKE + 2) == 0   # misaligned table
    # packed layout: the page fields are ignored
    assert paged(0, 0, 0, table=None) > 0


@host_only
def test_up_projection_arguments(dsa):
    lib = dsa.library()
    INV, UNS = dsa.DSA_ERR_INVALID_ARG, dsa.DSA_ERR_UNSUPPORTED
    assert lib.dsa_mla_up_proj(FAKE, FAKE, 0, 128, 512, 128, FAKE, None) == dsa.DSA_OK       # nothing to do
    assert lib.dsa_mla_up_proj(FAKE, FAKE, -1, 128, 512, 128, FAKE, None) == INV
    assert lib.dsa_mla_up_proj(FAKE + 8, FAKE, 4, 128, 512, 128, FAKE, None) == INV
    assert lib.dsa_mla_up_proj(FAKE, FAKE, 4, 128, 512, 128, None, None) == INV
    assert lib.dsa_mla_up_proj(FAKE, FAKE, 4, 64, 512, 128, FAKE, None) == UNS
    assert lib.dsa_mla_up_proj(FAKE, FAKE, 4, 128, 576, 128, FAKE, None) == UNS
    assert lib.dsa_mla_up_proj(FAKE, FAKE, 128 * 65536, 128, 512, 128, FAKE, None) == UNS


@host_only
def test_cache_append_arguments(dsa):
    """dsa_cache_append's host checks: paired buffers, alignment, supported
    shapes, the RoPE table and the index-key forms; a call with nothing to
    write returns DSA_OK without a launch."""
    lib = dsa.library()
    INV, UNS, OK = dsa.DSA_ERR_INVALID_ARG, dsa.DSA_ERR_UNSUPPORTED, dsa.DSA_OK
    BF16, AMAX, HAD = dsa.DSA_KQ_BF16, dsa.DSA_KQ_E4M3_AMAX, dsa.DSA_KQ_E4M3_HADAMARD
    v = varlen([0, 1, 2], [0, 300, 370])   # caches of 300 and 70 entries, one new token each

    def call(lat=None, kid=None, d_qk=576, d_v=512, idx_dim=128, rope=None, max_pos=0, kq=BF16,
             lat_c=None, k_c=None, k_s=None, layout=v):
        return lib.dsa_cache_append(lat, kid, layout, d_qk, d_v, idx_dim, rope, max_pos, kq, lat_c, k_c, k_s, None)

    assert call() == OK                                                  # nothing to write
    assert call(lat=FAKE, lat_c=FAKE, layout=varlen([0, 0], [0, 5])) == OK   # no new tokens
    assert call(lat=FAKE) == INV                                         # new latents without a cache
    assert call(lat_c=FAKE) == INV
    assert call(kid=FAKE) == INV                                         # new keys without a cache
    assert call(lat=FAKE + 8, lat_c=FAKE) == INV                         # misaligned rows
    assert call(kid=FAKE, k_c=FAKE + 8) == INV
    assert call(lat=FAKE, lat_c=FAKE, d_qk=512, d_v=512) == UNS          # not a supported MLA shape
    assert call(lat=FAKE, lat_c=FAKE, rope=FAKE + 4, max_pos=370) == INV  # table not 8-byte aligned
    assert call(rope=FAKE, max_pos=370) == INV                           # a table with no latents to rotate
    assert call(lat=FAKE, lat_c=FAKE, rope=FAKE, max_pos=299) == INV     # table shorter than the longest cache (300)
    assert call(kid=FAKE, k_c=FAKE, kq=7) == INV                         # unknown key form
    assert call(kid=FAKE, k_c=FAKE, idx_dim=64) == UNS                   # bf16 keys of an unsupported width
    for kq in (AMAX, HAD):
        assert call(kid=FAKE, k_c=FAKE, kq=kq) == INV                    # e4m3 keys need their scales
        assert call(kid=FAKE, k_c=FAKE, k_s=FAKE + 2, kq=kq) == INV      # scales not 4-byte aligned
        assert call(kid=FAKE, k_c=FAKE, k_s=FAKE, kq=kq, idx_dim=32) == UNS
    bad = varlen([0, 2], [0, 1])                                          # more new tokens than cache entries
    assert call(lat=FAKE, lat_c=FAKE, layout=bad) == INV


def test_wait_profile_is_a_profiling_build_feature(dsa):
    """The regular library has no wait counters: the diagnostic call answers
    DSA_ERR_UNSUPPORTED and touches neither array (no device access, so this
    also holds where a GPU is present)."""
    lib = dsa.library()
    cyc = (ctypes.c_uint64 * 4)(*([7] * 4))
    cnt = (ctypes.c_uint64 * 4)(*([9] * 4))
    assert lib.dsa_debug_wait_profile(cyc, cnt, 4, 1) == dsa.DSA_ERR_UNSUPPORTED
    assert list(cyc) == [7] * 4 and list(cnt) == [9] * 4
