"""Comparison helpers shared by the GPU parity tests.

Tolerances (stated once, used everywhere):
  scores     |gpu - oracle| <= 1e-3 * max(|oracle|, rms(row))   (exact on integer inputs)
  top-k      equal set sizes; every index in the symmetric difference of the
             GPU and oracle sets has |I(s) - tau| <= 1e-3 * max(|tau|, rms(row)),
             tau = the oracle's k-th score  (bit-exact sets on integer inputs)
  attention  |gpu - oracle| <= 2e-2 + 1e-2 * |oracle|   for out and lse
The score bound covers fp32 accumulation of exact bf16 x bf16 products over
d_I = 128 terms and 64 heads (worst case ~1e-4 relative to the row scale);
the attention bound covers bf16 inputs, fp32 accumulation, probabilities
rounded to bf16 for the PV product and a bf16 output.

The rms(row) floor in the score and top-k bounds is deliberate: it makes the
bound absolute near zero.  The fp32 rounding error of a score is bounded by
the magnitudes of the terms it sums (the |q.k| products weighted by |w|), not
by the score itself, and a score near zero (a k-th score tau near zero happens
whenever about half a row's scores are negative) is a sum of terms that
cancel.  A bound relative to |tau| alone would then ask for more than fp32
accumulation can give; rms(row) is the scale of those terms.

Every check records its worst error as a fraction of its limit (MARGINS);
the test session prints the largest fractions at its end, so a drift that
stays inside the bounds is still visible.
"""
import math

import numpy as np
import torch

SCORE_RTOL = 1e-3
ATT_ATOL, ATT_RTOL = 2e-2, 1e-2

MARGINS = []     # (check, worst error / its limit), one entry per call


def _margin(what, ratio):
    MARGINS.append((what, float(ratio)))


def row_positions(cu_q, cu_k):
    cu_q, cu_k = list(map(int, cu_q)), list(map(int, cu_k))
    pos = []
    for b in range(len(cu_q) - 1):
        ql, kl = cu_q[b + 1] - cu_q[b], cu_k[b + 1] - cu_k[b]
        pos += [kl - ql + i for i in range(ql)]
    return pos


def assert_scores_close(gpu_rows, oracle_rows, positions, exact=False):
    worst = 0.0
    for r, pos in enumerate(positions):
        g = gpu_rows[r, : pos + 1].astype(np.float64)
        o = oracle_rows[r, : pos + 1]
        if exact:
            assert np.array_equal(g, o), f"row {r}: scores differ"
            continue
        rho = math.sqrt(float(np.mean(o * o))) if o.size else 0.0
        tol = SCORE_RTOL * np.maximum(np.abs(o), rho)
        bad = ~(np.abs(g - o) <= tol)          # NaN (an unwritten score) fails too
        assert not bad.any(), f"row {r}: {int(bad.sum())} scores off, worst {np.abs(g - o).max():.3g}"
        worst = max(worst, float(np.max(np.abs(g - o) / np.maximum(tol, 1e-300)))) if o.size else worst
    if not exact:
        _margin("scores", worst)


def assert_index_sets(gpu_idx, oracle_idx, oracle_rows, positions, exact=False):
    """gpu_idx/oracle_idx [rows, k]; oracle_rows [rows, >= pos+1] float64 scores."""
    worst_set = 0.0
    for r, pos in enumerate(positions):
        g = set(int(v) for v in gpu_idx[r] if v >= 0)
        o = set(int(v) for v in oracle_idx[r] if v >= 0)
        assert len(g) == len(o), f"row {r}: {len(g)} vs {len(o)} selected"
        assert all(0 <= s <= pos for s in g), f"row {r}: index outside 0..pos"
        assert (gpu_idx[r] >= 0).sum() == len(g), f"row {r}: duplicate indices"
        if exact:
            assert g == o, f"row {r}: sets differ in {sorted(g ^ o)[:8]}"
            continue
        diff = g ^ o
        if not diff:
            continue
        sc = oracle_rows[r, : pos + 1]
        kth = np.sort(sc[sorted(o)])[0]
        rho = math.sqrt(float(np.mean(sc * sc)))
        tol = SCORE_RTOL * max(abs(kth), rho)
        worst = max(abs(sc[s] - kth) for s in diff)
        assert worst <= tol, f"row {r}: index set differs beyond tolerance ({worst:.3g} > {tol:.3g})"
        worst_set = max(worst_set, worst / tol)
    if not exact:
        _margin("top-k sets", worst_set)


def assert_attention_close(g_out, g_lse, o_out, o_lse, what=""):
    g_out = g_out.astype(np.float64)
    err = np.abs(g_out - o_out)
    lim = ATT_ATOL + ATT_RTOL * np.abs(o_out)
    assert np.all(np.isfinite(g_out)), f"{what}: non-finite output"
    assert (err <= lim).all(), f"{what}: out max err {err.max():.3g} (count {(~(err <= lim)).sum()})"
    _margin(f"attention out ({what})", np.max(err / lim) if err.size else 0.0)
    if g_lse is not None:
        g_lse = g_lse.astype(np.float64)
        fin = np.isfinite(o_lse)
        assert np.array_equal(fin, np.isfinite(g_lse)), f"{what}: lse finiteness differs"
        e = np.abs(g_lse[fin] - o_lse[fin])
        lim_l = ATT_ATOL + ATT_RTOL * np.abs(o_lse[fin])
        assert (e <= lim_l).all(), f"{what}: lse max err {e.max():.3g}"
        _margin(f"attention lse ({what})", np.max(e / lim_l) if e.size else 0.0)


def to_device(d, device="cuda"):
    out = {}
    for k, v in d.items():
        out[k] = v.to(device) if isinstance(v, torch.Tensor) and k not in ("cu_q", "cu_k") else v
    return out


def sample_rows(cu_q, n, seed=0):
    """First, last and seeded random rows of every sequence (at most n per sequence)."""
    cu_q = list(map(int, cu_q))
    g = np.random.default_rng(seed)
    rows = []
    for b in range(len(cu_q) - 1):
        lo, hi = cu_q[b], cu_q[b + 1]
        if hi <= lo:
            continue
        pick = {lo, hi - 1}
        if hi - lo > 2:
            pick |= set(int(x) for x in g.choice(np.arange(lo, hi), size=min(n, hi - lo) - 2 if n > 2 else 0,
                                                 replace=False))
        rows += sorted(pick)
    return rows
