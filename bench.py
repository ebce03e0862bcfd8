"""Benchmark of the DSA hot path (lightning indexer -> top-k -> sparse MLA).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step is one pass of the whole hot path over one batch of synthetic input.
The default workload is the 128K-context decode batch: 64 sequences, one new
query each, cached lengths uniform in [16384, 131072], e4m3 index-key cache with
one fp32 scale per token, top-2048, 128 heads, q/k dim 576, v dim 512.  Metric:
query tokens per second.  Inputs stay resident in HBM (index cache 0.6 GB,
latent cache 5.4 GB: both far larger than the 126 MB L2, so no flush is needed).

The step is issued as the three stage calls of the C ABI (exactly the launches
dsa_forward makes for a single chunk) with CUDA events between them, so the
per-kernel durations are measured inside the timed region.  `e2e` times the
public dsa_forward call with host buffers: the step's new inputs are copied
from pinned host memory, the outputs copied back.

For N > 1 (torchrun, one process per GPU) every rank runs its own batch
(sequences shard across GPUs with no exchange); timing is the max over ranks.
`--impl reference` times the CPU oracle on a bounded sample of the same
workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import dsa_inputs as di  # noqa: E402

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return PEAKS_FALLBACK, "fallback"


def dist_setup(n_gpus):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x, world):
    """The slowest rank's time (NCCL group: a device tensor; gloo, as in the CPU
    tests of this path: a host tensor)."""
    if world == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def rank_spec(spec, rank, world):
    """Weak scaling: every rank serves its own batch of the same shape (its own seed)."""
    if world == 1:
        return spec
    import dataclasses
    return dataclasses.replace(spec, seed=spec.seed + 1000 * rank)


def aggregate_throughput(tokens_per_rank, ms_per_step, world):
    """Whole-job query tokens/s: all ranks' tokens over the max-over-ranks step time."""
    return world * tokens_per_rank / (ms_per_step / 1e3)


# --------------------------------------------------------------------------- algorithmic work

def work_model(spec, idx_fp8):
    """Algorithmic bytes / flops per step, per stage (compulsory traffic only)."""
    H_I, d_I, k, H, dqk, dv = spec.H_I, spec.d_I, spec.topk, spec.H, spec.d_qk, spec.d_v
    pairs = 0          # causal (query, key) pairs
    rows_sel = 0       # selected rows over all queries
    score_cells = 0
    for ql, kl in zip(spec.q_lens, spec.kv_lens):
        for i in range(ql):
            pos = kl - ql + i
            pairs += pos + 1
            rows_sel += min(k, pos + 1)
    score_cells = pairs
    key_bytes = (d_I + 4) if idx_fp8 else 2 * d_I
    kv_total = sum(spec.kv_lens)
    T = spec.T
    idx_bytes = kv_total * key_bytes + T * (H_I * d_I * 2 + H_I * 4) + score_cells * 4
    topk_bytes = score_cells * 4 + T * k * 4
    att_bytes = rows_sel * dqk * 2 + T * (H * dqk * 2 + H * dv * 2 + H * 4) + T * k * 4
    return {
        "indexer": {"bytes": idx_bytes, "flops": pairs * 2 * H_I * d_I},
        "topk": {"bytes": topk_bytes, "flops": 0},
        "attention": {"bytes": att_bytes, "flops": rows_sel * 2 * H * (dqk + dv)},
    }


# --------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi sampling (200 ms) around the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        return False

    def summary(self):
        rows = []
        try:
            with open(self.path) as f:
                for line in f:
                    parts = [p.strip() for p in line.split(",")]
                    if len(parts) >= 9:
                        rows.append(parts)
        finally:
            os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# --------------------------------------------------------------------------- GPU arm

def describe(spec, idx_fp8):
    kv = spec.kv_lens
    return {
        "workload": spec.name,
        "batch": spec.B,
        "query_tokens": spec.T,
        "kv_len_min": min(kv), "kv_len_max": max(kv), "kv_len_mean": round(sum(kv) / len(kv), 1),
        "topk": spec.topk, "index_heads": spec.H_I, "index_dim": spec.d_I,
        "heads": spec.H, "d_qk": spec.d_qk, "d_v": spec.d_v,
        "index_cache": "e4m3 + fp32 scale per token" if idx_fp8 else "bf16",
        "l2": "inputs larger than L2 (no flush): index cache + latent cache stream from HBM",
    }


def pick_chunk(spec):
    ld = (max(spec.kv_lens) + 3) // 4 * 4
    budget = 4 << 30                      # fp32 score rows per pass
    rows = max(1, budget // (ld * 4))
    return 0 if rows >= spec.T else int(rows)


def gpu_arm(args, rank, world):
    import sparse_attention_long_07_b200 as dsa

    spec = rank_spec(di.config(args.workload), rank, world)   # each rank serves its own batch
    idx_fp8 = spec.kfp8
    dev = torch.device("cuda", torch.cuda.current_device())
    d = di.make_inputs(spec, device=dev)
    v = dsa.Varlen(d["cu_q"], d["cu_k"], dev)
    T, k = spec.T, spec.topk
    q_chunk = pick_chunk(spec)
    rows = T if q_chunk == 0 else q_chunk
    ld = (max(spec.kv_lens) + 3) // 4 * 4
    scores = torch.empty((rows, ld), dtype=torch.float32, device=dev)
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    out = torch.empty((T, spec.H, spec.d_v), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((T, spec.H), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    chunks = [(q0, min(T, q0 + rows)) for q0 in range(0, T, rows)]

    def step():
        for q0, q1 in chunks:
            dsa.dsa_indexer_scores(d["q_idx"], d["w"], d["k_idx"], d["k_scale"], v, q0, q1, scores, stream)
            dsa.dsa_topk(scores, v, q0, q1, k, idx[q0:q1], stream)
            dsa.dsa_sparse_mla_attn(d["q"], d["latent"], idx[q0:q1], v, q0, q1, spec.softmax_scale, out, lse,
                                    stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert dsa.dsa_device_error() == 0

    n_ev = args.steps * len(chunks)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n_ev)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        start.record(stream)
        i = 0
        for _ in range(args.steps):
            for q0, q1 in chunks:                  # one step = every chunk of the batch
                e = evs[i]
                i += 1
                e[0].record(stream)
                dsa.dsa_indexer_scores(d["q_idx"], d["w"], d["k_idx"], d["k_scale"], v, q0, q1, scores, stream)
                e[1].record(stream)
                dsa.dsa_topk(scores, v, q0, q1, k, idx[q0:q1], stream)
                e[2].record(stream)
                dsa.dsa_sparse_mla_attn(d["q"], d["latent"], idx[q0:q1], v, q0, q1, spec.softmax_scale, out, lse,
                                        stream=stream)
                e[3].record(stream)
        stop.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    elapsed_ms = max_over_ranks(start.elapsed_time(stop), world)
    assert dsa.dsa_device_error() == 0
    stage_ms = {"indexer": 0.0, "topk": 0.0, "attention": 0.0}
    for e in evs:
        stage_ms["indexer"] += e[0].elapsed_time(e[1])
        stage_ms["topk"] += e[1].elapsed_time(e[2])
        stage_ms["attention"] += e[2].elapsed_time(e[3])
    stage_ms = {n: t / args.steps for n, t in stage_ms.items()}   # per step
    ms_per_step = elapsed_ms / args.steps
    value = aggregate_throughput(T, ms_per_step, world)

    # ---------------------------------------------------------------- e2e (public API, host buffers)
    e2e = e2e_measure(dsa, spec, d, v, q_chunk, args, world)

    # ---------------------------------------------------------------- roofline of the dominant kernel
    peaks, peaks_src = load_peaks()
    work = work_model(spec, idx_fp8)
    dom = max(stage_ms, key=stage_ms.get)
    launches = len(chunks)
    per_launch_ms = stage_ms[dom] / launches
    w = work[dom]
    hbm_t = w["bytes"] / (peaks["hbm_gbs"] * 1e9)
    tc_peak = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    tc_t = w["flops"] / (tc_peak * 1e12)
    if hbm_t >= tc_t:
        achieved = w["bytes"] / launches / (per_launch_ms / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s"}
    else:
        achieved = w["flops"] / launches / (per_launch_ms / 1e3) / 1e12
        roof = {"bound": "tensor", "achieved": round(achieved, 1), "peak": tc_peak, "unit": "TFLOP/s"}
    roof["frac"] = round(roof["achieved"] / roof["peak"], 4)
    persistent = idx_fp8 and all(q == 1 for q in spec.q_lens) and spec.B <= 2048
    roof["kernel"] = {"indexer": "indexer_persistent_kernel" if persistent else "indexer_scores_kernel",
                      "topk": "topk_kernel", "attention": "sparse_mla_kernel"}[dom]
    roof["traffic"] = load_traffic(dom, spec.name, w["bytes"] / launches)
    roof["peak_source"] = f"{peaks_src} ({'MEASURED_PEAKS.json' if peaks_src == 'measured' else 'recipe fallback'})"
    # whole-step roofline: sum over stages of max(bytes / HBM, flops / TC)
    t_roof = sum(max(x["bytes"] / (peaks["hbm_gbs"] * 1e9), x["flops"] / (tc_peak * 1e12)) for x in work.values())
    clocks = clk.summary()
    return {
        "value": value, "ms_per_step": ms_per_step, "stage_ms": {n: round(t, 4) for n, t in stage_ms.items()},
        "roofline": roof, "step_roofline_frac": round(t_roof * 1e3 / ms_per_step, 4), "e2e": e2e,
        "gpu_launches": 3 * launches * args.steps, "clocks": clocks, "config": describe(spec, idx_fp8),
        "q_chunk": q_chunk, "inputs": d,
    }


def load_traffic(stage, workload, alg_bytes_per_launch):
    """DRAM bytes per launch of the kernel from the committed ncu summary, if it matches."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    try:
        with open(path) as f:
            t = json.load(f)
        e = t.get(f"{workload}/{stage}")
        return None if e is None else e.get("dram_bytes_per_launch")
    except (OSError, ValueError):
        return None


def e2e_measure(dsa, spec, d, v, q_chunk, args, world):
    """dsa_forward through the public API with the step's inputs in pinned host
    memory.  Decode: the step's new inputs are the query tensors and the new
    token's cache rows (the caches themselves are resident device state);
    prefill: every input tensor is the step's input."""
    dev = d["q"].device
    decode = all(q == 1 for q in spec.q_lens)
    cu_k = [int(x) for x in d["cu_k"]]
    new_rows = torch.tensor([c - 1 for c in cu_k[1:]], dtype=torch.long, device=dev) if decode else None
    names = ["q_idx", "w", "q"] + ([] if decode else ["k_idx", "latent"] + (["k_scale"] if spec.kfp8 else []))
    host = {n: d[n].cpu().pin_memory() for n in names}
    k_bytes = d["k_idx"].view(torch.uint8) if spec.kfp8 else d["k_idx"]
    if decode:
        host["k_rows"] = k_bytes[new_rows].cpu().pin_memory()
        host["lat_rows"] = d["latent"][new_rows].cpu().pin_memory()
        host["ks_rows"] = d["k_scale"][new_rows].cpu().pin_memory() if spec.kfp8 else None
    dev_in = {n: d[n] for n in names}
    out = torch.empty((spec.T, spec.H, spec.d_v), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((spec.T, spec.H), dtype=torch.float32, device=dev)
    out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    lse_h = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
    ws = torch.empty(dsa.dsa_forward_workspace_size(v, spec.topk, q_chunk), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    h2d = sum(t.numel() * t.element_size() for t in host.values() if t is not None)
    d2h = out_h.numel() * out_h.element_size() + lse_h.numel() * lse_h.element_size()

    def one():
        for n in names:
            dev_in[n].copy_(host[n], non_blocking=True)
        if decode:
            k_bytes.index_copy_(0, new_rows, host["k_rows"].to(dev, non_blocking=True))
            d["latent"].index_copy_(0, new_rows, host["lat_rows"].to(dev, non_blocking=True))
            if spec.kfp8:
                d["k_scale"].index_copy_(0, new_rows, host["ks_rows"].to(dev, non_blocking=True))
        dsa.dsa_forward(d["q_idx"], d["w"], d["k_idx"], d["k_scale"], d["q"], d["latent"], v, spec.topk,
                        spec.softmax_scale, out, lse, ws, q_chunk=q_chunk, stream=stream)
        out_h.copy_(out, non_blocking=True)
        lse_h.copy_(lse, non_blocking=True)

    for _ in range(max(3, args.warmup // 4)):
        one()
    torch.cuda.synchronize()
    n = max(3, args.steps // 4)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    a.record(stream)
    for _ in range(n):
        one()
    b.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(a.elapsed_time(b), world) / n
    return {"value": world * spec.T / (ms / 1e3), "unit": "query tokens/s", "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "ms_per_step": round(ms, 4), "steps": n}


# --------------------------------------------------------------------------- CPU oracle

def oracle_sample(spec, max_rows):
    """A bounded sample of the workload for the CPU oracle: whole sequences
    (their caches) with their query rows, at most max_rows query rows."""
    seqs, n = [], 0
    for b in range(spec.B):
        if n + spec.q_lens[b] > max_rows and seqs:
            break
        seqs.append(b)
        n += spec.q_lens[b]
        if n >= max_rows:
            break
    return seqs


def _slice_seqs(spec, d_full, seqs):
    """CPU copies of whole sequences of a device-resident workload."""
    cu_q = [int(x) for x in d_full["cu_q"]]
    cu_k = [int(x) for x in d_full["cu_k"]]
    out = {n: [] for n in ("q_idx", "w", "q", "k_idx", "k_scale", "latent")}
    for b in seqs:
        for n in ("q_idx", "w", "q"):
            out[n].append(d_full[n][cu_q[b]:cu_q[b + 1]].cpu())
        for n in ("k_idx", "latent") + (("k_scale",) if spec.kfp8 else ()):
            out[n].append(d_full[n][cu_k[b]:cu_k[b + 1]].cpu())
    d = {n: (torch.cat(v) if v else None) for n, v in out.items()}
    d["cu_q"] = di.cu_seqlens([spec.q_lens[b] for b in seqs])
    d["cu_k"] = di.cu_seqlens([spec.kv_lens[b] for b in seqs])
    return d


def run_oracle(spec, rows_target, d_full=None):
    """Time the oracle (as it stands) on a bounded sample of the workload."""
    import oracle
    oracle.build()
    decode = all(q == 1 for q in spec.q_lens)
    if decode:
        seqs = oracle_sample(spec, rows_target)
        d = _slice_seqs(spec, d_full, seqs) if d_full is not None else di.make_inputs(spec, seqs=seqs)
        rows = None
        sample = f"{len(seqs)} of {spec.B} decode sequences (whole caches), one query row each"
        n_rows = len(seqs)
    else:
        # the longest sequence's cache with its last query rows
        b = max(range(spec.B), key=lambda i: spec.kv_lens[i])
        d = _slice_seqs(spec, d_full, [b]) if d_full is not None else di.make_inputs(spec, seqs=[b])
        ql = spec.q_lens[b]
        rows = list(range(max(0, ql - rows_target), ql))
        sample = f"last {len(rows)} query rows of sequence {b} (kv_len {spec.kv_lens[b]})"
        n_rows = len(rows)
    t0 = time.perf_counter()
    oracle.forward(d["cu_q"], d["cu_k"], d["q_idx"], d["w"], d["k_idx"], d["k_scale"], d["q"], d["latent"],
                   spec.topk, spec.softmax_scale, spec.d_v, rows=rows)
    dt = time.perf_counter() - t0
    return n_rows / dt, dt, sample, min(oracle.num_threads(), n_rows)


def cpu_rows_target(cores):
    # one query row per host core, bounded so the oracle takes ~10-30 s
    return max(2, min(16, cores))


REFERENCE_BUDGET_S = 150.0     # oracle work of one whole --impl reference run, all steps


def _truncated_rows(spec, d_cpu, seqs, m):
    """One query row per sequence over the first min(kv_len, m) keys of its
    cache (the row's query placed at the last of those positions)."""
    cu_k = [int(x) for x in d_cpu["cu_k"]]
    cu_q = [int(x) for x in d_cpu["cu_q"]]
    out = {n: [] for n in ("q_idx", "w", "q", "k_idx", "k_scale", "latent")}
    lens = []
    for i, b in enumerate(seqs):
        n = min(spec.kv_lens[b], m)
        lens.append(n)
        for name in ("q_idx", "w", "q"):
            out[name].append(d_cpu[name][cu_q[i + 1] - 1:cu_q[i + 1]])
        for name in ("k_idx", "latent") + (("k_scale",) if spec.kfp8 else ()):
            out[name].append(d_cpu[name][cu_k[i]:cu_k[i] + n])
    d = {name: (torch.cat(v) if v else None) for name, v in out.items()}
    d["cu_q"] = di.cu_seqlens([1] * len(seqs))
    d["cu_k"] = di.cu_seqlens(lens)
    return d, lens


def reference_arm(args, rank, world):
    """The oracle as it stands, on the host cores.  Decode: every step runs one
    query row per core (the first sequences of the batch, in parallel).  With
    few steps the rows keep their whole caches; with many, each row's cache is
    cut to its first m keys, m sized so that all steps together cost about
    REFERENCE_BUDGET_S of oracle time, and the step is credited with the
    fraction of a whole-cache step it represents, from a per-row time model
    T(n) = a + b n + c min(k, n) fitted on three cut lengths (untimed)."""
    if rank != 0:
        return None
    spec = di.config(args.workload)
    import oracle
    oracle.build()
    cores = oracle.num_threads()
    rows = cpu_rows_target(cores)
    steps = max(1, args.steps)
    decode = all(q == 1 for q in spec.q_lens)
    times, tokens = [], 0.0
    if decode:
        seqs = oracle_sample(spec, rows)
        d_cpu = di.make_inputs(spec, seqs=seqs)     # generated once for all steps
        full = [spec.kv_lens[b] for b in seqs]

        def run(m):
            d, lens = _truncated_rows(spec, d_cpu, seqs, m)
            t0 = time.perf_counter()
            oracle.forward(d["cu_q"], d["cu_k"], d["q_idx"], d["w"], d["k_idx"], d["k_scale"], d["q"],
                           d["latent"], spec.topk, spec.softmax_scale, spec.d_v)
            return time.perf_counter() - t0, lens

        # Calibration (untimed): the step time of this sample as a function of the
        # cache length n, T(n) = a + b n + c min(k, n) (overhead, per-key work of
        # the indexer and top-k, per-selected-row work of the attention), fitted
        # exactly through three cut lengths.
        k = spec.topk
        pts = [max(64, k // 4), k, 4 * k]
        ts = [run(n)[0] for n in pts]
        n1, n2, n3 = pts
        bc = (ts[1] - ts[0]) / (n2 - n1)                     # b + c (n <= k)
        b_ = max((ts[2] - ts[1]) / (n3 - n2), 1e-12)          # n > k: only b grows
        c_ = max(bc - b_, 0.0)
        a_ = max(ts[0] - bc * n1, 0.0)

        def t_row(n):
            return a_ + b_ * n + c_ * min(k, n)

        per_step = REFERENCE_BUDGET_S / steps
        m = 64
        while m < max(full) and t_row(2 * m) <= per_step:
            m *= 2
        if t_row(max(full)) <= per_step:
            m = max(full)

        # A whole-cache step yields one token per row in the time of its longest
        # row (the rows run in parallel); a cut step is credited in proportion.
        t_full = max(t_row(f) for f in full)

        def frac_tokens(lens):
            return len(lens) * max(t_row(n) for n in lens) / t_full

        for _ in range(steps):
            dt, lens = run(m)
            times.append(dt)
            tokens += frac_tokens(lens)
        whole = m >= max(full)
        sample = (f"{len(seqs)} of {spec.B} decode sequences, one query row each, "
                  + ("whole caches" if whole else
                     f"caches cut to their first {m} keys; a step counts {len(seqs)} x T(cut)/T(whole) tokens, "
                     f"T(n) = a + b n + c min(k, n) per row fitted on cuts of {pts} keys "
                     f"(a={a_:.3g} s, b={b_:.3g} s/key, c={c_:.3g} s/row), T(whole) of the longest row"))
        used = min(cores, len(seqs))
    else:
        for _ in range(steps):
            v, dt, sample, used = run_oracle(spec, rows)
            times.append(dt)
            tokens += v * dt
    value = tokens / sum(times)
    ms = 1e3 * sum(times) / len(times)
    cb = {"value": value, "unit": "query tokens/s", "cores": used, "kind": "oracle", "sample": sample}
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "query tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": describe(spec, spec.kfp8), "cpu_baseline": cb,
        "e2e": {"value": value, "unit": "query tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


METRIC = "DSA query tokens/s (indexer+top-k+sparse MLA) at 128K ctx; % of roofline"


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=None)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", default="decode128k", choices=list(di.CONFIG_NAMES))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.impl == "reference":
        args.steps = 1 if args.steps is None else args.steps
        args.warmup = 0 if args.warmup is None else args.warmup
    else:
        args.steps = 2000 if args.steps is None else args.steps
        args.warmup = 20 if args.warmup is None else args.warmup
        args.warmup = max(3, args.warmup)
    rank, world, local = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
            line = reference_arm(args, rank, world)
            if line is not None:
                print(json.dumps(line), flush=True)
            return
        r = gpu_arm(args, rank, world)
        if rank != 0:
            return
        line = {
            "metric": METRIC, "value": r["value"], "unit": "query tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": r["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded counter-based generator; shapes of the released layer)",
            "config": {**r["config"], "parallelism": f"replicas x{world} (sequences sharded, no exchange)"},
            "roofline": r["roofline"], "step_roofline_frac": r["step_roofline_frac"],
            "stage_ms": r["stage_ms"], "e2e": r["e2e"], "gpu_launches": r["gpu_launches"], "clocks": r["clocks"],
        }
        if world == 1 and not args.no_cpu_baseline:
            spec = di.config(args.workload)
            import oracle
            oracle.build()
            cores = oracle.num_threads()
            v, dt, sample, used = run_oracle(spec, cpu_rows_target(cores), d_full=r["inputs"])
            line["cpu_baseline"] = {"value": v, "unit": "query tokens/s", "cores": used, "kind": "oracle",
                                    "sample": sample, "seconds": round(dt, 2)}
        print(json.dumps(line), flush=True)
    finally:
        if world > 1 and torch.distributed.is_initialized():
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
