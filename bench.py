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


SUSTAINED_AFTER_S = 2.0   # timed regions longer than this run into the power cap


def tc_peak_for(peaks, region_s):
    """bf16 tensor peak (TF/s) that applies to kernels timed in a region of
    region_s seconds: the burst figure for short regions, the sustained one
    for long ones."""
    if region_s >= SUSTAINED_AFTER_S and "bf16_tflops_sustained" in peaks:
        return peaks["bf16_tflops_sustained"], "sustained"
    return peaks["bf16_tflops"], "burst"


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

PART = 8   # keys per part maximum


def work_model(spec, idx_fp8):
    """Algorithmic bytes / flops per step, per stage (compulsory traffic only).

    The indexer writes every causal score and one part maximum per 8 keys.
    The top-k must read a row's part maxima and at least the k parts that
    hold the selection (8 scores each; the whole row when it is shorter), and
    write k indices per query."""
    H_I, d_I, k, H, dqk, dv = spec.H_I, spec.d_I, spec.topk, spec.H, spec.d_qk, spec.d_v
    pairs = 0          # causal (query, key) pairs
    rows_sel = 0       # selected rows over all queries
    parts = 0          # part maxima over all queries
    topk_read = 0      # scores the top-k must read
    for ql, kl in zip(spec.q_lens, spec.kv_lens):
        for i in range(ql):
            n = kl - ql + i + 1
            pairs += n
            rows_sel += min(k, n)
            parts += (n + PART - 1) // PART
            topk_read += min(n, PART * k)
    score_cells = pairs
    key_bytes = (d_I + 4) if idx_fp8 else 2 * d_I
    kv_total = sum(spec.kv_lens)
    T = spec.T
    idx_bytes = kv_total * key_bytes + T * (H_I * d_I * 2 + H_I * 4) + score_cells * 4 + parts * 4
    topk_bytes = parts * 4 + topk_read * 4 + T * k * 4
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
    part_max = torch.empty((rows, dsa.part_max_ld(ld)), dtype=torch.float32, device=dev)
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    out = torch.empty((T, spec.H, spec.d_v), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((T, spec.H), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    chunks = [(q0, min(T, q0 + rows)) for q0 in range(0, T, rows)]

    def step():
        for q0, q1 in chunks:
            dsa.dsa_indexer_scores(d["q_idx"], d["w"], d["k_idx"], d["k_scale"], v, q0, q1, scores, stream,
                                   part_max=part_max)
            dsa.dsa_topk(scores, v, q0, q1, k, idx[q0:q1], stream, part_max=part_max)
            dsa.dsa_sparse_mla_attn(d["q"], d["latent"], idx[q0:q1], v, q0, q1, spec.softmax_scale, out, lse,
                                    stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert dsa.dsa_device_error() == 0

    # Two timed regions on the same stream, the clocks sampled across both.
    # (1) The headline: K steps back to back, nothing between the launches, so
    # each kernel's launch overlaps its predecessor's end (the top-k and the
    # attention are programmatic dependents).  (2) The stage breakdown: up to
    # 500 more steps with an event between every two stages (which serialises
    # them): the per-kernel times behind stage_ms and the roofline.
    n_stage = min(args.steps, STAGE_STEPS)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n_stage * len(chunks))]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        start.record(stream)
        for _ in range(args.steps):
            step()
        stop.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        i = 0
        for _ in range(n_stage):
            for q0, q1 in chunks:                  # one step = every chunk of the batch
                e = evs[i]
                i += 1
                e[0].record(stream)
                dsa.dsa_indexer_scores(d["q_idx"], d["w"], d["k_idx"], d["k_scale"], v, q0, q1, scores, stream,
                                       part_max=part_max)
                e[1].record(stream)
                dsa.dsa_topk(scores, v, q0, q1, k, idx[q0:q1], stream, part_max=part_max)
                e[2].record(stream)
                dsa.dsa_sparse_mla_attn(d["q"], d["latent"], idx[q0:q1], v, q0, q1, spec.softmax_scale, out, lse,
                                        stream=stream)
                e[3].record(stream)
        torch.cuda.synchronize()
    barrier(world)
    elapsed_ms = max_over_ranks(start.elapsed_time(stop), world)
    assert dsa.dsa_device_error() == 0
    stage_ms = {"indexer": 0.0, "topk": 0.0, "attention": 0.0}
    for e in evs:
        stage_ms["indexer"] += e[0].elapsed_time(e[1])
        stage_ms["topk"] += e[1].elapsed_time(e[2])
        stage_ms["attention"] += e[2].elapsed_time(e[3])
    stage_ms = {n: t / n_stage for n, t in stage_ms.items()}   # per step
    ms_per_step = elapsed_ms / args.steps
    value = aggregate_throughput(T, ms_per_step, world)

    # ---------------------------------------------------------------- e2e (public API, host buffers)
    e2e = e2e_measure(dsa, spec, d, v, q_chunk, args, world)
    peaks, peaks_src = load_peaks()
    # the rows beyond the three stages (FP8 indexer, paged caches, RoPE, W_UV, append), 1 GPU only
    ext = None
    if world == 1 and not args.no_extensions and args.workload == "decode128k":
        ext = extensions_measure(dsa, spec, d, v, out, idx, peaks)
    # the indexer on a long causal prefill (its dense tensor-core regime), 1 GPU only
    idx_prefill = None
    if world == 1 and not args.no_indexer_prefill and args.workload == "decode128k":
        idx_prefill = indexer_prefill_measure(dsa, args, peaks)

    # ---------------------------------------------------------------- roofline of the dominant kernel
    work = work_model(spec, idx_fp8)
    dom = max(stage_ms, key=stage_ms.get)
    launches = len(chunks)
    per_launch_ms = stage_ms[dom] / launches
    w = work[dom]
    hbm_t = w["bytes"] / (peaks["hbm_gbs"] * 1e9)
    tc_peak, tc_kind = tc_peak_for(peaks, elapsed_ms / 1e3)
    tc_t = w["flops"] / (tc_peak * 1e12)
    if hbm_t >= tc_t:
        achieved = w["bytes"] / launches / (per_launch_ms / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s"}
    else:
        achieved = w["flops"] / launches / (per_launch_ms / 1e3) / 1e12
        roof = {"bound": "tensor", "achieved": round(achieved, 1), "peak": tc_peak, "unit": "TFLOP/s",
                "peak_kind": f"bf16 {tc_kind}"}
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
        "stage_ms_steps": n_stage,
        "roofline": roof, "step_roofline_frac": round(t_roof * 1e3 / ms_per_step, 4), "e2e": e2e,
        "gpu_launches": 3 * launches * args.steps, "clocks": clocks, "config": describe(spec, idx_fp8),
        "q_chunk": q_chunk, "inputs": d, "indexer_prefill": idx_prefill, "extensions": ext,
    }


def _time_ms(fn, n, stream):
    """Mean milliseconds of fn() over n launches (CUDA events on `stream`, after 3 warm-up calls)."""
    for _ in range(3):
        fn()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(n):
        fn()
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / n


def extensions_measure(dsa, spec, d, v, out, idx, peaks, n=50):
    """Decode128k with the scope rows that extend the three stages, each timed
    with CUDA events over n launches (inputs resident in HBM):
      fp8_indexer  the whole step with the FP8 indexer: the step's index queries
                   rotated and quantized to e4m3 (dsa_hadamard_quantize_fp8,
                   inside the step), keys prepared once the same way from the
                   bf16 keys of the workload (before their own e4m3 form);
      paged        the whole step on caches moved into a shuffled pool of
                   64-row pages (one block table for both caches);
      rope         the attention with RoPE applied to the queries' rope
                   columns while they load, against the same call without;
      up_proj      the per-head W_UV up-projection of the step's output;
      append       dsa_cache_append of the step's 64 new tokens (latent with
                   RoPE, index key quantized to e4m3 with an amax/448 scale)."""
    from dataclasses import replace
    stream = torch.cuda.current_stream()
    dev = out.device
    T, k = spec.T, spec.topk
    ld = (max(spec.kv_lens) + 3) // 4 * 4
    scores = torch.empty((T, ld), dtype=torch.float32, device=dev)
    pm = torch.empty((T, dsa.part_max_ld(ld)), dtype=torch.float32, device=dev)
    idx2 = torch.empty_like(idx)
    out2 = torch.empty_like(out)
    lse2 = torch.empty((T, spec.H), dtype=torch.float32, device=dev)
    hbm = peaks["hbm_gbs"] * 1e9
    res = {}

    # ---- FP8 indexer
    kb = di.make_inputs(replace(spec, kfp8=False), device=dev, tensors=("k_idx",))["k_idx"]
    kq, ks = dsa.dsa_hadamard_quantize_fp8(kb)
    del kb
    qb = d["q_idx"]
    qq = torch.empty(qb.shape, dtype=torch.float8_e4m3fn, device=dev)
    qs = torch.empty(qb.shape[:-1], dtype=torch.float32, device=dev)

    def fp8_indexer():
        dsa.dsa_hadamard_quantize_fp8(qb, qq, qs, stream=stream)
        dsa.dsa_indexer_scores(qq, d["w"], kq, ks, v, 0, T, scores, stream, part_max=pm, q_scale=qs)

    def fp8_step():
        fp8_indexer()
        dsa.dsa_topk(scores, v, 0, T, k, idx2, stream, part_max=pm)
        dsa.dsa_sparse_mla_attn(d["q"], d["latent"], idx2, v, 0, T, spec.softmax_scale, out2, lse2, stream=stream)

    ms_step = _time_ms(fp8_step, n, stream)
    ms_idx = _time_ms(fp8_indexer, n, stream)
    idx_bytes = work_model(spec, True)["indexer"]["bytes"]
    res["fp8_indexer"] = {
        "value": round(T / (ms_step / 1e3), 1), "unit": "query tokens/s", "ms_per_step": round(ms_step, 4),
        "indexer_ms": round(ms_idx, 4), "indexer_achieved_gbs": round(idx_bytes / (ms_idx / 1e3) / 1e9, 1),
        "indexer_hbm_frac": round(idx_bytes / (ms_idx / 1e3) / hbm, 4),
        "kernels": "hadamard_quantize_kernel + indexer_persistent_kernel (e4m3 x e4m3, kind::f8f6f4)"}
    del kq, ks, qq, qs
    torch.cuda.empty_cache()

    # ---- paged caches (64-row pages, shuffled)
    P = 64
    kv = list(spec.kv_lens)
    pps = max((x + P - 1) // P for x in kv)
    n_pages = sum((x + P - 1) // P for x in kv) + 8
    g = torch.Generator().manual_seed(7)
    perm = torch.randperm(n_pages, generator=g)
    bt = torch.full((len(kv), pps), -1, dtype=torch.int32)
    at = 0
    for b, x in enumerate(kv):
        np_b = (x + P - 1) // P
        bt[b, :np_b] = perm[at:at + np_b].to(torch.int32)
        at += np_b
    rows = torch.cat([(bt[b, torch.arange(x) // P].to(torch.int64) * P + torch.arange(x) % P)
                      for b, x in enumerate(kv)]).to(dev)
    lat_p = torch.zeros((n_pages * P, spec.d_qk), dtype=torch.bfloat16, device=dev)
    lat_p[rows] = d["latent"]
    k_p = torch.zeros((n_pages * P, spec.d_I), dtype=torch.uint8, device=dev)
    k_p[rows] = d["k_idx"].view(torch.uint8)
    ks_p = torch.zeros(n_pages * P, dtype=torch.float32, device=dev)
    ks_p[rows] = d["k_scale"]
    del rows
    vp = dsa.Varlen(d["cu_q"], d["cu_k"], dev, block_table=bt.to(dev), page_size=P, n_pages=n_pages)
    k_pv = k_p.view(torch.float8_e4m3fn)

    def paged_step():
        dsa.dsa_indexer_scores(d["q_idx"], d["w"], k_pv, ks_p, vp, 0, T, scores, stream, part_max=pm)
        dsa.dsa_topk(scores, vp, 0, T, k, idx2, stream, part_max=pm)
        dsa.dsa_sparse_mla_attn(d["q"], lat_p, idx2, vp, 0, T, spec.softmax_scale, out2, lse2, stream=stream)

    ms_paged = _time_ms(paged_step, n, stream)
    res["paged"] = {"value": round(T / (ms_paged / 1e3), 1), "unit": "query tokens/s",
                    "ms_per_step": round(ms_paged, 4), "page_size": P, "pages": n_pages}
    del lat_p, k_p, ks_p, k_pv
    torch.cuda.empty_cache()

    # ---- RoPE of the queries inside the attention
    i = torch.arange(32, dtype=torch.float64)
    ang = torch.arange(max(kv), dtype=torch.float64)[:, None] * (10000.0 ** (-2.0 * i / 64))[None, :]
    rope = torch.stack([torch.cos(ang), torch.sin(ang)], dim=-1).to(torch.float32).to(dev)
    ms_rope = _time_ms(lambda: dsa.dsa_sparse_mla_attn(d["q"], d["latent"], idx, v, 0, T, spec.softmax_scale,
                                                       out2, lse2, stream=stream, rope=rope), n, stream)
    ms_norope = _time_ms(lambda: dsa.dsa_sparse_mla_attn(d["q"], d["latent"], idx, v, 0, T, spec.softmax_scale,
                                                         out2, lse2, stream=stream), n, stream)
    res["rope"] = {"attention_ms_with_rope": round(ms_rope, 4), "attention_ms_without": round(ms_norope, 4)}

    # ---- W_UV up-projection of the step's output
    w_uv = di.make_w_uv(11, device=dev)
    y = torch.empty((T, spec.H, 128), dtype=torch.bfloat16, device=dev)
    ms_up = _time_ms(lambda: dsa.dsa_mla_up_proj(out, w_uv, y, stream=stream), n, stream)
    up_bytes = w_uv.numel() * 2 + out.numel() * 2 + y.numel() * 2
    res["up_proj"] = {"ms": round(ms_up, 4), "bytes": up_bytes,
                      "achieved_gbs": round(up_bytes / (ms_up / 1e3) / 1e9, 1),
                      "hbm_frac": round(up_bytes / (ms_up / 1e3) / hbm, 4),
                      "flops": 2 * T * spec.H * spec.d_v * 128, "kernel": "up_proj_kernel (tcgen05, M=128 rows)"}

    # ---- append of the step's new tokens (one per sequence) into the caches
    gg = torch.Generator().manual_seed(12)
    lat_new = torch.randn(T, spec.d_qk, generator=gg).to(torch.bfloat16).to(dev)
    k_new = torch.randn(T, spec.d_I, generator=gg).to(torch.bfloat16).to(dev)
    ms_app = _time_ms(lambda: dsa.dsa_cache_append(v, lat_new, d["latent"], k_new, d["k_idx"], d["k_scale"],
                                                   k_quant=dsa.DSA_KQ_E4M3_AMAX, rope=rope, stream=stream),
                      n, stream)
    res["append"] = {"ms": round(ms_app, 4), "tokens": T, "bytes_per_token": (spec.d_qk + spec.d_I) * 2 +
                     spec.d_qk * 2 + spec.d_I + 4}
    assert dsa.dsa_device_error() == 0
    del scores, pm, idx2, out2, lse2, rope, w_uv, y
    torch.cuda.empty_cache()
    return res


# The kernel of each stage (a substring of its name in an ncu launch list) and
# the sources it is compiled from: a recorded DRAM figure counts only while the
# digest of those sources is the one it was recorded with.
STAGE_KERNELS = {"indexer": "indexer", "topk": "topk_kernel", "attention": "sparse_mla"}
STAGE_SOURCES = {"indexer": ("indexer.cuh", "fp8.cuh"), "topk": ("topk.cuh",), "attention": ("sparse_mla.cuh",)}
COMMON_SOURCES = ("common.cuh", "sm100.cuh", "dsa.cu")
TRAFFIC_PATH = os.path.join(ROOT, "profiles", "traffic.json")


def code_text(src):
    """C/C++/CUDA source with its comments removed and every run of white
    space made one blank: what the compiler turns into code.  String and
    character literals are kept as they are (a comment marker inside one is
    not a comment)."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c == "/" and src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
            out.append(" ")
        elif c == "/" and src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        elif c in "\"'":
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def sources_digest(stage):
    """sha256 over the code (comments and layout ignored, code_text) of the
    stage kernel's own source files and the shared ones."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "sparse_attention_long_07_b200", "csrc")
    for name in STAGE_SOURCES[stage] + COMMON_SOURCES:
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            h.update(name.encode() + b"\0" + code_text(f.read()).encode())
    return h.hexdigest()


def load_traffic(stage, workload, alg_bytes_per_launch):
    """DRAM bytes per launch of the kernel from the committed ncu figures, or
    None when there is none for this stage and workload or the kernel's
    sources changed since it was taken."""
    if not os.path.exists(TRAFFIC_PATH):
        return None
    try:
        with open(TRAFFIC_PATH) as f:
            t = json.load(f)
        e = t.get(f"{workload}/{stage}")
        if e is None or e.get("sources_sha256") != sources_digest(stage):
            return None
        return e.get("dram_bytes_per_launch")
    except (OSError, ValueError):
        return None


def record_traffic(csv_path, workload):
    """Average DRAM bytes per launch of each stage's kernel from an ncu CSV
    (--metrics dram__bytes_read.sum,dram__bytes_write.sum ... --csv) into
    profiles/traffic.json, stamped with the current source digests."""
    import csv
    scale = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9, "KB": 1e3, "MB": 1e6, "GB": 1e9}
    launches = {}
    with open(csv_path) as f:
        rows = [ln for ln in f if ln.startswith('"')]
    for r in csv.DictReader(rows):
        m = r["Metric Name"]
        if m not in ("dram__bytes_read.sum", "dram__bytes_write.sum"):
            continue
        v = float(r["Metric Value"].replace(",", "")) * scale[r["Metric Unit"]]
        launches.setdefault((r["ID"], r["Kernel Name"]), {})[m] = v
    t = {}
    if os.path.exists(TRAFFIC_PATH):
        with open(TRAFFIC_PATH) as f:
            t = json.load(f)
    t["_note"] = ("DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per launch from ncu on the "
                  "full-size workload; an entry counts only while sources_sha256 matches the code (comments and "
                  "layout ignored) of the kernel's sources")
    for stage, pat in STAGE_KERNELS.items():
        got = [(name, v) for (_, name), v in launches.items() if pat in name and len(v) == 2]
        if not got:
            continue
        rd = sum(v["dram__bytes_read.sum"] for _, v in got) / len(got)
        wr = sum(v["dram__bytes_write.sum"] for _, v in got) / len(got)
        t[f"{workload}/{stage}"] = {"kernel": got[0][0].split("(")[0].replace("void ", ""), "launches": len(got),
                                    "dram_bytes_per_launch": int(round(rd + wr)), "read": int(round(rd)),
                                    "write": int(round(wr)), "sources_sha256": sources_digest(stage)}
    with open(TRAFFIC_PATH, "w") as f:
        json.dump(t, f, indent=1)
        f.write("\n")
    return t


INDEXER_PREFILL_WORKLOAD = "prefill32k"


def indexer_prefill_measure(dsa, args, peaks):
    """The indexer stage alone on the 32K-token causal prefill (the O(L^2)
    dense contraction of the method), timed with CUDA events over a few
    launches: flops = causal (query, key) pairs x 2 x H_I x d_I."""
    spec = di.config(INDEXER_PREFILL_WORKLOAD)
    dev = torch.device("cuda", torch.cuda.current_device())
    d = di.make_inputs(spec, device=dev, tensors=("q_idx", "w", "k_idx"))
    v = dsa.Varlen(d["cu_q"], d["cu_k"], dev)
    ld = (max(spec.kv_lens) + 3) // 4 * 4
    scores = torch.empty((spec.T, ld), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def launch():
        dsa.dsa_indexer_scores(d["q_idx"], d["w"], d["k_idx"], d["k_scale"], v, 0, spec.T, scores, stream)

    for _ in range(3):
        launch()
    torch.cuda.synchronize()
    n = 30
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clk:
        a.record(stream)
        for _ in range(n):
            launch()
        b.record(stream)
        torch.cuda.synchronize()
    assert dsa.dsa_device_error() == 0
    ms = a.elapsed_time(b) / n
    flops = work_model(spec, False)["indexer"]["flops"]
    tflops = flops / (ms / 1e3) / 1e12
    del d, scores
    torch.cuda.empty_cache()
    return {"workload": spec.name, "launches": n, "ms_per_launch": round(ms, 4), "tflops": round(tflops, 1),
            "flops_per_launch": flops, "kernel": "indexer_scores_kernel (4 queries per CTA)",
            "frac_of_burst_peak": round(tflops / peaks["bf16_tflops"], 4),
            "frac_of_sustained_peak": round(tflops / peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]), 4),
            "clocks": clk.summary()}


class _E2ELane:
    """One batch in flight for the end-to-end measurement.  Everything a step
    copies in sits in one device buffer with a pinned host twin (one copy per
    step), and so do its outputs (one copy back): decode steps bring the query
    tensors and the new token of every sequence (its index key and latent
    row, bf16), which dsa_cache_append writes into the resident caches;
    prefill steps bring every input tensor."""

    @staticmethod
    def _packed(tensors, dev):
        """One device buffer and one pinned host buffer holding the tensors at
        256-byte boundaries; returns (device views, host views, both buffers)."""
        offs, total = [], 0
        for _, t in tensors:
            offs.append(total)
            total += (t.numel() * t.element_size() + 255) // 256 * 256
        dbuf = torch.empty(max(total, 256), dtype=torch.uint8, device=dev)
        hbuf = torch.empty(max(total, 256), dtype=torch.uint8).pin_memory()
        dv, hv = {}, {}
        for (n, t), o in zip(tensors, offs):
            nb = t.numel() * t.element_size()
            dv[n] = dbuf[o:o + nb].view(t.dtype).view(t.shape)
            hv[n] = hbuf[o:o + nb].view(t.dtype).view(t.shape)
            dv[n].copy_(t)
            hv[n].copy_(t.cpu())
        return dv, hv, dbuf, hbuf

    def __init__(self, dsa, spec, d, v, q_chunk, decode):
        dev = d["q"].device
        self.spec, self.d, self.v, self.q_chunk, self.decode = spec, d, v, q_chunk, decode
        names = ["q_idx", "w", "q"] + ([] if decode else ["k_idx", "latent"] + (["k_scale"] if spec.kfp8 else []))
        staged = [(n, d[n]) for n in names]
        if decode:
            new_rows = torch.tensor([int(c) - 1 for c in d["cu_k"][1:]], dtype=torch.long, device=dev)
            k_new = d["k_idx"][new_rows]
            if spec.kfp8:   # the new tokens' index keys in bf16 (dsa_cache_append quantizes them)
                k_new = (k_new.float() * d["k_scale"][new_rows][:, None]).to(torch.bfloat16)
            staged += [("k_new", k_new.contiguous()), ("lat_new", d["latent"][new_rows].contiguous())]
        self.din, _, self.din_buf, self.hin_buf = self._packed(staged, dev)
        for n in names:
            d[n] = self.din[n]   # the forward reads the copied-in tensors
        outs = [("out", torch.empty((spec.T, spec.H, spec.d_v), dtype=torch.bfloat16, device=dev)),
                ("lse", torch.empty((spec.T, spec.H), dtype=torch.float32, device=dev))]
        dout, _, self.dout_buf, self.hout_buf = self._packed(outs, dev)
        self.out, self.lse = dout["out"], dout["lse"]
        self.ws = torch.empty(dsa.dsa_forward_workspace_size(v, spec.topk, q_chunk), dtype=torch.uint8, device=dev)
        self.h2d = self.hin_buf.numel()
        self.d2h = self.hout_buf.numel()
        self.k_quant = dsa.DSA_KQ_E4M3_AMAX if spec.kfp8 else dsa.DSA_KQ_BF16
        self.ev_in = torch.cuda.Event()        # inputs on the device
        self.ev_used = torch.cuda.Event()      # the forward that read them (and wrote out / lse) is done
        self.ev_out = torch.cuda.Event()       # out / lse copied back
        self.ev_used.record(torch.cuda.current_stream(dev))
        self.ev_out.record(torch.cuda.current_stream(dev))

    def step(self, dsa, s_in, s_comp, s_out):
        """One step: inputs in on s_in, the append and the forward on s_comp
        (every lane's on the same stream, so the kernels run one after another
        as in the device-timed step), outputs back on s_out."""
        d, spec = self.d, self.spec
        with torch.cuda.stream(s_in):
            s_in.wait_event(self.ev_used)     # the previous forward of this lane has read its inputs
            self.din_buf.copy_(self.hin_buf, non_blocking=True)
            self.ev_in.record(s_in)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(self.ev_in)
            s_comp.wait_event(self.ev_out)    # out / lse of this lane's previous step are back on the host
            if self.decode:
                dsa.dsa_cache_append(self.v, latent_new=self.din["lat_new"], latent_cache=d["latent"],
                                     kidx_new=self.din["k_new"], k_cache=d["k_idx"], k_scale=d["k_scale"],
                                     k_quant=self.k_quant, d_v=spec.d_v, stream=s_comp)
            dsa.dsa_forward(d["q_idx"], d["w"], d["k_idx"], d["k_scale"], d["q"], d["latent"], self.v, spec.topk,
                            spec.softmax_scale, self.out, self.lse, self.ws, q_chunk=self.q_chunk, stream=s_comp)
            self.ev_used.record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(self.ev_used)
            self.hout_buf.copy_(self.dout_buf, non_blocking=True)
            self.ev_out.record(s_out)


E2E_MIN_CALLS = 100
STAGE_STEPS = 500   # steps of the stage-breakdown region (events between the stages)


def e2e_measure(dsa, spec, d, v, q_chunk, args, world):
    """dsa_cache_append + dsa_forward through the public API, each step's
    inputs copied from pinned host memory and its outputs copied back.  Several batches are kept
    in flight, as a server would: lane 0 serves the benchmark's batch and the
    other lanes other batches of the same shape (other seeds), each with its
    own buffers, and the steps go round the lanes.  Host-to-device copies run
    on one stream, the forwards on a second (one after another, as in the
    device-timed step) and device-to-host copies on a third, so that the
    transfers of one step overlap the kernels of another.  Every step still
    copies its whole input in and its whole output out."""
    import dataclasses
    dev = d["q"].device
    decode = all(q == 1 for q in spec.q_lens)
    n_lanes = max(1, args.e2e_lanes)
    lanes = [_E2ELane(dsa, spec, d, v, q_chunk, decode)]
    for j in range(1, n_lanes):
        spec_j = dataclasses.replace(spec, seed=spec.seed + 500 + j)
        d_j = di.make_inputs(spec_j, device=dev)
        lanes.append(_E2ELane(dsa, spec_j, d_j, type(v)(d_j["cu_q"], d_j["cu_k"], dev), q_chunk, decode))
    s_in, s_comp, s_out = (torch.cuda.Stream(device=dev) for _ in range(3))
    for i in range(2 * n_lanes):
        lanes[i % n_lanes].step(dsa, s_in, s_comp, s_out)
    torch.cuda.synchronize()
    n = max(E2E_MIN_CALLS, min(args.steps, 1000))
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    start.record(s_in)
    s_comp.wait_event(start)
    s_out.wait_event(start)
    for i in range(n):
        lanes[i % n_lanes].step(dsa, s_in, s_comp, s_out)
    end.record(s_out)
    torch.cuda.synchronize()
    ms = max_over_ranks(start.elapsed_time(end), world) / n
    assert dsa.dsa_device_error() == 0
    h2d, d2h = lanes[0].h2d, lanes[0].d2h
    del lanes
    torch.cuda.empty_cache()
    return {"value": world * spec.T / (ms / 1e3), "unit": "query tokens/s", "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "ms_per_step": round(ms, 4), "steps": n,
            "api": "dsa_cache_append + dsa_forward" if decode else "dsa_forward",
            "batches_in_flight": n_lanes, "streams": "host-to-device, forward, device-to-host"}


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


REFERENCE_BUDGET_S = 240.0    # oracle time of one whole --impl reference run


def reference_arm(args, rank, world):
    """The oracle as it stands, on the host cores.  Every step runs it on the
    same bounded sample of the workload, whole caches: for decode one query
    row per host core (the first sequences of the batch, in parallel); for
    prefill the last rows of the longest sequence.  Steps stop once
    REFERENCE_BUDGET_S of oracle time has been spent (at least one step); the
    sample string says how many ran.  value = query rows timed / oracle time."""
    if rank != 0:
        return None
    spec = di.config(args.workload)
    import oracle
    oracle.build()
    cores = oracle.num_threads()
    rows_target = cpu_rows_target(cores)
    steps = max(1, args.steps)
    decode = all(q == 1 for q in spec.q_lens)
    if decode:
        seqs = oracle_sample(spec, rows_target)
        d = di.make_inputs(spec, seqs=seqs)         # generated once for all steps (untimed)
        rows = None
        sample = f"{len(seqs)} of {spec.B} decode sequences (whole caches), one query row each"
        n_rows = len(seqs)
    else:
        b = max(range(spec.B), key=lambda i: spec.kv_lens[i])
        d = di.make_inputs(spec, seqs=[b])
        ql = spec.q_lens[b]
        rows = list(range(max(0, ql - rows_target), ql))
        sample = f"last {len(rows)} query rows of sequence {b} (kv_len {spec.kv_lens[b]})"
        n_rows = len(rows)
    times = []
    for _ in range(steps):
        t0 = time.perf_counter()
        oracle.forward(d["cu_q"], d["cu_k"], d["q_idx"], d["w"], d["k_idx"], d["k_scale"], d["q"], d["latent"],
                       spec.topk, spec.softmax_scale, spec.d_v, rows=rows)
        times.append(time.perf_counter() - t0)
        if sum(times) >= REFERENCE_BUDGET_S:
            break
    value = n_rows * len(times) / sum(times)
    ms = 1e3 * sum(times) / len(times)
    used = min(cores, n_rows)
    sample += f"; {len(times)} of {steps} steps timed (budget {REFERENCE_BUDGET_S:.0f} s)"
    cb = {"value": value, "unit": "query tokens/s", "cores": used, "kind": "oracle", "sample": sample}
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "query tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {**describe(spec, spec.kfp8), "parallelism": parallelism(world)}, "cpu_baseline": cb,
        "e2e": {"value": value, "unit": "query tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def parallelism(world):
    return f"replicas x{world} (sequences sharded, no exchange)"


METRIC = "DSA query tokens/s (indexer+top-k+sparse MLA) at 128K ctx; % of roofline"


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=None)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", default="decode128k", choices=list(di.CONFIG_NAMES))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-indexer-prefill", action="store_true",
                    help="skip the secondary indexer measurement on the 32K prefill")
    ap.add_argument("--e2e-lanes", type=int, default=3,
                    help="batches in flight in the end-to-end measurement (one stream each)")
    ap.add_argument("--no-extensions", action="store_true",
                    help="skip the FP8-indexer, paged, RoPE, up-projection and append measurements")
    ap.add_argument("--record-traffic", metavar="NCU_CSV", default=None,
                    help="write profiles/traffic.json from an ncu DRAM-bytes CSV of --workload and exit")
    args = ap.parse_args()
    if args.record_traffic:
        print(json.dumps(record_traffic(args.record_traffic, args.workload), indent=1))
        return
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
            "config": {**r["config"], "parallelism": parallelism(world)},
            "roofline": r["roofline"], "step_roofline_frac": r["step_roofline_frac"],
            "stage_ms": r["stage_ms"], "stage_ms_steps": r["stage_ms_steps"], "e2e": r["e2e"],
            "gpu_launches": r["gpu_launches"], "clocks": r["clocks"],
        }
        if r.get("indexer_prefill"):
            line["indexer_prefill"] = r["indexer_prefill"]
        if r.get("extensions"):
            line["extensions"] = r["extensions"]
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
