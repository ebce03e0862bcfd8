"""Run one stage of the DSA hot path in a loop, for profilers (ncu).

    python profile_stage.py --workload decode128k \
        --seqs 16 --stage indexer --iters 3

--seqs keeps the first N sequences of the named workload (same values as the
full workload), so a capture can stay at a few GB of device memory while its
inputs remain larger than the L2 cache.  Prints the kernel's mean duration
(CUDA events, not under a profiler) and the sizes it ran on.
"""
from __future__ import annotations

import argparse
import json
import os
import sys

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import dsa_inputs as di  # noqa: E402
import sparse_attention_long_07_b200 as dsa  # noqa: E402


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="decode128k", choices=list(di.CONFIG_NAMES))
    ap.add_argument("--seqs", type=int, default=0, help="first N sequences only (0 = all)")
    ap.add_argument("--stage", default="indexer", choices=["indexer", "topk", "attention", "forward"])
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--fp8-indexer", action="store_true",
                    help="the FP8 indexer: queries and keys Hadamard-rotated and quantized to e4m3")
    ap.add_argument("--wait-profile", action="store_true",
                    help="print per-wait-site cycles (library built with --profile-waits)")
    args = ap.parse_args()
    spec = di.config(args.workload)
    seqs = list(range(spec.B)) if args.seqs <= 0 else list(range(min(args.seqs, spec.B)))
    dev = torch.device("cuda", 0)
    q_scale = None
    if args.fp8_indexer:
        from dataclasses import replace
        d = di.make_inputs(replace(spec, kfp8=False), device=dev, seqs=seqs)
        d["q_idx"], q_scale = dsa.dsa_hadamard_quantize_fp8(d["q_idx"])
        d["k_idx"], d["k_scale"] = dsa.dsa_hadamard_quantize_fp8(d["k_idx"])
    else:
        d = di.make_inputs(spec, device=dev, seqs=seqs)
    v = dsa.Varlen(d["cu_q"], d["cu_k"], dev)
    T, k = v.T, spec.topk
    ld = (v.max_kv + 3) // 4 * 4
    scores = torch.empty((T, ld), dtype=torch.float32, device=dev)
    part_max = torch.empty((T, dsa.part_max_ld(ld)), dtype=torch.float32, device=dev)
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    out = torch.empty((T, spec.H, spec.d_v), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((T, spec.H), dtype=torch.float32, device=dev)
    ws = torch.empty(dsa.dsa_forward_workspace_size(v, k), dtype=torch.uint8, device=dev)
    # inputs of the later stages
    dsa.dsa_indexer_scores(d["q_idx"], d["w"], d["k_idx"], d["k_scale"], v, 0, T, scores, part_max=part_max,
                           q_scale=q_scale)
    dsa.dsa_topk(scores, v, 0, T, k, idx, part_max=part_max)
    torch.cuda.synchronize()

    def run():
        if args.stage == "indexer":
            dsa.dsa_indexer_scores(d["q_idx"], d["w"], d["k_idx"], d["k_scale"], v, 0, T, scores, part_max=part_max,
                                   q_scale=q_scale)
        elif args.stage == "topk":
            dsa.dsa_topk(scores, v, 0, T, k, idx, part_max=part_max)
        elif args.stage == "attention":
            dsa.dsa_sparse_mla_attn(d["q"], d["latent"], idx, v, 0, T, spec.softmax_scale, out, lse)
        else:
            dsa.dsa_forward(d["q_idx"], d["w"], d["k_idx"], d["k_scale"], d["q"], d["latent"], v, k,
                            spec.softmax_scale, out, lse, ws, q_scale=q_scale)

    if args.wait_profile:
        dsa.dsa_debug_wait_profile(reset=True)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(args.iters):
        run()
    b.record()
    torch.cuda.synchronize()
    assert dsa.dsa_device_error() == 0
    if args.wait_profile:
        prof = dsa.dsa_debug_wait_profile(reset=True) or {}
        print(json.dumps({"wait_sites": {str(k): {"cycles_per_wait": round(c / max(n, 1), 1), "waits": n,
                                                  "cycles_total": c} for k, (c, n) in sorted(prof.items())}}))
    print(json.dumps({"workload": spec.name, "seqs": len(seqs), "stage": args.stage,
                      "indexer": "fp8" if args.fp8_indexer else "bf16 q", "query_rows": T,
                      "keys": v.S, "mean_ms": a.elapsed_time(b) / args.iters,
                      "device_bytes_allocated": torch.cuda.memory_allocated()}))


if __name__ == "__main__":
    main()
