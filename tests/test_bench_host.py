"""Host-side pieces of bench.py that the reported numbers rest on: the
algorithmic work model (bytes and flops per stage, the roofline numerators) and
the reference arm's cut-cache sample."""
import math

import pytest
import torch

import bench
import dsa_inputs as di


def test_work_model_counts_the_definitions():
    spec = di.config("decode128k")
    w = bench.work_model(spec, True)
    kv = sum(spec.kv_lens)
    # one query per sequence at position kv_len - 1: it scores every key of its cache
    assert w["indexer"]["flops"] == kv * 2 * spec.H_I * spec.d_I
    # e4m3 key (128 B) + fp32 scale per key, the query block and weights, one fp32 score per pair
    # and one fp32 part maximum per 8 keys
    parts = sum((n + 7) // 8 for n in spec.kv_lens)
    assert w["indexer"]["bytes"] == (kv * (spec.d_I + 4) + spec.T * (spec.H_I * spec.d_I * 2 + spec.H_I * 4)
                                     + kv * 4 + parts * 4)
    # every decode row here is longer than k: k selected rows per query
    assert all(n > spec.topk for n in spec.kv_lens)
    rows = spec.T * spec.topk
    assert w["attention"]["flops"] == rows * 2 * spec.H * (spec.d_qk + spec.d_v)
    assert w["attention"]["bytes"] == (rows * spec.d_qk * 2 + spec.T * (spec.H * spec.d_qk * 2 + spec.H * spec.d_v * 2
                                       + spec.H * 4) + spec.T * spec.topk * 4)
    # top-k: the part maxima, the k parts of 8 scores that hold the selection, k indices out
    assert w["topk"]["bytes"] == parts * 4 + spec.T * 8 * spec.topk * 4 + spec.T * spec.topk * 4


def test_work_model_prefill_counts_causal_pairs():
    spec = di.config("tiny")
    w = bench.work_model(spec, False)
    pairs = sum(sum(kl - ql + i + 1 for i in range(ql)) for ql, kl in zip(spec.q_lens, spec.kv_lens))
    sel = sum(sum(min(spec.topk, kl - ql + i + 1) for i in range(ql)) for ql, kl in zip(spec.q_lens, spec.kv_lens))
    assert w["indexer"]["flops"] == pairs * 2 * spec.H_I * spec.d_I
    assert w["attention"]["flops"] == sel * 2 * spec.H * (spec.d_qk + spec.d_v)


def test_reference_arm_times_whole_rows_and_names_its_workload(oracle_lib):
    """The reference arm on the tiny workload: an exact timing of whole rows,
    with the GPU line's config keys (parallelism included)."""
    import argparse
    args = argparse.Namespace(workload="tiny", steps=2, warmup=0)
    line = bench.reference_arm(args, 0, 1)
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["config"] == {**bench.describe(di.config("tiny"), False), "parallelism": bench.parallelism(1)}
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and "2 of 2 steps timed" in cb["sample"]
    assert line["e2e"]["value"] == line["value"]
    assert bench.reference_arm(args, 1, 2) is None           # only rank 0 runs it


def test_tensor_peak_follows_the_length_of_the_timed_region():
    peaks = {"hbm_gbs": 6538.3, "bf16_tflops": 1674.7, "bf16_tflops_sustained": 1364.1}
    assert bench.tc_peak_for(peaks, 0.007) == (1674.7, "burst")
    assert bench.tc_peak_for(peaks, 30.0) == (1364.1, "sustained")


def test_bench_line_carries_every_contract_key(monkeypatch, capsys):
    """The JSON line main() prints, with the GPU arm and the oracle timing
    replaced by fixed results (no device here)."""
    fake_roof = {"bound": "tensor", "achieved": 250.0, "peak": 1364.1, "unit": "TFLOP/s", "frac": 0.18,
                 "kernel": "sparse_mla_kernel", "traffic": 169466112, "peak_source": "measured"}
    spec = di.config("decode128k")

    def fake_gpu_arm(args, rank, world):
        return {"value": 1.0e5, "ms_per_step": 0.64, "stage_ms": {"indexer": 0.2, "topk": 0.1, "attention": 0.3},
                "stage_ms_steps": 5,
                "roofline": fake_roof, "step_roofline_frac": 0.3,
                "e2e": {"value": 5.0e4, "unit": "query tokens/s", "h2d_bytes_per_step": 1, "d2h_bytes_per_step": 2},
                "gpu_launches": 3 * args.steps, "clocks": {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []},
                "config": bench.describe(spec, spec.kfp8), "q_chunk": 0, "inputs": None}

    monkeypatch.setattr(bench, "gpu_arm", fake_gpu_arm)
    monkeypatch.setattr(bench, "run_oracle", lambda spec, rows, d_full=None: (1.5, 10.0, "sample", 8))
    monkeypatch.setattr(bench, "dist_setup", lambda n: (0, 1, 0))
    monkeypatch.setattr("sys.argv", ["bench.py", "--steps", "5", "--warmup", "3"])
    bench.main()
    import json
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks",
                "cpu_baseline"):
        assert key in line, key
    assert line["steps"] == 5 and line["warmup"] == 3 and line["n_gpus"] == 1
    assert line["higher_is_better"] is True and line["scaling"] == "weak"
    assert line["config"]["workload"] == "decode128k"
    for key in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
        assert key in line["roofline"], key
    for key in ("value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step"):
        assert key in line["e2e"], key
    for key in ("value", "unit", "cores", "kind", "sample"):
        assert key in line["cpu_baseline"], key
    assert line["cpu_baseline"]["kind"] == "oracle"


def test_traffic_counts_only_for_the_sources_it_was_recorded_with(tmp_path, monkeypatch):
    """profiles/traffic.json figures come from an ncu DRAM-bytes CSV; bench
    reports one only while the kernel's sources are unchanged."""
    hdr = ('"ID","Process ID","Process Name","Host Name","Kernel Name","Context","Stream","Block Size",'
           '"Grid Size","Device","CC","Section Name","Metric Name","Metric Unit","Metric Value"\n')
    rows = []
    for i, (name, rd, wr) in enumerate([("void indexer_persistent_kernel<X>(A)", "583909888", "19066112"),
                                        ("void indexer_persistent_kernel<X>(A)", "583909890", "19066110"),
                                        ("void topk_kernel(B)", "14.9", "0")]):
        unit = "Mbyte" if "topk" in name else "byte"
        for m, v in (("dram__bytes_read.sum", rd), ("dram__bytes_write.sum", wr)):
            rows.append(f'"{i}","1","python","h","{name}","1","7","(1, 1, 1)","(1, 1, 1)","0","10.0",'
                        f'"Command line profiler metrics","{m}","{unit}","{v}"\n')
    csv_path = tmp_path / "dram.csv"
    csv_path.write_text("==PROF== Connected\n" + hdr + "".join(rows))
    monkeypatch.setattr(bench, "TRAFFIC_PATH", str(tmp_path / "traffic.json"))
    t = bench.record_traffic(str(csv_path), "decode128k")
    assert t["decode128k/indexer"]["launches"] == 2
    assert t["decode128k/indexer"]["dram_bytes_per_launch"] == 583909889 + 19066111
    assert t["decode128k/topk"]["read"] == 14_900_000 and t["decode128k/topk"]["write"] == 0
    assert "decode128k/attention" not in t
    assert bench.load_traffic("indexer", "decode128k", 0) == 583909889 + 19066111
    assert bench.load_traffic("attention", "decode128k", 0) is None
    # a different source digest (a changed kernel) withdraws the figure
    monkeypatch.setattr(bench, "sources_digest", lambda stage: "0" * 64)
    assert bench.load_traffic("indexer", "decode128k", 0) is None


def test_traffic_digest_follows_the_code_not_its_comments():
    """A reworded comment or a reflowed line leaves the digest of a kernel's
    sources as it was; a changed token does not."""
    base = 'int f(int x) { // doubles x\n  return 2 * x; /* "twice" */ }\nconst char* s = "a // b";\n'
    reworded = '/* a new header\n   comment */\nint f(int x) {   // twice x\n  return 2 * x;  }\nconst char* s = "a // b";'
    changed = 'int f(int x) { // doubles x\n  return 3 * x; }\nconst char* s = "a // b";\n'
    in_string = 'int f(int x) { // doubles x\n  return 2 * x; }\nconst char* s = "a /* b";\n'
    assert bench.code_text(base) == bench.code_text(reworded)
    assert bench.code_text(base) != bench.code_text(changed)
    assert bench.code_text(base) != bench.code_text(in_string)
    assert '"a // b"' in bench.code_text(base)
