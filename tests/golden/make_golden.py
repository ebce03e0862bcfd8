"""Write tests/golden/tiny_expected.json from the CPU oracle alone.

The tiny workload (batch 1, L=256, H_I=4, d_I=32, topk=32, integer inputs in
[-3, 3]) has integer indexer scores, so the stored top-k sets are exact.  Run
from the repository root:  python tests/golden/make_golden.py
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import dsa_inputs as di  # noqa: E402
import oracle  # noqa: E402


def main():
    spec = di.config("tiny")
    d = di.make_inputs(spec)
    sc = oracle.indexer_scores(d["cu_q"], d["cu_k"], d["q_idx"], d["w"], d["k_idx"])
    ix = oracle.topk(d["cu_q"], d["cu_k"], sc, spec.topk)
    out, lse = oracle.sparse_mla(d["cu_q"], d["cu_k"], d["q"], d["latent"], ix, spec.softmax_scale, spec.d_v)
    rows = [0, 1, 31, 32, 33, 100, 255]
    doc = {
        "_source": "written by tests/golden/make_golden.py from the CPU oracle (tiny integer workload, seed 0)",
        "topk_sets": [sorted(int(v) for v in r if v >= 0) for r in ix],
        "score_rows": {str(t): [int(v) for v in sc[t, : t + 1]] for t in rows},
        "score_sum": int(np.nansum(np.where(np.isfinite(sc), sc, 0.0))),
        "lse_rows": {str(t): [float(v) for v in lse[t]] for t in rows},
        "out_row0_head0": [float(v) for v in out[0, 0]],
    }
    path = os.path.join(ROOT, "tests", "golden", "tiny_expected.json")
    with open(path, "w") as f:
        json.dump(doc, f, separators=(",", ":"))
        f.write("\n")
    print("wrote", path)


if __name__ == "__main__":
    main()
