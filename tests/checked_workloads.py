"""Workloads run by test_gpu_checked.py with the release and the checked
library (the latter in a child process, DSA_LIBRARY_VARIANT=checked): a tiny
and a released-shape forward on packed caches, the released shape on paged
caches with the persistent FP8 indexer, a cache append and an up-projection.
Prints one JSON line: the device error word after each workload and a digest
of every output."""
import hashlib
import json
import math
import sys

import numpy as np
import torch

import dsa_inputs as di
import sparse_attention_long_07_b200 as dsa

RELEASED = dict(H_I=64, d_I=128, topk=2048, H=128, d_qk=576, d_v=512, scale=1.0 / math.sqrt(192.0))


def _digest(*tensors):
    h = hashlib.sha256()
    for t in tensors:
        h.update(t.contiguous().view(torch.uint8).cpu().numpy().tobytes())
    return h.hexdigest()[:16]


def _forward(spec, d, v, q_scale=None, k_idx=None, k_scale=None, latent=None):
    dev = {k: (x.cuda() if isinstance(x, torch.Tensor) and k not in ("cu_q", "cu_k") else x) for k, x in d.items()}
    ws = torch.empty(dsa.dsa_forward_workspace_size(v, spec.topk), dtype=torch.uint8, device="cuda")
    out = torch.zeros((spec.T, spec.H, spec.d_v), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((spec.T, spec.H), dtype=torch.float32, device="cuda")
    idx = torch.zeros((spec.T, spec.topk), dtype=torch.int32, device="cuda")
    dsa.dsa_forward(dev["q_idx"], dev["w"], dev["k_idx"] if k_idx is None else k_idx,
                    dev["k_scale"] if k_scale is None else k_scale, dev["q"],
                    dev["latent"] if latent is None else latent, v, spec.topk, spec.softmax_scale, out, lse, ws,
                    idx_out=idx, q_scale=q_scale)
    torch.cuda.synchronize()
    return dsa.dsa_device_error(), _digest(out, lse, idx)


def run():
    res = {}
    spec = di.config("tiny")
    d = di.make_inputs(spec)
    res["tiny"] = _forward(spec, d, dsa.Varlen(d["cu_q"], d["cu_k"], "cuda"))
    spec = di.Spec("chk", (3, 1, 1), (2500, 700, 4100), seed=71, kfp8=True, **RELEASED)
    d = di.make_inputs(spec)
    res["released"] = _forward(spec, d, dsa.Varlen(d["cu_q"], d["cu_k"], "cuda"))
    # paged caches, FP8 indexer, one query per sequence (persistent schedule)
    spec = di.Spec("chk-paged", (1, 1, 1), (300, 5000, 2049), seed=72, **RELEASED)
    d = di.make_inputs(spec)
    qq, qs = dsa.dsa_hadamard_quantize_fp8(d["q_idx"].cuda())
    kq, ks = dsa.dsa_hadamard_quantize_fp8(d["k_idx"].cuda())
    d["q_idx"] = qq.cpu()
    P = 64
    kv = list(spec.kv_lens)
    pps = max((n + P - 1) // P for n in kv)
    n_pages = len(kv) * pps
    bt = torch.from_numpy(np.random.default_rng(73).permutation(n_pages).reshape(len(kv), pps).astype(np.int32))
    rows = []
    for b, n in enumerate(kv):
        rows += [int(bt[b, s // P]) * P + s % P for s in range(n)]
    rows = torch.tensor(rows, dtype=torch.long, device="cuda")
    lat = torch.zeros((n_pages * P, spec.d_qk), dtype=torch.bfloat16, device="cuda")
    lat[rows] = d["latent"].cuda()
    kp = torch.zeros((n_pages * P, spec.d_I), dtype=torch.uint8, device="cuda")
    kp[rows] = kq.view(torch.uint8)
    ksp = torch.zeros(n_pages * P, device="cuda")
    ksp[rows] = ks
    vp = dsa.Varlen(d["cu_q"], d["cu_k"], "cuda", block_table=bt.cuda(), page_size=P, n_pages=n_pages)
    res["paged-fp8"] = _forward(spec, d, vp, q_scale=qs, k_idx=kp.view(torch.float8_e4m3fn), k_scale=ksp,
                                latent=lat)
    # append of one decode token per sequence into the paged caches, then the up-projection
    g = torch.Generator().manual_seed(74)
    lat_new = torch.randn(3, spec.d_qk, generator=g).to(torch.bfloat16).cuda()
    k_new = torch.randn(3, spec.d_I, generator=g).to(torch.bfloat16).cuda()
    dsa.dsa_cache_append(vp, lat_new, lat, k_new, kp, ksp, k_quant=dsa.DSA_KQ_E4M3_HADAMARD)
    torch.cuda.synchronize()
    res["append"] = (dsa.dsa_device_error(), _digest(lat, kp, ksp))
    o = di.make_latent_out(75, 130).cuda()
    y = dsa.dsa_mla_up_proj(o, di.make_w_uv(76).cuda())
    torch.cuda.synchronize()
    res["up_proj"] = (dsa.dsa_device_error(), _digest(y))
    return res


if __name__ == "__main__":
    json.dump({"library": dsa.LIB_PATH, "results": run()}, sys.stdout)
    print()
