"""Planner report: the Auto shard degree for a memory budget and the per-token
time model of tensor parallelism at N = 1, 2, 4, 8, both computed by the
C-ABI's host functions (tpl_footprint_bytes, tpl_auto_t, tpl_decode_times,
tpl_tp_estimate_get).  Needs no GPU.

    python -m megatron_tensor_transformer_plan_b200.plan_report [--model 70b|7b] [--batch B] [--seq S]
        [--gpu-gb G] [--headroom H] [--latency-us L] [--link-gbs W] [--t-single-ms T]

Single-GPU terms: by default the roofline times of one decode step (every
weight and the cache read once at the HBM peak, one multiply-add per weight
per token at the bf16 peak; the measured peaks when MEASURED_PEAKS.json sits
at the repository root, else 6650 GB/s and 1590 TFLOP/s); --t-single-ms
replaces their sum with a measured step time.  The all-reduce: latency L
("Tensor parallel scaling curves", "The scaling math": 5-10 us per call on
NVLink) plus the ring's 2 (N-1)/N of a batch * hidden * 2-byte message at W.
"""
from __future__ import annotations

import argparse
import json
import os

MODELS = {"70b": (8192, 64, 8, 128, 28672, 80), "7b": (4096, 32, 32, 128, 11008, 32)}
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]) * 1e9, float(j["bf16_tflops"]) * 1e12, "measured"
    return 6650e9, 1590e12, "fallback"


def report(model="70b", batch=16, seq=8192, gpu_gb=180.0, headroom=0.1, latency_us=8.0, link_gbs=770.0,
           t_single_ms=None):
    from megatron_tensor_transformer_plan_b200 import tpl
    H, nq, nkv, d, F, L = MODELS[model]
    dims = tpl.make_dims(H, nq, nkv, d, F, L)
    budget = int(gpu_gb * 1e9)
    rows = [{"model": model, "batch": batch, "seq": seq, "gpu_bytes": budget, "headroom": headroom,
             "footprint_per_gpu": {t: tpl.footprint_bytes(dims, t, batch, seq) for t in (1, 2, 4, 8)},
             "auto_t": tpl.auto_t(dims, budget, headroom, batch, seq),
             "auto_t_blind_8_gpus": tpl.auto_t(dims, 0, headroom, batch, seq, 2, 8)}]
    hbm, flops, kind = peaks()
    tc, tm = tpl.decode_times(dims, batch, seq, 2, flops, hbm)
    if t_single_ms is not None:  # a measured step time stands for both terms
        tc, tm = 0.0, t_single_ms * 1e-3
    msg = batch * H * 2
    for n in (1, 2, 4, 8):
        e = tpl.tp_estimate(tc, tm, n, L, msg, latency_us * 1e-6, link_gbs * 1e9)
        rows.append({"n": n, "t_compute_ms": tc * 1e3, "t_memory_ms": tm * 1e3, "t_allreduce_us": e.t_allreduce * 1e6,
                     "t_comm_ms": e.t_comm * 1e3, "t_total_ms": e.t_total * 1e3, "speedup": e.speedup,
                     "comm_share": e.comm_share, "message_bytes": msg, "peaks": kind})
    return rows


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--model", choices=sorted(MODELS), default="70b")
    ap.add_argument("--batch", type=int, default=16)
    ap.add_argument("--seq", type=int, default=8192)
    ap.add_argument("--gpu-gb", type=float, default=180.0)
    ap.add_argument("--headroom", type=float, default=0.1)
    ap.add_argument("--latency-us", type=float, default=8.0)
    ap.add_argument("--link-gbs", type=float, default=770.0)
    ap.add_argument("--t-single-ms", type=float, default=None)
    a = ap.parse_args()
    from megatron_tensor_transformer_plan_b200 import build
    build.build()
    for r in report(a.model, a.batch, a.seq, a.gpu_gb, a.headroom, a.latency_us, a.link_gbs, a.t_single_ms):
        print(json.dumps(r))


if __name__ == "__main__":
    main()
