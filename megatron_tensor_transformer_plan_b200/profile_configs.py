"""Per-configuration decode timings through the C-ABI: microseconds per layer,
achieved HBM bandwidth against the measured copy peak, fused against separate
reduction, and each shard layout against the unsharded (t = 1) layer.

    python -m megatron_tensor_transformer_plan_b200.profile_configs [--iters N] [--only NAME]

Workloads (seeded synthetic tensors):
  tiny-mlp    hidden 256, ffn 688, t=2, 1 token, no norm/residual (MLP block)
  7b          hidden 4096, 32/32 heads, ffn 11008, KV 2048, B in {1, 16}, t in {1, 2, 4}
  70b         hidden 8192, 64/8 heads, ffn 28672, KV 8192, B=16, t in {1, 4, 8}
  70b-stack   one layer of the 80-layer stack: t=8, B=4, KV 4096
  70b-batch   hidden 8192, 64/8 heads, ffn 28672, t=4, KV 2048, B in {1..64}
              (above 16 tokens only the tensor-core projections apply)
Working sets under four times the L2 size rotate over several copies of the
weights and caches so that every timed call reads from HBM. Timing: CUDA
events around each call after 3 warm-up calls, median reported.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics

import torch

from megatron_tensor_transformer_plan_b200 import build, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
L2_BYTES = 126 * 1024 * 1024


def hbm_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def layer_bytes(H, nq, nkv, d, F, B, S, mlp_only=False):
    """Every weight once, the K/V cache once, the new K/V, x in and y out."""
    if mlp_only:
        return 3 * F * H * 2 + B * H * 2 * 2
    w = (nq + 2 * nkv) * d * H + H * nq * d + 3 * F * H
    return w * 2 + B * 2 * nkv * S * d * 2 + B * 2 * nkv * d * 2 + B * H * 2 * 2


def time_calls(fn, copies, iters, stream):
    for i in range(3):
        fn(copies[i % len(copies)])
    torch.cuda.synchronize()
    ts = []
    for i in range(iters):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn(copies[i % len(copies)])
        b.record(stream)
        ts.append((a, b))
    torch.cuda.synchronize()
    return statistics.median(a.elapsed_time(b) for a, b in ts) * 1e3  # us


def run_layer(tpl, H, nq, nkv, F, t, B, S, iters, mode, flags=None, mlp_only=False, gemv_mode=4, attn_mode=0):
    dev = torch.device("cuda")
    flags = (tpl.TPL_NORM | tpl.TPL_RESIDUAL) if flags is None else flags
    plan = tpl.Plan(tpl.make_dims(H, nq, nkv, 128, F, 1, 1e-5, flags), t)
    plan.set_option(tpl.TPL_OPT_GEMV_MODE, gemv_mode)
    plan.set_option(tpl.TPL_OPT_DECODE_ATTN, attn_mode)
    nbytes = layer_bytes(H, nq, nkv, 128, F, B, S, mlp_only)
    ncopies = max(1, min(8, -(-4 * L2_BYTES // nbytes)))
    copies = []
    for c in range(ncopies):
        w = synth.layer_weights(H, nq, nkv, 128, F, seed=c, device=dev, mlp_only=mlp_only)
        packed = plan.pack_layer(w)
        del w
        kv = None
        if not mlp_only:
            k, v = synth.kv_cache((t, B, nkv // t, S + 1, 128), seed=c, device=dev)
            kv = (k, v, tpl.Plan.kv(k, v, B, S + 1))
        copies.append((packed, kv))
    x = synth.activations(B, H, seed=0, device=dev)
    y = torch.empty_like(x)
    ws = plan.workspace(B, S, device=dev)
    st = torch.cuda.current_stream()
    m = tpl.TPL_REDUCE_FUSED if mode == "fused" else tpl.TPL_REDUCE_SEPARATE
    if mlp_only:
        fn = lambda c: plan.mlp_block(c[0], x, y, None, ws, m)
    else:
        fn = lambda c: plan.decode_layer(c[0], c[1][2], x, S, y, None, ws, m)
    us = time_calls(fn, copies, iters, st)
    rc = plan.last_device_error()
    del copies, plan
    torch.cuda.empty_cache()
    return us, nbytes, ncopies, rc


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--iters", type=int, default=30)
    ap.add_argument("--only", default="")
    ap.add_argument("--gemv-mode", type=int, default=4, help="TPL_OPT_GEMV_MODE of the plan (4: the default)")
    ap.add_argument("--rope", action="store_true", help="rotary embedding on (TPL_ROPE)")
    ap.add_argument("--attn-mode", type=int, default=0, help="TPL_OPT_DECODE_ATTN of the plan (0: the default)")
    args = ap.parse_args()
    build.build()
    from megatron_tensor_transformer_plan_b200 import tpl
    peak, kind = hbm_peak()
    cases = []
    cases += [("tiny-mlp", dict(H=256, nq=2, nkv=2, F=688, t=2, B=1, S=0, flags=0, mlp_only=True))]
    for B in (1, 16):
        for t in (1, 2, 4):
            cases.append(("7b", dict(H=4096, nq=32, nkv=32, F=11008, t=t, B=B, S=2048)))
    for t in (1, 4, 8):
        cases.append(("70b", dict(H=8192, nq=64, nkv=8, F=28672, t=t, B=16, S=8192)))
    cases.append(("70b-stack", dict(H=8192, nq=64, nkv=8, F=28672, t=8, B=4, S=4096)))
    for B in (1, 4, 8, 16, 24, 32, 48, 64):
        cases.append(("70b-batch", dict(H=8192, nq=64, nkv=8, F=28672, t=4, B=B, S=2048, only_fused=True)))
    for name, c in cases:
        if args.only and name != args.only:
            continue
        for mode in ("fused", "separate"):
            if (c["t"] == 1 or c.get("only_fused")) and mode == "separate":
                continue
            flags = c.get("flags")
            if args.rope and not c.get("mlp_only", False):
                flags = tpl.TPL_NORM | tpl.TPL_RESIDUAL | tpl.TPL_ROPE
            us, nbytes, ncopies, rc = run_layer(tpl, c["H"], c["nq"], c["nkv"], c["F"], c["t"], c["B"], c["S"],
                                                 args.iters, mode, flags, c.get("mlp_only", False),
                                                 args.gemv_mode, args.attn_mode)
            gbs = nbytes / (us * 1e-6) / 1e9
            tok_s = c["B"] / (us * 1e-6)
            print(json.dumps({"workload": name, "gemv_mode": args.gemv_mode, "attn_mode": args.attn_mode,
                              "rope": args.rope, "t": c["t"],
                              "B": c["B"], "S": c["S"],
                              "reduce": mode,
                              "us_per_layer": round(us, 2), "tokens_per_s_per_layer": round(tok_s, 1),
                              "algorithmic_bytes": nbytes, "gb_s": round(gbs, 1),
                              "frac_of_peak": round(gbs / peak, 4), "peak_gb_s": peak, "peak_kind": kind,
                              "weight_copies_rotated": ncopies, "device_status": rc}), flush=True)


if __name__ == "__main__":
    main()
