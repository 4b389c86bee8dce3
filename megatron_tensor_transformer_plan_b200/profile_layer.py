"""Run one decode layer a few times through the C-ABI: a small,
self-contained workload for profilers (2-3 GB on the device, five to seven
kernels per call).  Defaults: one layer of the 70B-shaped stack (t = 8,
batch 4, KV length 4096); the 70B single-layer workload is --t 4 --batch 16
--kv 8192, the 7B one --shape 7b --t 1 --batch 1 --kv 2048.

    python -m megatron_tensor_transformer_plan_b200.profile_layer [--calls N] [--mode fused|separate]
        [--shape 70b|7b] [--t T] [--batch B] [--kv S] [--gemv-mode M]
"""
from __future__ import annotations

import argparse

import torch

from megatron_tensor_transformer_plan_b200 import build, synth

D = 128
SHAPES = {"70b": (8192, 64, 8, 28672), "7b": (4096, 32, 32, 11008)}


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--calls", type=int, default=4)
    ap.add_argument("--mode", default="fused", choices=["fused", "separate"])
    ap.add_argument("--shape", default="70b", choices=sorted(SHAPES))
    ap.add_argument("--t", type=int, default=8)
    ap.add_argument("--batch", type=int, default=4)
    ap.add_argument("--kv", type=int, default=4096)
    ap.add_argument("--gemv-mode", type=int, default=4, help="TPL_OPT_GEMV_MODE of the plan (4: the default)")
    args = ap.parse_args()
    T, B, S = args.t, args.batch, args.kv
    H, NQ, NKV, F = SHAPES[args.shape]
    build.build()
    from megatron_tensor_transformer_plan_b200 import tpl
    dev = torch.device("cuda")
    plan = tpl.Plan(tpl.make_dims(H, NQ, NKV, D, F, 1), T)
    plan.set_option(tpl.TPL_OPT_GEMV_MODE, args.gemv_mode)
    w = synth.layer_weights(H, NQ, NKV, D, F, seed=0, device=dev)
    packed = plan.pack_layer(w)
    del w
    k, v = synth.kv_cache((T, B, NKV // T, S + 1, D), seed=0, device=dev)
    kv = tpl.Plan.kv(k, v, B, S + 1)
    x = synth.activations(B, H, seed=0, device=dev)
    y = torch.empty_like(x)
    ws = plan.workspace(B, S, device=dev)
    mode = tpl.TPL_REDUCE_FUSED if args.mode == "fused" else tpl.TPL_REDUCE_SEPARATE
    for _ in range(args.calls):
        plan.decode_layer(packed, kv, x, S, y, None, ws, mode)
    torch.cuda.synchronize()
    rc = plan.last_device_error()
    print(f"profile_layer: {args.calls} decode-layer calls, device status {rc}")
    del plan


if __name__ == "__main__":
    main()
