"""Run one 70B-shaped decode layer a few times through the C-ABI: a small,
self-contained workload for profilers (2-3 GB on the device, five kernels per
call).  Defaults: the stack's shape (t = 8, batch 4, KV length 4096); the
70B single-layer workload is --t 4 --batch 16 --kv 8192.

    python -m megatron_tensor_transformer_plan_b200.profile_layer [--calls N] [--mode fused|separate]
        [--t T] [--batch B] [--kv S]
"""
from __future__ import annotations

import argparse

import torch

from megatron_tensor_transformer_plan_b200 import build, synth

H, NQ, NKV, D, F = 8192, 64, 8, 128, 28672


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--calls", type=int, default=4)
    ap.add_argument("--mode", default="fused", choices=["fused", "separate"])
    ap.add_argument("--t", type=int, default=8)
    ap.add_argument("--batch", type=int, default=4)
    ap.add_argument("--kv", type=int, default=4096)
    args = ap.parse_args()
    T, B, S = args.t, args.batch, args.kv
    build.build()
    from megatron_tensor_transformer_plan_b200 import tpl
    dev = torch.device("cuda")
    plan = tpl.Plan(tpl.make_dims(H, NQ, NKV, D, F, 1), T)
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
