"""Run one decode layer of the 70B-shaped stack (t = 8, batch 4, KV length
4096) a few times through the C-ABI: a small, self-contained workload for
profilers (about 2 GB on the device, five kernels per call).

    python -m megatron_tensor_transformer_plan_b200.profile_layer [--calls N] [--mode fused|separate]
"""
from __future__ import annotations

import argparse

import torch

from megatron_tensor_transformer_plan_b200 import build, synth

H, NQ, NKV, D, F, T, B, S = 8192, 64, 8, 128, 28672, 8, 4, 4096


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--calls", type=int, default=4)
    ap.add_argument("--mode", default="fused", choices=["fused", "separate"])
    args = ap.parse_args()
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
