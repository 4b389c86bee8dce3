"""Run the 70B-shaped layer prefill (t = 8, a chunk of 2048 tokens, causal
attention inside the chunk) through the C-ABI: a self-contained workload for
profilers and for timing (about 5 GB on the device, eight kernels per call).

    python -m megatron_tensor_transformer_plan_b200.profile_prefill [--calls N] [--mode fused|separate]
        [--time] [--tokens T]

With --time it reports the CUDA-event time per call (after 3 warm-up calls)
and the algorithmic FLOP rate: 2*T per weight for the four projections plus
4*d per (query head, key) pair that the causal mask keeps.
"""
from __future__ import annotations

import argparse
import json

import torch

from megatron_tensor_transformer_plan_b200 import build, synth

H, NQ, NKV, D, F, TP = 8192, 64, 8, 128, 28672, 8


def prefill_flops(T: int, H=H, nq=NQ, nkv=NKV, d=D, F=F) -> tuple[float, float]:
    params = H * (nq + 2 * nkv) * d + H * nq * d + 3 * H * F
    linear = 2.0 * T * params
    attn = 4.0 * d * nq * (T * (T + 1) // 2)
    return linear, attn


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--calls", type=int, default=3)
    ap.add_argument("--tokens", type=int, default=2048)
    ap.add_argument("--mode", default="fused", choices=["fused", "separate"])
    ap.add_argument("--time", action="store_true")
    args = ap.parse_args()
    build.build()
    from megatron_tensor_transformer_plan_b200 import tpl
    dev = torch.device("cuda")
    T = args.tokens
    plan = tpl.Plan(tpl.make_dims(H, NQ, NKV, D, F, 1), TP)
    w = synth.layer_weights(H, NQ, NKV, D, F, seed=0, device=dev)
    packed = plan.pack_layer(w)
    torch.cuda.synchronize()
    del w
    torch.cuda.empty_cache()
    n = NKV * T * D
    k = torch.zeros(n, dtype=torch.bfloat16, device=dev)
    v = torch.zeros(n, dtype=torch.bfloat16, device=dev)
    kv = tpl.Plan.kv(k, v, 1, T)
    x = synth.activations(T, H, seed=0, device=dev)
    y = torch.empty_like(x)
    ws = plan.prefill_workspace(T, device=dev)
    mode = tpl.TPL_REDUCE_FUSED if args.mode == "fused" else tpl.TPL_REDUCE_SEPARATE
    if not args.time:
        for _ in range(args.calls):
            plan.prefill_layer(packed, kv, x, y, None, ws, mode)
        torch.cuda.synchronize()
        print(f"profile_prefill: {args.calls} prefill calls, device status {plan.last_device_error()}")
        return
    st = torch.cuda.current_stream()
    for _ in range(3):
        plan.prefill_layer(packed, kv, x, y, None, ws, mode)
    torch.cuda.synchronize()
    times = []
    for _ in range(args.calls):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(st)
        plan.prefill_layer(packed, kv, x, y, None, ws, mode)
        e1.record(st)
        e1.synchronize()
        times.append(e0.elapsed_time(e1))
    lin, att = prefill_flops(T)
    times.sort()
    med = times[len(times) // 2]
    print(json.dumps({"workload": f"70B layer prefill t={TP} T={T} ({args.mode})", "ms_median": med,
                      "ms_min": times[0], "tflops": (lin + att) / (med * 1e-3) / 1e12,
                      "device_status": plan.last_device_error()}))


if __name__ == "__main__":
    main()
