"""Run the 70B-shaped layer prefill (t = 8, a chunk of 2048 tokens, causal
attention inside the chunk) through the C-ABI: a self-contained workload for
profilers and for timing (about 5 GB on the device, seven kernels per call).

    python -m megatron_tensor_transformer_plan_b200.profile_prefill [--calls N] [--mode fused|separate]
        [--time] [--tokens T] [--start P0] [--rope] [--whole-tiles]

--start P0 makes the call a chunk at position P0 of a cache already holding P0
tokens (tpl_prefill_chunk); --rope turns on the rotary embedding; --whole-tiles
keeps every GEMM output tile whole (TPL_OPT_PREFILL_TAIL 0).  With --time
it reports the CUDA-event time per call (after 3 warm-up calls) and the
algorithmic FLOP rate: 2*T per weight for the four projections plus 4*d per
(query head, key) pair that the causal mask keeps (T*P0 + T(T+1)/2 pairs per
head).
"""
from __future__ import annotations

import argparse
import json

import torch

from megatron_tensor_transformer_plan_b200 import build, synth

H, NQ, NKV, D, F, TP = 8192, 64, 8, 128, 28672, 8


def prefill_flops(T: int, H=H, nq=NQ, nkv=NKV, d=D, F=F, start=0) -> tuple[float, float]:
    params = H * (nq + 2 * nkv) * d + H * nq * d + 3 * H * F
    linear = 2.0 * T * params
    attn = 4.0 * d * nq * (T * start + T * (T + 1) // 2)
    return linear, attn


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--calls", type=int, default=3)
    ap.add_argument("--tokens", type=int, default=2048)
    ap.add_argument("--mode", default="fused", choices=["fused", "separate"])
    ap.add_argument("--time", action="store_true")
    ap.add_argument("--start", type=int, default=0)
    ap.add_argument("--rope", action="store_true")
    ap.add_argument("--whole-tiles", action="store_true",
                    help="keep every GEMM output tile whole (no half tiles in a partial last wave)")
    args = ap.parse_args()
    build.build()
    from megatron_tensor_transformer_plan_b200 import tpl
    dev = torch.device("cuda")
    T, P0 = args.tokens, args.start
    flags = tpl.TPL_NORM | tpl.TPL_RESIDUAL | (tpl.TPL_ROPE if args.rope else 0)
    plan = tpl.Plan(tpl.make_dims(H, NQ, NKV, D, F, 1, 1e-5, flags), TP)
    if args.whole_tiles:
        plan.set_option(tpl.TPL_OPT_PREFILL_TAIL, 0)
    w = synth.layer_weights(H, NQ, NKV, D, F, seed=0, device=dev)
    packed = plan.pack_layer(w)
    torch.cuda.synchronize()
    del w
    torch.cuda.empty_cache()
    n = NKV * (P0 + T) * D
    k, v = synth.kv_cache((n,), seed=1, device=dev)  # the earlier tokens' keys and values
    kv = tpl.Plan.kv(k, v, 1, P0 + T)
    x = synth.activations(T, H, seed=0, device=dev)
    y = torch.empty_like(x)
    ws = plan.prefill_workspace(T, device=dev)
    mode = tpl.TPL_REDUCE_FUSED if args.mode == "fused" else tpl.TPL_REDUCE_SEPARATE

    def call():
        plan.prefill_chunk(packed, kv, x, P0, y, None, ws, mode)

    if not args.time:
        for _ in range(args.calls):
            call()
        torch.cuda.synchronize()
        print(f"profile_prefill: {args.calls} prefill calls, device status {plan.last_device_error()}")
        return
    st = torch.cuda.current_stream()
    for _ in range(3):
        call()
    torch.cuda.synchronize()
    times = []
    for _ in range(args.calls):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(st)
        call()
        e1.record(st)
        e1.synchronize()
        times.append(e0.elapsed_time(e1))
    lin, att = prefill_flops(T, start=P0)
    times.sort()
    med = times[len(times) // 2]
    rope = ", rope" if args.rope else ""
    whole = ", whole tiles" if args.whole_tiles else ""
    print(json.dumps({"workload": f"70B layer prefill t={TP} T={T} start={P0} ({args.mode}{rope}{whole})",
                      "ms_median": med,
                      "ms_min": times[0], "tflops": (lin + att) / (med * 1e-3) / 1e12,
                      "device_status": plan.last_device_error()}))


if __name__ == "__main__":
    main()
