#!/usr/bin/env python
"""Decode throughput of the 70B-shaped 80-layer stack in the t = 8 shard
layout on one GPU (batch 4, KV length 4096), through the C-ABI library.

One step = one decode token for each of the B sequences through all 80
layers: per layer the column-parallel QKV, the owned-head attention, the
row-parallel O projection with its fused shard sum, the column-parallel
gate/up with SwiGLU and the row-parallel down projection with its fused
shard sum (160 reduction points per step).  Weights (137 GB) and KV caches
(5.4 GB) are seeded synthetic tensors resident in HBM; every step reads all
of them, so the working set is far larger than L2 and no flush is needed.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (under torchrun) every rank runs an independent replica of the
stack on its own GPU (the path has no cross-GPU exchange in this build);
value = all tokens / the slowest rank's time.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode tokens/s (70B-shaped layer stack, 1 GPU); achieved HBM GB/s vs peak"
H, NQ, NKV, D, F, L = 8192, 64, 8, 128, 28672, 80
T_SHARDS, BATCH, KV_LEN = 8, 4, 4096
WORKLOAD = "70B-shaped 80-layer decode stack, t=8 shard layout"


def config_dict():
    return {"workload": WORKLOAD, "hidden": H, "n_q_heads": NQ, "n_kv_heads": NKV, "head_dim": D, "ffn": F,
            "layers": L, "t": T_SHARDS, "batch": BATCH, "kv_len": KV_LEN, "reduce": "fused",
            "reductions_per_step": 2 * L,
            "l2": "no flush: every step streams 142 GB of weights and KV, far above the 126 MB L2"}


def algorithmic_bytes_per_step():
    w = (NQ + 2 * NKV) * D * H + H * NQ * D + 2 * F * H + H * F  # params per layer
    per_layer = (w * 2                                   # every weight once (bf16)
                 + BATCH * 2 * NKV * KV_LEN * D * 2      # K and V cache read
                 + BATCH * 2 * NKV * D * 2               # new K/V written and read back
                 + BATCH * H * 2 * 2)                    # x in, y out
    return L * per_layer


def gate_up_bytes_per_launch():
    return 2 * F * H * 2 + BATCH * H * 4 + BATCH * F * 2  # weights + h (fp32) + act (bf16)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def load_tensor_peak():
    """Dense bf16 TFLOP/s for a kernel sequence timed on its own (burst)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        if "bf16_tflops" in j:
            return float(j["bf16_tflops"]), "measured"
    return 1590.0, "fallback"


PREFILL_T = 2048


def prefill_flops(T=PREFILL_T):
    """Algorithmic FLOP of one layer prefill over T tokens: 2*T per weight of
    the four projections, plus 4*d per (query head, key) pair the causal mask
    keeps (QK^T and PV)."""
    params = (NQ + 2 * NKV) * D * H + H * NQ * D + 3 * F * H
    return 2.0 * T * params + 4.0 * D * NQ * (T * (T + 1) // 2)


# the sources the decode gate/up kernel and its launch are built from
DECODE_SOURCES = ("tpl_common.cuh", "tpl_device.cu", "tpl_gemm.cuh", "tpl_gemv.cuh", "tpl_gemv_tc.cuh",
                  "tpl_internal.h", "tpl_norm.cuh", "tpl_plan.cpp", "tpl_tma.h")


def _code_only(text: str) -> str:
    """Source text without comments and with whitespace collapsed, so that a
    change to comments alone keeps the recorded capture valid."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def kernel_source_hash():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "megatron_tensor_transformer_plan_b200", "csrc")
    for name in DECODE_SOURCES:
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            h.update(name.encode())
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic():
    """dram bytes per gate/up launch from the committed ncu summary, valid only
    while the kernel sources are unchanged since the capture."""
    p = os.path.join(ROOT, "profiles", "gemv_gate_up_stack.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        j = json.load(f)
    if j.get("source_hash") != kernel_source_hash():
        return None
    return j.get("dram_bytes_per_launch")


class Clocks:
    """nvidia-smi sampled every 200 ms during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu_index = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "200", "-i", str(self.gpu_index)],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx.append(float(parts[2]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_init():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(value: float, ws: int, device=None) -> float:
    """The largest value over all ranks (a one-element all-reduce; the
    process group is already initialised when ws > 1)."""
    if ws <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def run_reference(args, ws, rank):
    """The oracle (plain fp64 C, as it stands) on the host cores, on a bounded
    sample of the same workload: one decoder layer of the stack per step,
    scaled to the 80-layer stack's tokens/s."""
    if rank != 0:
        return 0
    import numpy as np
    import torch
    import oracle
    from megatron_tensor_transformer_plan_b200 import synth
    threads = os.cpu_count() or 1
    oracle.set_threads(threads)
    dims = oracle.Dims(H, NQ, NKV, D, F)
    w = synth.layer_weights(H, NQ, NKV, D, F, seed=0, layer=0, dtype=torch.bfloat16, device="cpu")
    wb = {k: synth.bits(v) for k, v in w.items()}
    x = synth.activations(BATCH, H, seed=0, dtype=torch.bfloat16).float().numpy().astype(np.float64)
    kl, vl = synth.kv_cache((BATCH, NKV, KV_LEN + 1, D), seed=0)
    kb, vb = synth.bits(kl), synth.bits(vl)
    for _ in range(args.warmup):
        oracle.decode_layer(dims, wb, x, kb, vb, KV_LEN)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle.decode_layer(dims, wb, x, kb, vb, KV_LEN)
        times.append(time.perf_counter() - t0)
    t_layer = sum(times) / len(times)
    step_s = t_layer * L
    value = BATCH / step_s
    cpu = {"value": value, "unit": "tokens/s", "cores": oracle.get_threads(), "kind": "oracle",
           "sample": f"one decoder layer (B={BATCH}, KV {KV_LEN}) per step, fp64, x{L} layers extrapolated"}
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config_dict(),
            "cpu_baseline": cpu,
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def build_stack(plan, tpl, synth, torch, dev, seed=0):
    packed, kvs, keep = [], [], []
    nkv_s = NKV // T_SHARDS
    for l in range(L):
        w = synth.layer_weights(H, NQ, NKV, D, F, seed=seed, layer=l, dtype=torch.bfloat16, device=dev)
        packed.append(plan.pack_layer(w))
        del w
        k, v = synth.kv_cache((T_SHARDS, BATCH, nkv_s, KV_LEN + 1, D), seed=seed, layer=l, device=dev)
        keep.append((k, v))
        kvs.append(tpl.Plan.kv(k, v, BATCH, KV_LEN + 1))
    torch.cuda.synchronize()
    return packed, kvs, keep


def run_tp(args, ws, rank, local):
    """The stack with its shards on the N GPUs of the job (N = t, one shard
    per rank): each rank holds its slice of every layer (its heads, ffn
    columns and kv heads) and its cache shard, runs the library's steps on a
    one-shard plan of those dimensions, and the two row-parallel partial sums
    of every layer are added by an NCCL all-reduce (2L per step).  Reported
    against the pages' time model T(N) = T(1)/N + 2L*T_allreduce(N)
    ("Tensor parallel scaling curves", "The scaling math").  value = the B
    tokens of one step / the slowest rank's step time (strong scaling: the
    model is the same at every N)."""
    import datetime

    import torch
    import torch.distributed as dist
    from megatron_tensor_transformer_plan_b200 import build
    build.build()
    from megatron_tensor_transformer_plan_b200 import synth, tpl
    from megatron_tensor_transformer_plan_b200.tp_dist import (CudaOps, ShardSpec, decode_stack_tp, shard_cache,
                                                                shard_weights)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    t = ws
    spec = ShardSpec(H, NQ, NKV, D, F, t, rank)
    layers, keep = [], []
    wsb = None
    for l in range(L):
        w = synth.layer_weights(H, NQ, NKV, D, F, seed=0, layer=l, dtype=torch.bfloat16, device=dev)
        kl, vl = synth.kv_cache((BATCH, NKV, KV_LEN + 1, D), seed=0, layer=l, device=dev)
        if wsb is None:
            probe = tpl.Plan(tpl.make_dims(H, spec.nq_s, spec.nkv_s, D, spec.ffn_s, 1, 1e-5,
                                           tpl.TPL_NORM | tpl.TPL_RESIDUAL), 1)
            wsb = CudaOps.make_workspace(probe, BATCH, KV_LEN + 1, dev)
        layers.append(CudaOps(spec, shard_weights(w, spec), shard_cache(kl, spec), shard_cache(vl, spec), BATCH,
                              KV_LEN + 1, workspace=wsb))
        del w, kl, vl
    x = synth.activations(BATCH, H, seed=0, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()

    def all_reduce(P):
        if ws > 1:
            dist.all_reduce(P)

    def no_reduce(P):
        pass

    def barrier():
        if ws > 1:
            dist.barrier()

    def timed(steps, reduce):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(steps):
            decode_stack_tp(layers, x, KV_LEN, reduce)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        return max_over_ranks(e0.elapsed_time(e1) / steps, ws, dev)

    for _ in range(args.warmup):
        decode_stack_tp(layers, x, KV_LEN, all_reduce)
    torch.cuda.synchronize()
    for op in layers:
        assert op.plan.last_device_error() == tpl.TPL_OK
    clocks = Clocks(local)
    clocks.start()
    time.sleep(0.3)
    ms = timed(args.steps, all_reduce)
    clk = clocks.stop()
    # the decomposition the model needs (not the reported value): the same
    # steps with the collectives left out, and one all-reduce of a layer's
    # partial (B x H fp32) timed alone
    ms_local = timed(max(3, args.steps // 2), no_reduce)
    ar_us = 0.0
    if ws > 1:
        P = torch.zeros((1, BATCH, H), dtype=torch.float32, device=dev)
        for _ in range(10):
            dist.all_reduce(P)
        n_ar = 200
        barrier()
        torch.cuda.synchronize()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for _ in range(n_ar):
            dist.all_reduce(P)
        a1.record(stream)
        torch.cuda.synchronize()
        ar_us = max_over_ranks(a0.elapsed_time(a1) / n_ar * 1e3, ws, dev)
    predicted_ms = ms_local + 2 * L * ar_us / 1e3
    if rank == 0:
        line = {"metric": METRIC + " [tensor-parallel over the job's GPUs]", "value": BATCH / (ms / 1e3),
                "unit": "tokens/s", "n_gpus": ws, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
                "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic (seeded N(0,0.02) weights, N(0,1) x/KV)",
                "config": dict(config_dict(), t=t, workload=f"70B-shaped 80-layer decode stack, t={t} shards on "
                               f"{t} GPU(s), NCCL all-reduce of the partials", reduce="nccl all-reduce"),
                "tp_model": {"step_ms_without_collectives": ms_local, "allreduce_us_per_call": ar_us,
                             "allreduces_per_step": 2 * L,
                             "predicted_ms": predicted_ms,
                             "measured_over_predicted": ms / predicted_ms,
                             "model": "T(N) = T(1)/N + 2L*T_allreduce(N), with T(1)/N taken as this rank's step "
                                      "without collectives"},
                "gpu_launches": sum(op.plan.decode_kernel_count(BATCH, tpl.TPL_REDUCE_SEPARATE) for op in layers)
                * args.steps,
                "clocks": clk}
        print(json.dumps(line), flush=True)
    if ws > 1:
        dist.destroy_process_group()
    return 0


def run_ours(args, ws, rank, local):
    import torch
    from megatron_tensor_transformer_plan_b200 import build
    build.build()
    from megatron_tensor_transformer_plan_b200 import synth, tpl
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600), device_id=dev)

    dims = tpl.make_dims(H, NQ, NKV, D, F, L, 1e-5, tpl.TPL_NORM | tpl.TPL_RESIDUAL)
    plan = tpl.Plan(dims, T_SHARDS)
    packed, kvs, keep = build_stack(plan, tpl, synth, torch, dev)
    x = synth.activations(BATCH, H, seed=0, dtype=torch.bfloat16, device=dev)
    y = torch.empty_like(x)
    wsb = plan.workspace(BATCH, KV_LEN, device=dev)
    stream = torch.cuda.Stream(device=dev)
    arr = (ctypes.c_void_p * L)(*[p.data_ptr() for p in packed])
    kva = (tpl.tpl_kv * L)(*kvs)

    def step(xin, yout):
        tpl.check(tpl.tpl_decode_stack(plan.handle, arr, kva, xin.data_ptr(), BATCH, KV_LEN, yout.data_ptr(), None,
                                       wsb.data_ptr(), wsb.numel(), tpl.TPL_REDUCE_FUSED, stream.cuda_stream),
                  "tpl_decode_stack")

    def barrier():
        if ws > 1:
            import torch.distributed as dist
            dist.barrier()

    # ---- device-resident throughput ----
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step(x, y)
    torch.cuda.synchronize()
    assert plan.last_device_error() == tpl.TPL_OK
    y_direct = y.clone()
    plan.reset_counters()
    # one CUDA graph per step: the 401 launches of tpl_decode_stack captured
    # once (their programmatic-dependent-launch edges included) and replayed;
    # the reductions are counted by the host call, so during the capture
    graph = None
    if not args.no_graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            step(x, y)
        y.zero_()
        with torch.cuda.stream(stream):
            for _ in range(args.warmup):
                graph.replay()
        torch.cuda.synchronize()
        assert plan.last_device_error() == tpl.TPL_OK
        assert torch.equal(y, y_direct), "graph replay differs from the direct calls"
        reductions = plan.reduction_count() * args.steps
    run_step = (lambda: graph.replay()) if graph is not None else (lambda: step(x, y))
    clocks = Clocks(local)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    e0.record(stream)
    with torch.cuda.stream(stream):
        for _ in range(args.steps):
            run_step()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, ws, dev)
    if graph is None:
        reductions = plan.reduction_count()
    tokens_per_s = ws * BATCH / (ms / 1e3)

    # ---- end to end: pinned host x in, y back to the host, every step ----
    xh = x.cpu().pin_memory()
    yh = torch.empty_like(xh).pin_memory()
    xd = torch.empty_like(x)
    e2e_step = lambda: step(xd, y)
    if graph is not None:
        graph_e2e = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph_e2e, stream=stream):
            step(xd, y)
        e2e_step = lambda: graph_e2e.replay()
    with torch.cuda.stream(stream):
        for _ in range(2):
            xd.copy_(xh, non_blocking=True)
            e2e_step()
            yh.copy_(y, non_blocking=True)
    torch.cuda.synchronize()
    barrier()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    e2e_steps = max(3, args.steps // 4)
    with torch.cuda.stream(stream):
        for _ in range(e2e_steps):
            xd.copy_(xh, non_blocking=True)
            e2e_step()
            yh.copy_(y, non_blocking=True)
    f1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(f0.elapsed_time(f1) / e2e_steps, ws, dev)

    # ---- the dominant kernel (gate/up) timed alone, one launch per layer ----
    act = torch.empty((BATCH, F), dtype=torch.bfloat16, device=dev)
    hbuf = torch.randn((BATCH, H), dtype=torch.float32, device=dev)
    with torch.cuda.stream(stream):
        for l in range(3):
            plan.gate_up(packed[l], hbuf, act, wsb)
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(L)]
    with torch.cuda.stream(stream):
        for l in range(L):
            evs[l][0].record(stream)
            plan.gate_up(packed[l], hbuf, act, wsb)
            evs[l][1].record(stream)
    torch.cuda.synchronize()
    gu_ms = sum(a.elapsed_time(b) for a, b in evs) / L
    # ---- the prefill row: one 70B layer over a 2048-token chunk (layer 0's
    # weights, its cache rows 0..2047 of sequence 0), timed alone ----
    xp = synth.activations(PREFILL_T, H, seed=0, layer=1000, dtype=torch.bfloat16, device=dev)
    yp = torch.empty_like(xp)
    wsp = plan.prefill_workspace(PREFILL_T, device=dev)
    with torch.cuda.stream(stream):
        for _ in range(3):
            plan.prefill_layer(packed[0], kvs[0], xp, yp, None, wsp)
    torch.cuda.synchronize()
    pf_times = []
    with torch.cuda.stream(stream):
        for _ in range(10):
            a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a_.record(stream)
            plan.prefill_layer(packed[0], kvs[0], xp, yp, None, wsp)
            b_.record(stream)
            pf_times.append((a_, b_))
    torch.cuda.synchronize()
    assert plan.last_device_error() == tpl.TPL_OK
    pf_ms = max_over_ranks(statistics.median(a_.elapsed_time(b_) for a_, b_ in pf_times), ws, dev)
    tpeak, tpeak_kind = load_tensor_peak()
    pf_tflops = prefill_flops() / (pf_ms / 1e3) / 1e12
    del wsp, xp, yp

    peak, peak_kind = load_peaks()
    configs = None
    if ws == 1 and not args.no_configs:
        del arr, kva, kvs, keep, packed, wsb
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
        configs = run_configs(tpl, peak, peak_kind, local, args.config_iters)
    gu_gbs = gate_up_bytes_per_launch() / (gu_ms / 1e3) / 1e9
    per_step = plan.decode_kernel_count(BATCH, n_layers=L)
    if plan.decode_kernel_count(BATCH) == 6:  # the tensor-core family: the gate/up call is two kernels
        gu_kernel = ("gate/up call: scale_split_kernel (h * gamma as bf16 hi + lo) + gemv_tc_kernel<16, true> "
                     "(tcgen05 gate/up, 1/rms and SwiGLU in the epilogue); timed together, traffic of the GEMV "
                     "kernel; inside the layer the O kernel writes that operand and no extra kernel runs")
    else:
        gu_kernel = "gemv_kernel<3, false> (gate/up + SwiGLU, activation as bf16 hi+lo)"
    step_gbs = algorithmic_bytes_per_step() / (ms / 1e3) / 1e9

    if rank == 0:
        line = {"metric": METRIC, "value": tokens_per_s, "unit": "tokens/s", "n_gpus": ws, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,0.02) weights, N(0,1) x/KV)",
                "config": dict(config_dict(), step_hbm_gbs=step_gbs, step_hbm_frac=step_gbs / peak,
                               algorithmic_bytes_per_step=algorithmic_bytes_per_step(),
                               reductions_counted=reductions // max(1, args.steps),
                               launch=("one CUDA graph per step (tpl_decode_stack captured once, replayed; "
                                       "bit-identical to direct calls)") if graph is not None
                               else "tpl_decode_stack called every step"),
                "roofline": {"bound": "hbm", "kernel": gu_kernel, "achieved": gu_gbs,
                             "peak": peak, "peak_kind": peak_kind + " (burst copy, kernel timed alone)",
                             "unit": "GB/s", "frac": gu_gbs / peak, "traffic": recorded_traffic(),
                             "algorithmic_bytes_per_launch": gate_up_bytes_per_launch(), "launch_ms": gu_ms},
                "e2e": {"value": ws * BATCH / (e2e_ms / 1e3), "unit": "tokens/s",
                        "h2d_bytes_per_step": x.numel() * 2, "d2h_bytes_per_step": y.numel() * 2},
                "gpu_launches": per_step * args.steps,
                "clocks": clk,
                "prefill": {"workload": f"70B-shaped layer prefill, t={T_SHARDS}, {PREFILL_T} tokens, causal in chunk",
                            "ms_per_layer": pf_ms, "tokens_per_s": ws * PREFILL_T / (pf_ms / 1e3),
                            "flop_per_layer": prefill_flops(), "achieved_tflops": pf_tflops,
                            "peak_tflops": tpeak, "peak_kind": tpeak_kind + " (dense bf16 burst)",
                            "frac": pf_tflops / tpeak, "timing": "median of 10 calls, CUDA events, after 3 warm-ups",
                            "kernels_per_layer": 7}}
        if configs is not None:
            line["configs"] = configs
        if ws == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline_sample()
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


# Per-configuration decode layers (the per-configuration targets): one layer call
# per timed iteration, CUDA events on the launching stream, median of
# `iters` after 3 warm-ups; working sets under 4 x L2 rotate over copies of
# the weights and caches so that every call reads from HBM.
CONFIG_CASES = [
    # name, H, nq, nkv, F, t, B, S, reduce, extra
    ("config 1: tiny MLP block", 256, 2, 2, 688, 2, 1, 0, "fused", dict(flags=0, mlp_only=True)),
    ("config 1: tiny MLP block", 256, 2, 2, 688, 2, 1, 0, "separate", dict(flags=0, mlp_only=True)),
] + [
    ("config 2: 7B layer", 4096, 32, 32, 11008, t, B, 2048, mode, {})
    for B in (1, 16) for t in (1, 2, 4) for mode in (("fused",) if t == 1 else ("fused", "separate"))
] + [
    ("config 3: 70B layer", 8192, 64, 8, 28672, t, 16, 8192, mode, {})
    for t in (1, 4, 8) for mode in (("fused", "separate") if t == 4 else ("fused",))
] + [
    ("config 5: one stack layer", 8192, 64, 8, 28672, 8, 4, 4096, "fused", {}),
]


def attach_overheads(rows):
    """Give every fused row with t > 1 its time over the same workload's
    unsharded (t = 1, fused) row at the same batch: the fused-reduction
    overhead (at most 5% is the target)."""
    base = {(r["workload"], r["batch"]): r["us_per_layer"] for r in rows if r["t"] == 1 and r["reduce"] == "fused"}
    for r in rows:
        b = base.get((r["workload"], r["batch"]))
        if b is not None and r["reduce"] == "fused" and r["t"] > 1:
            r["overhead_vs_t1"] = r["us_per_layer"] / b - 1.0
    return rows


def run_configs(tpl, peak, peak_kind, gpu_index, iters):
    """Microseconds per layer, algorithmic GB/s and fraction of the copy
    peak for each case, and each shard layout's fused time against the same
    workload's unsharded (t = 1) layer."""
    from megatron_tensor_transformer_plan_b200 import profile_configs as pc
    clocks = Clocks(gpu_index)
    clocks.start()
    rows = []
    for name, Hc, nq, nkv, Fc, t, B, S, mode, extra in CONFIG_CASES:
        us, nbytes, ncopies, rc = pc.run_layer(tpl, Hc, nq, nkv, Fc, t, B, S, iters, mode, extra.get("flags"),
                                               extra.get("mlp_only", False))
        if rc != tpl.TPL_OK:
            raise RuntimeError(f"{name}: device status {rc}")
        gbs = nbytes / (us * 1e-6) / 1e9
        rows.append({"workload": name, "hidden": Hc, "ffn": Fc, "t": t, "batch": B, "kv_len": S, "reduce": mode,
                     "us_per_layer": us, "tokens_per_s": B / (us * 1e-6), "algorithmic_bytes": nbytes,
                     "gb_s": gbs, "frac": gbs / peak, "copies_rotated": ncopies})
    clk = clocks.stop()
    attach_overheads(rows)
    return {"peak_gbs": peak, "peak_kind": peak_kind + " (burst copy)",
            "timing": f"CUDA events around each layer call, median of {iters} after 3 warm-ups",
            "bytes": "every weight once, the K/V cache once, new K/V, x and y",
            "rows": rows, "clocks": clk}


def _cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def _time_oracle(fn, min_runs=1, budget_s=10.0):
    """Mean seconds per call of fn over at least min_runs calls, stopping
    once budget_s has passed."""
    t0 = time.perf_counter()
    n = 0
    while True:
        fn()
        n += 1
        if n >= min_runs and time.perf_counter() - t0 > budget_s:
            break
        if n >= 5:
            break
    return (time.perf_counter() - t0) / n, n


def cpu_baseline_sample():
    """The oracle as it stands (plain fp64 C loops) on the host cores, on
    bounded samples of the workloads: single-threaded and on every core.

    All cores: config 1 (tiny MLP) and config 2 (7B layer, B = 1 and 16) and
    config 3 (70B layer, B = 16, KV 8192) in full, config 4 (70B prefill) on
    a 256-token chunk scaled to 2048 tokens by the FLOP count, and one layer
    of the 80-layer stack scaled by 80 (the bench workload).  One thread: the
    same, except that the larger cases run one sequence and scale by the
    batch (each sequence is independent work in the oracle) and the prefill
    is left out.  Each sample says what it ran."""
    import numpy as np
    import torch
    import oracle
    from megatron_tensor_transformer_plan_b200 import synth
    threads = os.cpu_count() or 1
    f64 = lambda t: t.float().numpy().astype(np.float64)

    def layer(H, nq, nkv, F, seed=0, mlp_only=False):
        w = synth.layer_weights(H, nq, nkv, D, F, seed=seed, dtype=torch.bfloat16, device="cpu", mlp_only=mlp_only)
        return {k: synth.bits(v) for k, v in w.items()}

    def kv(B, nkv, S, seed=0):
        kl, vl = synth.kv_cache((B, nkv, S + 1, D), seed=seed)
        return synth.bits(kl), synth.bits(vl)

    out = {"cpu_model": _cpu_model(), "nproc": threads, "entries": []}

    def add(name, cores, secs, n, unit_per_s, unit, sample):
        out["entries"].append({"workload": name, "cores": cores, "seconds_per_call": secs, "runs": n,
                               "value": unit_per_s, "unit": unit, "sample": sample})

    # config 1: tiny MLP block, t = 2 (the oracle's unsharded MLP; flags 0)
    d1 = oracle.Dims(256, 2, 2, D, 688, flags=0)
    w1 = layer(256, 2, 2, 688, mlp_only=True)
    x1 = f64(synth.activations(1, 256, seed=0))
    for cores in (1, threads):
        oracle.set_threads(cores)
        secs, n = _time_oracle(lambda: oracle.mlp_sharded(d1, w1, 1, x1), 5, 0.5)
        add("config 1: tiny MLP H=256 F=688, 1 token", cores, secs, n, 1 / secs, "tokens/s", "full")
    # config 2: 7B layer (t does not change the unsharded oracle), KV 2048
    d2 = oracle.Dims(4096, 32, 32, D, 11008)
    w2 = layer(4096, 32, 32, 11008)
    k2, v2 = kv(16, 32, 2048)
    for B in (1, 16):
        x2 = f64(synth.activations(B, 4096, seed=0))
        for cores in (1, threads):
            oracle.set_threads(cores)
            Bs = 1 if (cores == 1 and B > 1) else B
            secs, n = _time_oracle(lambda: oracle.decode_layer(d2, w2, x2[:Bs], k2[:Bs], v2[:Bs], 2048), 1, 2.0)
            secs *= B / Bs
            add(f"config 2: 7B layer B={B} KV 2048", cores, secs, n, B / secs, "tokens/s",
                "full" if Bs == B else f"{Bs} of {B} sequences, x{B // Bs}")
    del w2, k2, v2
    # config 3: 70B layer, B = 16, KV 8192
    d3 = oracle.Dims(H, NQ, NKV, D, F)
    w3 = layer(H, NQ, NKV, F)
    k3, v3 = kv(16, NKV, 8192)
    x3 = f64(synth.activations(16, H, seed=0))
    for cores in (threads, 1):
        oracle.set_threads(cores)
        Bs = 1 if cores == 1 else 16
        secs, n = _time_oracle(lambda: oracle.decode_layer(d3, w3, x3[:Bs], k3[:Bs], v3[:Bs], 8192), 1, 2.0)
        secs *= 16 / Bs
        add("config 3: 70B layer B=16 KV 8192", cores, secs, n, 16 / secs, "tokens/s",
            "full" if Bs == 16 else "1 of 16 sequences, x16")
    del k3, v3
    # the bench workload: one layer of the stack (B = 4, KV 4096), x80 layers
    k5, v5 = kv(BATCH, NKV, KV_LEN)
    x5 = f64(synth.activations(BATCH, H, seed=0))
    for cores in (threads, 1):
        oracle.set_threads(cores)
        Bs = BATCH if cores > 1 else 1
        secs, n = _time_oracle(lambda: oracle.decode_layer(d3, w3, x5[:Bs], k5[:Bs], v5[:Bs], KV_LEN), 1, 2.0)
        secs *= BATCH / Bs
        add(f"config 5: 80-layer stack B={BATCH} KV {KV_LEN}", cores, secs * L, n, BATCH / (secs * L), "tokens/s",
            f"one layer{'' if Bs == BATCH else f', 1 of {BATCH} sequences x{BATCH}'}, x{L} layers extrapolated")
    del k5, v5
    # config 4: prefill, a 256-token chunk, scaled to 2048 tokens by FLOPs
    oracle.set_threads(threads)
    Tp = 256
    xp = f64(synth.activations(Tp, H, seed=0, layer=1000))
    secs, n = _time_oracle(lambda: oracle.prefill_layer(d3, w3, xp), 1, 0.0)
    secs_full = secs * prefill_flops(PREFILL_T) / prefill_flops(Tp)
    add(f"config 4: 70B prefill {PREFILL_T} tokens", threads, secs_full, n, PREFILL_T / secs_full, "tokens/s",
        f"one {Tp}-token chunk, scaled to {PREFILL_T} tokens by the FLOP count "
        f"({prefill_flops(PREFILL_T) / prefill_flops(Tp):.2f}x)")
    oracle.set_threads(threads)
    stack = [e for e in out["entries"] if e["workload"].startswith("config 5") and e["cores"] == threads][0]
    out.update({"value": stack["value"], "unit": "tokens/s", "cores": threads, "kind": "oracle",
                "sample": stack["sample"]})
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip the per-configuration layer timings")
    ap.add_argument("--tp", action="store_true",
                    help="shard the stack over the job's GPUs (one shard per rank, NCCL all-reduce) instead of "
                         "running an independent replica per GPU")
    ap.add_argument("--config-iters", type=int, default=30)
    ap.add_argument("--no-graph", action="store_true",
                    help="call tpl_decode_stack every step instead of replaying one captured CUDA graph")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    ws, rank, local = dist_init()
    if args.impl == "reference":
        return run_reference(args, ws, rank)
    if args.tp:
        return run_tp(args, ws, rank, local)
    return run_ours(args, ws, rank, local)


if __name__ == "__main__":
    sys.exit(main())
