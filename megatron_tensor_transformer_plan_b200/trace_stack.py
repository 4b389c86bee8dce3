"""Per-kernel timeline of a chained decode stack, from the traced build of the
library (libtpl_trace.so: one record per CTA with global-timer marks at entry,
after the dependency wait, at the end of the main loop and at exit).

For every launch in the chain it reports, relative to the end of the launch
before it (the last CTA's exit):
  exposed   its own last exit minus the previous launch's last exit: the time
            the chain spends on it;
  release   its last CTA's wait-passed mark minus the previous last exit
            (how long after the producer finished the last consumer CTA ran);
  loop      the slowest CTA's main-loop end minus the release;
  tail      its last exit minus the slowest main-loop end (the cross-CTA
            combines and epilogues that finish the kernel);
  spread    the slowest minus the median main-loop end over CTAs.
Medians over the layers of the stack.

    python -m megatron_tensor_transformer_plan_b200.trace_stack [--layers N] [--t T] [--batch B] [--kv S]
        [--shape 70b|7b] [--gemv-mode M] [--attn-mode A] [--steps K]
"""
from __future__ import annotations

import argparse
import json
import os
import statistics

import torch

from megatron_tensor_transformer_plan_b200 import build, synth

D = 128
SHAPES = {"70b": (8192, 64, 8, 28672), "7b": (4096, 32, 32, 11008)}


def launches(records):
    """Group per-CTA records into launches: all CTAs of a grid start before
    any CTA of the next dependent grid, so launches are runs of one tag in
    entry order, each holding `grid` records."""
    recs = sorted(records, key=lambda r: r[4][0])
    out, cur = [], None
    for r in recs:
        tag, grid = r[0], r[3]
        if cur is None or cur["tag"] != tag or len(cur["ctas"]) >= cur["grid"]:
            cur = {"tag": tag, "grid": grid, "ctas": []}
            out.append(cur)
        cur["ctas"].append(r)
    return out


def epilogue_stats(L, epi):
    """The tensor-core projections' epilogue marks of the launch's last shared
    tiles (publish, arrival counted, pieces listed, tile finished)."""
    t2 = [c[4][2] for c in L["ctas"] if c[4][2]]
    if not epi or not t2:
        return {}
    last_issue = max(t2)
    lasts = [e for e in epi if e[4][2] > e[4][1]]
    out = {"publish_after_issue": (max(e[4][0] for e in epi) - last_issue) / 1e3,
           "count": statistics.median((e[4][1] - e[4][0]) / 1e3 for e in epi)}
    if lasts:
        out["list"] = statistics.median((e[4][2] - e[4][1]) / 1e3 for e in lasts)
        out["combine"] = statistics.median((e[4][3] - e[4][2]) / 1e3 for e in lasts)
        out["combine_max"] = max((e[4][3] - e[4][2]) / 1e3 for e in lasts)
        out["lasts"] = len(lasts)
    return out


def summarise(ls, epi_records=()):
    rows = []
    prev_end = None
    for L in ls:
        t0 = [c[4][0] for c in L["ctas"]]
        t1 = [c[4][1] for c in L["ctas"] if c[4][1]]
        t2 = [c[4][2] for c in L["ctas"] if c[4][2]]
        t3 = [c[4][3] for c in L["ctas"]]
        end = max(t3)
        row = {"kernel": L["tag"], "ctas": len(L["ctas"]), "grid": L["grid"]}
        if prev_end is not None:
            row["exposed"] = (end - prev_end) / 1e3
            row["first_entry"] = (min(t0) - prev_end) / 1e3
            if t1:
                row["release"] = (max(t1) - prev_end) / 1e3
            if t2 and t1:
                row["loop"] = (max(t2) - max(t1)) / 1e3
                row["tail"] = (end - max(t2)) / 1e3
                row["spread"] = (max(t2) - statistics.median(t2)) / 1e3
        start = min(t0)
        epi = [e for e in epi_records if e[0] == L["tag"] + ".epi" and start <= e[4][0] <= end]
        row.update({"epi_" + k: v for k, v in epilogue_stats(L, epi).items()})
        rows.append(row)
        prev_end = end
    return rows


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--layers", type=int, default=6)
    ap.add_argument("--shape", default="70b", choices=sorted(SHAPES))
    ap.add_argument("--t", type=int, default=8)
    ap.add_argument("--batch", type=int, default=4)
    ap.add_argument("--kv", type=int, default=4096)
    ap.add_argument("--gemv-mode", type=int, default=4)
    ap.add_argument("--attn-mode", type=int, default=0, help="TPL_OPT_DECODE_ATTN of the plan (0: the default)")
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--json", default="")
    args = ap.parse_args()
    if not os.environ.get("TPL_LIB"):  # another traced build may be named explicitly
        os.environ["TPL_LIB"] = build.build(trace=True)
    from megatron_tensor_transformer_plan_b200 import tpl
    H, NQ, NKV, F = SHAPES[args.shape]
    T, B, S, NL = args.t, args.batch, args.kv, args.layers
    dev = torch.device("cuda")
    plan = tpl.Plan(tpl.make_dims(H, NQ, NKV, D, F, NL, 1e-5, tpl.TPL_NORM | tpl.TPL_RESIDUAL), T)
    plan.set_option(tpl.TPL_OPT_GEMV_MODE, args.gemv_mode)
    plan.set_option(tpl.TPL_OPT_DECODE_ATTN, args.attn_mode)
    packed, kvs, keep = [], [], []
    for l in range(NL):
        w = synth.layer_weights(H, NQ, NKV, D, F, seed=0, layer=l, device=dev)
        packed.append(plan.pack_layer(w))
        del w
        k, v = synth.kv_cache((T, B, NKV // T, S + 1, D), seed=0, layer=l, device=dev)
        keep.append((k, v))
        kvs.append(tpl.Plan.kv(k, v, B, S + 1))
    x = synth.activations(B, H, seed=0, device=dev)
    y = torch.empty_like(x)
    ws = plan.workspace(B, S, device=dev)
    for _ in range(2):
        plan.decode_stack(packed, kvs, x, S, y, None, ws)
    torch.cuda.synchronize()
    tpl.trace_read()  # drop the warm-up records
    per_kind = {}
    clk = {}
    for _ in range(args.steps):
        plan.decode_stack(packed, kvs, x, S, y, None, ws)
        torch.cuda.synchronize()
        recs = tpl.trace_read()
        main_recs = [r for r in recs if not r[0].endswith((".epi", ".clk"))]
        epi_recs = [r for r in recs if r[0].endswith(".epi")]
        for r in recs:  # combine phases in SM cycles: list, loads and sums, final write
            if r[0].endswith(".clk") and r[4][3] >= r[4][0] > 0:
                t = r[4]
                clk.setdefault(r[0], []).append((t[1] - t[0], t[2] - t[1], t[3] - t[2]))
        rows = summarise(launches(main_recs), epi_recs)
        for r in rows[1:]:  # the first launch has no predecessor in this step
            per_kind.setdefault(r["kernel"], []).append(r)
    assert plan.last_device_error() == tpl.TPL_OK
    out = {"shape": args.shape, "t": T, "batch": B, "kv": S, "layers": NL, "gemv_mode": args.gemv_mode,
           "attn_mode": args.attn_mode,
           "kernels": {}}
    order = ["operand", "qkv", "attention", "o_proj", "gate_up", "down"]
    print(f"{'kernel':10s} {'n':>4s} {'exposed':>8s} {'release':>8s} {'loop':>8s} {'tail':>8s} {'spread':>8s}  (us)")
    for k in order + sorted(set(per_kind) - set(order)):
        rs = per_kind.get(k)
        if not rs:
            continue
        fields = sorted({f for r in rs for f in r if f not in ("kernel", "ctas", "grid")})
        med = {f: statistics.median(r[f] for r in rs if f in r) for f in fields}
        out["kernels"][k] = dict(med, launches=len(rs))
        print(f"{k:10s} {len(rs):4d} " + " ".join(f"{med.get(f, float('nan')):8.1f}" for f in
                                                  ("exposed", "release", "loop", "tail", "spread")))
        ep = {f: v for f, v in med.items() if f.startswith("epi_")}
        if ep:
            print("           epilogue: " + ", ".join(f"{f[4:]} {v:.1f}" for f, v in sorted(ep.items())))
    for k, v in sorted(clk.items()):
        print(f"{k:14s} combine cycles (median of {len(v)}): list {statistics.median(x[0] for x in v):.0f}, "
              f"loads+sums {statistics.median(x[1] for x in v):.0f}, final {statistics.median(x[2] for x in v):.0f}; "
              f"slowest total {max(sum(x) for x in v):.0f}")
    print(f"sum of median exposed times per layer: {sum(v['exposed'] for k, v in out['kernels'].items() if k != 'operand'):.1f} us")
    if args.json:
        with open(args.json, "w") as f:
            json.dump(out, f, indent=1)


if __name__ == "__main__":
    main()
