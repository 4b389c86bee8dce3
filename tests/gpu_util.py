"""Helpers for the GPU parity tests: build a layer on the device from the
seeded generators, run it through the C-ABI, and evaluate the oracle on the
same input bits."""
from __future__ import annotations

import os
from dataclasses import dataclass

import numpy as np
import torch

import oracle
from megatron_tensor_transformer_plan_b200 import synth, tpl

TOL = 2e-2  # |gpu - oracle| <= TOL * (|oracle| + RMS(oracle)), per element

oracle.set_threads(os.cpu_count() or 1)


def close_rel(gpu, ref, tol=TOL):
    """Return (ok, worst normalised error)."""
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    bound = tol * (np.abs(ref) + rms)
    err = np.abs(gpu - ref)
    worst = float(np.max(err / np.maximum(bound, 1e-300) * tol)) if ref.size else 0.0
    return bool(np.all(err <= bound)) and np.all(np.isfinite(gpu)), worst


def assert_close_rel(gpu, ref, tol=TOL, what=""):
    ok, worst = close_rel(gpu, ref, tol)
    assert ok, f"{what}: worst normalised error {worst:.3e} > {tol}"
    return worst


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


@dataclass
class Layer:
    plan: tpl.Plan
    dims: tpl.tpl_dims
    t: int
    B: int
    S: int
    S_cap: int
    w: dict
    packed: torch.Tensor
    x: torch.Tensor
    kv_logical: tuple
    k: torch.Tensor
    v: torch.Tensor
    kv: tpl.tpl_kv
    ws: torch.Tensor


def make_layer(H, nq, nkv, d, F, t, B, S, *, flags=tpl.TPL_NORM | tpl.TPL_RESIDUAL, seed=0, layer=0,
               S_cap=None, gamma_std=0.0, n_layers=1, mlp_only=False, device="cuda") -> Layer:
    fp32 = bool(flags & tpl.TPL_FP32_WEIGHTS)
    dt = torch.float32 if fp32 else torch.bfloat16
    dims = tpl.make_dims(H, nq, nkv, d, F, n_layers, 1e-5, flags)
    plan = tpl.Plan(dims, t)
    w = synth.layer_weights(H, nq, nkv, d, F, seed=seed, layer=layer, dtype=dt, device=device,
                            gamma_std=gamma_std, mlp_only=mlp_only)
    packed = plan.pack_layer(w)
    x = synth.activations(B, H, seed=seed, layer=layer, dtype=dt, device=device)
    S_cap = S_cap or (S + 1)
    kl, vl = synth.kv_cache((B, nkv, S_cap, d), seed=seed, layer=layer, device=device)
    k = plan.pack_kv(kl)
    v = plan.pack_kv(vl)
    kv = tpl.Plan.kv(k, v, B, S_cap)
    ws = plan.workspace(B, S, device=device)
    torch.cuda.synchronize()
    return Layer(plan, dims, t, B, S, S_cap, w, packed, x, (kl, vl), k, v, kv, ws)


def oracle_weights(L: Layer) -> dict:
    out = {k: synth.bits(v) for k, v in L.w.items() if k.startswith("w")}
    out["gamma_attn"] = synth.bits(L.w["gamma_attn"])
    out["gamma_mlp"] = synth.bits(L.w["gamma_mlp"])
    return out


def oracle_dims(L: Layer) -> oracle.Dims:
    d = L.dims
    return oracle.Dims(d.hidden, d.n_q_heads, d.n_kv_heads, d.head_dim, d.ffn, eps=float(d.rms_eps),
                       flags=int(d.flags) & (tpl.TPL_NORM | tpl.TPL_RESIDUAL | tpl.TPL_ROPE),
                       rope_base=float(d.rope_base))


def oracle_decode(L: Layer, x=None):
    x = L.x if x is None else x
    return oracle.decode_layer(oracle_dims(L), oracle_weights(L), to_np(x), synth.bits(L.kv_logical[0]),
                               synth.bits(L.kv_logical[1]), L.S, trace=True)


def run_steps(L: Layer, mode=tpl.TPL_REDUCE_FUSED):
    """Run the layer step by step through the per-step entry points and
    return every intermediate (the same kernels tpl_decode_layer runs)."""
    p, d = L.plan, L.dims
    B, H, F = L.B, d.hidden, d.ffn
    nqd = d.n_q_heads * d.head_dim
    dt = p.act_dtype
    dev = L.x.device
    q = torch.empty((B, d.n_q_heads, d.head_dim), dtype=torch.float32, device=dev)
    o = torch.empty((B, nqd), dtype=dt, device=dev)
    h = torch.empty((B, H), dtype=torch.float32, device=dev)
    act = torch.empty((B, F), dtype=dt, device=dev)
    y = torch.empty((B, H), dtype=dt, device=dev)
    y32 = torch.empty((B, H), dtype=torch.float32, device=dev)
    resid = bool(d.flags & tpl.TPL_RESIDUAL)
    kn = torch.empty((B, d.n_kv_heads, d.head_dim), dtype=torch.float32, device=dev)
    vn = torch.empty_like(kn)
    p.qkv(L.packed, L.kv, L.x, L.S, q, L.ws, kn, vn)
    p.attn_decode(L.kv, q, L.S, o, L.ws, kn, vn)
    if mode == tpl.TPL_REDUCE_FUSED:
        p.o_proj(L.packed, o, L.x, h=h, ws=L.ws)
    else:
        P = torch.empty((L.t, B, H), dtype=torch.float32, device=dev)
        p.o_proj(L.packed, o, None, partials=P, ws=L.ws)
        p.reduce_partials(P, L.x if resid else None, False if dt == torch.bfloat16 else True, out32=h)
    p.gate_up(L.packed, h, act, L.ws)
    P2 = None
    if mode == tpl.TPL_REDUCE_FUSED:
        p.down_proj(L.packed, act, h, y=y, y32=y32, ws=L.ws)
    else:
        P2 = torch.empty((L.t, B, H), dtype=torch.float32, device=dev)
        p.down_proj(L.packed, act, None, partials=P2, ws=L.ws)
        p.reduce_partials(P2, h if resid else None, True, out32=y32, out_act=y)
    torch.cuda.synchronize()
    return {"q": q, "k_new": kn, "v_new": vn, "attn": o, "h": h, "act": act, "y": y, "y32": y32,
            "down_partials": P2}


def new_kv_slot(L: Layer):
    """The k/v the layer wrote at slot S, gathered back to [B][n_kv*d]."""
    d = L.dims
    t, B, nkv_s = L.t, L.B, d.n_kv_heads // L.t
    kk = L.k.view(t, B, nkv_s, L.S_cap, d.head_dim)[:, :, :, L.S, :]  # [t][B][nkv_s][d]
    vv = L.v.view(t, B, nkv_s, L.S_cap, d.head_dim)[:, :, :, L.S, :]
    kk = kk.permute(1, 0, 2, 3).reshape(B, d.n_kv_heads * d.head_dim)
    vv = vv.permute(1, 0, 2, 3).reshape(B, d.n_kv_heads * d.head_dim)
    return kk, vv
