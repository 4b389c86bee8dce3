"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle.

This module holds no arithmetic of the method: it only draws random tensors
(weights ~ N(0, 0.02), activations and KV cache ~ N(0, 1), norm gains = 1 or
1 + N(0, 0.02)) from torch generators keyed by (seed, layer, tensor id), so
that the same call always yields the same bits.  Large tensors are drawn in
fixed-size chunks so that the result does not depend on free memory.

Shapes follow the nn.Linear orientation W[out][in]:
  wq [n_q*d][H], wk/wv [n_kv*d][H], wo [H][n_q*d], wg/wu [F][H], wd [H][F].
"""
from __future__ import annotations

import torch

TENSOR_IDS = {"wq": 1, "wk": 2, "wv": 3, "wo": 4, "wg": 5, "wu": 6, "wd": 7,
              "gamma_attn": 8, "gamma_mlp": 9, "x": 10, "k_cache": 11, "v_cache": 12}

_CHUNK = 1 << 26  # elements drawn per generator call


def sub_seed(seed: int, layer: int, tensor_id: int) -> int:
    """A fixed 63-bit mixing of (seed, layer, tensor id)."""
    v = (seed * 0x9E3779B97F4A7C15 + (layer + 1) * 0xBF58476D1CE4E5B9 + tensor_id * 0x94D049BB133111EB)
    v &= (1 << 64) - 1
    v ^= v >> 31
    return v & ((1 << 63) - 1)


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def normal_(out: torch.Tensor, std: float, seed: int, mean: float = 0.0) -> torch.Tensor:
    """Fill `out` (any float dtype) with N(mean, std^2) drawn in float32 chunks."""
    g = _gen(out.device, seed)
    flat = out.view(-1)
    n = flat.numel()
    for s in range(0, n, _CHUNK):
        e = min(n, s + _CHUNK)
        tmp = torch.randn(e - s, generator=g, device=out.device, dtype=torch.float32)
        if std != 1.0:
            tmp.mul_(std)
        if mean != 0.0:
            tmp.add_(mean)
        flat[s:e].copy_(tmp)
    return out


def layer_weight_shapes(H: int, nq: int, nkv: int, d: int, F: int) -> dict:
    return {"wq": (nq * d, H), "wk": (nkv * d, H), "wv": (nkv * d, H), "wo": (H, nq * d),
            "wg": (F, H), "wu": (F, H), "wd": (H, F)}


def layer_weights(H: int, nq: int, nkv: int, d: int, F: int, *, seed: int = 0, layer: int = 0,
                  dtype=torch.bfloat16, device="cpu", std: float = 0.02,
                  gamma_std: float = 0.0, mlp_only: bool = False) -> dict:
    """Unsharded weights of one layer.  gamma_* are float32 (ones when
    gamma_std == 0, else 1 + N(0, gamma_std^2))."""
    shapes = layer_weight_shapes(H, nq, nkv, d, F)
    names = ("wg", "wu", "wd") if mlp_only else tuple(shapes)
    w = {}
    for name in names:
        t = torch.empty(shapes[name], dtype=dtype, device=device)
        normal_(t, std, sub_seed(seed, layer, TENSOR_IDS[name]))
        w[name] = t
    for name in ("gamma_attn", "gamma_mlp"):
        gmm = torch.ones(H, dtype=torch.float32, device=device)
        if gamma_std:
            normal_(gmm, gamma_std, sub_seed(seed, layer, TENSOR_IDS[name]), mean=1.0)
        w[name] = gmm
    return w


def activations(B: int, H: int, *, seed: int = 0, layer: int = 0, dtype=torch.bfloat16,
                device="cpu") -> torch.Tensor:
    x = torch.empty((B, H), dtype=dtype, device=device)
    return normal_(x, 1.0, sub_seed(seed, layer, TENSOR_IDS["x"]))


def kv_cache(shape, *, seed: int = 0, layer: int = 0, device="cpu"):
    """K and V caches (bf16, N(0, 1)) of the given shape."""
    k = torch.empty(shape, dtype=torch.bfloat16, device=device)
    v = torch.empty(shape, dtype=torch.bfloat16, device=device)
    normal_(k, 1.0, sub_seed(seed, layer, TENSOR_IDS["k_cache"]))
    normal_(v, 1.0, sub_seed(seed, layer, TENSOR_IDS["v_cache"]))
    return k, v


def bits(t: torch.Tensor):
    """Raw bit view of a bf16 tensor as a numpy uint16 array (host copy), or
    a float32 numpy array for float32 tensors."""
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view("uint16")
    if t.dtype == torch.float32:
        return t.numpy()
    raise TypeError(t.dtype)
