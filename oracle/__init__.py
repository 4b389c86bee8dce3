"""Oracle for the single-device Megatron-style tensor-parallel layer.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The product library
never calls into it, and it shares no code with the CUDA path: the arithmetic
lives in ``tpl_oracle.c`` (plain fp64 loops), this module only marshals numpy
arrays through ctypes.

Every function cites the page passage it follows, by page title and section:

* "Tensor parallel scaling curves", section "What tensor parallelism actually
  splits" -- head-wise column split of Q/K/V, each shard attending over its own
  heads without exchange,
  row split of the output projection, gate/up column split, down row split,
  partial sums added (two per layer, 2L per pass).
* "Tensor Parallelism Fundamentals", sections "Mechanics of Matrix Slicing" and
  "Memory Overhead and Communication Bottlenecks" -- column-then-row slicing,
  weights divided by t, the per-GPU KV formula.

Parity status: every function here is pinned by ``tests/test_oracle.py``
(closed forms, exact integer identities, the pages' worked numbers and an
independent numpy float64 evaluation).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "tpl_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

NORM = 1
RESIDUAL = 2
ROPE = 8


def build(force: bool = False) -> str:
    """Compile the C oracle (gcc, -O2, no fast-math, no FP contraction)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
               "-std=c11", "-o", _LIB_PATH + ".tmp", _SRC, "-lm"]
        subprocess.check_call(cmd)
        os.replace(_LIB_PATH + ".tmp", _LIB_PATH)
    return _LIB_PATH


class _Dims(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int32), ("n_q_heads", ctypes.c_int32),
                ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("ffn", ctypes.c_int32), ("eps", ctypes.c_double), ("flags", ctypes.c_uint32),
                ("rope_base", ctypes.c_double)]


class _Weights(ctypes.Structure):
    _fields_ = [("wq", ctypes.c_void_p), ("wk", ctypes.c_void_p), ("wv", ctypes.c_void_p),
                ("wo", ctypes.c_void_p), ("wg", ctypes.c_void_p), ("wu", ctypes.c_void_p),
                ("wd", ctypes.c_void_p), ("gamma_attn", ctypes.c_void_p),
                ("gamma_mlp", ctypes.c_void_p), ("wtype", ctypes.c_int32)]


class _Trace(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("k_new", ctypes.c_void_p), ("v_new", ctypes.c_void_p),
                ("attn", ctypes.c_void_p), ("h", ctypes.c_void_p), ("act", ctypes.c_void_p)]


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        L = _lib
        L.orc_decode_layer.restype = ctypes.c_int
        L.orc_prefill_layer.restype = ctypes.c_int
        L.orc_prefill_chunk.restype = ctypes.c_int
        L.orc_mlp_sharded.restype = ctypes.c_int
        L.orc_attn_sharded.restype = ctypes.c_int
        L.orc_plan_maps.restype = ctypes.c_int
        L.orc_kv_bytes_per_shard.restype = ctypes.c_longlong
        L.orc_kv_bytes_per_shard.argtypes = [ctypes.c_longlong] * 7
        L.orc_layer_params_per_shard.restype = ctypes.c_longlong
        L.orc_reductions_per_pass.restype = ctypes.c_longlong
        L.orc_reductions_per_pass.argtypes = [ctypes.c_longlong]
        L.orc_silu.restype = ctypes.c_double
        L.orc_silu.argtypes = [ctypes.c_double]
        L.orc_get_threads.restype = ctypes.c_int
        L.orc_set_threads.argtypes = [ctypes.c_int]
    return _lib


def set_threads(n: int) -> None:
    lib().orc_set_threads(int(n))


def get_threads() -> int:
    return int(lib().orc_get_threads())


@dataclass
class Dims:
    hidden: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    ffn: int
    eps: float = 1e-5
    flags: int = NORM | RESIDUAL
    rope_base: float = 500000.0

    def c(self) -> _Dims:
        return _Dims(self.hidden, self.n_q_heads, self.n_kv_heads, self.head_dim, self.ffn,
                     float(self.eps), int(self.flags), float(self.rope_base))


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _weights_struct(w: dict):
    """w: numpy arrays in nn.Linear orientation: wq, wk, wv, wo, wg, wu, wd as
    uint16 (raw bf16 bits) or float32; optional gamma_attn, gamma_mlp float32."""
    keep = {}
    wtype = None
    for k in ("wq", "wk", "wv", "wo", "wg", "wu", "wd"):
        a = w.get(k)
        if a is None:
            keep[k] = None
            continue
        a = np.ascontiguousarray(a)
        t = 0 if a.dtype == np.uint16 else 1
        if a.dtype not in (np.uint16, np.float32):
            raise TypeError(f"{k}: weights must be uint16 (bf16 bits) or float32, got {a.dtype}")
        if wtype is None:
            wtype = t
        elif wtype != t:
            raise TypeError("all weights must share one dtype")
        keep[k] = a
    for k in ("gamma_attn", "gamma_mlp"):
        a = w.get(k)
        keep[k] = None if a is None else np.ascontiguousarray(a, dtype=np.float32)
    s = _Weights(*[_p(keep[k]) for k in ("wq", "wk", "wv", "wo", "wg", "wu", "wd",
                                          "gamma_attn", "gamma_mlp")], wtype or 0)
    return s, keep


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of raw bf16 bit patterns to float64."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def decode_layer(dims: Dims, w: dict, x: np.ndarray, kc: np.ndarray, vc: np.ndarray, S: int,
                 trace: bool = False):
    """Unsharded decode layer ("Tensor parallel scaling curves", "What tensor
    parallelism actually splits", read unsharded).  x [B][H] float64; kc/vc
    uint16 [B][n_kv][S_cap][d]; S cached tokens.  Returns y [B][H] (float64)
    and, if trace, a dict of q, k_new, v_new, attn, h, act."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    B, H = x.shape
    kc = np.ascontiguousarray(kc, dtype=np.uint16)
    vc = np.ascontiguousarray(vc, dtype=np.uint16)
    S_cap = kc.shape[2]
    y = np.empty((B, H), np.float64)
    ws, keep = _weights_struct(w)
    tr = None
    tr_arrays = {}
    if trace:
        nqd = dims.n_q_heads * dims.head_dim
        nkd = dims.n_kv_heads * dims.head_dim
        tr_arrays = {"q": np.empty((B, nqd)), "k_new": np.empty((B, nkd)),
                     "v_new": np.empty((B, nkd)), "attn": np.empty((B, nqd)),
                     "h": np.empty((B, H)), "act": np.empty((B, dims.ffn))}
        tr = _Trace(*[_p(tr_arrays[k]) for k in ("q", "k_new", "v_new", "attn", "h", "act")])
    rc = lib().orc_decode_layer(ctypes.byref(dims.c()), ctypes.byref(ws), ctypes.c_long(B), _p(x),
                                _p(kc), _p(vc), ctypes.c_long(S_cap), ctypes.c_long(S), _p(y),
                                ctypes.byref(tr) if tr is not None else None)
    if rc != 0:
        raise ValueError(f"orc_decode_layer failed ({rc})")
    return (y, tr_arrays) if trace else y


def prefill_layer(dims: Dims, w: dict, x: np.ndarray, trace: bool = False):
    """Unsharded prefill layer over a chunk starting at position 0, causal
    inside the chunk ("Tensor parallel scaling curves", "Prefill vs decode").
    Returns y [T][H], k [T][n_kv*d], v [T][n_kv*d] (and a trace dict)."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    T, H = x.shape
    nkd = dims.n_kv_heads * dims.head_dim
    y = np.empty((T, H))
    k = np.empty((T, nkd))
    v = np.empty((T, nkd))
    ws, keep = _weights_struct(w)
    tr = None
    tr_arrays = {}
    if trace:
        nqd = dims.n_q_heads * dims.head_dim
        tr_arrays = {"q": np.empty((T, nqd)), "attn": np.empty((T, nqd)), "h": np.empty((T, H)),
                     "act": np.empty((T, dims.ffn))}
        tr = _Trace(_p(tr_arrays["q"]), None, None, _p(tr_arrays["attn"]), _p(tr_arrays["h"]),
                    _p(tr_arrays["act"]))
    rc = lib().orc_prefill_layer(ctypes.byref(dims.c()), ctypes.byref(ws), ctypes.c_long(T), _p(x),
                                 _p(y), _p(k), _p(v), ctypes.byref(tr) if tr is not None else None)
    if rc != 0:
        raise ValueError(f"orc_prefill_layer failed ({rc})")
    return (y, k, v, tr_arrays) if trace else (y, k, v)


def rope(v: np.ndarray, pos: int, base: float) -> np.ndarray:
    """Rotary position embedding of head vectors v[..., d] at one position."""
    out = np.ascontiguousarray(v, dtype=np.float64).copy()
    d = out.shape[-1]
    flat = out.reshape(-1, d)
    f = lib().orc_rope
    f.restype = None
    for r in range(flat.shape[0]):
        row = np.ascontiguousarray(flat[r])
        f(_p(row), ctypes.c_long(d), ctypes.c_long(pos), ctypes.c_double(base))
        flat[r] = row
    return out


def prefill_chunk(dims: Dims, w: dict, x: np.ndarray, P0: int, kc=None, vc=None, rows=None, trace: bool = False):
    """The prefill layer over a chunk of one sequence whose cache holds P0
    tokens: token i at position P0 + i attends the cached keys and the chunk's
    keys 0..i.  kc/vc uint16 (bf16 bits) [n_kv][S_cap][d] (or [1][n_kv][S_cap][d])
    holding the P0 cached tokens.  rows: the token rows whose outputs are
    wanted (default all).  Returns y [len(rows)][H], k, v [max(rows)+1][n_kv*d]
    (and a trace dict with q, attn, h, act at the listed rows)."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    T, H = x.shape
    r = np.arange(T, dtype=np.int64) if rows is None else np.asarray(rows, dtype=np.int64)
    r = np.ascontiguousarray(r)
    n = len(r)
    R = int(r.max()) + 1 if n else 0
    nkd = dims.n_kv_heads * dims.head_dim
    S_cap = 0
    if kc is not None:
        kc = np.ascontiguousarray(kc, dtype=np.uint16)
        vc = np.ascontiguousarray(vc, dtype=np.uint16)
        if kc.ndim == 4:
            kc, vc = kc[0], vc[0]
        S_cap = kc.shape[1]
    y = np.empty((n, H))
    k = np.empty((R, nkd))
    v = np.empty((R, nkd))
    ws, keep = _weights_struct(w)
    tr = None
    tr_arrays = {}
    if trace:
        nqd = dims.n_q_heads * dims.head_dim
        tr_arrays = {"q": np.empty((n, nqd)), "attn": np.empty((n, nqd)), "h": np.empty((n, H)),
                     "act": np.empty((n, dims.ffn))}
        tr = _Trace(_p(tr_arrays["q"]), None, None, _p(tr_arrays["attn"]), _p(tr_arrays["h"]),
                    _p(tr_arrays["act"]))
    rc = lib().orc_prefill_chunk(ctypes.byref(dims.c()), ctypes.byref(ws), ctypes.c_long(T), _p(x),
                                 ctypes.c_long(P0), _p(kc), _p(vc), ctypes.c_long(S_cap), ctypes.c_long(n),
                                 r.ctypes.data_as(ctypes.POINTER(ctypes.c_long)), _p(y), _p(k), _p(v),
                                 ctypes.byref(tr) if tr is not None else None)
    if rc != 0:
        raise ValueError(f"orc_prefill_chunk failed ({rc})")
    return (y, k, v, tr_arrays) if trace else (y, k, v)


def prefill_rows(dims: Dims, w: dict, x: np.ndarray, rows, trace: bool = False):
    """The prefill layer's outputs at the listed token rows only (keys and
    values for every token up to the last listed row).  Returns y
    [len(rows)][H], k and v [max(rows)+1][n_kv*d] (and a trace dict with
    q, attn, h, act at the listed rows)."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    T, H = x.shape
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    n = len(r)
    R = int(r.max()) + 1 if n else 0
    nkd = dims.n_kv_heads * dims.head_dim
    y = np.empty((n, H))
    k = np.empty((R, nkd))
    v = np.empty((R, nkd))
    ws, keep = _weights_struct(w)
    tr = None
    tr_arrays = {}
    if trace:
        nqd = dims.n_q_heads * dims.head_dim
        tr_arrays = {"q": np.empty((n, nqd)), "attn": np.empty((n, nqd)), "h": np.empty((n, H)),
                     "act": np.empty((n, dims.ffn))}
        tr = _Trace(_p(tr_arrays["q"]), None, None, _p(tr_arrays["attn"]), _p(tr_arrays["h"]),
                    _p(tr_arrays["act"]))
    rc = lib().orc_prefill_rows(ctypes.byref(dims.c()), ctypes.byref(ws), ctypes.c_long(T), _p(x),
                                ctypes.c_long(n), r.ctypes.data_as(ctypes.POINTER(ctypes.c_long)), _p(y), _p(k),
                                _p(v), ctypes.byref(tr) if tr is not None else None)
    if rc != 0:
        raise ValueError(f"orc_prefill_rows failed ({rc})")
    return (y, k, v, tr_arrays) if trace else (y, k, v)


def mlp_sharded(dims: Dims, w: dict, t: int, x: np.ndarray, partials: bool = False):
    """MLP pair sharded t ways, partials summed in ascending shard order
    ("Tensor Parallelism Fundamentals", "Mechanics of Matrix Slicing")."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    B, H = x.shape
    y = np.empty((B, H))
    parts = np.empty((t, B, H)) if partials else None
    ws, keep = _weights_struct(w)
    rc = lib().orc_mlp_sharded(ctypes.byref(dims.c()), ctypes.byref(ws), ctypes.c_int32(t),
                               ctypes.c_long(B), _p(x), _p(y), _p(parts))
    if rc != 0:
        raise ValueError(f"orc_mlp_sharded failed ({rc})")
    return (y, parts) if partials else y


def attn_sharded(dims: Dims, w: dict, t: int, x: np.ndarray, a: np.ndarray, kc, vc, S: int,
                 partials: bool = False):
    """Attention block sharded t ways by whole heads ("Tensor parallel scaling
    curves", "What tensor parallelism actually splits"): h = x + sum_s
    partial_s in ascending s (residual only if flagged)."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    a = np.ascontiguousarray(a, dtype=np.float64)
    B, H = x.shape
    kc = np.ascontiguousarray(kc, dtype=np.uint16)
    vc = np.ascontiguousarray(vc, dtype=np.uint16)
    h = np.empty((B, H))
    parts = np.empty((t, B, H)) if partials else None
    ws, keep = _weights_struct(w)
    rc = lib().orc_attn_sharded(ctypes.byref(dims.c()), ctypes.byref(ws), ctypes.c_int32(t),
                                ctypes.c_long(B), _p(x), _p(a), _p(kc), _p(vc),
                                ctypes.c_long(kc.shape[2]), ctypes.c_long(S), _p(h), _p(parts))
    if rc != 0:
        raise ValueError(f"orc_attn_sharded failed ({rc})")
    return (h, parts) if partials else h


def plan_maps(dims: Dims, t: int):
    """Shard maps from the ownership rule: shard s owns the contiguous block of
    query heads [s*n_q/t, (s+1)*n_q/t) ("Tensor parallel scaling curves",
    "What tensor parallelism actually splits").  Returns None when t is not
    admissible."""
    q_shard = np.empty(dims.n_q_heads, np.int32)
    q_local = np.empty(dims.n_q_heads, np.int32)
    kv_shard = np.empty(dims.n_kv_heads, np.int32)
    ffn_shard = np.empty(dims.ffn, np.int32)
    rc = lib().orc_plan_maps(ctypes.byref(dims.c()), ctypes.c_int32(t), _p(q_shard), _p(q_local),
                             _p(kv_shard), _p(ffn_shard))
    if rc != 0:
        return None
    return {"q_shard": q_shard, "q_local": q_local, "kv_shard": kv_shard, "ffn_shard": ffn_shard}


def kv_bytes_per_shard(layers, kv_heads, head_dim, seq, bytes_per_elem, batch, t) -> int:
    """Per-GPU KV bytes ("Tensor Parallelism Fundamentals", "Memory Overhead and
    Communication Bottlenecks")."""
    return int(lib().orc_kv_bytes_per_shard(layers, kv_heads, head_dim, seq, bytes_per_elem, batch, t))


def layer_params_per_shard(dims: Dims, t: int) -> int:
    return int(lib().orc_layer_params_per_shard(ctypes.byref(dims.c()), ctypes.c_int32(t)))


def reductions_per_pass(layers: int) -> int:
    """2L sums per forward pass ("Tensor parallel scaling curves")."""
    return int(lib().orc_reductions_per_pass(layers))


def footprint_per_gpu(dims: Dims, layers: int, t: int, batch: int, seq: int, bytes_per_elem: int = 2) -> int:
    """Per-GPU weight + KV bytes at shard degree t (-1 if t does not divide)."""
    f = lib().orc_footprint_per_gpu
    f.restype = ctypes.c_longlong
    return int(f(ctypes.byref(dims.c()), ctypes.c_longlong(layers), ctypes.c_int(t), ctypes.c_longlong(batch),
                 ctypes.c_longlong(seq), ctypes.c_longlong(bytes_per_elem)))


def auto_t(dims: Dims, layers: int, budget_bytes: int, headroom: float, batch: int, seq: int,
           bytes_per_elem: int = 2, max_t: int = 8) -> int:
    """Smallest power-of-two shard degree that fits ("Tensor Parallelism" docs, "Auto")."""
    f = lib().orc_auto_t
    f.restype = ctypes.c_int
    return int(f(ctypes.byref(dims.c()), ctypes.c_longlong(layers), ctypes.c_longlong(budget_bytes),
                 ctypes.c_double(headroom), ctypes.c_longlong(batch), ctypes.c_longlong(seq),
                 ctypes.c_longlong(bytes_per_elem), ctypes.c_int(max_t)))


def allreduce_time(n: int, message_bytes: float, latency_s: float, link_bytes_per_s: float) -> float:
    f = lib().orc_allreduce_time
    f.restype = ctypes.c_double
    return float(f(ctypes.c_int(n), ctypes.c_double(message_bytes), ctypes.c_double(latency_s),
                   ctypes.c_double(link_bytes_per_s)))


def tp_time(t_single: float, n: int, layers: int, t_allreduce: float) -> float:
    """T(N) = T_single/N + 2L * T_allreduce ("Tensor parallel scaling curves", "The scaling math")."""
    f = lib().orc_tp_time
    f.restype = ctypes.c_double
    return float(f(ctypes.c_double(t_single), ctypes.c_int(n), ctypes.c_longlong(layers), ctypes.c_double(t_allreduce)))


def silu(z: float) -> float:
    return float(lib().orc_silu(float(z)))


def rmsnorm(x: np.ndarray, gamma, eps: float) -> np.ndarray:
    """RMSNorm of one vector: x * gamma / sqrt(mean(x^2) + eps) (pre-norm reading
    of the Llama-shaped layer the pages size; the pages do not name the norm)."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty_like(x)
    g = None if gamma is None else np.ascontiguousarray(gamma, dtype=np.float32)
    L = lib()
    L.orc_rmsnorm.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_long, ctypes.c_double,
                              ctypes.c_void_p]
    L.orc_rmsnorm(_p(x), _p(g), x.size, float(eps), _p(out))
    return out
