"""ctypes binding of libtpl (the C-ABI in include/tpl.h).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  The module fails loudly at import if libtpl.so has not been built
(run ``python -m megatron_tensor_transformer_plan_b200.build`` or
``__graft_entry__.build()``); there is no fallback path.

The functions with the C names take raw integers (device pointers as ints,
streams as ints); ``Plan`` wraps them for torch tensors.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
# TPL_LIB may name the timeline-traced build (libtpl_trace.so) instead
LIB_PATH = os.environ.get("TPL_LIB") or os.path.join(_HERE, "libtpl.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libtpl.so not built at {LIB_PATH}; run megatron_tensor_transformer_plan_b200/build.py")
_lib = ctypes.CDLL(LIB_PATH)

(TPL_OK, TPL_EINVAL, TPL_EINDIVISIBLE, TPL_EWORKSPACE, TPL_ENOMEM, TPL_ECUDA, TPL_EDEVICE, TPL_EUNSUPPORTED,
 TPL_ENOFIT) = range(9)
TPL_NORM, TPL_RESIDUAL, TPL_FP32_WEIGHTS, TPL_ROPE = 1, 2, 4, 8
TPL_REDUCE_FUSED, TPL_REDUCE_SEPARATE = 0, 1
TPL_OPT_GEMV_MODE = 1
TPL_OPT_PREFILL_ATTN = 2
TPL_OPT_DECODE_ATTN = 3
TPL_OPT_PREFILL_SPLIT = 4
TPL_OPT_PREFILL_TAIL = 5
TPL_SPLIT_QKV, TPL_SPLIT_O, TPL_SPLIT_GU = 1, 2, 4
TPL_SPLIT_DEFAULT = TPL_SPLIT_QKV | TPL_SPLIT_O | TPL_SPLIT_GU
TPL_ATTN_STATIC_SCRATCH_BYTES = 4 * 1024 * 1024

c_int32, c_int64, c_size_t, c_void_p, c_uint32 = ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_uint32
P = ctypes.POINTER


class tpl_dims(ctypes.Structure):
    _fields_ = [("hidden", c_int32), ("n_q_heads", c_int32), ("n_kv_heads", c_int32), ("head_dim", c_int32),
                ("ffn", c_int32), ("n_layers", c_int32), ("rms_eps", ctypes.c_float), ("flags", c_uint32),
                ("rope_base", ctypes.c_float)]


class tpl_tp_estimate(ctypes.Structure):
    _fields_ = [(n, ctypes.c_double) for n in ("t_compute", "t_memory", "t_allreduce", "t_comm", "t_total",
                                                "speedup", "comm_share")]


class tpl_plan_info(ctypes.Structure):
    _fields_ = [("t", c_int32), ("q_heads_per_shard", c_int32), ("kv_heads_per_shard", c_int32),
                ("ffn_per_shard", c_int32), ("group_size", c_int32), ("qkv_rows_per_shard", c_int32),
                ("elem_bytes", c_int32), ("layer_params_per_shard", c_int64),
                ("layer_weight_bytes_per_shard", c_int64), ("packed_layer_bytes", c_int64),
                ("reductions_per_step", c_int64)]


class tpl_layer_weights(ctypes.Structure):
    _fields_ = [("wq", c_void_p), ("wk", c_void_p), ("wv", c_void_p), ("wo", c_void_p), ("wg", c_void_p),
                ("wu", c_void_p), ("wd", c_void_p), ("gamma_attn", c_void_p), ("gamma_mlp", c_void_p)]


class tpl_kv(ctypes.Structure):
    _fields_ = [("k", c_void_p), ("v", c_void_p), ("batch_cap", c_int32), ("seq_cap", c_int64)]


def _sig(name, restype, *argtypes):
    f = getattr(_lib, name)
    f.restype = restype
    f.argtypes = list(argtypes)
    globals()[name] = f
    return f


_plan_p = c_void_p
_sig("tpl_plan_create", ctypes.c_int, P(tpl_dims), c_int32, P(c_void_p))
_sig("tpl_plan_destroy", None, _plan_p)
_sig("tpl_plan_info_get", ctypes.c_int, _plan_p, P(tpl_plan_info))
_sig("tpl_plan_maps", ctypes.c_int, _plan_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p)
_sig("tpl_plan_set_option", ctypes.c_int, _plan_p, c_int32, c_int32)
_sig("tpl_kv_bytes", c_int64, P(tpl_dims), c_int32, c_int64, c_int64, c_int32)
_sig("tpl_footprint_bytes", c_int64, P(tpl_dims), c_int32, c_int64, c_int64, c_int32)
_sig("tpl_auto_t", ctypes.c_int, P(tpl_dims), c_int64, ctypes.c_double, c_int64, c_int64, c_int32, c_int32, P(c_int32))
_sig("tpl_tp_estimate_get", ctypes.c_int, ctypes.c_double, ctypes.c_double, c_int32, c_int32, ctypes.c_double,
     ctypes.c_double, ctypes.c_double, P(tpl_tp_estimate))
_sig("tpl_decode_times", ctypes.c_int, P(tpl_dims), c_int64, c_int64, c_int32, ctypes.c_double, ctypes.c_double,
     P(ctypes.c_double), P(ctypes.c_double))
_sig("tpl_kv_layer_bytes", c_int64, _plan_p, c_int32, c_int64)
_sig("tpl_workspace_size", ctypes.c_int, _plan_p, c_int32, c_int64, P(c_size_t))
_sig("tpl_workspace_init", ctypes.c_int, _plan_p, c_void_p, c_size_t, c_void_p)
_sig("tpl_prefill_workspace_size", ctypes.c_int, _plan_p, c_int32, P(c_size_t))
_sig("tpl_prefill_intermediates", ctypes.c_int, _plan_p, c_int32, P(c_size_t))
_sig("tpl_pack_layer", ctypes.c_int, _plan_p, P(tpl_layer_weights), c_void_p, c_size_t, c_void_p)
_sig("tpl_pack_kv", ctypes.c_int, _plan_p, c_void_p, c_void_p, c_int32, c_int64, c_void_p)
_sig("tpl_decode_layer", ctypes.c_int, _plan_p, c_void_p, P(tpl_kv), c_void_p, c_int32, c_int64, c_void_p, c_void_p,
     c_void_p, c_size_t, c_int32, c_void_p)
_sig("tpl_decode_stack", ctypes.c_int, _plan_p, P(c_void_p), P(tpl_kv), c_void_p, c_int32, c_int64, c_void_p,
     c_void_p, c_void_p, c_size_t, c_int32, c_void_p)
_sig("tpl_prefill_layer", ctypes.c_int, _plan_p, c_void_p, P(tpl_kv), c_void_p, c_int32, c_void_p, c_void_p,
     c_void_p, c_size_t, c_int32, c_void_p)
_sig("tpl_prefill_chunk", ctypes.c_int, _plan_p, c_void_p, P(tpl_kv), c_void_p, c_int32, c_int64, c_void_p,
     c_void_p, c_void_p, c_size_t, c_int32, c_void_p)
_sig("tpl_qkv", ctypes.c_int, _plan_p, c_void_p, P(tpl_kv), c_void_p, c_int32, c_int64, c_void_p, c_void_p,
     c_void_p, c_void_p, c_size_t, c_void_p)
_sig("tpl_attn_decode", ctypes.c_int, _plan_p, P(tpl_kv), c_void_p, c_void_p, c_void_p, c_int32, c_int64, c_void_p,
     c_void_p, c_size_t, c_void_p)
_sig("tpl_attn_decode_static", ctypes.c_int, _plan_p, P(tpl_kv), c_void_p, c_void_p, c_void_p, c_int32, c_int64,
     c_void_p, c_void_p)
_sig("tpl_o_proj", ctypes.c_int, _plan_p, c_void_p, c_void_p, c_void_p, c_int32, c_void_p, c_void_p, c_void_p,
     c_size_t, c_void_p)
_sig("tpl_gate_up", ctypes.c_int, _plan_p, c_void_p, c_void_p, c_int32, c_int32, c_void_p, c_void_p, c_size_t,
     c_void_p)
_sig("tpl_down_proj", ctypes.c_int, _plan_p, c_void_p, c_void_p, c_void_p, c_int32, c_void_p, c_void_p, c_void_p,
     c_void_p, c_size_t, c_void_p)
_sig("tpl_reduce_partials", ctypes.c_int, _plan_p, c_void_p, c_void_p, c_int32, c_int32, c_void_p, c_void_p,
     c_void_p)
_sig("tpl_mlp_block", ctypes.c_int, _plan_p, c_void_p, c_void_p, c_int32, c_void_p, c_void_p, c_void_p, c_size_t,
     c_int32, c_void_p)
_sig("tpl_reduction_count", c_int64, _plan_p)
_sig("tpl_decode_kernel_count", ctypes.c_int, _plan_p, c_int32, c_int32, c_int32, P(c_int32))
_sig("tpl_reset_counters", None, _plan_p)
_sig("tpl_last_device_error", ctypes.c_int, _plan_p, c_void_p)
_sig("tpl_trace_read", ctypes.c_int, c_void_p, c_int32, P(c_int32))


class tpl_trace_rec(ctypes.Structure):
    _fields_ = [("tag", c_uint32), ("cta", c_uint32), ("smid", c_uint32), ("grid", c_uint32),
                ("t", ctypes.c_uint64 * 4)]


TRACE_TAGS = {1: "qkv", 2: "attention", 3: "o_proj", 4: "gate_up", 5: "down", 6: "operand", 7: "reduce",
              101: "qkv.epi", 103: "o_proj.epi", 104: "gate_up.epi", 105: "down.epi",
              201: "qkv.clk", 203: "o_proj.clk", 204: "gate_up.clk", 205: "down.clk",
              202: "attention.clk", 212: "attention_last.clk"}


def trace_read(max_records: int = 1 << 18):
    """Records of the traced build since the last read, as a list of
    (tag name, cta, smid, grid, [t0, t1, t2, t3] in ns)."""
    buf = (tpl_trace_rec * max_records)()
    n = c_int32()
    check(tpl_trace_read(ctypes.cast(buf, c_void_p), max_records, ctypes.byref(n)), "tpl_trace_read")
    return [(TRACE_TAGS.get(r.tag, str(r.tag)), r.cta, r.smid, r.grid, list(r.t)) for r in buf[:n.value]]
_sig("tpl_status_string", ctypes.c_char_p, ctypes.c_int)


class TplError(RuntimeError):
    def __init__(self, code: int, where: str = ""):
        self.code = code
        super().__init__(f"{where}: {tpl_status_string(code).decode()} (status {code})")


def check(code: int, where: str = "") -> None:
    if code != TPL_OK:
        raise TplError(code, where)


def make_dims(hidden, n_q_heads, n_kv_heads, head_dim, ffn, n_layers=1, rms_eps=1e-5,
              flags=TPL_NORM | TPL_RESIDUAL, rope_base=500000.0) -> tpl_dims:
    return tpl_dims(hidden, n_q_heads, n_kv_heads, head_dim, ffn, n_layers, rms_eps, flags, rope_base)


def footprint_bytes(dims: tpl_dims, t: int, batch: int, seq: int, bytes_per_elem: int = 2) -> int:
    """Per-GPU weight + KV bytes at degree t (-1 when t does not divide)."""
    return int(tpl_footprint_bytes(ctypes.byref(dims), t, batch, seq, bytes_per_elem))


def auto_t(dims: tpl_dims, budget_bytes: int, headroom: float, batch: int, seq: int, bytes_per_elem: int = 2,
           max_t: int = 8) -> int:
    """The smallest power-of-two degree that fits the budget (0 when none does)."""
    out = c_int32(0)
    rc = tpl_auto_t(ctypes.byref(dims), budget_bytes, headroom, batch, seq, bytes_per_elem, max_t, ctypes.byref(out))
    if rc == TPL_ENOFIT:
        return 0
    check(rc, "tpl_auto_t")
    return int(out.value)


def tp_estimate(t_compute: float, t_memory: float, n: int, layers: int, message_bytes: float, latency_s: float,
                link_bytes_per_s: float) -> tpl_tp_estimate:
    out = tpl_tp_estimate()
    check(tpl_tp_estimate_get(t_compute, t_memory, n, layers, message_bytes, latency_s, link_bytes_per_s,
                              ctypes.byref(out)), "tpl_tp_estimate_get")
    return out


def decode_times(dims: tpl_dims, batch: int, seq: int, bytes_per_elem: int, flops_per_s: float,
                 hbm_bytes_per_s: float):
    tc, tm = ctypes.c_double(), ctypes.c_double()
    check(tpl_decode_times(ctypes.byref(dims), batch, seq, bytes_per_elem, flops_per_s, hbm_bytes_per_s,
                           ctypes.byref(tc), ctypes.byref(tm)), "tpl_decode_times")
    return tc.value, tm.value


# --------------------------------------------------------------------------
# torch-facing wrapper
# --------------------------------------------------------------------------

def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream():
    import torch
    return torch.cuda.current_stream().cuda_stream


class Plan:
    """A shard plan.  Tensors passed in must be contiguous CUDA tensors of the
    types the C-ABI documents (bf16 activations, or fp32 with
    TPL_FP32_WEIGHTS)."""

    def __init__(self, dims: tpl_dims, t: int):
        self.dims = dims
        self.t = t
        h = c_void_p()
        check(tpl_plan_create(ctypes.byref(dims), t, ctypes.byref(h)), "tpl_plan_create")
        self.handle = h

    def __del__(self):
        h = getattr(self, "handle", None)
        destroy = globals().get("tpl_plan_destroy")
        if h is not None and h.value and destroy is not None:
            destroy(h)
            self.handle = None

    # ---- host queries ----
    def info(self) -> tpl_plan_info:
        out = tpl_plan_info()
        check(tpl_plan_info_get(self.handle, ctypes.byref(out)), "tpl_plan_info_get")
        return out

    def maps(self):
        import numpy as np
        d = self.dims
        q_shard = np.empty(d.n_q_heads, np.int32)
        q_local = np.empty(d.n_q_heads, np.int32)
        kv_shard = np.empty(d.n_kv_heads, np.int32)
        ffn_shard = np.empty(d.ffn, np.int32)
        offs = np.empty(4 * self.t + 2, np.int64)
        check(tpl_plan_maps(self.handle, q_shard.ctypes.data, q_local.ctypes.data, kv_shard.ctypes.data,
                            ffn_shard.ctypes.data, offs.ctypes.data), "tpl_plan_maps")
        return {"q_shard": q_shard, "q_local": q_local, "kv_shard": kv_shard, "ffn_shard": ffn_shard,
                "packed_offsets": offs}

    def workspace_size(self, B: int, S: int) -> int:
        out = c_size_t()
        check(tpl_workspace_size(self.handle, B, S, ctypes.byref(out)), "tpl_workspace_size")
        return out.value

    def prefill_workspace_size(self, T: int) -> int:
        out = c_size_t()
        check(tpl_prefill_workspace_size(self.handle, T, ctypes.byref(out)), "tpl_prefill_workspace_size")
        return out.value

    def prefill_intermediates(self, T: int) -> dict:
        """Byte offsets of q, o (high part), h, act, o_lo inside a prefill
        workspace for T tokens."""
        offs = (c_size_t * 5)()
        check(tpl_prefill_intermediates(self.handle, T, offs), "tpl_prefill_intermediates")
        return dict(zip(("q", "o", "h", "act", "o_lo"), list(offs)))

    def kv_layer_bytes(self, batch_cap: int, seq_cap: int) -> int:
        return tpl_kv_layer_bytes(self.handle, batch_cap, seq_cap)

    def set_option(self, option: int, value: int) -> None:
        check(tpl_plan_set_option(self.handle, option, value), "tpl_plan_set_option")

    def reduction_count(self) -> int:
        return tpl_reduction_count(self.handle)

    def decode_kernel_count(self, B: int, mode=TPL_REDUCE_FUSED, n_layers: int = 1) -> int:
        """Kernels a decode call launches for B tokens (n_layers > 1: a stack)."""
        n = c_int32(0)
        check(tpl_decode_kernel_count(self.handle, B, mode, n_layers, ctypes.byref(n)), "tpl_decode_kernel_count")
        return int(n.value)

    def reset_counters(self) -> None:
        tpl_reset_counters(self.handle)

    # ---- device helpers ----
    def workspace(self, B: int, S: int, device="cuda"):
        import torch
        n = self.workspace_size(B, S)
        ws = torch.zeros(n, dtype=torch.uint8, device=device)
        check(tpl_workspace_init(self.handle, ws.data_ptr(), n, _stream()), "tpl_workspace_init")
        return ws

    @property
    def act_dtype(self):
        import torch
        return torch.float32 if (self.dims.flags & TPL_FP32_WEIGHTS) else torch.bfloat16

    def pack_layer(self, w: dict, out=None):
        """w: unsharded device tensors wq, wk, wv, wo, wg, wu, wd (activation
        type) and optional fp32 gamma_attn, gamma_mlp."""
        import torch
        n = self.info().packed_layer_bytes
        dev = w["wg"].device
        if out is None:
            out = torch.empty(n, dtype=torch.uint8, device=dev)
        lw = tpl_layer_weights(*[_ptr(w.get(k)) for k in ("wq", "wk", "wv", "wo", "wg", "wu", "wd",
                                                           "gamma_attn", "gamma_mlp")])
        check(tpl_pack_layer(self.handle, ctypes.byref(lw), out.data_ptr(), out.numel() * out.element_size(),
                             _stream()), "tpl_pack_layer")
        return out

    def pack_kv(self, unsharded, out=None):
        """[B_cap][n_kv][S_cap][d] bf16 -> the shard-major layout of tpl_kv."""
        import torch
        if out is None:
            out = torch.empty_like(unsharded)
        check(tpl_pack_kv(self.handle, unsharded.data_ptr(), out.data_ptr(), unsharded.shape[0], unsharded.shape[2],
                          _stream()), "tpl_pack_kv")
        return out

    @staticmethod
    def kv(k, v, batch_cap: int, seq_cap: int) -> tpl_kv:
        return tpl_kv(k.data_ptr(), v.data_ptr(), batch_cap, seq_cap)

    def decode_layer(self, packed, kv: tpl_kv, x, S: int, y, y32=None, ws=None, mode=TPL_REDUCE_FUSED):
        B = x.shape[0]
        check(tpl_decode_layer(self.handle, packed.data_ptr(), ctypes.byref(kv), x.data_ptr(), B, S, _ptr(y),
                               _ptr(y32), ws.data_ptr(), ws.numel(), mode, _stream()), "tpl_decode_layer")

    def prefill_workspace(self, T: int, device="cuda"):
        import torch
        return torch.empty(self.prefill_workspace_size(T), dtype=torch.uint8, device=device)

    def prefill_layer(self, packed, kv: tpl_kv, x, y, y32=None, ws=None, mode=TPL_REDUCE_FUSED):
        T = x.shape[0]
        check(tpl_prefill_layer(self.handle, packed.data_ptr(), ctypes.byref(kv), x.data_ptr(), T, _ptr(y),
                                _ptr(y32), ws.data_ptr(), ws.numel(), mode, _stream()), "tpl_prefill_layer")

    def prefill_chunk(self, packed, kv: tpl_kv, x, start: int, y, y32=None, ws=None, mode=TPL_REDUCE_FUSED):
        T = x.shape[0]
        check(tpl_prefill_chunk(self.handle, packed.data_ptr(), ctypes.byref(kv), x.data_ptr(), T, start, _ptr(y),
                                _ptr(y32), ws.data_ptr(), ws.numel(), mode, _stream()), "tpl_prefill_chunk")

    def decode_stack(self, packed_list, kv_list, x, S: int, y, y32=None, ws=None, mode=TPL_REDUCE_FUSED):
        L = len(packed_list)
        if L != self.dims.n_layers or len(kv_list) != L:
            raise ValueError(f"decode_stack: the plan has {self.dims.n_layers} layers, got {L} packed layers and "
                             f"{len(kv_list)} caches")
        arr = (c_void_p * L)(*[p.data_ptr() for p in packed_list])
        kvs = (tpl_kv * L)(*kv_list)
        B = x.shape[0]
        check(tpl_decode_stack(self.handle, arr, kvs, x.data_ptr(), B, S, _ptr(y), _ptr(y32), ws.data_ptr(),
                               ws.numel(), mode, _stream()), "tpl_decode_stack")

    def qkv(self, packed, kv: tpl_kv, x, S: int, q, ws, k_new=None, v_new=None):
        check(tpl_qkv(self.handle, packed.data_ptr(), ctypes.byref(kv), x.data_ptr(), x.shape[0], S, q.data_ptr(),
                      _ptr(k_new), _ptr(v_new), ws.data_ptr(), ws.numel(), _stream()), "tpl_qkv")

    def attn_decode(self, kv: tpl_kv, q, S: int, o, ws, k_new=None, v_new=None):
        check(tpl_attn_decode(self.handle, ctypes.byref(kv), q.data_ptr(), _ptr(k_new), _ptr(v_new), q.shape[0], S,
                              o.data_ptr(), ws.data_ptr(), ws.numel(), _stream()), "tpl_attn_decode")

    def o_proj(self, packed, o, x, h=None, partials=None, ws=None):
        check(tpl_o_proj(self.handle, packed.data_ptr(), o.data_ptr(), _ptr(x), o.shape[0], _ptr(h), _ptr(partials),
                         ws.data_ptr(), ws.numel(), _stream()), "tpl_o_proj")

    def gate_up(self, packed, h, act, ws, h_is_act=False):
        check(tpl_gate_up(self.handle, packed.data_ptr(), h.data_ptr(), int(h_is_act), h.shape[0], act.data_ptr(),
                          ws.data_ptr(), ws.numel(), _stream()), "tpl_gate_up")

    def down_proj(self, packed, act, h, y=None, y32=None, partials=None, ws=None):
        check(tpl_down_proj(self.handle, packed.data_ptr(), act.data_ptr(), _ptr(h), act.shape[0], _ptr(y),
                            _ptr(y32), _ptr(partials), ws.data_ptr(), ws.numel(), _stream()), "tpl_down_proj")

    def reduce_partials(self, partials, resid, resid_is_f32: bool, out32=None, out_act=None):
        B = partials.shape[1]
        check(tpl_reduce_partials(self.handle, partials.data_ptr(), _ptr(resid), int(resid_is_f32), B, _ptr(out32),
                                  _ptr(out_act), _stream()), "tpl_reduce_partials")

    def mlp_block(self, packed, x, y=None, y32=None, ws=None, mode=TPL_REDUCE_FUSED):
        check(tpl_mlp_block(self.handle, packed.data_ptr(), x.data_ptr(), x.shape[0], _ptr(y), _ptr(y32),
                            ws.data_ptr(), ws.numel(), mode, _stream()), "tpl_mlp_block")

    def last_device_error(self) -> int:
        return tpl_last_device_error(self.handle, _stream())
