"""Tensor parallelism across t GPUs, one rank per GPU: each rank holds one
shard's weights and KV cache and runs the single-device library's step kernels
on its slice, and the two row-parallel partial sums of a layer are added by an
all-reduce over torch.distributed (NCCL) instead of the on-device fused sum
("Tensor parallel scaling curves", section "What tensor parallelism actually
splits": Q/K/V and gate/up split by columns so that rank r owns the query
heads [r*n_q/t, (r+1)*n_q/t), O and down split by rows, two all-reduces per
layer; "Tensor Parallelism Fundamentals", section "Mechanics of Matrix
Slicing").

Per rank and layer, for the B tokens of a decode step:

    q, k, v   = column-parallel QKV of RMSNorm(x) for the rank's heads   (tpl_qkv)
    o         = attention over the rank's heads and its cache shard      (tpl_attn_decode)
    P         = o Wo[:, rank's columns]^T, a full-size partial           (tpl_o_proj, partials)
    P         = all_reduce(P)                                            (NCCL)
    h         = x + P                                                    (tpl_reduce_partials)
    act       = SwiGLU of RMSNorm(h) for the rank's ffn columns          (tpl_gate_up)
    P2        = act Wd[:, rank's columns]^T                              (tpl_down_proj, partials)
    P2        = all_reduce(P2)
    y         = h + P2                                                   (tpl_reduce_partials)

Each rank's local plan is a one-shard plan of the sliced dimensions (hidden,
n_q/t heads, n_kv/t kv heads, ffn/t), so every kernel is the one the
single-device layer runs.  The all-reduce adds the partials in NCCL's order,
so results match the single-device layer within fp32 rounding, not bit for
bit.  The step order is the same on every rank, so the collectives match.

`DecodeStepOps` is the set of per-rank steps; `CudaOps` runs them through the
C ABI.  Tests drive the same orchestration with other implementations of the
steps on the CPU.
"""
from __future__ import annotations

from dataclasses import dataclass


@dataclass(frozen=True)
class ShardSpec:
    """Rank `rank` of `t`: the q heads, kv heads and ffn columns it owns."""
    hidden: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    ffn: int
    t: int
    rank: int

    def __post_init__(self):
        if self.t < 1 or not 0 <= self.rank < self.t:
            raise ValueError("rank must be in [0, t)")
        if self.n_q_heads % self.t or self.n_kv_heads % self.t or self.ffn % self.t:
            raise ValueError("t must divide the q heads, the kv heads and ffn")
        if self.n_q_heads % self.n_kv_heads:
            raise ValueError("n_kv_heads must divide n_q_heads")

    @property
    def nq_s(self) -> int:
        return self.n_q_heads // self.t

    @property
    def nkv_s(self) -> int:
        return self.n_kv_heads // self.t

    @property
    def ffn_s(self) -> int:
        return self.ffn // self.t

    def q_heads(self) -> range:
        return range(self.rank * self.nq_s, (self.rank + 1) * self.nq_s)

    def kv_heads(self) -> range:
        return range(self.rank * self.nkv_s, (self.rank + 1) * self.nkv_s)

    def ffn_cols(self) -> range:
        return range(self.rank * self.ffn_s, (self.rank + 1) * self.ffn_s)


def shard_weights(w: dict, spec: ShardSpec) -> dict:
    """The rank's slices of one layer's weights (nn.Linear orientation
    W[out][in]; numpy arrays or torch tensors): rows of Wq, Wk, Wv for its
    heads, columns of Wo for its q heads, rows of Wg and Wu for its ffn
    columns, columns of Wd; the RMSNorm gains whole (every rank normalises the
    full hidden vector)."""
    d = spec.head_dim
    q0, q1 = spec.q_heads().start * d, spec.q_heads().stop * d
    k0, k1 = spec.kv_heads().start * d, spec.kv_heads().stop * d
    f0, f1 = spec.ffn_cols().start, spec.ffn_cols().stop
    out = {
        "wq": w["wq"][q0:q1],
        "wk": w["wk"][k0:k1],
        "wv": w["wv"][k0:k1],
        "wo": w["wo"][:, q0:q1],
        "wg": w["wg"][f0:f1],
        "wu": w["wu"][f0:f1],
        "wd": w["wd"][:, f0:f1],
    }
    for k in ("gamma_attn", "gamma_mlp"):
        if w.get(k) is not None:
            out[k] = w[k]
    return out


def shard_cache(cache, spec: ShardSpec):
    """The rank's kv heads of an unsharded cache [B][n_kv][S_cap][d]."""
    return cache[:, spec.kv_heads().start:spec.kv_heads().stop]


class DecodeStepOps:
    """The per-rank steps of one decode layer; arrays are whatever the
    implementation uses (device tensors for CudaOps)."""

    def qkv(self, x, S):  # -> (q, k_new, v_new) of the rank's heads
        raise NotImplementedError

    def attn(self, q, k_new, v_new, S):  # -> o [B][nq_s*d]
        raise NotImplementedError

    def o_partial(self, o):  # -> P [B][H] fp32 (no residual)
        raise NotImplementedError

    def add_resid(self, P, resid, resid_is_f32):  # -> resid + P, fp32
        raise NotImplementedError

    def gate_up(self, h):  # -> act [B][ffn_s]
        raise NotImplementedError

    def down_partial(self, act):  # -> P2 [B][H] fp32
        raise NotImplementedError

    def add_resid_out(self, P, h):  # -> (y32, y) = h + P
        raise NotImplementedError


def decode_layer_tp(ops: DecodeStepOps, x, S: int, all_reduce, residual: bool = True):
    """One tensor-parallel decode layer on this rank: the steps in the same
    order on every rank, with `all_reduce(tensor)` summing a partial in place
    across the t ranks (torch.distributed.all_reduce for the NCCL group)."""
    q, kn, vn = ops.qkv(x, S)
    o = ops.attn(q, kn, vn, S)
    P = ops.o_partial(o)
    all_reduce(P)                                   # reduction point 1
    h = ops.add_resid(P, x if residual else None, False)
    act = ops.gate_up(h)
    P2 = ops.down_partial(act)
    all_reduce(P2)                                  # reduction point 2
    return ops.add_resid_out(P2, h if residual else None)


def decode_stack_tp(ops_per_layer, x, S: int, all_reduce, residual: bool = True):
    """n_layers tensor-parallel decode layers on this rank: layer l reads
    layer l-1's output (the replicated y, in the activation type), 2 *
    n_layers all-reduces per step ("Tensor parallel scaling curves": 2L per
    forward pass).  Returns the last layer's (y32, y)."""
    out = None
    cur = x
    for ops in ops_per_layer:
        out = decode_layer_tp(ops, cur, S, all_reduce, residual)
        cur = out[1]
    return out


class CudaOps(DecodeStepOps):
    """The steps through the C ABI on the rank's GPU: a one-shard plan of the
    sliced dimensions, the rank's packed weights and KV cache shard.

    Every per-step buffer (q, new k/v, o, the partials, h, act, y) and the
    workspace are allocated once here, the workspace for the largest S the
    cache holds (its size does not shrink with S), so a decode loop never
    enters the allocator.  The step methods return these buffers: a layer's
    output stays valid until that layer's next step.  `workspace` may be
    shared by the layers of one rank (their steps run in order on one
    stream)."""

    def __init__(self, spec: ShardSpec, weights_local: dict, k_local, v_local, batch: int, seq_cap: int,
                 rms_eps: float = 1e-5, flags=None, rope_base: float = 500000.0, workspace=None):
        import torch

        from megatron_tensor_transformer_plan_b200 import tpl
        self.tpl, self.torch = tpl, torch
        flags = (tpl.TPL_NORM | tpl.TPL_RESIDUAL) if flags is None else flags
        self.dims = tpl.make_dims(spec.hidden, spec.nq_s, spec.nkv_s, spec.head_dim, spec.ffn_s, 1, rms_eps, flags,
                                  rope_base)
        self.plan = tpl.Plan(self.dims, 1)
        self.spec = spec
        # column slices of Wo and Wd are strided views: the library takes dense rows
        self.packed = self.plan.pack_layer({k: v.contiguous() for k, v in weights_local.items()})
        self.k, self.v = self.plan.pack_kv(k_local.contiguous()), self.plan.pack_kv(v_local.contiguous())
        self.kv = tpl.Plan.kv(self.k, self.v, batch, seq_cap)
        self.B = batch
        self.seq_cap = seq_cap
        self.dev = self.packed.device
        self.ws = workspace if workspace is not None else self.make_workspace(self.plan, batch, seq_cap, self.dev)
        if self.ws.numel() < self.plan.workspace_size(batch, seq_cap - 1):
            raise ValueError("workspace smaller than the plan needs at the cache's capacity")
        B, sp, f32, act = batch, spec, torch.float32, self.plan.act_dtype
        self.q = torch.empty((B, sp.nq_s, sp.head_dim), dtype=f32, device=self.dev)
        self.kn = torch.empty((B, sp.nkv_s, sp.head_dim), dtype=f32, device=self.dev)
        self.vn = torch.empty_like(self.kn)
        self.o = torch.empty((B, sp.nq_s * sp.head_dim), dtype=act, device=self.dev)
        self.P = torch.empty((1, B, sp.hidden), dtype=f32, device=self.dev)
        self.h = torch.empty((B, sp.hidden), dtype=f32, device=self.dev)
        self.act = torch.empty((B, sp.ffn_s), dtype=act, device=self.dev)
        self.P2 = torch.empty((1, B, sp.hidden), dtype=f32, device=self.dev)
        self.y32 = torch.empty((B, sp.hidden), dtype=f32, device=self.dev)
        self.y = torch.empty((B, sp.hidden), dtype=act, device=self.dev)

    @staticmethod
    def make_workspace(plan, batch: int, seq_cap: int, device):
        """A workspace for every S up to seq_cap - 1 (the largest needed)."""
        return plan.workspace(batch, seq_cap - 1, device=device)

    def _check_S(self, S):
        if not 0 <= S < self.seq_cap:
            raise ValueError(f"S = {S} outside the cache's capacity {self.seq_cap}")

    def qkv(self, x, S):
        self._check_S(S)
        self.plan.qkv(self.packed, self.kv, x, S, self.q, self.ws, self.kn, self.vn)
        return self.q, self.kn, self.vn

    def attn(self, q, kn, vn, S):
        self._check_S(S)
        self.plan.attn_decode(self.kv, q, S, self.o, self.ws, kn, vn)
        return self.o

    def o_partial(self, o):
        self.plan.o_proj(self.packed, o, None, partials=self.P, ws=self.ws)
        return self.P

    def add_resid(self, P, resid, resid_is_f32):
        self.plan.reduce_partials(P, resid, resid_is_f32, out32=self.h)
        return self.h

    def gate_up(self, h):
        self.plan.gate_up(self.packed, h, self.act, self.ws)
        return self.act

    def down_partial(self, act):
        self.plan.down_proj(self.packed, act, None, partials=self.P2, ws=self.ws)
        return self.P2

    def add_resid_out(self, P, h):
        self.plan.reduce_partials(P, h, True, out32=self.y32, out_act=self.y)
        return self.y32, self.y
