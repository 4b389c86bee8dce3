"""The multi-GPU tensor-parallel decode layer's host logic (tp_dist) on the
CPU: the rank's weight and cache slices follow the ownership rule of "Tensor
parallel scaling curves" ("What tensor parallelism actually splits") and agree
with the oracle's shard maps; and the orchestration -- the rank's steps, the
two all-reduces (gloo, world size 2 and 4), the residual adds after them --
reproduces the oracle's unsharded layer.  The steps are done here in float64
numpy on the rank's slices (a stand-in for the kernels, which need a GPU)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from megatron_tensor_transformer_plan_b200.tp_dist import (DecodeStepOps, ShardSpec, decode_layer_tp,
                                                            decode_stack_tp, shard_cache, shard_weights)

H, NQ, NKV, D, F, B, S = 64, 8, 4, 16, 48, 2, 5
EPS = 1e-5


def _inputs(seed=7):
    r = np.random.default_rng(seed)
    f = lambda *s: (r.standard_normal(s) * 0.2).astype(np.float32)
    w = {"wq": f(NQ * D, H), "wk": f(NKV * D, H), "wv": f(NKV * D, H), "wo": f(H, NQ * D),
         "wg": f(F, H), "wu": f(F, H), "wd": f(H, F),
         "gamma_attn": (1 + 0.1 * r.standard_normal(H)).astype(np.float32),
         "gamma_mlp": (1 + 0.1 * r.standard_normal(H)).astype(np.float32)}
    x = r.standard_normal((B, H))
    kc = (r.standard_normal((B, NKV, S + 1, D)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    vc = (r.standard_normal((B, NKV, S + 1, D)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    return w, x, kc, vc


def _bf16(a):
    return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


class NumpyOps(DecodeStepOps):
    """The rank's steps in float64 on its slices (test stand-in)."""

    def __init__(self, spec, w, kc, vc):
        self.s, self.w = spec, {k: np.asarray(v, np.float64) for k, v in w.items()}
        self.kc, self.vc = _bf16(kc), _bf16(vc)

    @staticmethod
    def _norm(v, g):
        return v / np.sqrt(np.mean(v * v, axis=-1, keepdims=True) + EPS) * g

    def qkv(self, x, S_):
        a = self._norm(x, self.w["gamma_attn"])
        return a @ self.w["wq"].T, a @ self.w["wk"].T, a @ self.w["wv"].T

    def attn(self, q, k, v, S_):
        sp, d = self.s, D
        g = sp.nq_s // sp.nkv_s
        o = np.zeros((B, sp.nq_s * d))
        for b in range(B):
            for h in range(sp.nq_s):
                j = h // g
                keys = np.concatenate([self.kc[b, j, :S_], k[b, j * d:(j + 1) * d][None]])
                vals = np.concatenate([self.vc[b, j, :S_], v[b, j * d:(j + 1) * d][None]])
                z = keys @ q[b, h * d:(h + 1) * d] / np.sqrt(d)
                p = np.exp(z - z.max())
                o[b, h * d:(h + 1) * d] = (p / p.sum()) @ vals
        return o

    def o_partial(self, o):
        return torch.from_numpy((o @ self.w["wo"].T)[None].copy())

    def add_resid(self, P, resid, resid_is_f32):
        return P[0].numpy() + (resid if resid is not None else 0.0)

    def gate_up(self, h):
        m = self._norm(h, self.w["gamma_mlp"])
        gg, uu = m @ self.w["wg"].T, m @ self.w["wu"].T
        return gg / (1 + np.exp(-gg)) * uu

    def down_partial(self, act):
        return torch.from_numpy((act @ self.w["wd"].T)[None].copy())

    def add_resid_out(self, P, h):
        y = P[0].numpy() + (h if h is not None else 0.0)
        return y, y


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, t, port, q):
    import datetime
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=t, timeout=datetime.timedelta(seconds=60))
    try:
        w, x, kc, vc = _inputs()
        spec = ShardSpec(H, NQ, NKV, D, F, t, rank)
        ops = NumpyOps(spec, shard_weights(w, spec), shard_cache(kc, spec), shard_cache(vc, spec))
        y32, _ = decode_layer_tp(ops, x, S, lambda T: dist.all_reduce(T, op=dist.ReduceOp.SUM))
        q.put((rank, y32))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("t", [2, 4])
def test_tp_layer_over_gloo_matches_the_unsharded_oracle(t):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, t, port, q)) for r in range(t)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = dict(q.get(timeout=5) for _ in range(t))
    w, x, kc, vc = _inputs()
    ref = oracle.decode_layer(oracle.Dims(H, NQ, NKV, D, F, eps=EPS), w, x, kc, vc, S)
    for r in range(t):
        np.testing.assert_allclose(res[r], ref, rtol=1e-10, atol=1e-10 * np.abs(ref).max())
    # every rank ends with the same (replicated) output
    for r in range(1, t):
        np.testing.assert_array_equal(res[r], res[0])


@pytest.mark.parametrize("t", [1, 2, 4])
def test_slices_follow_the_ownership_rule_and_the_oracle_maps(t):
    w, _, kc, _ = _inputs()
    m = oracle.plan_maps(oracle.Dims(H, NQ, NKV, D, F), t)
    q_shard, kv_shard, ffn_shard = m["q_shard"], m["kv_shard"], m["ffn_shard"]
    parts = [shard_weights(w, ShardSpec(H, NQ, NKV, D, F, t, r)) for r in range(t)]
    for r in range(t):
        spec = ShardSpec(H, NQ, NKV, D, F, t, r)
        assert list(spec.q_heads()) == [h for h in range(NQ) if q_shard[h] == r]
        assert list(spec.kv_heads()) == [j for j in range(NKV) if kv_shard[j] == r]
        assert list(spec.ffn_cols()) == [c for c in range(F) if ffn_shard[c] == r]
        assert shard_cache(kc, spec).shape == (B, NKV // t, S + 1, D)
    # the slices put back together are the unsharded weights, exactly
    np.testing.assert_array_equal(np.concatenate([p["wq"] for p in parts]), w["wq"])
    np.testing.assert_array_equal(np.concatenate([p["wk"] for p in parts]), w["wk"])
    np.testing.assert_array_equal(np.concatenate([p["wo"] for p in parts], axis=1), w["wo"])
    np.testing.assert_array_equal(np.concatenate([p["wg"] for p in parts]), w["wg"])
    np.testing.assert_array_equal(np.concatenate([p["wd"] for p in parts], axis=1), w["wd"])
    for p in parts:
        np.testing.assert_array_equal(p["gamma_mlp"], w["gamma_mlp"])


def test_shard_spec_rejects_bad_degrees():
    with pytest.raises(ValueError):
        ShardSpec(H, NQ, NKV, D, F, 3, 0)
    with pytest.raises(ValueError):
        ShardSpec(H, NQ, NKV, D, F, 2, 2)
    with pytest.raises(ValueError):
        ShardSpec(H, NQ, 3, D, F, 1, 0)


def _stack_worker(rank, t, port, q):
    import datetime
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=t, timeout=datetime.timedelta(seconds=60))
    try:
        spec = ShardSpec(H, NQ, NKV, D, F, t, rank)
        ops = []
        for layer in range(3):
            w, _, kc, vc = _inputs(seed=100 + layer)
            ops.append(NumpyOps(spec, shard_weights(w, spec), shard_cache(kc, spec), shard_cache(vc, spec)))
        count = [0]

        def ar(T):
            count[0] += 1
            dist.all_reduce(T, op=dist.ReduceOp.SUM)
        _, x, _, _ = _inputs(seed=7)
        y32, _ = decode_stack_tp(ops, x, S, ar)
        q.put((rank, y32, count[0]))
    finally:
        dist.destroy_process_group()


def test_tp_stack_over_gloo_matches_a_sequence_of_oracle_layers():
    """Three layers, two ranks: 2L = 6 all-reduces, and the output of the
    oracle's layers applied in sequence."""
    t = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_stack_worker, args=(r, t, port, q)) for r in range(t)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = {r: (y, n) for r, y, n in (q.get(timeout=5) for _ in range(t))}
    _, cur, _, _ = _inputs(seed=7)
    for layer in range(3):
        w, _, kc, vc = _inputs(seed=100 + layer)
        cur = oracle.decode_layer(oracle.Dims(H, NQ, NKV, D, F, eps=EPS), w, cur, kc, vc, S)
    for r in range(t):
        y, n = res[r]
        assert n == 6
        np.testing.assert_allclose(y, cur, rtol=1e-9, atol=1e-9 * np.abs(cur).max())
