"""The multi-GPU tensor-parallel layer's device steps (tp_dist.CudaOps) on one
GPU: the t ranks run as threads of one process, each with its own one-shard
plan, packed slice and cache shard; the all-reduce is emulated on the host
(the partials summed in rank order, then copied back to every rank).  No
kernel waits for another rank's.  Every rank's output matches the oracle's
unsharded layer."""
import threading

import numpy as np
import pytest
import torch

from tests.conftest import has_gpu

pytestmark = pytest.mark.gpu

if has_gpu():
    import oracle
    from megatron_tensor_transformer_plan_b200 import synth, tpl
    from megatron_tensor_transformer_plan_b200.tp_dist import (CudaOps, ShardSpec, decode_layer_tp, shard_cache,
                                                                shard_weights)
    from tests.gpu_util import assert_close_rel, to_np


@pytest.mark.parametrize("t", [1, 2, 4])
def test_tp_ranks_on_one_gpu_match_the_oracle(gpu, t):
    H, nq, nkv, d, F, B, S = 1024, 16, 4, 128, 2816, 3, 77
    w = synth.layer_weights(H, nq, nkv, d, F, seed=31, device=gpu)
    kl, vl = synth.kv_cache((B, nkv, S + 1, d), seed=31, device=gpu)
    x = synth.activations(B, H, seed=31, device=gpu)
    ops = []
    for r in range(t):
        spec = ShardSpec(H, nq, nkv, d, F, t, r)
        ops.append(CudaOps(spec, shard_weights(w, spec), shard_cache(kl, spec), shard_cache(vl, spec), B, S + 1))
    torch.cuda.synchronize()
    bar = threading.Barrier(t, timeout=60)
    slots, shared, out, errs = [None] * t, {}, [None] * t, []

    def make_all_reduce(r):
        def all_reduce(P):
            torch.cuda.synchronize()
            slots[r] = P
            bar.wait()
            if r == 0:
                tot = slots[0].clone()
                for i in range(1, t):
                    tot += slots[i]
                torch.cuda.synchronize()
                shared["sum"] = tot
            bar.wait()
            P.copy_(shared["sum"])
            torch.cuda.synchronize()
            bar.wait()
        return all_reduce

    def run(r):
        try:
            torch.cuda.set_device(gpu)
            y32, _ = decode_layer_tp(ops[r], x, S, make_all_reduce(r))
            torch.cuda.synchronize()
            out[r] = y32.clone()
        except Exception as e:  # noqa: BLE001 - reported below
            errs.append(e)
            bar.abort()

    threads = [threading.Thread(target=run, args=(r,)) for r in range(t)]
    for th in threads:
        th.start()
    for th in threads:
        th.join(timeout=120)
    assert not errs, errs
    for o in ops:
        assert o.plan.last_device_error() == tpl.TPL_OK
    wb = {k: synth.bits(v) for k, v in w.items()}
    ref = oracle.decode_layer(oracle.Dims(H, nq, nkv, d, F), wb, to_np(x), synth.bits(kl), synth.bits(vl), S)
    for r in range(t):
        assert_close_rel(to_np(out[r]), ref, what=f"y32 rank {r}")
        assert torch.equal(out[r], out[0])
