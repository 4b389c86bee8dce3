"""GPU parity of the decode layer with the projections on the 5th-generation
tensor cores (TPL_OPT_GEMV_MODE 3: weights streamed by TMA, tcgen05.mma,
stream-K work division): the same oracle checks as the default kernels, the
fused and separate row-split sums bit for bit, the stack as a sequence of
layers, and repeatable bits."""
import numpy as np
import pytest
import torch

from tests.conftest import has_gpu
from tests.test_gpu_parity import SMALL, _check_layer

pytestmark = pytest.mark.gpu

if has_gpu():
    import oracle
    from megatron_tensor_transformer_plan_b200 import tpl
    from tests.gpu_util import (assert_close_rel, make_layer, oracle_decode, oracle_dims, oracle_weights,
                                run_steps, to_np)

TC = 3


def tc_layer(*args, **kw):
    L = make_layer(*args, **kw)
    L.plan.set_option(tpl.TPL_OPT_GEMV_MODE, TC)
    return L


@pytest.mark.parametrize("case", SMALL)
def test_decode_layer_small_tc(gpu, case):
    H, nq, nkv, F, t, B, S, gs = case
    L = tc_layer(H, nq, nkv, 128, F, t, B, S, gamma_std=gs, S_cap=S + 3)
    ref_y, tr = oracle_decode(L)
    _check_layer(L, ref_y, tr)


@pytest.mark.parametrize("B", [1, 4, 8, 9, 16])
def test_batch_sizes_tc(gpu, B):
    """Every operand height: B <= 8 (16-column accumulators) and 9..16 (32)."""
    L = tc_layer(1024, 16, 8, 128, 2816, 8, B, 200)
    ref_y, tr = oracle_decode(L)
    _check_layer(L, ref_y, tr)


def test_config1_tiny_mlp_block_tc(gpu):
    H, F, t = 256, 688, 2
    L = tc_layer(H, 2, 2, 128, F, t, 1, 0, flags=0, mlp_only=True)
    w = oracle_weights(L)
    od = oracle_dims(L)
    ref = oracle.mlp_sharded(od, w, t, to_np(L.x))
    y = torch.empty((1, H), dtype=torch.bfloat16, device=gpu)
    y32 = torch.empty((1, H), dtype=torch.float32, device=gpu)
    L.plan.mlp_block(L.packed, L.x, y, y32, L.ws, tpl.TPL_REDUCE_FUSED)
    ys, ys32 = torch.empty_like(y), torch.empty_like(y32)
    L.plan.mlp_block(L.packed, L.x, ys, ys32, L.ws, tpl.TPL_REDUCE_SEPARATE)
    torch.cuda.synchronize()
    assert_close_rel(to_np(y32), ref, what="y32")
    assert torch.equal(y32, ys32) and torch.equal(y, ys)


@pytest.mark.parametrize("t", [1, 2, 4])
@pytest.mark.parametrize("B", [1, 16])
def test_config2_7b_layer_tc(gpu, t, B):
    L = tc_layer(4096, 32, 32, 128, 11008, t, B, 2048, seed=0)
    ref_y, tr = oracle_decode(L)
    _check_layer(L, ref_y, tr, mode_both=(B == 16))


@pytest.mark.slow
def test_config3_70b_layer_tc(gpu):
    L = tc_layer(8192, 64, 8, 128, 28672, 4, 16, 8192, seed=0)
    ref_y, tr = oracle_decode(L)
    _check_layer(L, ref_y, tr)


@pytest.mark.slow
def test_stack_shape_layer_tc(gpu):
    L = tc_layer(8192, 64, 8, 128, 28672, 8, 4, 4096, seed=0, layer=39)
    ref_y, tr = oracle_decode(L)
    _check_layer(L, ref_y, tr)


def test_tc_matches_default_kernels(gpu):
    """Both kernel families on the same layer: close (different summation
    order only)."""
    L = make_layer(1024, 16, 8, 128, 2816, 4, 5, 300)
    L.plan.set_option(tpl.TPL_OPT_GEMV_MODE, 0)  # the mma.sync family
    a = run_steps(L)
    L.plan.set_option(tpl.TPL_OPT_GEMV_MODE, TC)
    b = run_steps(L)
    # fp32 outputs to 2e-3; act is bf16, where the two may round one step apart
    for k, tol in (("q", 2e-3), ("h", 2e-3), ("act", 1e-2), ("y32", 2e-3)):
        assert_close_rel(to_np(b[k]), to_np(a[k]), tol=tol, what=k)


def test_stack_equals_layer_sequence_tc(gpu):
    H, nq, nkv, F, t, B, S, NL = 512, 8, 4, 1024, 4, 2, 50, 4
    layers = [tc_layer(H, nq, nkv, 128, F, t, B, S, seed=5, layer=l, n_layers=NL) for l in range(NL)]
    plan = layers[0].plan
    x = layers[0].x
    ws = plan.workspace(B, S)
    snaps = [(L.k.clone(), L.v.clone()) for L in layers]
    y_stack = torch.empty_like(x)
    plan.reset_counters()
    plan.decode_stack([L.packed for L in layers], [L.kv for L in layers], x, S, y_stack, None, ws)
    torch.cuda.synchronize()
    assert plan.reduction_count() == 2 * NL
    for L, (k, v) in zip(layers, snaps):
        L.k.copy_(k)
        L.v.copy_(v)
    cur = x
    for L in layers:
        nxt = torch.empty_like(x)
        plan.decode_layer(L.packed, L.kv, cur, S, nxt, None, ws)
        cur = nxt
    torch.cuda.synchronize()
    assert torch.equal(cur, y_stack)
    ys = torch.empty_like(x)
    plan.decode_stack([L.packed for L in layers], [L.kv for L in layers], x, S, ys, None, ws,
                      tpl.TPL_REDUCE_SEPARATE)
    torch.cuda.synchronize()
    assert torch.equal(ys, y_stack)


def test_stack_captured_in_cuda_graph(gpu):
    """The decode stack captured once into a CUDA graph (its launches and
    their programmatic-dependent-launch edges) and replayed gives the bits of
    the direct call, replay after replay (every arrival counter resets itself
    inside the kernels)."""
    H, nq, nkv, F, t, B, S, NL = 2048, 16, 4, 5632, 2, 4, 300, 3
    layers = [tc_layer(H, nq, nkv, 128, F, t, B, S, seed=9, layer=l, n_layers=NL) for l in range(NL)]
    plan = layers[0].plan
    x = layers[0].x
    ws = plan.workspace(B, S)
    snaps = [(L.k.clone(), L.v.clone()) for L in layers]
    y = torch.empty_like(x)
    plan.decode_stack([L.packed for L in layers], [L.kv for L in layers], x, S, y, None, ws)
    torch.cuda.synchronize()
    y_direct = y.clone()
    stream = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        plan.decode_stack([L.packed for L in layers], [L.kv for L in layers], x, S, y, None, ws)
    for _ in range(3):
        for L, (k, v) in zip(layers, snaps):
            L.k.copy_(k)
            L.v.copy_(v)
        y.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(y, y_direct)
    assert plan.last_device_error() == tpl.TPL_OK


def test_repeated_calls_are_deterministic_tc(gpu):
    L = tc_layer(1024, 16, 8, 128, 2816, 8, 16, 500)
    a = run_steps(L)["y32"].clone()
    for _ in range(3):
        b = run_steps(L)["y32"]
        assert torch.equal(a, b)
    assert L.plan.last_device_error() == tpl.TPL_OK
