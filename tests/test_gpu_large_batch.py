"""GPU parity of decode with 17..64 tokens per call, where every projection
runs on the tensor-core kernel (token columns up to 128: 64 hi + 64 lo rows of
the split activation) and its epilogue walks the tokens in chunks of 16: the
oracle checks of every intermediate, fused = separate bit for bit, the
step-by-step calls = the one-call layer, the stack = a sequence of layers."""
import pytest
import torch

from tests.conftest import has_gpu
from tests.test_gpu_parity import _check_layer

pytestmark = pytest.mark.gpu

if has_gpu():
    from megatron_tensor_transformer_plan_b200 import tpl
    from tests.gpu_util import make_layer, oracle_decode, run_steps


@pytest.mark.parametrize("B", [17, 24, 32, 33, 48, 64])
def test_batch_sizes_above_16(gpu, B):
    """Every operand width: 64-column (B <= 32) and 128-column (B <= 64)
    accumulators, ragged 16-token chunks."""
    L = make_layer(1024, 16, 8, 128, 2816, 8, B, 200, seed=21)
    ref_y, tr = oracle_decode(L)
    _check_layer(L, ref_y, tr)


@pytest.mark.parametrize("t", [1, 4])
def test_7b_layer_batch_64(gpu, t):
    L = make_layer(4096, 32, 32, 128, 11008, t, 64, 2048, seed=22)
    ref_y, tr = oracle_decode(L)
    _check_layer(L, ref_y, tr)


def test_gemv_mode_does_not_matter_above_16(gpu):
    """Above 16 tokens only the tensor-core kernel applies: modes 0, 3 and 4
    give the same bits."""
    L = make_layer(1024, 16, 8, 128, 2816, 4, 40, 100, seed=23)
    outs = []
    for mode in (0, 3, 4):
        L.plan.set_option(tpl.TPL_OPT_GEMV_MODE, mode)
        outs.append(run_steps(L)["y32"].clone())
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[1], outs[2])


def test_rope_batch_64(gpu):
    L = make_layer(1024, 16, 4, 128, 2816, 4, 64, 700, seed=24,
                   flags=tpl.TPL_NORM | tpl.TPL_RESIDUAL | tpl.TPL_ROPE)
    ref_y, tr = oracle_decode(L)
    _check_layer(L, ref_y, tr)


def test_stack_equals_layer_sequence_batch_64(gpu):
    H, nq, nkv, F, t, B, S, NL = 512, 8, 4, 1024, 4, 64, 50, 3
    layers = [make_layer(H, nq, nkv, 128, F, t, B, S, seed=25, layer=l, n_layers=NL) for l in range(NL)]
    plan, x = layers[0].plan, layers[0].x
    ws = plan.workspace(B, S)
    snaps = [(L.k.clone(), L.v.clone()) for L in layers]
    y_stack = torch.empty_like(x)
    plan.decode_stack([L.packed for L in layers], [L.kv for L in layers], x, S, y_stack, None, ws)
    torch.cuda.synchronize()
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
    assert plan.last_device_error() == tpl.TPL_OK


def test_repeated_calls_are_deterministic_batch_64(gpu):
    L = make_layer(1024, 16, 8, 128, 2816, 8, 64, 300, seed=26)
    a = run_steps(L)["y32"].clone()
    for _ in range(2):
        assert torch.equal(a, run_steps(L)["y32"])


@pytest.mark.slow
def test_70b_layer_batch_64(gpu):
    L = make_layer(8192, 64, 8, 128, 28672, 4, 64, 2048, seed=27)
    ref_y, tr = oracle_decode(L)
    _check_layer(L, ref_y, tr)
